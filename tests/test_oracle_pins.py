"""Pins for the fp64 oracle, checked against what the HARP pages and mathematics fix.

Source: "HARP: Hadamard-Preconditioned Adaptive Rotation Processor for Extreme LLM
Quantization" (gist.science): Sec. 2.1 (stride stages of block-diagonal orthogonal
B_t between stride permutations), Sec. 2.2 (B = Q(theta) G_2, Givens Q, normalised
Sylvester G_2; Theta = 0 recovers the randomized Hadamard transform), Sec. 1 and 5
(an exact, orthogonal change of basis that preserves the full-precision layer).
Each test is chosen so that a plausible slip in the oracle (a dropped stage, a
wrong sign, a transposed factor, a mis-numbered pair, a wrong rounding rule) fails.
"""
import math

import numpy as np
import pytest
import scipy.linalg

from conftest import read_golden

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand_theta(rng, n, w, scale):
    m = int(math.log2(w))
    return rng.uniform(-scale, scale, size=(m, n // 2))


def _rand_sign(rng, n):
    return (rng.integers(0, 2, n) * 2 - 1).astype(np.int8)


def _dense(ora, n, w, theta, sign, inv=False):
    f = ora.butterfly_inv if inv else ora.butterfly_fwd
    # column j of the matrix is F e_j; the oracle acts on rows of a batch
    return f(np.eye(n), theta, sign, w).T


# ------------------------------------------------------------------ fp16 rounding
def test_f16_conversion_matches_numpy(ora):
    """The oracle's own fp64 -> fp16 rounding agrees with numpy's correctly rounded
    conversion on random values, exact ties, subnormals and the overflow edge."""
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(3000) * 0.02, rng.standard_normal(1000) * 300.0,
        rng.uniform(-1e-4, 1e-4, 1000), rng.uniform(-7e-8, 7e-8, 300),
        # exact midpoints between neighbouring fp16 values (ties to even)
        (np.arange(1024, 1100) + 0.5) * 2.0 ** -10, (np.arange(1, 60) + 0.5) * 2.0 ** -24,
        [65504.0, 65519.0, 65519.999, 65520.0, 70000.0, -65520.0, 2.0 ** -24, 2.0 ** -25,
         3 * 2.0 ** -26, 2.0 ** -14, 0.0, -0.0, 1.0 / 3.0],
    ])
    got = ora.f16_from_f64(vals)
    want = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, want)


def test_f16_decode_all_bit_patterns(ora):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    got = ora.f16_to_f64(bits)
    want = bits.view(np.float16).astype(np.float64)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], want[~nan])


# ------------------------------------------------------------------ P1: Theta = 0
@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64])
def test_theta0_is_sylvester_hadamard(ora, n):
    """F(0, s, n) = H_n diag(s) / sqrt(n) with H_n the Sylvester Hadamard matrix."""
    rng = np.random.default_rng(n)
    s = _rand_sign(rng, n)
    M = _dense(ora, n, n, np.zeros((int(math.log2(n)), n // 2)), s)
    want = scipy.linalg.hadamard(n) @ np.diag(s.astype(float)) / math.sqrt(n)
    assert np.max(np.abs(M - want)) < 1e-14


@pytest.mark.parametrize("n", [1024, 2048])
def test_theta0_hadamard_spot(ora, n):
    rng = np.random.default_rng(7)
    s = _rand_sign(rng, n)
    x = rng.standard_normal((3, n))
    got = ora.butterfly_fwd(x, np.zeros((int(math.log2(n)), n // 2)), s, n)
    want = (x * s) @ scipy.linalg.hadamard(n).T / math.sqrt(n)
    assert np.max(np.abs(got - want)) < 1e-12


def test_theta0_block_diagonal_hadamard(ora):
    n, w = 64, 16
    s = _rand_sign(np.random.default_rng(3), n)
    M = _dense(ora, n, w, np.zeros((4, n // 2)), s)
    want = np.kron(np.eye(n // w), scipy.linalg.hadamard(w)) @ np.diag(s.astype(float)) / 4.0
    assert np.max(np.abs(M - want)) < 1e-14


# ------------------------------------------------------------------ golden values
def test_golden_butterfly(ora):
    for (nw, th, sg, x, want) in read_golden("butterfly_examples.txt"):
        n, w = int(nw[0]), int(nw[1])
        theta = np.array([float(t) for t in th]).reshape(int(math.log2(w)), n // 2)
        got = ora.butterfly_fwd(np.array([float(t) for t in x]), theta,
                                np.array([int(t) for t in sg], np.int8), w)
        assert np.allclose(got, [float(t) for t in want], rtol=0, atol=1e-15), (nw, got, want)


# ------------------------------------------------------------------ P2: orthogonality
@pytest.mark.parametrize("n,w,scale", [(4096, 4096, 0.05), (11008, 256, 0.05),
                                       (2048, 512, 3.0), (28672, 4096, 0.05)])
def test_orthogonal_norm_and_inverse(ora, n, w, scale):
    rng = np.random.default_rng(n + w)
    th, s = _rand_theta(rng, n, w, scale), _rand_sign(rng, n)
    x = rng.standard_normal((2, n))
    y = ora.butterfly_fwd(x, th, s, w)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13, atol=0)
    assert np.max(np.abs(ora.butterfly_inv(y, th, s, w) - x)) < 1e-12
    assert np.max(np.abs(ora.butterfly_fwd(ora.butterfly_inv(x, th, s, w), th, s, w) - x)) < 1e-12


@pytest.mark.parametrize("n,w", [(16, 16), (64, 64), (64, 8)])
def test_dense_orthogonal_and_transpose(ora, n, w):
    rng = np.random.default_rng(11)
    th, s = _rand_theta(rng, n, w, 1.0), _rand_sign(rng, n)
    M = _dense(ora, n, w, th, s)
    assert np.max(np.abs(M.T @ M - np.eye(n))) < 1e-14
    assert np.max(np.abs(_dense(ora, n, w, th, s, inv=True) - M.T)) < 1e-14


# ------------------------------------------------------------------ structure of the stages
def _stride_perm(n, w, t):
    """Permutation matrix P that lists, block by block of 2^(t+1) coordinates, the
    pairs (i, i + 2^t) next to each other (interleaving the two halves of the block)."""
    h = 1 << t
    order = []
    for base in range(0, n, 2 * h):
        for i in range(h):
            order += [base + i, base + i + h]
    P = np.zeros((n, n))
    P[np.arange(n), order] = 1.0
    return P


def _page_block(theta):
    """B(theta) = Q(theta) G_2: Givens rotation times the normalised Sylvester H_2."""
    c, s = math.cos(theta), math.sin(theta)
    Q = np.array([[c, -s], [s, c]])
    G2 = np.array([[1.0, 1.0], [1.0, -1.0]]) / math.sqrt(2.0)
    return Q @ G2


def _page_butterfly(n, w, theta, sign):
    """Dense F built from the pages' description: D first, then for t = 0..m-1 the
    block-diagonal B_t conjugated by the stride permutation of stage t; pair c of
    stage t takes theta[t][c]."""
    m = int(math.log2(w))
    F = np.diag(sign.astype(float))
    for t in range(m):
        P = _stride_perm(n, w, t)
        Bt = scipy.linalg.block_diag(*[_page_block(theta[t][c]) for c in range(n // 2)])
        F = P.T @ Bt @ P @ F
    return F


@pytest.mark.parametrize("n,w", [(8, 8), (16, 16), (32, 32), (32, 8), (64, 16)])
def test_stages_match_stride_permutation_construction(ora, n, w):
    rng = np.random.default_rng(n * 7 + w)
    th, s = _rand_theta(rng, n, w, 1.5), _rand_sign(rng, n)
    assert np.max(np.abs(_dense(ora, n, w, th, s) - _page_butterfly(n, w, th, s))) < 1e-13


def test_single_angle_moves_only_its_pair(ora):
    """Changing theta[t][p] alone changes the output exactly as the page block predicts."""
    n = w = 16
    rng = np.random.default_rng(5)
    s = _rand_sign(rng, n)
    base = np.zeros((4, n // 2))
    for t in range(4):
        for p in (0, 3, 7):
            th = base.copy()
            th[t, p] = 0.3
            assert np.max(np.abs(_dense(ora, n, w, th, s) - _page_butterfly(n, w, th, s))) < 1e-14


# ------------------------------------------------------------------ P6: block diagonal
def test_block_diagonal_equals_independent_blocks(ora):
    n, w = 11008, 256
    rng = np.random.default_rng(9)
    th, s = _rand_theta(rng, n, w, 0.05), _rand_sign(rng, n)
    x = rng.standard_normal(n)
    got = ora.butterfly_fwd(x, th, s, w)
    for k in (0, 17, 42):
        sl = slice(k * w, (k + 1) * w)
        th_k = th[:, k * (w // 2):(k + 1) * (w // 2)]
        assert np.max(np.abs(got[sl] - ora.butterfly_fwd(x[sl], th_k, s[sl], w))) < 1e-15


# ------------------------------------------------------------------ theta = -pi/4: diagonal
def test_theta_minus_quarter_pi_is_diagonal(ora):
    """psi = 0 makes every block diag(1, -1): F = diag(s_i (-1)^popcount(i mod w))."""
    n, w = 256, 64
    s = _rand_sign(np.random.default_rng(2), n)
    th = np.full((6, n // 2), -math.pi / 4)
    x = np.random.default_rng(3).standard_normal(n)
    par = np.array([(-1.0) ** bin(i % w).count("1") for i in range(n)])
    assert np.max(np.abs(ora.butterfly_fwd(x, th, s, w) - s * par * x)) < 1e-15


# ------------------------------------------------------------------ P3: exact change of basis
@pytest.mark.parametrize("n_out,n_in,w_in,w_out", [(256, 512, 512, 256), (384, 256, 256, 128),
                                                   (128, 1024, 64, 128)])
def test_rotation_is_exact_change_of_basis(ora, n_out, n_in, w_in, w_out):
    rng = np.random.default_rng(n_out + n_in)
    W = rng.standard_normal((n_out, n_in)) * 0.02
    thV, sV = _rand_theta(rng, n_in, w_in, 0.5), _rand_sign(rng, n_in)
    thU, sU = _rand_theta(rng, n_out, w_out, 0.5), _rand_sign(rng, n_out)
    Wr = ora.rotate_weights(W, thV, sV, w_in, thU, sU, w_out)
    x = rng.standard_normal((3, n_in))
    y = ora.dense_rotated_fwd(Wr, thV, sV, w_in, thU, sU, w_out, x)
    want = x @ W.T
    assert np.linalg.norm(y - want) / np.linalg.norm(want) < 1e-12
    # and W' = U W V^T with V = F_V, U = F_U^T built from the pages' construction
    if n_out <= 256 and n_in <= 512:
        FV = _page_butterfly(n_in, w_in, thV, sV)
        FU = _page_butterfly(n_out, w_out, thU, sU)
        assert np.max(np.abs(Wr - FU.T @ W @ FV.T)) < 1e-13


# ------------------------------------------------------------------ P4: quantizer
def _deq(q, s16, z16, ora, group=64):
    s = ora.f16_to_f64(s16).repeat(group, axis=1)
    z = ora.f16_to_f64(z16).repeat(group, axis=1)
    return s * q + z, s, z


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_quantizer_is_nearest_level(ora, bits):
    rng = np.random.default_rng(bits)
    W = rng.standard_normal((48, 512)) * 0.02
    W[:, 5] *= 20.0
    W[3, 64:128] = 0.125           # constant group -> scale 1
    W[4, 128:192] = rng.standard_normal(64) * 1e-7   # tiny range
    q, s16, z16 = ora.quantize(W, bits)
    L = (1 << bits) - 1
    assert q.max() <= L
    mn = W.reshape(48, 8, 64).min(-1)
    mx = W.reshape(48, 8, 64).max(-1)
    want_z = mn.astype(np.float16).view(np.uint16)
    want_s = ((mx - mn) / L).astype(np.float16).view(np.uint16)
    want_s = np.where(want_s == 0, np.uint16(0x3C00), want_s)
    assert np.array_equal(z16, want_z) and np.array_equal(s16, want_s)
    deq, s, z = _deq(q, s16, z16, ora)
    levels = s[..., None] * np.arange(L + 1) + z[..., None]
    dist = np.abs(W[..., None] - levels)
    best = dist.min(-1)
    mine = np.abs(W - deq)
    assert np.all(mine <= best * (1 + 1e-12) + 1e-300)
    unclamped = (q > 0) & (q < L)
    assert np.all(mine[unclamped] <= s[unclamped] / 2 * (1 + 1e-9))
    ulp_z = np.abs(np.spacing(z.astype(np.float16)).astype(np.float64))
    assert np.all(mine <= s / 2 * (1 + 1e-9) + ulp_z + 1e-300)


def test_golden_quantize(ora):
    for (bits, vals, sb, zb, codes) in read_golden("quantize_examples.txt"):
        b = int(bits[0])
        W = np.array([[float(v) for v in vals]])
        assert W.shape == (1, 64)
        q, s16, z16 = ora.quantize(W, b)
        assert s16[0, 0] == int(sb[0], 16) and z16[0, 0] == int(zb[0], 16)
        assert q[0].tolist() == [int(c) for c in codes]


# ------------------------------------------------------------------ P5: packing
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_pack_roundtrip(ora, bits):
    rng = np.random.default_rng(40 + bits)
    q = rng.integers(0, 1 << bits, (12, 320)).astype(np.uint8)
    p = ora.pack(q, bits)
    assert p.size == 12 * 320 * bits // 8
    assert np.array_equal(ora.unpack(p, 12, 320, bits), q)


def test_golden_pack(ora):
    for (bits, codes, want) in read_golden("pack_examples.txt"):
        b = int(bits[0])
        q = np.array([[int(c) for c in codes]], np.uint8)
        assert q.shape == (1, 64)
        assert ora.pack(q, b).tolist() == [int(h, 16) for h in want]


# ------------------------------------------------------------------ P8: brute-force linear
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_linear_matches_dense_brute_force(ora, bits):
    n_out, n_in, w_in, w_out = 64, 128, 64, 32
    rng = np.random.default_rng(100 + bits)
    W = rng.standard_normal((n_out, n_in)) * 0.02
    thV, sV = _rand_theta(rng, n_in, w_in, 0.3), _rand_sign(rng, n_in)
    thU, sU = _rand_theta(rng, n_out, w_out, 0.3), _rand_sign(rng, n_out)
    lay, q, s16, z16, Wr = ora.prepare_layer(W, bits, w_in, w_out, thV, sV, thU, sU)
    deq, _, _ = _deq(q, s16, z16, ora)
    FV = _page_butterfly(n_in, w_in, thV, sV)
    FU = _page_butterfly(n_out, w_out, thU, sU)
    x = rng.standard_normal((4, n_in))
    want = (FU @ deq @ FV @ x.T).T
    got = ora.linear_fwd(lay, x)
    assert np.max(np.abs(got - want)) < 1e-13 * np.max(np.abs(want))
    # quantization error stays at the level the half-step bound allows
    assert np.linalg.norm(got - x @ W.T) / np.linalg.norm(x @ W.T) < {2: 0.6, 3: 0.3, 4: 0.15}[bits]


def test_linear_integer_special_case(ora):
    """theta = -pi/4 (diagonal butterflies), scale 1, zero 0: y = D_U Q D_V x exactly."""
    n_out, n_in = 64, 128
    rng = np.random.default_rng(8)
    q = rng.integers(0, 4, (n_out, n_in)).astype(np.uint8)
    sz = np.zeros((n_out, n_in // 64, 2), np.uint16)
    sz[..., 0] = 0x3C00
    thV = np.full((7, n_in // 2), -math.pi / 4)
    thU = np.full((6, n_out // 2), -math.pi / 4)
    sV, sU = _rand_sign(rng, n_in), _rand_sign(rng, n_out)
    lay = ora.Layer(n_in, n_out, 2, n_in, n_out, thV, sV, thU, sU, ora.pack(q, 2), sz)
    x = rng.integers(-8, 9, (2, n_in)).astype(float)
    dV = sV * np.array([(-1.0) ** bin(i).count("1") for i in range(n_in)])
    dU = sU * np.array([(-1.0) ** bin(i).count("1") for i in range(n_out)])
    want = ((q.astype(float) @ (x * dV).T).T) * dU
    assert np.array_equal(ora.linear_fwd(lay, x), want)


# ------------------------------------------------------------------ stack step
def _tiny_stack(ora, n_layers, zero=(), seed=0):
    hidden, ffn, nh, nkv, hd = 128, 192, 4, 2, 32
    shapes = [(nh * hd, hidden), (nkv * hd, hidden), (nkv * hd, hidden), (hidden, nh * hd),
              (ffn, hidden), (ffn, hidden), (hidden, ffn)]
    rng = np.random.default_rng(seed)
    layers = []
    for l in range(n_layers):
        for i, (n_out, n_in) in enumerate(shapes):
            W = rng.standard_normal((n_out, n_in)) * 0.05
            if i in zero:
                W[:] = 0.0
            w_in, w_out = (64 if n_in == ffn else n_in), (64 if n_out == ffn else n_out)
            thV, sV = _rand_theta(rng, n_in, w_in, 0.05), _rand_sign(rng, n_in)
            thU, sU = _rand_theta(rng, n_out, w_out, 0.05), _rand_sign(rng, n_out)
            layers.append(ora.prepare_layer(W, 2, w_in, w_out, thV, sV, thU, sU)[0])
    return layers, (hidden, ffn, nh, nkv, hd)


def test_stack_zero_output_projections_is_identity(ora):
    """With o_proj and down_proj weights all zero both residual branches vanish."""
    layers, dims = _tiny_stack(ora, 2, zero=(3, 6))
    x = np.random.default_rng(1).standard_normal((2, dims[0]))
    assert np.array_equal(ora.stack_step(layers, *dims, x), x)


def test_stack_q_k_do_not_reach_output(ora):
    """A one-key attention returns its value: q_proj and k_proj cannot change the step."""
    a, dims = _tiny_stack(ora, 1, seed=3)
    b, _ = _tiny_stack(ora, 1, seed=4)
    mixed = [b[0], b[1]] + a[2:]
    x = np.random.default_rng(2).standard_normal((1, dims[0]))
    assert np.array_equal(ora.stack_step(a, *dims, x), ora.stack_step(mixed, *dims, x))


def test_stack_zero_up_kills_mlp(ora):
    """silu(g) * 0 = 0: with up_proj zero the MLP branch is exactly zero."""
    layers, dims = _tiny_stack(ora, 1, zero=(5,), seed=6)
    ref, _ = _tiny_stack(ora, 1, zero=(5, 6), seed=6)
    x = np.random.default_rng(7).standard_normal((1, dims[0]))
    assert np.array_equal(ora.stack_step(layers, *dims, x), ora.stack_step(ref, *dims, x))


def _sparse_exact_layer(ora, n_out, n_in, w_in, w_out, entries, rng):
    """A layer whose dequantized rotated matrix is exactly known: theta = -pi/4 makes both
    butterflies diagonal (+-1, see test_linear_integer_special_case), scale 1 and zero 0
    make dequant(q) = q, and `entries` maps output row i -> (input column j, code value).
    Returns the oracle layer and the effective dense matrix D_U Q D_V."""
    q = np.zeros((n_out, n_in), np.uint8)
    for i, (j, v) in entries.items():
        q[i, j] = v
    sz = np.zeros((n_out, n_in // 64, 2), np.uint16)
    sz[..., 0] = 0x3C00  # fp16 1.0
    mV, mU = int(math.log2(w_in)), int(math.log2(w_out))
    thV = np.full((mV, n_in // 2), -math.pi / 4)
    thU = np.full((mU, n_out // 2), -math.pi / 4)
    sV, sU = _rand_sign(rng, n_in), _rand_sign(rng, n_out)
    dV = sV * np.array([(-1.0) ** bin(i % w_in).count("1") for i in range(n_in)])
    dU = sU * np.array([(-1.0) ** bin(i % w_out).count("1") for i in range(n_out)])
    lay = ora.Layer(n_in, n_out, 2, w_in, w_out, thV, sV, thU, sU, ora.pack(q, 2), sz)
    return lay, dU[:, None] * q.astype(float) * dV[None, :]


def test_stack_glue_closed_form(ora):
    """Every linear is a sparse exact map and the input a constant vector, so each glue
    step reduces to a scalar closed form:
    - RMSNorm of c*1 is c / sqrt(c^2 + eps) per element;
    - the one-key attention copies kv head h // rep into query head h;
    - SiLU(g) = g / (1 + e^-g) gates the up value.
    A swapped gate/up, a sigmoid in place of SiLU, eps outside the root, a missing residual
    or the kv groups taken modulo instead of by division each change the result."""
    hidden, ffn, nh, nkv, hd = 128, 192, 4, 2, 32
    dq, dkv, rep = nh * hd, nkv * hd, nh // nkv
    eps, c = 1e-5, 0.75
    rng = np.random.default_rng(21)
    # q, k: anything (a one-key attention ignores them)
    lq, _ = _sparse_exact_layer(ora, dq, hidden, hidden, dq, {0: (1, 1)}, rng)
    lk, _ = _sparse_exact_layer(ora, dkv, hidden, hidden, dkv, {0: (2, 3)}, rng)
    # v: kv head 1, dim 5 <- input 7 (code 2); o: output 9 <- query head 2, dim 5 (code 3);
    # head 2 reads kv head 2 // rep = 1 (2 % rep would be kv head 0, which is all zero)
    lv, Mv = _sparse_exact_layer(ora, dkv, hidden, hidden, dkv, {32 + 5: (7, 2)}, rng)
    lo, Mo = _sparse_exact_layer(ora, hidden, dq, dq, hidden, {9: (2 * hd + 5, 3)}, rng)
    # gate/up rows 10 and 70 read inputs 9 and 40; down output 20 <- ffn rows 10 and 70
    lg, Mg = _sparse_exact_layer(ora, ffn, hidden, hidden, 64, {10: (9, 1), 70: (40, 2)}, rng)
    lu, Mu = _sparse_exact_layer(ora, ffn, hidden, hidden, 64, {10: (40, 3), 70: (9, 1)}, rng)
    ld, Md = _sparse_exact_layer(ora, hidden, ffn, 64, hidden, {20: (10, 1), 21: (70, 2)}, rng)
    x = np.full((1, hidden), c)
    got = ora.stack_step([lq, lk, lv, lo, lg, lu, ld], hidden, ffn, nh, nkv, hd, x, eps=eps)

    a1 = c / math.sqrt(c * c + eps)                      # RMSNorm of a constant vector
    v = Mv[32 + 5, 7] * a1                               # the only nonzero of v
    # query head 2 reads kv head 2 // rep = 1: its dim 5 carries v
    o9 = Mo[9, 2 * hd + 5] * v
    h1 = np.full(hidden, c)
    h1[9] += o9
    r2 = 1.0 / math.sqrt(float(np.mean(h1 * h1)) + eps)
    n9, n40 = h1[9] * r2, h1[40] * r2
    g10, g70 = Mg[10, 9] * n9, Mg[70, 40] * n40
    u10, u70 = Mu[10, 40] * n40, Mu[70, 9] * n9
    silu = lambda t: t / (1.0 + math.exp(-t))
    m10, m70 = silu(g10) * u10, silu(g70) * u70
    want = h1.copy()
    want[20] += Md[20, 10] * m10
    want[21] += Md[21, 70] * m70
    assert np.max(np.abs(got[0] - want)) < 1e-13
    assert o9 != 0 and m10 != 0 and m70 != 0  # the case exercises every branch


# ------------------------------------------------------------------ calibration objective
def _calib_case(seed, n_out=128, n_in=256, w_in=128, w_out=64, bits=2):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((n_out, n_in)) * 0.02
    W[:, 7] *= 20.0  # an outlier input column, as in the workloads
    thV, thU = _rand_theta(rng, n_in, w_in, 0.05), _rand_theta(rng, n_out, w_out, 0.05)
    sV, sU = _rand_sign(rng, n_in), _rand_sign(rng, n_out)
    return W, bits, w_in, w_out, thV, sV, thU, sU


def _spd(rng, n):
    """A Hessian proxy X^T X / N of heavy-tailed activations with two outlier channels."""
    X = rng.standard_t(4, size=(3 * n, n))
    X[:, 3] *= 8.0
    X[:, n - 5] *= 5.0
    return X.T @ X / X.shape[0]


def _off_group(M, group=64):
    n = M.shape[0]
    blk = np.arange(n) // group
    return float(np.sum(np.where(blk[:, None] != blk[None, :], M * M, 0.0)))


def test_calib_identity_hessian_is_the_rotated_quantization_error(ora):
    """H = I: d = 1 and R_bd = 0, so L_diag is the quantization error of W' itself,
    formed here from rotate_weights and quantize."""
    W, bits, w_in, w_out, thV, sV, thU, sU = _calib_case(1)
    Wr = ora.rotate_weights(W, thV, sV, w_in, thU, sU, w_out)
    q, s16, z16 = ora.quantize(Wr, bits)
    s = np.repeat(s16.view(np.float16).astype(np.float64), 64, axis=1)
    z = np.repeat(z16.view(np.float16).astype(np.float64), 64, axis=1)
    want = float(np.sum((Wr - (s * q + z)) ** 2))
    Lf, Ld, Rb = ora.calib_fit(W, bits, w_in, w_out, thV, sV, thU, sU, lambda_bd=7.0)
    assert abs(Ld - want) <= 1e-10 * want and Rb == 0.0 and Lf == Ld
    Lf2, Ld2, Rb2 = ora.calib_fit(W, bits, w_in, w_out, thV, sV, thU, sU, H=np.eye(W.shape[1]), lambda_bd=7.0)
    assert abs(Ld2 - want) <= 1e-10 * want and Rb2 < 1e-24


def test_calib_identity_hessian_matches_the_linear(ora):
    """The butterflies are orthogonal, so with H = I L_diag is also ||W - W^||_F^2 with W^
    the dequantized layer: its columns are linear_fwd of the unit vectors, on the linear's
    own path (F_U(deq . F_V(x)), codes unpacked on the fly)."""
    W, bits, w_in, w_out, thV, sV, thU, sU = _calib_case(2)
    lay = ora.prepare_layer(W, bits, w_in, w_out, thV, sV, thU, sU)[0]
    What = ora.linear_fwd(lay, np.eye(W.shape[1])).T
    want = float(np.sum((W - What) ** 2))
    got = ora.calib_fit(W, bits, w_in, w_out, thV, sV, thU, sU)[1]
    assert abs(got - want) <= 1e-9 * want


def test_calib_diagonal_weight_under_the_hadamard_transform(ora):
    """Theta_V = 0 and w_in = n_in make V a signed Sylvester Hadamard matrix / sqrt(n), all
    of whose entries square to 1/n: for H = diag(a), every d_j = mean(a), so L_diag is
    mean(a) times the unweighted error."""
    W, bits, _, w_out, _, sV, thU, sU = _calib_case(3)
    n_in = W.shape[1]
    zero = np.zeros((int(np.log2(n_in)), n_in // 2))
    a = np.random.default_rng(5).uniform(0.1, 9.0, n_in)
    L1 = ora.calib_fit(W, bits, n_in, w_out, zero, sV, thU, sU)[1]
    La = ora.calib_fit(W, bits, n_in, w_out, zero, sV, thU, sU, H=np.diag(a))[1]
    assert abs(La - a.mean() * L1) <= 1e-10 * La


def test_calib_block_penalty_invariants(ora):
    """R_bd(c I) = 0 for any rotation (V V^T = I); R_bd is quadratic and L_diag linear in H;
    with butterfly blocks inside the 64-column groups (w_in = 32) V mixes only within a
    group, so R_bd equals the off-group energy of H itself."""
    rng = np.random.default_rng(6)
    W, bits, w_in, w_out, thV, sV, thU, sU = _calib_case(4)
    n_in = W.shape[1]
    H = _spd(rng, n_in)
    assert ora.calib_fit(W, bits, w_in, w_out, thV, sV, thU, sU, H=3.0 * np.eye(n_in))[2] < 1e-20
    _, Ld1, Rb1 = ora.calib_fit(W, bits, w_in, w_out, thV, sV, thU, sU, H=H)
    _, Ld2, Rb2 = ora.calib_fit(W, bits, w_in, w_out, thV, sV, thU, sU, H=2.0 * H)
    assert Rb1 > 0 and abs(Rb2 - 4.0 * Rb1) <= 1e-10 * Rb2 and abs(Ld2 - 2.0 * Ld1) <= 1e-10 * Ld2
    th32 = _rand_theta(rng, n_in, 32, 0.3)
    Rb = ora.calib_fit(W, bits, 32, w_out, th32, sV, thU, sU, H=H)[2]
    want = _off_group(H)
    assert abs(Rb - want) <= 1e-10 * want
    # and a 128-wide V does move energy across groups
    assert abs(Rb1 - want) > 1e-3 * want


@pytest.mark.parametrize("theta_scale", [0.0, 0.05])
def test_calib_gradient_matches_finite_differences(ora, theta_scale):
    """dL_fit/dtheta against central differences of the loss with the code target frozen,
    written densely here: V, U as matrices (butterflies of the unit vectors),
    W' = U W V^T, H' = V H V^T, L = sum d_j (W' - T)^2 + lambda sum_off H'^2. Checked along
    random directions and on single angles of both butterflies, at the Hadamard start
    (Theta = 0) and away from it."""
    rng = np.random.default_rng(7)
    n_out, n_in, w_in, w_out, bits, lam = 64, 256, 128, 32, 2, 0.3  # V blocks span two groups
    W = rng.standard_normal((n_out, n_in)) * 0.02
    W[:, 9] *= 15.0
    thV = _rand_theta(rng, n_in, w_in, theta_scale)
    thU = _rand_theta(rng, n_out, w_out, theta_scale)
    sV, sU = _rand_sign(rng, n_in), _rand_sign(rng, n_out)
    H = _spd(rng, n_in)
    (Lf, Ld, Rb), gV, gU = ora.calib_fit(W, bits, w_in, w_out, thV, sV, thU, sU, H=H, lambda_bd=lam, grad=True)
    Wr = ora.rotate_weights(W, thV, sV, w_in, thU, sU, w_out)
    q, s16, z16 = ora.quantize(Wr, bits)
    T = np.repeat(s16.view(np.float16).astype(np.float64), 64, axis=1) * q + \
        np.repeat(z16.view(np.float16).astype(np.float64), 64, axis=1)

    def loss(tV, tU):
        V = _dense(ora, n_in, w_in, tV, sV)
        U = _dense(ora, n_out, w_out, tU, sU).T
        Wp = U @ W @ V.T
        Hp = V @ H @ V.T
        return float(np.sum(np.diag(Hp)[None, :] * (Wp - T) ** 2)) + lam * _off_group(Hp)

    assert abs(loss(thV, thU) - Lf) <= 1e-10 * Lf
    eps = 1e-5
    for k in range(3):
        dV, dU = rng.standard_normal(thV.shape), rng.standard_normal(thU.shape)
        fd = (loss(thV + eps * dV, thU + eps * dU) - loss(thV - eps * dV, thU - eps * dU)) / (2 * eps)
        an = float(np.sum(gV * dV) + np.sum(gU * dU))
        assert abs(fd - an) <= 1e-6 * max(abs(an), 1e-3), (k, fd, an)
    for (side, t, p) in [("V", 0, 3), ("V", 5, 40), ("U", 0, 1), ("U", 4, 17)]:
        dV, dU = np.zeros_like(thV), np.zeros_like(thU)
        (dV if side == "V" else dU)[t, p] = 1.0
        fd = (loss(thV + eps * dV, thU + eps * dU) - loss(thV - eps * dV, thU - eps * dU)) / (2 * eps)
        an = float((gV if side == "V" else gU)[t, p])
        assert abs(fd - an) <= 1e-6 * max(abs(an), 1e-2), (side, t, p, fd, an)


def test_calib_degenerate_cases(ora):
    """Zero for W = 0 with H = I (every group constant, exact); more bits reduce L_diag."""
    W, bits, w_in, w_out, thV, sV, thU, sU = _calib_case(8)
    assert ora.calib_fit(np.zeros_like(W), bits, w_in, w_out, thV, sV, thU, sU) == (0.0, 0.0, 0.0)
    errs = [ora.calib_fit(W, b, w_in, w_out, thV, sV, thU, sU)[1] for b in (2, 3, 4)]
    assert errs[0] > errs[1] > errs[2]


# ------------------------------------------------------------------ int8 angles
def test_angle_q8_hand_example(ora):
    """Hand-computed: stage 0 has max |theta| = 0.127, so delta = fp32(0.001), and
    0.127 -> 127, -0.0636 -> -63.6 -> -64, 0.001 -> 0.99999995 -> 1, 0 -> 0. An all-zero
    stage has delta 0 and codes 0."""
    th = np.array([[0.127, -0.0636, 0.001, 0.0], [0.0, 0.0, 0.0, 0.0]])
    q, d = ora.quantize_angles(th)
    assert q.tolist() == [[127, -64, 1, 0], [0, 0, 0, 0]]
    assert d[0] == np.float32(0.001) and d[1] == 0.0


def test_angle_q8_is_the_nearest_code(ora):
    """Brute force over all 255 codes of each stage's step: the chosen code is the nearest
    (ties to even), so |theta^ - theta| <= delta / 2, and the largest angle of a stage
    reaches +-127."""
    rng = np.random.default_rng(21)
    th = rng.uniform(-0.05, 0.05, (6, 96)) * rng.uniform(0.1, 3.0, (6, 1))
    th[2, 5] = 0.0
    th[3] = np.round(th[3] * 1e3) / 1e3  # many values on exact grid points
    q, d = ora.quantize_angles(th)
    codes = np.arange(-127, 128, dtype=np.float64)
    for t in range(th.shape[0]):
        dist = np.abs(th[t][:, None] - float(d[t]) * codes[None, :])
        best = dist.min(axis=1)
        mine = np.abs(th[t] - float(d[t]) * q[t])
        assert np.all(mine <= best + 1e-18)
        assert np.all(mine <= float(d[t]) / 2 * (1 + 1e-12))
        assert np.abs(q[t]).max() == 127
    assert np.array_equal(ora.dequantize_angles(q, d), d.astype(np.float64)[:, None] * q)


def test_angle_q8_butterfly_error_bound(ora):
    """Each 2x2 block moves by at most |d theta| in operator norm (its derivative in the
    angle is orthogonal), so ||F(theta^) x - F(theta) x|| <= sum_t max_p |d theta_tp| ||x||,
    and with the nearest code that is at most sum_t delta_t / 2."""
    rng = np.random.default_rng(22)
    n, w = 1024, 1024
    th = _rand_theta(rng, n, w, 0.05)
    s = _rand_sign(rng, n)
    q, d = ora.quantize_angles(th)
    thq = ora.dequantize_angles(q, d)
    x = rng.standard_normal((4, n))
    diff = np.linalg.norm(ora.butterfly_fwd(x, thq, s, w) - ora.butterfly_fwd(x, th, s, w), axis=1)
    bound = np.abs(thq - th).max(axis=1).sum()
    assert np.all(diff <= bound * np.linalg.norm(x, axis=1) * (1 + 1e-9))
    assert bound <= d.astype(np.float64).sum() / 2 * (1 + 1e-12)
    assert diff.max() > 0


# ------------------------------------------------------------------ mixed-radix schedules
def _mr_theta(rng, radices, scale):
    return rng.uniform(-scale, scale, oracle_mr_size(radices))


def oracle_mr_size(radices):
    d = int(np.prod(radices))
    return sum((d // b) * (1 if b == 2 else b * (b - 1) // 2) for b in radices)


def _gauss(rng, radices):
    return [None if (b & (b - 1)) == 0 else rng.standard_normal((b, b)) for b in radices]


def _mr_dense(ora, radices, theta, sign, gauss=None, inverse=False):
    d = int(np.prod(radices))
    f = ora.mr_butterfly_inv if inverse else ora.mr_butterfly_fwd
    return f(np.eye(d), radices, theta, sign, gauss).T


def test_mr_all_radix2_is_the_butterfly(ora):
    """Every b_t = 2: the mixed-radix schedule is the radix-2 butterfly, parameters in the
    same stage-major, pair-numbered order."""
    rng = np.random.default_rng(31)
    d = 256
    th = _rand_theta(rng, d, d, 0.3)
    s = _rand_sign(rng, d)
    x = rng.standard_normal((3, d))
    rad = [2] * 8
    assert np.allclose(ora.mr_butterfly_fwd(x, rad, th.reshape(-1), s), ora.butterfly_fwd(x, th, s, d), atol=1e-13)
    assert np.allclose(ora.mr_butterfly_inv(x, rad, th.reshape(-1), s), ora.butterfly_inv(x, th, s, d), atol=1e-13)


@pytest.mark.parametrize("radices", [(8, 8), (4, 2, 8), (16, 4), (2, 32), (64,)])
def test_mr_hadamard_start_power_of_two(ora, radices):
    """Theta = 0 with power-of-two radices: every block is a Sylvester H_b / sqrt(b) and
    their Kronecker product over the digits is H_d (Sec. 2.2: HARP starts at the fixed
    randomized Hadamard transform)."""
    from scipy.linalg import hadamard
    rng = np.random.default_rng(32)
    d = int(np.prod(radices))
    s = _rand_sign(rng, d)
    F = _mr_dense(ora, radices, np.zeros(oracle_mr_size(radices)), s)
    assert np.allclose(F, hadamard(d) * s[None, :] / np.sqrt(d), atol=1e-13)


def test_mr_hadamard_start_kronecker_with_odd_radices(ora):
    """Theta = 0, schedule (3, 4, 5): stage t mixes digit t (stride b_0...b_{t-1}), so F is
    kron(G_5, G_4, G_3) D with the slowest digit's mixer leftmost."""
    rng = np.random.default_rng(33)
    rad = (3, 4, 5)
    g = _gauss(rng, rad)
    s = _rand_sign(rng, 60)
    F = _mr_dense(ora, rad, np.zeros(oracle_mr_size(rad)), s, g)
    G3, G4, G5 = ora.mr_mixer(3, g[0]), ora.mr_mixer(4), ora.mr_mixer(5, g[2])
    assert np.allclose(F, np.kron(G5, np.kron(G4, G3)) * s[None, :], atol=1e-13)


def test_mr_stages_as_stride_permutations(ora):
    """The page's construction written independently with numpy axes: index i is the array
    position (i_{m-1}, ..., i_0) of a C-ordered tensor; stage t moves axis m-1-t last (the
    stride permutation), applies block c = B_{t,c} to row c of the remaining axes in C order,
    and moves the axis back. Blocks from cayley() and mr_mixer()."""
    rng = np.random.default_rng(34)
    rad = (3, 2, 4, 5)
    d = int(np.prod(rad))
    th = _mr_theta(rng, rad, 0.4)
    g = _gauss(rng, rad)
    s = _rand_sign(rng, d)
    x = rng.standard_normal(d)
    v = (x * s).reshape(tuple(reversed(rad)))
    off = 0
    for t, b in enumerate(rad):
        ax = len(rad) - 1 - t
        rows = np.moveaxis(v, ax, -1).reshape(-1, b)
        out = np.empty_like(rows)
        for c in range(rows.shape[0]):
            if b == 2:
                p = np.pi / 4 + th[off + c]
                B = np.array([[np.cos(p), np.sin(p)], [np.sin(p), -np.cos(p)]])
            else:
                k = b * (b - 1) // 2
                B = ora.cayley(th[off + c * k: off + (c + 1) * k], b) @ ora.mr_mixer(b, g[t])
            out[c] = B @ rows[c]
        off += (d // b) * (1 if b == 2 else b * (b - 1) // 2)
        shape = list(np.moveaxis(v, ax, -1).shape)
        v = np.moveaxis(out.reshape(shape), -1, ax)
    assert np.allclose(ora.mr_butterfly_fwd(x, rad, th, s, g), v.reshape(-1), atol=1e-13)


def test_cayley_closed_forms(ora):
    """Q(0) = I; for b = 2, A = [[0, a], [-a, 0]] gives [[1 - a^2, -2a], [2a, 1 - a^2]] / (1 + a^2);
    Q is orthogonal with det +1; Q(-theta) = Q(theta)^T."""
    assert np.allclose(ora.cayley(np.zeros(10), 5), np.eye(5), atol=0)
    a = 0.37
    want = np.array([[1 - a * a, -2 * a], [2 * a, 1 - a * a]]) / (1 + a * a)
    assert np.allclose(ora.cayley([a], 2), want, atol=1e-15)
    rng = np.random.default_rng(35)
    for b in (3, 5, 8, 43):
        th = rng.uniform(-0.8, 0.8, b * (b - 1) // 2)
        Q = ora.cayley(th, b)
        assert np.allclose(Q.T @ Q, np.eye(b), atol=1e-12)
        assert abs(np.linalg.det(Q) - 1.0) < 1e-10
        assert np.allclose(ora.cayley(-th, b), Q.T, atol=1e-12)


def test_mr_mixer_properties(ora):
    """Powers of two: H_b / sqrt(b). Otherwise G is orthogonal and G^T M is upper triangular
    with a positive diagonal, which fixes G uniquely for an invertible M."""
    from scipy.linalg import hadamard
    for b in (2, 4, 16):
        assert np.allclose(ora.mr_mixer(b), hadamard(b) / np.sqrt(b), atol=1e-15)
    rng = np.random.default_rng(36)
    for b in (3, 5, 7, 43):
        M = rng.standard_normal((b, b))
        G = ora.mr_mixer(b, M)
        assert np.allclose(G.T @ G, np.eye(b), atol=1e-12)
        R = G.T @ M
        assert np.allclose(np.tril(R, -1), 0.0, atol=1e-11)
        assert np.all(np.diag(R) > 0)


@pytest.mark.parametrize("radices", [(8, 8, 8, 5, 2), (2, 2, 2, 2, 2, 2, 2, 2, 43)])
def test_mr_orthogonal_at_page_sizes(ora, radices):
    """The page's example schedule for d = 5120 (8, 8, 8, 5, 2), and 11008 = 2^8 43: norms are
    kept and F^T undoes F, for random angles."""
    rng = np.random.default_rng(37)
    d = int(np.prod(radices))
    th = _mr_theta(rng, radices, 0.2)
    g = _gauss(rng, radices)
    s = _rand_sign(rng, d)
    x = rng.standard_normal((2, d))
    y = ora.mr_butterfly_fwd(x, radices, th, s, g)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    assert np.allclose(ora.mr_butterfly_inv(y, radices, th, s, g), x, atol=1e-12)


def _mr_side(ora, rng, radices, scale=0.2):
    d = int(np.prod(radices))
    return ora.MixedRadixSide(radices, rng.uniform(-scale, scale, oracle_mr_size(radices)), _rand_sign(rng, d),
                              _gauss(rng, radices))


def test_mr_linear_exact_change_of_basis(ora):
    """Sec. 5 with mixed-radix sides: F_U(W' F_V x) = W x for the unquantized W' = U W V^T,
    with odd radices on both sides (n_in = 192 = 3 4 16, n_out = 40 = 5 8)."""
    rng = np.random.default_rng(41)
    V, U = _mr_side(ora, rng, (3, 4, 16)), _mr_side(ora, rng, (5, 8))
    W = rng.standard_normal((40, 192))
    Wr = ora.mr_rotate_weights(W, V, U)
    x = rng.standard_normal((3, 192))
    assert np.allclose(U.fwd(V.fwd(x) @ Wr.T), x @ W.T, atol=1e-12)


def test_mr_linear_all_radix2_is_the_linear(ora):
    """All-radix-2 sides: the mixed-radix layer is the radix-2 layer of the same angles,
    codes and output."""
    rng = np.random.default_rng(42)
    n_in, n_out = 256, 128
    thV, thU = _rand_theta(rng, n_in, n_in, 0.05), _rand_theta(rng, n_out, n_out, 0.05)
    sV, sU = _rand_sign(rng, n_in), _rand_sign(rng, n_out)
    W = rng.standard_normal((n_out, n_in)) * 0.02
    V = ora.MixedRadixSide([2] * 8, thV.reshape(-1), sV)
    U = ora.MixedRadixSide([2] * 7, thU.reshape(-1), sU)
    mr, _ = ora.mr_prepare_layer(W, 2, V, U)
    lay = ora.prepare_layer(W, 2, n_in, n_out, thV, sV, thU, sU)[0]
    assert np.array_equal(mr["packed"], lay.packed) and np.array_equal(mr["sz"], lay.sz)
    x = rng.standard_normal((2, n_in))
    assert np.allclose(ora.mr_linear_fwd(mr, x), ora.linear_fwd(lay, x), atol=1e-12)


def test_mr_linear_dequantizes_its_own_codes(ora):
    """The mixed-radix linear applies exactly scale16 q + zero16 of quantize()'s output,
    through its packed codes and scale/zero words."""
    rng = np.random.default_rng(43)
    V, U = _mr_side(ora, rng, (3, 64)), _mr_side(ora, rng, (5, 8))
    W = rng.standard_normal((40, 192)) * 0.02
    mr, Wr = ora.mr_prepare_layer(W, 3, V, U)
    q, s16, z16 = ora.quantize(Wr, 3)
    deq = np.repeat(s16.view(np.float16).astype(np.float64), 64, axis=1) * q + \
        np.repeat(z16.view(np.float16).astype(np.float64), 64, axis=1)
    x = rng.standard_normal((2, 192))
    assert np.allclose(ora.mr_linear_fwd(mr, x), U.fwd(V.fwd(x) @ deq.T), atol=1e-12)
