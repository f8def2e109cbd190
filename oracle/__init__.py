"""fp64 CPU oracle for the rotated low-bit linear -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package. It is a ctypes front end to ``harp_oracle.c`` (plain fp64 C, see that
file's header for the passages of "HARP: Hadamard-Preconditioned Adaptive Rotation
Processor for Extreme LLM Quantization" each function follows). It shares nothing
with the CUDA library: no code, headers, tables or helpers.

Parity status: every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (Sylvester-Hadamard identity, orthogonality, exact
change of basis, brute-force quantizer argmin, pack round trip with hand-built
bytes, block-diagonal split, the theta = -pi/4 diagonal case, a dense
stride-permutation construction and hand-computed golden fixtures).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_i64 = ctypes.c_int64
_int = ctypes.c_int
_dp = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i8p = ctypes.POINTER(ctypes.c_int8)
_u16p = ctypes.POINTER(ctypes.c_uint16)


class _Linear(ctypes.Structure):
    _fields_ = [("n_in", _i64), ("n_out", _i64), ("w_in", _i64), ("w_out", _i64),
                ("bits", _i64), ("group", _i64),
                ("thV", _dp), ("sV", _i8p), ("thU", _dp), ("sU", _i8p),
                ("packed", _u8p), ("scale_zero", _u16p)]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.ora_butterfly_fwd.argtypes = [_i64, _i64, _i64, _dp, _i8p, _dp]
        L.ora_butterfly_inv.argtypes = [_i64, _i64, _i64, _dp, _i8p, _dp]
        L.ora_rotate_weights.argtypes = [_i64, _i64, _i64, _i64, _dp, _i8p, _dp, _i8p, _dp]
        L.ora_quantize.argtypes = [_i64, _i64, _int, _int, _dp, _u8p, _u16p, _u16p]
        L.ora_pack.argtypes = [_i64, _i64, _int, _u8p, _u8p]
        L.ora_unpack.argtypes = [_i64, _i64, _int, _u8p, _u8p]
        L.ora_packed_bytes.argtypes = [_i64, _i64, _int]
        L.ora_packed_bytes.restype = _i64
        L.ora_linear_fwd.argtypes = [ctypes.POINTER(_Linear), _i64, _dp, _dp]
        L.ora_dense_rotated_fwd.argtypes = [_i64, _i64, _i64, _i64, _dp, _i8p, _dp, _i8p, _dp,
                                            _i64, _dp, _dp]
        L.ora_stack_step.argtypes = [_i64, ctypes.POINTER(_Linear), _i64, _i64, _i64, _i64, _i64,
                                     ctypes.c_double, _i64, _dp, _dp]
        L.ora_f16_from_f64.argtypes = [ctypes.c_double]
        L.ora_f16_from_f64.restype = ctypes.c_uint16
        L.ora_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.ora_f16_to_f64.restype = ctypes.c_double
        L.ora_set_threads.argtypes = [_int]
        L.ora_mr_mixer.argtypes = [_int, _dp, _dp]
        L.ora_cayley.argtypes = [_int, _dp, _dp]
        L.ora_mr_butterfly.argtypes = [_i64, _int, ctypes.POINTER(ctypes.c_int), _dp, _i8p, _dp, _int, _i64, _dp]
        L.ora_quantize_angles.argtypes = [_i64, _i64, _dp, _i8p, ctypes.POINTER(ctypes.c_float)]
        L.ora_calib_fit.argtypes = [_i64, _i64, _int, _int, _i64, _i64, _dp, _i8p, _dp, _i8p, _dp, _dp,
                                    ctypes.c_double, _dp, _dp, _dp]
        L.ora_get_threads.restype = _int
        _lib = L
    return _lib


def _d(a):
    return a.ctypes.data_as(_dp)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i8(a):
    return np.ascontiguousarray(a, dtype=np.int8)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


def set_threads(n: int) -> None:
    lib().ora_set_threads(int(n))


def get_threads() -> int:
    return int(lib().ora_get_threads())


# ---------------------------------------------------------------- fp16 bits
def f16_from_f64(v) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64)
    f = lib().ora_f16_from_f64
    return np.array([f(float(t)) for t in v.ravel()], dtype=np.uint16).reshape(v.shape)


def f16_to_f64(h) -> np.ndarray:
    h = np.asarray(h, dtype=np.uint16)
    f = lib().ora_f16_to_f64
    return np.array([f(int(t)) for t in h.ravel()], dtype=np.float64).reshape(h.shape)


# ---------------------------------------------------------------- butterfly
def _bfly(fn, x, theta, sign, w):
    x = _f64(x).copy()
    one = x.ndim == 1
    x2 = x.reshape(1, -1) if one else x
    n = x2.shape[1]
    th = _f64(theta)
    sg = _i8(sign)
    assert th.size == (n // 2) * int(np.log2(w)) and sg.size == n
    _check(fn(n, int(w), x2.shape[0], _d(th), sg.ctypes.data_as(_i8p), _d(x2)), "butterfly")
    return x2.reshape(-1) if one else x2


def butterfly_fwd(x, theta, sign, w):
    """F(theta, s, w) x: signs first, then stages of stride 1, 2, ..., w/2."""
    return _bfly(lib().ora_butterfly_fwd, x, theta, sign, w)


def butterfly_inv(x, theta, sign, w):
    """F(theta, s, w)^T x: stages of stride w/2, ..., 1, then signs."""
    return _bfly(lib().ora_butterfly_inv, x, theta, sign, w)


# ---------------------------------------------------------------- offline prep
def rotate_weights(W, thV, sV, w_in, thU, sU, w_out):
    """W' = U W V^T with V = F_V and U^T = F_U."""
    Wr = _f64(W).copy()
    n_out, n_in = Wr.shape
    thV, thU = _f64(thV), _f64(thU)
    sV, sU = _i8(sV), _i8(sU)
    _check(lib().ora_rotate_weights(n_out, n_in, int(w_in), int(w_out), _d(thV),
                                    sV.ctypes.data_as(_i8p), _d(thU), sU.ctypes.data_as(_i8p),
                                    _d(Wr)), "rotate")
    return Wr


def quantize(Wr, bits, group=64):
    """Returns (q uint8 [n_out, n_in], scale16 uint16 [n_out, ng], zero16 uint16 [n_out, ng])."""
    Wr = _f64(Wr)
    n_out, n_in = Wr.shape
    q = np.zeros((n_out, n_in), np.uint8)
    s = np.zeros((n_out, n_in // group), np.uint16)
    z = np.zeros((n_out, n_in // group), np.uint16)
    _check(lib().ora_quantize(n_out, n_in, int(bits), int(group), _d(Wr), q.ctypes.data_as(_u8p),
                              s.ctypes.data_as(_u16p), z.ctypes.data_as(_u16p)), "quantize")
    return q, s, z


def pack(q, bits):
    q = np.ascontiguousarray(q, dtype=np.uint8)
    n_out, n_in = q.shape
    out = np.zeros(int(lib().ora_packed_bytes(n_out, n_in, int(bits))), np.uint8)
    _check(lib().ora_pack(n_out, n_in, int(bits), q.ctypes.data_as(_u8p), out.ctypes.data_as(_u8p)),
           "pack")
    return out


def unpack(packed, n_out, n_in, bits):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    q = np.zeros((n_out, n_in), np.uint8)
    _check(lib().ora_unpack(n_out, n_in, int(bits), packed.ctypes.data_as(_u8p),
                            q.ctypes.data_as(_u8p)), "unpack")
    return q


def scale_zero(scale16, zero16):
    """Interleaves the fp16 bits into the [n_out][n_in/group] {scale, zero} pair layout."""
    return np.ascontiguousarray(np.stack([scale16, zero16], axis=-1).astype(np.uint16))


# ---------------------------------------------------------------- layers
class Layer:
    """One rotated low-bit linear as the oracle sees it (all arrays host numpy)."""

    def __init__(self, n_in, n_out, bits, w_in, w_out, thV, sV, thU, sU, packed, sz, group=64):
        self.n_in, self.n_out, self.bits, self.group = int(n_in), int(n_out), int(bits), int(group)
        self.w_in, self.w_out = int(w_in), int(w_out)
        self.thV, self.thU = _f64(thV), _f64(thU)
        self.sV, self.sU = _i8(sV), _i8(sU)
        self.packed = np.ascontiguousarray(packed, dtype=np.uint8)
        self.sz = np.ascontiguousarray(sz, dtype=np.uint16)
        assert self.packed.size == n_out * n_in * bits // 8
        assert self.sz.size == n_out * (n_in // group) * 2

    def cstruct(self):
        return _Linear(self.n_in, self.n_out, self.w_in, self.w_out, self.bits, self.group,
                       _d(self.thV), self.sV.ctypes.data_as(_i8p), _d(self.thU),
                       self.sU.ctypes.data_as(_i8p), self.packed.ctypes.data_as(_u8p),
                       self.sz.ctypes.data_as(_u16p))


def prepare_layer(W, bits, w_in, w_out, thV, sV, thU, sU, group=64):
    """Rotate, quantize and pack a weight matrix; returns (Layer, q, scale16, zero16, W')."""
    n_out, n_in = np.shape(W)
    Wr = rotate_weights(W, thV, sV, w_in, thU, sU, w_out)
    q, s, z = quantize(Wr, bits, group)
    lay = Layer(n_in, n_out, bits, w_in, w_out, thV, sV, thU, sU, pack(q, bits), scale_zero(s, z),
                group)
    return lay, q, s, z, Wr


def linear_fwd(layer: Layer, x):
    """y = F_U(dequant(codes) . F_V(x)); x [batch, n_in] -> y [batch, n_out] (fp64)."""
    x = _f64(x)
    one = x.ndim == 1
    x2 = x.reshape(1, -1) if one else x
    y = np.zeros((x2.shape[0], layer.n_out), np.float64)
    st = layer.cstruct()
    _check(lib().ora_linear_fwd(ctypes.byref(st), x2.shape[0], _d(x2), _d(y)), "linear")
    return y.reshape(-1) if one else y


def dense_rotated_fwd(Wr, thV, sV, w_in, thU, sU, w_out, x):
    """F_U(W' F_V(x)) with an unquantized rotated matrix."""
    Wr = _f64(Wr)
    n_out, n_in = Wr.shape
    x = _f64(x)
    one = x.ndim == 1
    x2 = x.reshape(1, -1) if one else x
    y = np.zeros((x2.shape[0], n_out), np.float64)
    thV, thU, sV, sU = _f64(thV), _f64(thU), _i8(sV), _i8(sU)
    _check(lib().ora_dense_rotated_fwd(n_out, n_in, int(w_in), int(w_out), _d(thV),
                                       sV.ctypes.data_as(_i8p), _d(thU), sU.ctypes.data_as(_i8p),
                                       _d(Wr), x2.shape[0], _d(x2), _d(y)), "dense")
    return y.reshape(-1) if one else y


def stack_step(layers, hidden, ffn, n_heads, n_kv_heads, head_dim, x, eps=1e-5):
    """One decode step through len(layers)//7 blocks (q, k, v, o, gate, up, down each)."""
    assert len(layers) % 7 == 0
    arr = (_Linear * len(layers))(*[l.cstruct() for l in layers])
    x = _f64(x)
    one = x.ndim == 1
    x2 = x.reshape(1, -1) if one else x
    out = np.zeros_like(x2)
    _check(lib().ora_stack_step(len(layers) // 7, arr, hidden, ffn, n_heads, n_kv_heads, head_dim,
                                float(eps), x2.shape[0], _d(x2), _d(out)), "stack")
    return out.reshape(-1) if one else out


def mr_param_count(b: int) -> int:
    """Parameters of one b x b block: 1 angle for b = 2, b(b-1)/2 Cayley parameters above."""
    return 1 if b == 2 else b * (b - 1) // 2


def mr_theta_size(radices) -> int:
    d = int(np.prod(radices))
    return sum((d // b) * mr_param_count(b) for b in radices)


def mr_mixer(b, M=None):
    """G_b: Sylvester H_b / sqrt(b) for powers of two, else the positive-diagonal QR factor
    of the fixed Gaussian M (HARP Sec. 2.2, base mixer)."""
    G = np.zeros((b, b))
    MM = _f64(M) if M is not None else None
    _check(lib().ora_mr_mixer(int(b), _d(MM) if MM is not None else None, _d(G)), "mr_mixer")
    return G


def cayley(theta, b):
    """(I - A)(I + A)^-1 for the skew-symmetric A of the b(b-1)/2 parameters (upper triangle,
    row by row)."""
    th = _f64(theta).reshape(-1)
    assert th.size == b * (b - 1) // 2
    Q = np.zeros((b, b))
    _check(lib().ora_cayley(int(b), _d(th), _d(Q)), "cayley")
    return Q


def _mr(x, radices, theta, sign, gauss, inverse):
    v = np.array(x, dtype=np.float64, copy=True, order="C")
    d = v.shape[-1]
    r = (ctypes.c_int * len(radices))(*[int(b) for b in radices])
    th = _f64(theta).reshape(-1)
    assert th.size == mr_theta_size(radices)
    g = None
    if gauss is not None:
        g = np.concatenate([np.zeros(b * b) if m is None else _f64(m).reshape(-1) for b, m in zip(radices, gauss)])
    sg = _i8(sign)
    _check(lib().ora_mr_butterfly(d, len(radices), r, _d(th), sg.ctypes.data_as(_i8p), _d(g) if g is not None else None,
                                  int(inverse), v.size // d, _d(v)), "mr_butterfly")
    return v


def mr_butterfly_fwd(x, radices, theta, sign, gauss=None):
    """Mixed-radix F(theta, s, b) x over the last dimension (HARP Sec. 2.1): signs, then stage
    t = 0..m-1 mixing the b_t coordinates that differ in mixed-radix digit t. gauss: one
    b_t x b_t Gaussian per stage (None entries for powers of two)."""
    return _mr(x, radices, theta, sign, gauss, False)


def mr_butterfly_inv(x, radices, theta, sign, gauss=None):
    """F^T x: the stage transposes from t = m-1 down to 0, then the signs."""
    return _mr(x, radices, theta, sign, gauss, True)


class MixedRadixSide:
    """One side of a linear with a mixed-radix butterfly: radices, parameters (stage after
    stage), signs and one Gaussian per stage (None for powers of two)."""

    def __init__(self, radices, theta, sign, gauss=None):
        self.radices = [int(b) for b in radices]
        self.theta = _f64(theta).reshape(-1)
        self.sign = _i8(sign)
        self.gauss = gauss

    def fwd(self, x):
        return mr_butterfly_fwd(x, self.radices, self.theta, self.sign, self.gauss)

    def inv(self, x):
        return mr_butterfly_inv(x, self.radices, self.theta, self.sign, self.gauss)


def mr_rotate_weights(W, V: MixedRadixSide, U: MixedRadixSide):
    """W' = U W V^T with V = F_V and U = F_U^T: rows through F_V, then columns through F_U^T."""
    Wr = V.fwd(_f64(W))
    return np.ascontiguousarray(U.inv(np.ascontiguousarray(Wr.T)).T)


def mr_prepare_layer(W, bits, V: MixedRadixSide, U: MixedRadixSide, group=64):
    """Rotate with mixed-radix sides, quantize and pack; returns (layer dict, W')."""
    Wr = mr_rotate_weights(W, V, U)
    q, s, z = quantize(Wr, bits, group)
    return dict(V=V, U=U, bits=int(bits), group=int(group), packed=pack(q, bits), sz=scale_zero(s, z),
                n_out=Wr.shape[0], n_in=Wr.shape[1]), Wr


def mr_linear_fwd(layer, x):
    """y = F_U(deq(codes) F_V(x)) for a mixed-radix layer: the codes are unpacked, each
    dequantized to scale16 q + zero16 of its group, and applied as a dense matrix."""
    x = _f64(x)
    one = x.ndim == 1
    x2 = x.reshape(1, -1) if one else x
    n_out, n_in, g = layer["n_out"], layer["n_in"], layer["group"]
    q = unpack(layer["packed"], n_out, n_in, layer["bits"]).astype(np.float64)
    sz = np.asarray(layer["sz"], np.uint16).reshape(n_out, n_in // g, 2)
    # fp16 -> fp64 is exact; numpy's conversion serves as the library step
    s = np.repeat(np.ascontiguousarray(sz[:, :, 0]).view(np.float16).astype(np.float64), g, axis=1)
    z = np.repeat(np.ascontiguousarray(sz[:, :, 1]).view(np.float16).astype(np.float64), g, axis=1)
    y = layer["U"].fwd((layer["V"].fwd(x2)) @ (s * q + z).T)
    return y.reshape(-1) if one else y


def quantize_angles(theta):
    """int8 angle storage: (q int8 [m, n/2], delta fp32 [m]) with one symmetric step per
    stage, delta_t = fp32(max |theta_t| / 127), q = RNE(theta / delta_t) clamped to +-127."""
    th = _f64(theta)
    m, half = th.shape
    q = np.zeros((m, half), np.int8)
    d = np.zeros(m, np.float32)
    _check(lib().ora_quantize_angles(m, half, _d(th), q.ctypes.data_as(_i8p),
                                     d.ctypes.data_as(ctypes.POINTER(ctypes.c_float))), "quantize_angles")
    return q, d


def dequantize_angles(q, delta):
    """theta^ = delta_t * q_tp in fp64 (the angles a layer stored in int8 applies)."""
    return np.asarray(delta, np.float64)[:, None] * np.asarray(q, np.float64)


def calib_fit(W, bits, w_in, w_out, thV, sV, thU, sU, H=None, lambda_bd=0.0, grad=False, group=64):
    """The page's per-layer fitting loss L_fit = L_diag + lambda_bd R_bd (HARP Sec. 2.3).

    H: the input-side Hessian proxy [n_in, n_in] (None: identity). Returns
    (L_fit, L_diag, R_bd), and with grad=True also (dL_fit/dtheta_V, dL_fit/dtheta_U)
    with the code target held constant."""
    W = _f64(W)
    n_out, n_in = W.shape
    thV, thU, sV, sU = _f64(thV), _f64(thU), _i8(sV), _i8(sU)
    HH = _f64(H) if H is not None else None
    out = np.zeros(3)
    gV = np.zeros_like(thV) if grad else None
    gU = np.zeros_like(thU) if grad else None
    _check(lib().ora_calib_fit(n_out, n_in, int(bits), int(group), int(w_in), int(w_out), _d(thV),
                               sV.ctypes.data_as(_i8p), _d(thU), sU.ctypes.data_as(_i8p), _d(W),
                               _d(HH) if HH is not None else None, float(lambda_bd), _d(out),
                               _d(gV) if grad else None, _d(gU) if grad else None), "calib_fit")
    loss = (float(out[0]), float(out[1]), float(out[2]))
    return (loss, gV, gU) if grad else loss
