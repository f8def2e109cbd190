/*
 * harp_oracle.c -- TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow, fp64 CPU statement of what the rotated low-bit linear computes.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg load it.
 * It shares no code, header, table or helper with the CUDA library; the two meet
 * only through the seeded input generators.
 *
 * Source: "HARP: Hadamard-Preconditioned Adaptive Rotation Processor for Extreme
 * LLM Quantization" (gist.science explanation of arXiv 2605.29843):
 *   Sec. 2.1 (Arquitetura Central)  -- the rotation is a product of sparse stride
 *                                      stages, each a block-diagonal orthogonal B_t
 *                                      between stride permutations; radix-2 here.
 *   Sec. 2.2 (Pre-condicionamento)  -- block B_{t,c}(theta) = Q_{t,c}(theta) G_2 with
 *                                      Q a Givens rotation and G_2 the normalised
 *                                      Sylvester Hadamard; Theta = 0 gives the fixed
 *                                      randomized Hadamard transform.
 *   Sec. 5 (Exatidao vs. Aproximacao) -- an exact change of basis: the full-precision
 *                                      layer is preserved, only the quantizer's
 *                                      coordinates change.
 * The pages leave the codebook to the backend (Sec. 2.4, Compatibilidade); the
 * quantizer below is this library's stand-in: group-wise uniform scalar codes,
 * b in {2,3,4} bits, an fp16 scale and an fp16 zero per group of 64 columns.
 *
 * Readings taken where the pages are silent (each is listed in the design notes):
 *   - 2x2 block: Givens(theta) * H_2 = [[cos p, sin p], [sin p, -cos p]], p = pi/4 + theta.
 *   - F = S_{m-1} ... S_1 S_0 D: the sign diagonal D first, then stage t = 0..m-1
 *     pairs (i, i + 2^t) inside each w-wide block; pairs are numbered, per stage,
 *     in increasing order of their first index.
 *   - n not a power of two: F is block-diagonal with w-wide blocks (w a power of two).
 *   - Every 2x2 block is symmetric, so F^T applies the stages in reverse, then D.
 *
 * Arithmetic is fp64 throughout; fp32/bf16 inputs convert to fp64 exactly.
 * Parallelism (OpenMP) only splits independent rows or vectors; it never changes
 * the order of any sum.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORA_OK 0
#define ORA_EINVAL 1

static const double ORA_PI = 3.14159265358979323846264338327950288;

static int ora_log2_exact(int64_t w) {
  if (w < 1) return -1;
  int m = 0;
  while (((int64_t)1 << m) < w) ++m;
  return (((int64_t)1 << m) == w) ? m : -1;
}

/* ------------------------------------------------------------------ threads */
void ora_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int ora_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------ fp16
 * IEEE 754 binary16 from fp64, round to nearest, ties to even, written from the
 * format's definition (1 sign bit, 5 exponent bits with bias 15, 10 fraction bits;
 * subnormals below 2^-14; overflow to infinity at and above 65520).
 */
uint16_t ora_f16_from_f64(double v) {
  uint16_t sign = 0;
  if (signbit(v)) { sign = 0x8000u; v = -v; }
  if (isnan(v)) return (uint16_t)(sign | 0x7e00u);
  if (v == 0.0) return sign;
  int e2;
  frexp(v, &e2);            /* v = f * 2^e2, f in [0.5, 1) -> exponent of v is e2 - 1 */
  int e = e2 - 1;
  if (e < -14) e = -14;      /* subnormal range shares the quantum 2^-24 */
  double quantum = ldexp(1.0, e - 10);
  double m = v / quantum;    /* exact: division by a power of two */
  double r = nearbyint(m);   /* default rounding mode: nearest, ties to even */
  /* r in [1024, 2048] for normals; rounding may carry into the next binade */
  if (r >= 2048.0) { r = r / 2.0; e += 1; }
  if (e > 15) return (uint16_t)(sign | 0x7c00u);
  if (r < 1024.0) {          /* subnormal (only possible when e == -14) */
    return (uint16_t)(sign | (uint16_t)r);
  }
  uint16_t exp_bits = (uint16_t)(e + 15);
  uint16_t frac = (uint16_t)((int)r - 1024);
  return (uint16_t)(sign | (exp_bits << 10) | frac);
}

double ora_f16_to_f64(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 0x1f, f = h & 0x3ff;
  double v;
  if (e == 0) v = ldexp((double)f, -24);
  else if (e == 31) v = f ? NAN : INFINITY;
  else v = ldexp((double)(1024 + f), e - 25);
  return s ? -v : v;
}

/* ------------------------------------------------------------------ butterfly
 * theta: [m][n/2] (m = log2 w), sign: [n] of +-1, x: [batch][n], in place.
 */
static void ora_stage(int64_t n, int64_t w, int t, const double* theta_t, double* x) {
  const int64_t h = (int64_t)1 << t;
  for (int64_t k = 0; k < n / w; ++k) {
    double* blk = x + k * w;
    for (int64_t i = 0; i < w; ++i) {
      if (i & h) continue;
      const int64_t p = k * (w / 2) + ((i >> (t + 1)) << t) + (i & (h - 1));
      const double psi = ORA_PI / 4.0 + theta_t[p];
      const double c = cos(psi), s = sin(psi);
      const double a = blk[i], b = blk[i + h];
      blk[i] = c * a + s * b;
      blk[i + h] = s * a - c * b;
    }
  }
}

static int ora_check_bfly(int64_t n, int64_t w) {
  if (n <= 0 || w < 2 || n % w) return -1;
  return ora_log2_exact(w);
}

int ora_butterfly_fwd(int64_t n, int64_t w, int64_t batch, const double* theta,
                      const int8_t* sign, double* x) {
  const int m = ora_check_bfly(n, w);
  if (m < 1 || batch < 0) return ORA_EINVAL;
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < batch; ++b) {
    double* v = x + b * n;
    for (int64_t i = 0; i < n; ++i) v[i] *= (double)sign[i];
    for (int t = 0; t < m; ++t) ora_stage(n, w, t, theta + (int64_t)t * (n / 2), v);
  }
  return ORA_OK;
}

int ora_butterfly_inv(int64_t n, int64_t w, int64_t batch, const double* theta,
                      const int8_t* sign, double* x) {
  const int m = ora_check_bfly(n, w);
  if (m < 1 || batch < 0) return ORA_EINVAL;
#pragma omp parallel for schedule(static)
  for (int64_t b = 0; b < batch; ++b) {
    double* v = x + b * n;
    for (int t = m - 1; t >= 0; --t) ora_stage(n, w, t, theta + (int64_t)t * (n / 2), v);
    for (int64_t i = 0; i < n; ++i) v[i] *= (double)sign[i];
  }
  return ORA_OK;
}

/* ------------------------------------------------------------------ rotate
 * W' = U W V^T with V = F(theta_V, s_V, w_in) and U^T = F(theta_U, s_U, w_out):
 * every row r becomes F_V(W_r), then every column j becomes F_U^T(W'_{:,j}).
 * W: [n_out][n_in] row-major, in place.
 */
int ora_rotate_weights(int64_t n_out, int64_t n_in, int64_t w_in, int64_t w_out,
                       const double* thV, const int8_t* sV, const double* thU,
                       const int8_t* sU, double* W) {
  if (ora_check_bfly(n_in, w_in) < 1 || ora_check_bfly(n_out, w_out) < 1) return ORA_EINVAL;
  int rc = ora_butterfly_fwd(n_in, w_in, n_out, thV, sV, W);
  if (rc) return rc;
  int bad = 0;
#pragma omp parallel
  {
    double* col = (double*)malloc(sizeof(double) * (size_t)n_out);
    if (!col) {
#pragma omp atomic write
      bad = 1;
    } else {
#pragma omp for schedule(static)
      for (int64_t j = 0; j < n_in; ++j) {
        for (int64_t r = 0; r < n_out; ++r) col[r] = W[r * n_in + j];
        ora_butterfly_inv(n_out, w_out, 1, thU, sU, col);
        for (int64_t r = 0; r < n_out; ++r) W[r * n_in + j] = col[r];
      }
      free(col);
    }
  }
  return bad ? ORA_EINVAL : ORA_OK;
}

/* ------------------------------------------------------------------ quantize
 * Per row r and group g (group consecutive columns of W'):
 *   zero16  = fp16(min), scale16 = fp16((max - min) / (2^b - 1)), 1 if that is 0,
 *   q       = clamp(round_half_even((w - zero16) / scale16), 0, 2^b - 1),
 *   dequant = scale16 * q + zero16.
 * q: [n_out][n_in] one code per byte; scale16, zero16: [n_out][n_in/group] fp16 bits.
 */
int ora_quantize(int64_t n_out, int64_t n_in, int bits, int group, const double* Wr,
                 uint8_t* q, uint16_t* scale16, uint16_t* zero16) {
  if (bits < 2 || bits > 4 || group < 1 || n_in % group) return ORA_EINVAL;
  const double L = (double)((1 << bits) - 1);
  const int64_t ng = n_in / group;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_out; ++r) {
    for (int64_t g = 0; g < ng; ++g) {
      const double* w = Wr + r * n_in + g * group;
      double mn = w[0], mx = w[0];
      for (int j = 1; j < group; ++j) {
        if (w[j] < mn) mn = w[j];
        if (w[j] > mx) mx = w[j];
      }
      uint16_t zb = ora_f16_from_f64(mn);
      uint16_t sb = ora_f16_from_f64((mx - mn) / L);
      if (ora_f16_to_f64(sb) == 0.0) sb = 0x3c00u; /* 1.0 */
      const double z = ora_f16_to_f64(zb), s = ora_f16_to_f64(sb);
      for (int j = 0; j < group; ++j) {
        double v = nearbyint((w[j] - z) / s);
        if (!(v >= 0.0)) v = 0.0; /* also maps NaN to 0 */
        if (v > L) v = L;
        q[r * n_in + g * group + j] = (uint8_t)v;
      }
      scale16[r * ng + g] = sb;
      zero16[r * ng + g] = zb;
    }
  }
  return ORA_OK;
}

/* ------------------------------------------------------------------ pack
 * Canonical packed layout, row-major by output row; e = r * n_in + j:
 *   b = 2 or 4: code e sits in little-endian 32-bit word (e * b) / 32 at bit (e * b) % 32;
 *   b = 3     : a 2-bit plane of (q & 3) laid out as for b = 2 (n_out*n_in/4 bytes),
 *               then a 1-bit plane of (q >> 2): word e / 32, bit e % 32.
 * Total bytes: n_out * n_in * b / 8.
 */
static void ora_put_bits(uint8_t* buf, int64_t bitpos, unsigned v, int nb) {
  for (int k = 0; k < nb; ++k) {
    const int64_t p = bitpos + k;
    const uint8_t bit = (uint8_t)((v >> k) & 1u);
    /* little-endian words: bit p of the stream is bit (p % 8) of byte p / 8 */
    buf[p >> 3] = (uint8_t)((buf[p >> 3] & ~(1u << (p & 7))) | (bit << (p & 7)));
  }
}

static unsigned ora_get_bits(const uint8_t* buf, int64_t bitpos, int nb) {
  unsigned v = 0;
  for (int k = 0; k < nb; ++k) {
    const int64_t p = bitpos + k;
    v |= (unsigned)((buf[p >> 3] >> (p & 7)) & 1u) << k;
  }
  return v;
}

int64_t ora_packed_bytes(int64_t n_out, int64_t n_in, int bits) {
  return n_out * n_in * bits / 8;
}

int ora_pack(int64_t n_out, int64_t n_in, int bits, const uint8_t* q, uint8_t* packed) {
  if (bits < 2 || bits > 4 || n_in % 32) return ORA_EINVAL;
  const int64_t N = n_out * n_in;
  memset(packed, 0, (size_t)ora_packed_bytes(n_out, n_in, bits));
  if (bits == 3) {
    uint8_t* hi = packed + N / 4;
    for (int64_t e = 0; e < N; ++e) {
      ora_put_bits(packed, e * 2, q[e] & 3u, 2);
      ora_put_bits(hi, e, (q[e] >> 2) & 1u, 1);
    }
  } else {
    for (int64_t e = 0; e < N; ++e) ora_put_bits(packed, e * bits, q[e], bits);
  }
  return ORA_OK;
}

int ora_unpack(int64_t n_out, int64_t n_in, int bits, const uint8_t* packed, uint8_t* q) {
  if (bits < 2 || bits > 4 || n_in % 32) return ORA_EINVAL;
  const int64_t N = n_out * n_in;
  if (bits == 3) {
    const uint8_t* hi = packed + N / 4;
    for (int64_t e = 0; e < N; ++e)
      q[e] = (uint8_t)(ora_get_bits(packed, e * 2, 2) | (ora_get_bits(hi, e, 1) << 2));
  } else {
    for (int64_t e = 0; e < N; ++e) q[e] = (uint8_t)ora_get_bits(packed, e * bits, bits);
  }
  return ORA_OK;
}

/* ------------------------------------------------------------------ linear */
typedef struct {
  int64_t n_in, n_out, w_in, w_out;
  int64_t bits, group;
  const double* thV;
  const int8_t* sV;
  const double* thU;
  const int8_t* sU;
  const uint8_t* packed;      /* canonical layout above */
  const uint16_t* scale_zero; /* [n_out][n_in/group][2]: {scale16, zero16} */
} ora_linear;

/* code of element (r, j) read straight from the canonical packed layout */
static unsigned ora_code_at(const ora_linear* L, int64_t r, int64_t j) {
  const int64_t e = r * L->n_in + j;
  if (L->bits == 3) {
    const uint8_t* hi = L->packed + (L->n_out * L->n_in) / 4;
    return ora_get_bits(L->packed, e * 2, 2) | (ora_get_bits(hi, e, 1) << 2);
  }
  return ora_get_bits(L->packed, e * L->bits, (int)L->bits);
}

/* y = F_U( dequant(codes) . F_V(x) ), x: [batch][n_in], y: [batch][n_out] */
int ora_linear_fwd(const ora_linear* L, int64_t batch, const double* x, double* y) {
  if (ora_check_bfly(L->n_in, L->w_in) < 1 || ora_check_bfly(L->n_out, L->w_out) < 1) return ORA_EINVAL;
  if (L->group < 1 || L->n_in % L->group) return ORA_EINVAL;
  const int64_t n_in = L->n_in, n_out = L->n_out, ng = n_in / L->group;
  double* xt = (double*)malloc(sizeof(double) * (size_t)(batch * n_in));
  if (!xt && batch) return ORA_EINVAL;
  memcpy(xt, x, sizeof(double) * (size_t)(batch * n_in));
  ora_butterfly_fwd(n_in, L->w_in, batch, L->thV, L->sV, xt);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_out; ++r) {
    for (int64_t b = 0; b < batch; ++b) {
      double acc = 0.0;
      for (int64_t j = 0; j < n_in; ++j) {
        const int64_t g = j / L->group;
        const double s = ora_f16_to_f64(L->scale_zero[(r * ng + g) * 2 + 0]);
        const double z = ora_f16_to_f64(L->scale_zero[(r * ng + g) * 2 + 1]);
        const double wdq = s * (double)ora_code_at(L, r, j) + z;
        acc += wdq * xt[b * n_in + j];
      }
      y[b * n_out + r] = acc;
    }
  }
  free(xt);
  return ora_butterfly_fwd(n_out, L->w_out, batch, L->thU, L->sU, y);
}

/* Same composition with an unquantized rotated matrix Wr (used to check that the
 * rotation is an exact change of basis: F_U(Wr F_V(x)) must equal W x). */
int ora_dense_rotated_fwd(int64_t n_out, int64_t n_in, int64_t w_in, int64_t w_out,
                          const double* thV, const int8_t* sV, const double* thU,
                          const int8_t* sU, const double* Wr, int64_t batch,
                          const double* x, double* y) {
  if (ora_check_bfly(n_in, w_in) < 1 || ora_check_bfly(n_out, w_out) < 1) return ORA_EINVAL;
  double* xt = (double*)malloc(sizeof(double) * (size_t)(batch * n_in));
  if (!xt && batch) return ORA_EINVAL;
  memcpy(xt, x, sizeof(double) * (size_t)(batch * n_in));
  ora_butterfly_fwd(n_in, w_in, batch, thV, sV, xt);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < n_out; ++r)
    for (int64_t b = 0; b < batch; ++b) {
      double acc = 0.0;
      for (int64_t j = 0; j < n_in; ++j) acc += Wr[r * n_in + j] * xt[b * n_in + j];
      y[b * n_out + r] = acc;
    }
  free(xt);
  return ora_butterfly_fwd(n_out, w_out, batch, thU, sU, y);
}

/* ------------------------------------------------------------------ stack step
 * One decode step through n_layers Llama-shaped blocks whose seven linears are all
 * rotated low-bit layers, in the order q, k, v, o, gate, up, down:
 *   n1 = rms(x); v = v_proj(n1); a = v repeated per key/value group (a one-key
 *   attention returns its value; q_proj and k_proj are evaluated all the same);
 *   h = x + o_proj(a); n2 = rms(h); x' = h + down(silu(gate(n2)) * up(n2)),
 *   rms(u) = u / sqrt(mean(u^2) + eps), silu(g) = g / (1 + exp(-g)).
 * x, out: [batch][hidden].
 */
static void ora_rms(int64_t n, double eps, const double* u, double* o) {
  double ss = 0.0;
  for (int64_t i = 0; i < n; ++i) ss += u[i] * u[i];
  const double inv = 1.0 / sqrt(ss / (double)n + eps);
  for (int64_t i = 0; i < n; ++i) o[i] = u[i] * inv;
}

int ora_stack_step(int64_t n_layers, const ora_linear* lin, int64_t hidden, int64_t ffn,
                   int64_t n_heads, int64_t n_kv_heads, int64_t head_dim, double eps,
                   int64_t batch, const double* x, double* out) {
  if (n_kv_heads < 1 || n_heads % n_kv_heads) return ORA_EINVAL;
  const int64_t dq = n_heads * head_dim, dkv = n_kv_heads * head_dim, rep = n_heads / n_kv_heads;
  const size_t B = (size_t)batch;
  double* h = (double*)malloc(sizeof(double) * B * (size_t)hidden);
  double* nrm = (double*)malloc(sizeof(double) * B * (size_t)hidden);
  double* q = (double*)malloc(sizeof(double) * B * (size_t)dq);
  double* k = (double*)malloc(sizeof(double) * B * (size_t)dkv);
  double* v = (double*)malloc(sizeof(double) * B * (size_t)dkv);
  double* a = (double*)malloc(sizeof(double) * B * (size_t)dq);
  double* o = (double*)malloc(sizeof(double) * B * (size_t)hidden);
  double* g = (double*)malloc(sizeof(double) * B * (size_t)ffn);
  double* u = (double*)malloc(sizeof(double) * B * (size_t)ffn);
  int rc = ORA_OK;
  if (!h || !nrm || !q || !k || !v || !a || !o || !g || !u) { rc = ORA_EINVAL; goto done; }
  memcpy(out, x, sizeof(double) * B * (size_t)hidden);
  for (int64_t l = 0; l < n_layers && rc == ORA_OK; ++l) {
    const ora_linear* L = lin + 7 * l;
    for (int64_t b = 0; b < batch; ++b) ora_rms(hidden, eps, out + b * hidden, nrm + b * hidden);
    rc |= ora_linear_fwd(&L[0], batch, nrm, q);
    rc |= ora_linear_fwd(&L[1], batch, nrm, k);
    rc |= ora_linear_fwd(&L[2], batch, nrm, v);
    for (int64_t b = 0; b < batch; ++b)
      for (int64_t hh = 0; hh < n_heads; ++hh)
        for (int64_t d = 0; d < head_dim; ++d)
          a[b * dq + hh * head_dim + d] = v[b * dkv + (hh / rep) * head_dim + d];
    rc |= ora_linear_fwd(&L[3], batch, a, o);
    for (size_t i = 0; i < B * (size_t)hidden; ++i) h[i] = out[i] + o[i];
    for (int64_t b = 0; b < batch; ++b) ora_rms(hidden, eps, h + b * hidden, nrm + b * hidden);
    rc |= ora_linear_fwd(&L[4], batch, nrm, g);
    rc |= ora_linear_fwd(&L[5], batch, nrm, u);
    for (size_t i = 0; i < B * (size_t)ffn; ++i) g[i] = g[i] / (1.0 + exp(-g[i])) * u[i];
    rc |= ora_linear_fwd(&L[6], batch, g, o);
    for (size_t i = 0; i < B * (size_t)hidden; ++i) out[i] = h[i] + o[i];
  }
done:
  free(h); free(nrm); free(q); free(k); free(v); free(a); free(o); free(g); free(u);
  return rc;
}

/* ------------------------------------------------------------------ mixed-radix schedules
 * HARP page, Sec. 2.1 (Suporte a Misto-Raiz) and Sec. 2.2: for d = b_0 b_1 ... b_{m-1},
 * stage t applies a block-diagonal orthogonal matrix to groups of b_t coordinates that
 * stride permutations bring together. Read here as mixed-radix digits:
 *   stride s_t = b_0 ... b_{t-1}; index i has digit i_t = (i / s_t) mod b_t;
 *   group c of stage t is the b_t indices base_c + j s_t (j = 0..b_t-1) that share every
 *   other digit, groups numbered in increasing order of base_c:
 *   base_c = (c mod s_t) + (c div s_t) s_t b_t.
 * With every b_t = 2 this is the radix-2 butterfly above (pairs (i, i + 2^t)).
 * Block B_{t,c} = Q_{t,c}(theta) G_{b_t}:
 *   b = 2: the Givens block of the radix-2 butterfly, one angle offset;
 *   b > 2: Q = (I - A)(I + A)^-1 (the Cayley map) of the skew-symmetric A whose strict upper
 *          triangle holds the b(b-1)/2 parameters row by row (A_ij = theta, A_ji = -theta);
 *          G_b = H_b / sqrt(b) (Sylvester) when b is a power of two, else the orthogonal
 *          factor of the QR factorisation of a fixed Gaussian matrix M_b, with R's diagonal
 *          made positive (which makes the factor unique).
 * theta: stage after stage, group after group, the group's parameters in the order above.
 * F = B_{m-1} ... B_0 D (signs first); F^T applies B_t^T from t = m-1 down to 0, then D.
 */
static int ora_mr_params(int b) { return b == 2 ? 1 : b * (b - 1) / 2; }

static int ora_is_pow2(int b) { return b >= 1 && (b & (b - 1)) == 0; }

/* G_b [b][b]: Sylvester H_b / sqrt(b), or the Q factor of M (row-major b x b) by modified
 * Gram-Schmidt on its columns, each column orthogonalised twice, R's diagonal positive. */
int ora_mr_mixer(int b, const double* M, double* G) {
  if (b < 2) return ORA_EINVAL;
  if (ora_is_pow2(b)) {
    const double sc = 1.0 / sqrt((double)b);
    for (int i = 0; i < b; ++i)
      for (int j = 0; j < b; ++j) G[i * b + j] = (__builtin_popcount((unsigned)(i & j)) & 1) ? -sc : sc;
    return ORA_OK;
  }
  if (!M) return ORA_EINVAL;
  double* q = (double*)malloc(sizeof(double) * (size_t)b);
  if (!q) return ORA_EINVAL;
  for (int j = 0; j < b; ++j) {
    for (int i = 0; i < b; ++i) q[i] = M[i * b + j];
    for (int pass = 0; pass < 2; ++pass)
      for (int k = 0; k < j; ++k) {
        double dot = 0.0;
        for (int i = 0; i < b; ++i) dot += G[i * b + k] * q[i];
        for (int i = 0; i < b; ++i) q[i] -= dot * G[i * b + k];
      }
    double nrm = 0.0;
    for (int i = 0; i < b; ++i) nrm += q[i] * q[i];
    nrm = sqrt(nrm);
    if (!(nrm > 0.0)) { free(q); return ORA_EINVAL; }
    for (int i = 0; i < b; ++i) G[i * b + j] = q[i] / nrm;
  }
  free(q);
  return ORA_OK;
}

/* Q = (I - A)(I + A)^-1 for the skew-symmetric A of the b(b-1)/2 parameters th;
 * (I + A) is inverted by Gauss-Jordan elimination with partial pivoting. */
int ora_cayley(int b, const double* th, double* Q) {
  if (b < 2) return ORA_EINVAL;
  const size_t bb = (size_t)b * (size_t)b;
  double* A = (double*)calloc(bb, sizeof(double));
  double* P = (double*)malloc(sizeof(double) * bb);   /* I + A, reduced in place */
  double* X = (double*)malloc(sizeof(double) * bb);   /* becomes (I + A)^-1 */
  if (!A || !P || !X) { free(A); free(P); free(X); return ORA_EINVAL; }
  int k = 0;
  for (int i = 0; i < b; ++i)
    for (int j = i + 1; j < b; ++j, ++k) {
      A[i * b + j] = th[k];
      A[j * b + i] = -th[k];
    }
  for (int i = 0; i < b; ++i)
    for (int j = 0; j < b; ++j) {
      P[i * b + j] = (i == j ? 1.0 : 0.0) + A[i * b + j];
      X[i * b + j] = i == j ? 1.0 : 0.0;
    }
  for (int col = 0; col < b; ++col) {
    int piv = col;
    for (int r = col + 1; r < b; ++r)
      if (fabs(P[r * b + col]) > fabs(P[piv * b + col])) piv = r;
    if (piv != col)
      for (int j = 0; j < b; ++j) {
        double t = P[col * b + j]; P[col * b + j] = P[piv * b + j]; P[piv * b + j] = t;
        t = X[col * b + j]; X[col * b + j] = X[piv * b + j]; X[piv * b + j] = t;
      }
    const double dv = P[col * b + col];
    for (int j = 0; j < b; ++j) { P[col * b + j] /= dv; X[col * b + j] /= dv; }
    for (int r = 0; r < b; ++r) {
      if (r == col) continue;
      const double f = P[r * b + col];
      if (f == 0.0) continue;
      for (int j = 0; j < b; ++j) { P[r * b + j] -= f * P[col * b + j]; X[r * b + j] -= f * X[col * b + j]; }
    }
  }
  for (int i = 0; i < b; ++i)
    for (int j = 0; j < b; ++j) {
      double acc = 0.0;
      for (int l = 0; l < b; ++l) acc += ((i == l ? 1.0 : 0.0) - A[i * b + l]) * X[l * b + j];
      Q[i * b + j] = acc;
    }
  free(A); free(P); free(X);
  return ORA_OK;
}

/* The stage blocks B_{t,c} [groups][b][b] of one stage (b = 2 included, as a 2 x 2 matrix). */
static int ora_mr_stage_blocks(int64_t d, int b, const double* th, const double* M, double* Bs) {
  const int64_t groups = d / b;
  const size_t bb = (size_t)b * (size_t)b;
  if (b == 2) {
    for (int64_t c = 0; c < groups; ++c) {
      const double psi = ORA_PI / 4.0 + th[c], cs = cos(psi), sn = sin(psi);
      double* B = Bs + (size_t)c * 4;
      B[0] = cs; B[1] = sn; B[2] = sn; B[3] = -cs;
    }
    return ORA_OK;
  }
  double* G = (double*)malloc(sizeof(double) * bb);
  double* Q = (double*)malloc(sizeof(double) * bb);
  int rc = (G && Q) ? ora_mr_mixer(b, M, G) : ORA_EINVAL;
  for (int64_t c = 0; c < groups && rc == ORA_OK; ++c) {
    rc = ora_cayley(b, th + (size_t)c * (size_t)ora_mr_params(b), Q);
    double* B = Bs + (size_t)c * bb;
    for (int i = 0; i < b && rc == ORA_OK; ++i)
      for (int j = 0; j < b; ++j) {
        double acc = 0.0;
        for (int l = 0; l < b; ++l) acc += Q[i * b + l] * G[l * b + j];
        B[i * b + j] = acc;
      }
  }
  free(G); free(Q);
  return rc;
}

/* x [batch][d] in place. radix [m]; theta: every stage's parameters, stage after stage;
 * gauss: every stage's b_t x b_t Gaussian, stage after stage (read only for radices that
 * are not powers of two; may be NULL when there are none). */
int ora_mr_butterfly(int64_t d, int m, const int* radix, const double* theta, const int8_t* sign,
                     const double* gauss, int inverse, int64_t batch, double* x) {
  if (m < 1 || d < 2 || batch < 0) return ORA_EINVAL;
  int64_t prod = 1;
  for (int t = 0; t < m; ++t) {
    if (radix[t] < 2 || radix[t] > 256) return ORA_EINVAL;
    prod *= radix[t];
  }
  if (prod != d) return ORA_EINVAL;
  double** blocks = (double**)calloc((size_t)m, sizeof(double*));
  if (!blocks) return ORA_EINVAL;
  int rc = ORA_OK;
  size_t toff = 0, goff = 0;
  for (int t = 0; t < m && rc == ORA_OK; ++t) {
    const int b = radix[t];
    blocks[t] = (double*)malloc(sizeof(double) * (size_t)(d / b) * (size_t)b * (size_t)b);
    if (!blocks[t]) { rc = ORA_EINVAL; break; }
    rc = ora_mr_stage_blocks(d, b, theta + toff, gauss ? gauss + goff : NULL, blocks[t]);
    toff += (size_t)(d / b) * (size_t)ora_mr_params(b);
    goff += (size_t)b * (size_t)b;
  }
  if (rc == ORA_OK) {
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < batch; ++r) {
      double* v = x + r * d;
      double tmp[256], out[256];
      if (!inverse)
        for (int64_t i = 0; i < d; ++i) v[i] *= (double)sign[i];
      for (int step = 0; step < m; ++step) {
        const int t = inverse ? m - 1 - step : step;
        const int b = radix[t];
        int64_t st = 1;
        for (int k = 0; k < t; ++k) st *= radix[k];
        for (int64_t c = 0; c < d / b; ++c) {
          const int64_t base = (c % st) + (c / st) * st * b;
          const double* B = blocks[t] + (size_t)c * (size_t)b * (size_t)b;
          for (int j = 0; j < b; ++j) tmp[j] = v[base + j * st];
          for (int i = 0; i < b; ++i) {
            double acc = 0.0;
            for (int j = 0; j < b; ++j) acc += (inverse ? B[j * b + i] : B[i * b + j]) * tmp[j];
            out[i] = acc;
          }
          for (int i = 0; i < b; ++i) v[base + i * st] = out[i];
        }
      }
      if (inverse)
        for (int64_t i = 0; i < d; ++i) v[i] *= (double)sign[i];
    }
  }
  for (int t = 0; t < m; ++t) free(blocks[t]);
  free(blocks);
  return rc;
}

/* ------------------------------------------------------------------ int8 angles
 * The HARP page stores its parameters in int8 (Sec. 2.4, Armazenamento; Sec. 4, 2.00 ->
 * 2.05 bits per parameter at 2 bits). The format is this library's reading:
 * every stage t of a butterfly has one symmetric step, and the angle offsets become
 *   delta_t = fp32(max_p |theta_tp| / 127),
 *   q_tp    = clamp(round_half_even(theta_tp / delta_t), -127, 127)   (0 when delta_t = 0),
 *   theta^  = delta_t * q_tp.
 * A layer stored this way is the layer built from theta^: W' is rotated with theta^.
 */
int ora_quantize_angles(int64_t m, int64_t half, const double* theta, int8_t* q, float* delta) {
  if (m < 1 || half < 1) return ORA_EINVAL;
  for (int64_t t = 0; t < m; ++t) {
    const double* th = theta + t * half;
    double mx = 0.0;
    for (int64_t p = 0; p < half; ++p) mx = fabs(th[p]) > mx ? fabs(th[p]) : mx;
    const float d = (float)(mx / 127.0);
    delta[t] = d;
    for (int64_t p = 0; p < half; ++p) {
      double v = d > 0.0f ? rint(th[p] / (double)d) : 0.0;
      if (v > 127.0) v = 127.0;
      if (v < -127.0) v = -127.0;
      q[t * half + p] = (int8_t)v;
    }
  }
  return ORA_OK;
}

/* ------------------------------------------------------------------ calibration objective
 * The per-layer fitting loss of the HARP page, Sec. 2.3 (Objetivo de Otimizacao):
 *   L_fit(Theta) = L_diag(Theta) + lambda_bd * R_bd(Theta_V).
 * H is the input-side Hessian proxy [n_in][n_in] (symmetric; NULL: the identity). In the
 * rotated coordinates the layer sees inputs V x, so its proxy there is H' = V H V^T.
 *   L_diag = sum_{r,j} d_j (W'_rj - T_rj)^2,   d = diag(H'),
 *            W' = U W V^T and T = deq(Q(W')) its blockwise code target;
 *   R_bd   = sum of H'_ij^2 over i, j in different quantizer groups (floor(i / group)).
 * The gradient treats T as a constant (the page stops gradients through the discrete
 * code assignment) and is taken with respect to the angle offsets theta of both
 * butterflies, through W' (U and V), d (V) and R_bd (V).
 *
 * Backward through one 2x2 block: the stage maps (a, b) to (u, v) = (c a + s b, s a - c b)
 * with c = cos p, s = sin p, p = pi/4 + theta. Its derivative in p is (-v, u), so
 * dL/dtheta = g_v u - g_u v from the block's outputs and their gradients alone, and
 * since the block is its own inverse, (a, b) and (g_a, g_b) are the block applied to
 * (u, v) and (g_u, g_v).
 */
typedef struct {
  int64_t n, w;
  int m;
  double* c; /* [m][n/2] cos(pi/4 + theta), then sin */
  double* s;
} ora_tab;

static int ora_tab_make(ora_tab* T, int64_t n, int64_t w, const double* theta) {
  T->n = n;
  T->w = w;
  T->m = ora_check_bfly(n, w);
  T->c = T->s = NULL;
  if (T->m < 1) return ORA_EINVAL;
  const size_t k = (size_t)T->m * (size_t)(n / 2);
  T->c = (double*)malloc(sizeof(double) * k);
  T->s = (double*)malloc(sizeof(double) * k);
  if (!T->c || !T->s) return ORA_EINVAL;
  for (size_t i = 0; i < k; ++i) {
    const double psi = ORA_PI / 4.0 + theta[i];
    T->c[i] = cos(psi);
    T->s[i] = sin(psi);
  }
  return ORA_OK;
}

static void ora_tab_free(ora_tab* T) { free(T->c); free(T->s); }

/* One stage t of one w-wide block k, run backwards on a row: y holds the stage's
 * outputs and becomes its inputs, g likewise for the gradients; dth gets the angle
 * gradients of the stage's pairs. */
static void ora_stage_back(const ora_tab* T, int t, int64_t k, double* y, double* g, double* dth) {
  const int64_t h = (int64_t)1 << t, w = T->w;
  for (int64_t i = k * w; i < (k + 1) * w; ++i) {
    const int64_t il = i - k * w;
    if (il & h) continue;
    const int64_t p = (int64_t)t * (T->n / 2) + k * (w / 2) + ((il >> (t + 1)) << t) + (il & (h - 1));
    const double c = T->c[p], s = T->s[p];
    const double u = y[i], v = y[i + h], gu = g[i], gv = g[i + h];
    dth[p] += gv * u - gu * v;
    y[i] = c * u + s * v;
    y[i + h] = s * u - c * v;
    g[i] = c * gu + s * gv;
    g[i + h] = s * gu - c * gv;
  }
}

/* Backward of `batch` rows that went through F (inverse = 0) or F^T (inverse = 1):
 * y: the rows' outputs, replaced by their inputs; g: dL/dy, replaced by dL/dx;
 * dth [m][n/2] += dL/dtheta. Blocks are independent (disjoint pairs) and run in
 * parallel; rows run in index order, so every angle's sum has one fixed order. */
static void ora_bfly_back(const ora_tab* T, int64_t batch, const int8_t* sign, int inverse, double* y, double* g,
                          double* dth) {
  const int64_t n = T->n, nb = n / T->w;
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < nb; ++k) {
    for (int64_t r = 0; r < batch; ++r) {
      double* yr = y + r * n;
      double* gr = g + r * n;
      if (inverse) { /* F^T = D S_0 ... S_{m-1}: undo D, then S_0 first */
        for (int64_t i = k * T->w; i < (k + 1) * T->w; ++i) { yr[i] *= (double)sign[i]; gr[i] *= (double)sign[i]; }
        for (int t = 0; t < T->m; ++t) ora_stage_back(T, t, k, yr, gr, dth);
      } else { /* F = S_{m-1} ... S_0 D: S_{m-1} first, then D */
        for (int t = T->m - 1; t >= 0; --t) ora_stage_back(T, t, k, yr, gr, dth);
        for (int64_t i = k * T->w; i < (k + 1) * T->w; ++i) { yr[i] *= (double)sign[i]; gr[i] *= (double)sign[i]; }
      }
    }
  }
}

static void ora_transpose(int64_t R, int64_t C, const double* in, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t c = 0; c < C; ++c)
    for (int64_t r = 0; r < R; ++r) out[c * R + r] = in[r * C + c];
}

/* out[0] = L_fit, out[1] = L_diag, out[2] = R_bd. gV [log2 w_in][n_in/2] and
 * gU [log2 w_out][n_out/2] receive dL_fit/dtheta when non-NULL. */
int ora_calib_fit(int64_t n_out, int64_t n_in, int bits, int group, int64_t w_in, int64_t w_out,
                  const double* thV, const int8_t* sV, const double* thU, const int8_t* sU, const double* W,
                  const double* H, double lambda_bd, double* out, double* gV, double* gU) {
  if (bits < 2 || bits > 4 || group < 1 || n_in % group) return ORA_EINVAL;
  const int mi = ora_check_bfly(n_in, w_in), mo = ora_check_bfly(n_out, w_out);
  if (mi < 1 || mo < 1) return ORA_EINVAL;
  const size_t nw = (size_t)n_out * (size_t)n_in, nh = (size_t)n_in * (size_t)n_in;
  const int64_t ng = n_in / group;
  const int grad = gV || gU;
  double *Wr = NULL, *E = NULL, *A = NULL, *Hp = NULL, *Hq = NULL, *K = NULL, *d = NULL, *e = NULL, *row = NULL;
  uint8_t* q = NULL;
  uint16_t *s16 = NULL, *z16 = NULL;
  ora_tab TV = {0}, TU = {0};
  int rc = ORA_OK;
  Wr = (double*)malloc(sizeof(double) * nw);
  E = (double*)malloc(sizeof(double) * nw);
  q = (uint8_t*)malloc(nw);
  s16 = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)n_out * (size_t)ng);
  z16 = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)n_out * (size_t)ng);
  d = (double*)malloc(sizeof(double) * (size_t)n_in);
  e = (double*)malloc(sizeof(double) * (size_t)n_in);
  row = (double*)malloc(sizeof(double) * (size_t)n_out);
  if (!Wr || !E || !q || !s16 || !z16 || !d || !e || !row) { rc = ORA_EINVAL; goto done; }

  /* W', its code target T and the residual E = W' - T */
  memcpy(Wr, W, sizeof(double) * nw);
  if ((rc = ora_rotate_weights(n_out, n_in, w_in, w_out, thV, sV, thU, sU, Wr))) goto done;
  if ((rc = ora_quantize(n_out, n_in, bits, group, Wr, q, s16, z16))) goto done;
  for (int64_t r = 0; r < n_out; ++r)
    for (int64_t j = 0; j < n_in; ++j) {
      const int64_t g = r * ng + j / group;
      E[r * n_in + j] = Wr[r * n_in + j] - (ora_f16_to_f64(s16[g]) * (double)q[r * n_in + j] + ora_f16_to_f64(z16[g]));
    }

  /* H' = V H V^T: rows of H through F_V give B = H V^T; rows of B^T through F_V give H' */
  if (H) {
    Hp = (double*)malloc(sizeof(double) * nh);
    Hq = (double*)malloc(sizeof(double) * nh);
    if (!Hp || !Hq) { rc = ORA_EINVAL; goto done; }
    memcpy(Hp, H, sizeof(double) * nh);
    if ((rc = ora_butterfly_fwd(n_in, w_in, n_in, thV, sV, Hp))) goto done;
    ora_transpose(n_in, n_in, Hp, Hq);
    if ((rc = ora_butterfly_fwd(n_in, w_in, n_in, thV, sV, Hq))) goto done;
    for (int64_t j = 0; j < n_in; ++j) d[j] = Hq[j * n_in + j];
  } else {
    for (int64_t j = 0; j < n_in; ++j) d[j] = 1.0;
  }

  /* the loss, summed row by row in index order */
  {
    double Ld = 0.0, Rb = 0.0;
    for (int64_t r = 0; r < n_out; ++r) {
      double acc = 0.0;
      for (int64_t j = 0; j < n_in; ++j) acc += d[j] * E[r * n_in + j] * E[r * n_in + j];
      Ld += acc;
    }
    if (H)
      for (int64_t i = 0; i < n_in; ++i) {
        double acc = 0.0;
        for (int64_t j = 0; j < n_in; ++j)
          if (i / group != j / group) acc += Hq[i * n_in + j] * Hq[i * n_in + j];
        Rb += acc;
      }
    out[0] = Ld + lambda_bd * Rb;
    out[1] = Ld;
    out[2] = Rb;
  }
  if (!grad) goto done;

  if ((rc = ora_tab_make(&TV, n_in, w_in, thV)) || (rc = ora_tab_make(&TU, n_out, w_out, thU))) goto done;
  double* dV = (double*)calloc((size_t)mi * (size_t)(n_in / 2), sizeof(double));
  double* dU = (double*)calloc((size_t)mo * (size_t)(n_out / 2), sizeof(double));
  A = (double*)malloc(sizeof(double) * nw);
  if (!dV || !dU || !A) { free(dV); free(dU); rc = ORA_EINVAL; goto done; }

  /* dL_diag/dW' = 2 d_j E_rj (T constant); e_j = sum_r E_rj^2 = dL_diag/dd_j */
  for (int64_t j = 0; j < n_in; ++j) {
    double acc = 0.0;
    for (int64_t r = 0; r < n_out; ++r) acc += E[r * n_in + j] * E[r * n_in + j];
    e[j] = acc;
  }
  for (int64_t r = 0; r < n_out; ++r)
    for (int64_t j = 0; j < n_in; ++j) E[r * n_in + j] *= 2.0 * d[j];

  /* columns: W'_{:,j} = F_U^T A_{:,j}; back through it, one column at a time */
  for (int64_t j = 0; j < n_in; ++j) {
    double* gcol = A; /* scratch: the column's gradient, then written back into E */
    for (int64_t r = 0; r < n_out; ++r) { row[r] = Wr[r * n_in + j]; gcol[r] = E[r * n_in + j]; }
    ora_bfly_back(&TU, 1, sU, 1, row, gcol, dU);
    for (int64_t r = 0; r < n_out; ++r) E[r * n_in + j] = gcol[r];
  }
  /* rows: A_r = F_V W_r (recomputed), back through F_V with dL/dA in E */
  memcpy(A, W, sizeof(double) * nw);
  if ((rc = ora_butterfly_fwd(n_in, w_in, n_out, thV, sV, A))) { free(dV); free(dU); goto done; }
  ora_bfly_back(&TV, n_out, sV, 0, A, E, dV);

  if (H) {
    /* dL/dH' = 2 lambda_bd H' (off-group entries) + diag(e) */
    K = (double*)malloc(sizeof(double) * nh);
    if (!K) { free(dV); free(dU); rc = ORA_EINVAL; goto done; }
    for (int64_t i = 0; i < n_in; ++i)
      for (int64_t j = 0; j < n_in; ++j)
        K[i * n_in + j] = (i / group != j / group ? 2.0 * lambda_bd * Hq[i * n_in + j] : 0.0) + (i == j ? e[i] : 0.0);
    /* second pass: rows of H' came from rows of B^T; Hq becomes B^T, K its gradient */
    ora_bfly_back(&TV, n_in, sV, 0, Hq, K, dV);
    /* first pass: rows of B came from rows of H */
    ora_transpose(n_in, n_in, Hq, Hp);
    ora_transpose(n_in, n_in, K, Hq);
    ora_bfly_back(&TV, n_in, sV, 0, Hp, Hq, dV);
  }
  if (gV) memcpy(gV, dV, sizeof(double) * (size_t)mi * (size_t)(n_in / 2));
  if (gU) memcpy(gU, dU, sizeof(double) * (size_t)mo * (size_t)(n_out / 2));
  free(dV);
  free(dU);
done:
  free(Wr); free(E); free(A); free(Hp); free(Hq); free(K); free(d); free(e); free(row);
  free(q); free(s16); free(z16);
  ora_tab_free(&TV);
  ora_tab_free(&TU);
  return rc;
}
