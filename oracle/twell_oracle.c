/*
 * twell_oracle.c — plain, slow, fp64 CPU oracle for the activation-sparse gated
 * FFN and its TwELL (tile-wise ELLPACK) packing.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no code, header, table or helper with the CUDA library.
 *
 * Sources (the only description of the method; they print no code, no worked
 * example and no kernel internals):
 *   [aimodelsnavi] "How TwELL by Sakana AI and NVIDIA Accelerates LLMs by 20%
 *                  Using Unstructured Sparsity" (aimodelsnavi.com)
 *   [aivizor]      "Sakana AI и NVIDIA представили TwELL — формат и CUDA-ядра,
 *                  превращающие активную разреженность в реальные ускорения LLM"
 *                  (edge.aivizor.me), paragraphs 1-4
 *
 * What is computed, and where it is stated:
 *   - gated FFN with gate / up / down projections ([aivizor] ¶2), ReLU gate
 *     ([aimodelsnavi] "Technical Explanation"), a gate bias b_g:
 *         z = X W_g^T + b_g,  g = ReLU(z),  u = X W_u^T,  h = g * u,  Y = h W_d^T
 *   - TwELL: the hidden dimension is cut into horizontal tiles of width T_n and
 *     nonzeros are packed locally inside each tile ([aivizor] ¶2; ELLPACK per
 *     tile, [aimodelsnavi] "Core of TwELL"): per (row, tile) a count and up to K
 *     (value, in-tile column) pairs.
 *   - hybrid format: a row goes to the compact ELL store, or, if it overflows K,
 *     to a dense backup block ([aivizor] ¶2 and ¶4 on non-uniform sparsity).
 *   - L1 term on the gate activations ([aivizor] ¶1): loss adds lambda * sum(g).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   active  <=> z > 0 (z == 0 is inactive, ReLU'(0) = 0);
 *   slot order = ascending in-tile column; the first min(count, K) actives are
 *   kept; unused slots are (value 0, column 0); count holds the true count even
 *   when it exceeds K; a row overflows when any of its tiles has count > K, and
 *   overflow rows are listed in ascending row order; stored values are
 *   bfloat16 round-to-nearest-even of z; the L1 term is a plain sum over g.
 *
 * Arithmetic: every input is a bfloat16 bit pattern converted exactly to double;
 * every sum runs in ascending index order in double precision; terms with g == 0
 * are skipped, which leaves each sum unchanged. Build with -ffp-contract=off and
 * without -ffast-math so that no sum is re-associated or fused.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- bfloat16 */

/* bfloat16 bits -> double, exact (bfloat16 is the top half of a binary32). */
double oracle_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* double -> bfloat16 bits, round to nearest, ties to even.
 * bfloat16 keeps 8 significant bits and the binary32 exponent range. For
 * |x| = m 2^e with m in [0.5, 1), the spacing of representable values is
 * 2^(e-8) while 2^(e-1) is a normal number (e-1 >= -126), and 2^-133 below it
 * (subnormals). x / spacing is exact in double; rounding it with nearbyint under
 * the default round-to-nearest-even mode and scaling back gives the result,
 * which is exactly representable in binary32, whose top 16 bits are the answer. */
uint16_t oracle_bf16_round(double x) {
  if (isnan(x)) return 0x7FC0;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  if (isinf(a)) return (uint16_t)(sign | 0x7F80);
  int e;
  (void)frexp(a, &e);
  int q_exp = (e - 1 >= -126) ? (e - 8) : -133;
  double q = ldexp(a, -q_exp);
  double r = nearbyint(q);
  double v = ldexp(r, q_exp);
  if (v >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);
  float fv = (float)v;
  uint32_t u;
  memcpy(&u, &fv, sizeof u);
  return (uint16_t)(sign | (uint16_t)(u >> 16));
}

void oracle_bf16_round_array(const double* in, uint16_t* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_round(in[i]);
}

void oracle_bf16_to_double_array(const uint16_t* in, double* out, int64_t n) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_to_double(in[i]);
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

static double* to_double(const uint16_t* b, int64_t n) {
  double* d = (double*)malloc((size_t)n * sizeof(double));
  if (d) oracle_bf16_to_double_array(b, d, n);
  return d;
}

/* [rows x cols] bf16 -> [cols x rows] double (so that a loop over the original
 * row index runs over contiguous memory). */
static double* to_double_transposed(const uint16_t* b, int64_t rows, int64_t cols) {
  double* d = (double*)malloc((size_t)(rows * cols) * sizeof(double));
  if (!d) return NULL;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) d[c * rows + r] = oracle_bf16_to_double(b[r * cols + c]);
  return d;
}

/* ------------------------------------------------------------- 8-bit weights */

/* Combining the method with 8-bit quantisation is the pages' outlook
 * ([aimodelsnavi] "Industry Impact", long-term impact). Reading taken here: the
 * weights the sparse kernels gather (W_u and W_d) are stored per hidden unit j
 * (row j of W_u, column j of W_d) as FP8 E4M3 codes with one power-of-two scale
 * 2^e_j per unit and matrix. E4M3 (the OCP 8-bit floating-point format with a
 * 4-bit exponent, bias 7, and a 3-bit mantissa; no infinities; code 0x7F/0xFF is
 * NaN; largest finite value 448): code s eeee mmm is (-1)^s (8 + m) 2^(e - 10)
 * for e >= 1 and (-1)^s m 2^-9 for e = 0.
 *   e_j  = the smallest integer with max_k |w_jk| <= 448 * 2^e_j (0 for a zero unit)
 *   q_jk = w_jk / 2^e_j rounded to the nearest E4M3 value, ties to even mantissa
 *   w~_jk = value(q_jk) * 2^e_j, which has at most 4 significant bits and is
 *          therefore a bf16 value exactly
 * The FFN with 8-bit weights is the definition above evaluated on w~. */

double oracle_e4m3_value(uint8_t code) {
  const int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  const double v = e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
  return s ? -v : v;
}

/* Nearest E4M3 code of x (ties to even); |x| > 448 saturates to +-448. Within a
 * binade [2^k, 2^(k+1)), k >= -6, the E4M3 values are spaced 2^(k-3); below
 * 2^-6 (the subnormals) they are spaced 2^-9. a / spacing is exact, nearbyint
 * rounds it half to even (an even integer is an even mantissa), and a result
 * of 2^(k+1) moves to the next binade with mantissa 0. */
uint8_t oracle_e4m3_round(double x) {
  if (isnan(x)) return 0x7F;
  const uint8_t sign = signbit(x) ? 0x80 : 0;
  const double a = fabs(x);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  if (a == 0.0) return sign;
  int E;
  (void)frexp(a, &E); /* a in [2^(E-1), 2^E) */
  const int k = E - 1;
  const double spacing = k >= -6 ? ldexp(1.0, k - 3) : ldexp(1.0, -9);
  const double r = nearbyint(a / spacing) * spacing;
  if (r == 0.0) return sign;
  if (r < ldexp(1.0, -6)) return (uint8_t)(sign | (int)ldexp(r, 9));
  int E2;
  (void)frexp(r, &E2);
  const int k2 = E2 - 1;
  const int m = (int)ldexp(r, 3 - k2) - 8;
  return (uint8_t)(sign | ((k2 + 7) << 3) | m);
}

/* Quantises `units` units of `len` bf16 weights each; element k of unit j is
 * W[j * su + k * sk]. Writes q[j * len + k] (unit-major codes), exps[j] = e_j and
 * deq[j * su + k * sk] = bf16 bits of w~_jk (the input's layout). */
void oracle_quantize_units(const uint16_t* W, int64_t units, int64_t len, int64_t su, int64_t sk, uint8_t* q,
                           int32_t* exps, uint16_t* deq) {
  for (int64_t j = 0; j < units; ++j) {
    double amax = 0.0;
    for (int64_t k = 0; k < len; ++k) {
      const double v = fabs(oracle_bf16_to_double(W[j * su + k * sk]));
      if (v > amax) amax = v;
    }
    int e = 0;
    if (amax > 0.0) {
      int E;
      (void)frexp(amax, &E);
      e = E - 12; /* 448 * 2^(E - 12) < 2^(E - 1) <= amax: start below the answer */
      while (amax > ldexp(448.0, e)) ++e;
    }
    exps[j] = e;
    for (int64_t k = 0; k < len; ++k) {
      const uint8_t c = oracle_e4m3_round(ldexp(oracle_bf16_to_double(W[j * su + k * sk]), -e));
      q[j * len + k] = c;
      deq[j * su + k * sk] = oracle_bf16_round(ldexp(oracle_e4m3_value(c), e));
    }
  }
}

/* -------------------------------------------------------------------- gate */

/* z_ij = sum_k x_ik W_g[j,k] (k ascending) + b_j for one row i.
 * Loop order k outer, j inner: each z_ij still accumulates its terms in
 * ascending k; the inner loop runs over contiguous memory of W_g^T. */
static void gate_row(const double* x, const double* WgT, const double* b, int64_t d, int64_t f,
                     double* z) {
  for (int64_t j = 0; j < f; ++j) z[j] = 0.0;
  for (int64_t k = 0; k < d; ++k) {
    const double xk = x[k];
    const double* w = WgT + k * f;
    for (int64_t j = 0; j < f; ++j) z[j] += xk * w[j];
  }
  for (int64_t j = 0; j < f; ++j) z[j] += b[j];
}

/* Dot product in ascending k. */
static double dot(const double* a, const double* b, int64_t n) {
  double s = 0.0;
  for (int64_t k = 0; k < n; ++k) s += a[k] * b[k];
  return s;
}

/* Gate pre-activation Z [nrows x f] for rows[0..nrows) (rows == NULL: all M rows).
 * Returns 0, or 1 on allocation failure. */
int oracle_gate(const uint16_t* X, const uint16_t* Wg, const uint16_t* bg, int64_t M, int64_t d,
                int64_t f, const int32_t* rows, int64_t nrows, double* Z) {
  if (!rows) nrows = M;
  double* WgT = to_double_transposed(Wg, f, d);
  double* b = to_double(bg, f);
  if (!WgT || !b) { free(WgT); free(b); return 1; }
  int err = 0;
#pragma omp parallel
  {
    double* x = (double*)malloc((size_t)d * sizeof(double));
    if (!x) {
#pragma omp atomic write
      err = 1;
    } else {
#pragma omp for schedule(dynamic, 4)
      for (int64_t r = 0; r < nrows; ++r) {
        const int64_t i = rows ? rows[r] : r;
        oracle_bf16_to_double_array(X + i * d, x, d);
        gate_row(x, WgT, b, d, f, Z + r * f);
      }
      free(x);
    }
  }
  free(WgT);
  free(b);
  return err;
}

/* -------------------------------------------------------------------- pack */

/* TwELL + hybrid routing of a dense gate pre-activation Z [M x f].
 * Per (row i, tile t) over columns [t*T_n, (t+1)*T_n):
 *   count[i,t] = #{c : Z[i, t*T_n + c] > 0}
 *   the first min(count, K) active c in ascending order fill slots 0.. with
 *   val = bf16(Z), col = c; the remaining slots are (0, 0).
 * Row i overflows (row_ovf[i] = 1) when some tile has count > K, or, with
 * dense_min > 0, when its active units (the sum of its counts) number at least
 * dense_min (rows whose gathers cost more than a dense row). Overflow rows
 * are listed in ascending order in ovf_rows; the first `cap` of them get a dense
 * row g_ovf[s, :] = bf16(ReLU(Z[i, :])) (bits 0 where Z <= 0).
 * *n_ovf_total receives the number of overflow rows. Returns 0, 3 when that
 * number exceeds cap (rows beyond cap are counted but not stored), or 1 when
 * the shape is not packable (in-tile columns are bytes, so 1 <= T_n <= 256,
 * and d_ff must be a whole number of tiles). */
int oracle_pack(const double* Z, int64_t M, int64_t f, int32_t T_n, int32_t K, int64_t cap, int64_t dense_min,
                uint16_t* count, uint16_t* val, uint8_t* col, uint8_t* row_ovf, int32_t* ovf_rows,
                int64_t* n_ovf_total, uint16_t* g_ovf) {
  if (T_n < 1 || T_n > 256 || K < 1 || f % T_n != 0) return 1;
  const int64_t T = f / T_n;
  int64_t n = 0;
  for (int64_t i = 0; i < M; ++i) {
    int ovf = 0;
    int64_t active = 0;
    for (int64_t t = 0; t < T; ++t) {
      const double* z = Z + i * f + t * T_n;
      uint16_t* v = val + (i * T + t) * K;
      uint8_t* c8 = col + (i * T + t) * K;
      for (int32_t s = 0; s < K; ++s) { v[s] = 0; c8[s] = 0; }
      int32_t cnt = 0;
      for (int32_t c = 0; c < T_n; ++c) {
        if (z[c] > 0.0) {
          if (cnt < K) { v[cnt] = oracle_bf16_round(z[c]); c8[cnt] = (uint8_t)c; }
          ++cnt;
        }
      }
      count[i * T + t] = (uint16_t)cnt;
      if (cnt > K) ovf = 1;
      active += cnt;
    }
    if (dense_min > 0 && active >= dense_min) ovf = 1;
    row_ovf[i] = (uint8_t)ovf;
    if (ovf) {
      if (n < cap) {
        ovf_rows[n] = (int32_t)i;
        for (int64_t j = 0; j < f; ++j) {
          const double zj = Z[i * f + j];
          g_ovf[n * f + j] = zj > 0.0 ? oracle_bf16_round(zj) : 0;
        }
      }
      ++n;
    }
  }
  *n_ovf_total = n;
  return n > cap ? 3 : 0;
}

/* Dense bf16 ReLU(Z) [M x f] rebuilt from the hybrid format: ELL slots for rows
 * with row_ovf == 0, the dense backup row for the others. */
void oracle_unpack(const uint16_t* count, const uint16_t* val, const uint8_t* col,
                   const uint8_t* row_ovf, const int32_t* ovf_rows, int64_t n_ovf,
                   const uint16_t* g_ovf, int64_t M, int64_t f, int32_t T_n, int32_t K,
                   uint16_t* G) {
  const int64_t T = f / T_n;
  memset(G, 0, (size_t)(M * f) * sizeof(uint16_t));
  for (int64_t i = 0; i < M; ++i) {
    if (row_ovf[i]) continue;
    for (int64_t t = 0; t < T; ++t) {
      int32_t cnt = count[i * T + t];
      if (cnt > K) cnt = K;
      for (int32_t s = 0; s < cnt; ++s)
        G[i * f + t * T_n + col[(i * T + t) * K + s]] = val[(i * T + t) * K + s];
    }
  }
  for (int64_t s = 0; s < n_ovf; ++s) memcpy(G + (int64_t)ovf_rows[s] * f, g_ovf + s * f, (size_t)f * 2);
}

/* ----------------------------------------------------------------- forward */

/* Y [nrows x d] for rows[0..nrows) (rows == NULL: all), by the definition:
 *   z_ij = x_i . W_g[j] + b_j;  active_ij = (mask ? mask[r, j] : z_ij > 0)
 *   g_ij = active ? (round_g ? bf16(z_ij) : z_ij) : 0
 *   u_ij = x_i . W_u[j];  h_ij = g_ij u_ij;  Y_ic = sum_j h_ij W_d[c, j]  (j ascending)
 * mask, when given, is [nrows x f] bytes and replaces the z > 0 test (used to
 * evaluate the definition on another implementation's active set).
 * gmat, when given, is [nrows x f] bf16 bits of g itself: active_ij = (gmat != 0)
 * and g_ij = gmat_ij (used to evaluate the definition on the g values another
 * implementation stored, i.e. with its z > 0 and bf16 rounding decisions).
 * Returns 0, or 1 on allocation failure. */
int oracle_ffn_fwd(const uint16_t* X, const uint16_t* Wg, const uint16_t* bg, const uint16_t* Wu,
                   const uint16_t* Wd, int64_t M, int64_t d, int64_t f, const int32_t* rows,
                   int64_t nrows, const uint8_t* mask, int32_t round_g, const uint16_t* gmat, double* Y) {
  if (!rows) nrows = M;
  const int given = (mask != NULL) || (gmat != NULL);
  double* WgT = given ? NULL : to_double_transposed(Wg, f, d);
  double* Wgd = given ? to_double(Wg, f * d) : NULL;
  double* Wud = to_double(Wu, f * d);
  double* WdT = to_double_transposed(Wd, d, f); /* WdT[j*d + c] = W_d[c, j] */
  double* b = to_double(bg, f);
  int err = (!(WgT || Wgd) || !Wud || !WdT || !b);
  if (!err) {
#pragma omp parallel
    {
      double* x = (double*)malloc((size_t)d * sizeof(double));
      double* z = (double*)malloc((size_t)f * sizeof(double));
      if (!x || !z) {
#pragma omp atomic write
        err = 1;
      } else {
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < nrows; ++r) {
          const int64_t i = rows ? rows[r] : r;
          oracle_bf16_to_double_array(X + i * d, x, d);
          if (!given) gate_row(x, WgT, b, d, f, z);
          double* y = Y + r * d;
          for (int64_t c = 0; c < d; ++c) y[c] = 0.0;
          for (int64_t j = 0; j < f; ++j) {
            double zj;
            if (gmat) {
              if (gmat[r * f + j] == 0) continue;
              zj = oracle_bf16_to_double(gmat[r * f + j]);
            } else if (mask) {
              if (!mask[r * f + j]) continue;
              zj = dot(x, Wgd + j * d, d) + b[j];
            } else {
              zj = z[j];
              if (!(zj > 0.0)) continue;
            }
            const double g = (round_g && !gmat) ? oracle_bf16_to_double(oracle_bf16_round(zj)) : zj;
            const double u = dot(x, Wud + j * d, d);
            const double h = g * u;
            const double* w = WdT + j * d;
            for (int64_t c = 0; c < d; ++c) y[c] += h * w[c];
          }
        }
      }
      free(x);
      free(z);
    }
  }
  free(WgT); free(Wgd); free(Wud); free(WdT); free(b);
  return err;
}

/* Y [M x d] computed from the hybrid representation instead of from z:
 * for a row with row_ovf == 0 the active units are the ELL slots
 * (unit t*T_n + col, g = val); for an overflow row they are the nonzeros of its
 * dense backup row. u and Y follow the same definition as oracle_ffn_fwd.
 * Returns 0, or 1 on allocation failure. */
int oracle_ffn_fwd_hybrid(const uint16_t* X, const uint16_t* Wu, const uint16_t* Wd,
                          const uint16_t* count, const uint16_t* val, const uint8_t* col,
                          const uint8_t* row_ovf, const int32_t* ovf_rows, int64_t n_ovf,
                          const uint16_t* g_ovf, int64_t M, int64_t d, int64_t f, int32_t T_n,
                          int32_t K, double* Y) {
  const int64_t T = f / T_n;
  int64_t* slot_of_row = (int64_t*)malloc((size_t)(M > 0 ? M : 1) * sizeof(int64_t));
  double* Wud = to_double(Wu, f * d);
  double* WdT = to_double_transposed(Wd, d, f);
  int err = (!slot_of_row || !Wud || !WdT);
  if (!err) {
    for (int64_t i = 0; i < M; ++i) slot_of_row[i] = -1;
    for (int64_t s = 0; s < n_ovf; ++s) slot_of_row[ovf_rows[s]] = s;
#pragma omp parallel
    {
      double* x = (double*)malloc((size_t)d * sizeof(double));
      if (!x) {
#pragma omp atomic write
        err = 1;
      } else {
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < M; ++i) {
          oracle_bf16_to_double_array(X + i * d, x, d);
          double* y = Y + i * d;
          for (int64_t c = 0; c < d; ++c) y[c] = 0.0;
          if (row_ovf[i]) {
            const int64_t s = slot_of_row[i];
            if (s < 0) continue; /* not stored (capacity exceeded) */
            for (int64_t j = 0; j < f; ++j) {
              const double g = oracle_bf16_to_double(g_ovf[s * f + j]);
              if (g == 0.0) continue;
              const double h = g * dot(x, Wud + j * d, d);
              for (int64_t c = 0; c < d; ++c) y[c] += h * WdT[j * d + c];
            }
          } else {
            for (int64_t t = 0; t < T; ++t) {
              int32_t cnt = count[i * T + t];
              if (cnt > K) cnt = K;
              for (int32_t sl = 0; sl < cnt; ++sl) {
                const int64_t j = t * T_n + col[(i * T + t) * K + sl];
                const double g = oracle_bf16_to_double(val[(i * T + t) * K + sl]);
                const double h = g * dot(x, Wud + j * d, d);
                for (int64_t c = 0; c < d; ++c) y[c] += h * WdT[j * d + c];
              }
            }
          }
        }
        free(x);
      }
    }
  }
  free(slot_of_row); free(Wud); free(WdT);
  return err;
}

/* ---------------------------------------------------------------- backward */

/* Gradients of L = sum_ic Y_ic dY_ic + lambda * sum_ij g_ij, by calculus on the
 * forward definition (g = ReLU(z) with ReLU'(z) = [z > 0]):
 *   dH_ij = sum_c dY_ic W_d[c, j]                       (c ascending)
 *   dU_ij = dH_ij g_ij
 *   dZ_ij = (dH_ij u_ij + lambda) [active_ij]
 *   dX_ik = sum_j (dU_ij W_u[j, k] + dZ_ij W_g[j, k])   (j ascending)
 *   dW_d[c, j] = sum_i dY_ic h_ij;  dW_u[j, k] = sum_i dU_ij x_ik
 *   dW_g[j, k] = sum_i dZ_ij x_ik;  db_g[j] = sum_i dZ_ij   (i ascending)
 * mask [M x f] (nullable) replaces the z > 0 test as in oracle_ffn_fwd; round_g
 * uses bf16(z) for g; gmat [M x f] (nullable) gives g itself as in
 * oracle_ffn_fwd. db_g may be NULL. Returns 0, or 1 on allocation failure. */
int oracle_ffn_bwd(const uint16_t* X, const uint16_t* Wg, const uint16_t* bg, const uint16_t* Wu,
                   const uint16_t* Wd, const uint16_t* dY, double lambda, int64_t M, int64_t d,
                   int64_t f, const uint8_t* mask, int32_t round_g, const uint16_t* gmat, double* dX,
                   double* dWg, double* dWu, double* dWd, double* dbg) {
  const int given = (mask != NULL) || (gmat != NULL);
  double* WgT = given ? NULL : to_double_transposed(Wg, f, d);
  double* Wgd = to_double(Wg, f * d);
  double* Wud = to_double(Wu, f * d);
  double* WdT = to_double_transposed(Wd, d, f);
  double* b = to_double(bg, f);
  /* per-row active lists: unit index and (h, dU, dZ) */
  int64_t* nact = (int64_t*)calloc((size_t)(M > 0 ? M : 1), sizeof(int64_t));
  int32_t** act_j = (int32_t**)calloc((size_t)(M > 0 ? M : 1), sizeof(int32_t*));
  double** act_v = (double**)calloc((size_t)(M > 0 ? M : 1), sizeof(double*));
  int err = ((!given && !WgT) || !Wgd || !Wud || !WdT || !b || !nact || !act_j || !act_v);
  if (!err) {
#pragma omp parallel
    {
      double* x = (double*)malloc((size_t)d * sizeof(double));
      double* dy = (double*)malloc((size_t)d * sizeof(double));
      double* z = (double*)malloc((size_t)f * sizeof(double));
      if (!x || !dy || !z) {
#pragma omp atomic write
        err = 1;
      } else {
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < M; ++i) {
          oracle_bf16_to_double_array(X + i * d, x, d);
          oracle_bf16_to_double_array(dY + i * d, dy, d);
          if (!given) gate_row(x, WgT, b, d, f, z);
          int64_t n = 0;
          for (int64_t j = 0; j < f; ++j)
            n += gmat ? (gmat[i * f + j] != 0) : mask ? (mask[i * f + j] != 0) : (z[j] > 0.0);
          nact[i] = n;
          act_j[i] = (int32_t*)malloc((size_t)(n > 0 ? n : 1) * sizeof(int32_t));
          act_v[i] = (double*)malloc((size_t)(n > 0 ? 3 * n : 1) * sizeof(double));
          if (!act_j[i] || !act_v[i]) {
#pragma omp atomic write
            err = 1;
            continue;
          }
          double* dx = dX + i * d;
          for (int64_t k = 0; k < d; ++k) dx[k] = 0.0;
          int64_t a = 0;
          for (int64_t j = 0; j < f; ++j) {
            double zj;
            if (gmat) {
              if (gmat[i * f + j] == 0) continue;
              zj = oracle_bf16_to_double(gmat[i * f + j]);
            } else if (mask) {
              if (!mask[i * f + j]) continue;
              zj = dot(x, Wgd + j * d, d) + b[j];
            } else {
              zj = z[j];
              if (!(zj > 0.0)) continue;
            }
            const double g = (round_g && !gmat) ? oracle_bf16_to_double(oracle_bf16_round(zj)) : zj;
            const double u = dot(x, Wud + j * d, d);
            const double dh = dot(dy, WdT + j * d, d);
            const double du = dh * g;
            const double dz = dh * u + lambda;
            const double* wu = Wud + j * d;
            const double* wg = Wgd + j * d;
            for (int64_t k = 0; k < d; ++k) {
              dx[k] += du * wu[k];
              dx[k] += dz * wg[k];
            }
            act_j[i][a] = (int32_t)j;
            act_v[i][3 * a + 0] = g * u;
            act_v[i][3 * a + 1] = du;
            act_v[i][3 * a + 2] = dz;
            ++a;
          }
        }
      }
      free(x); free(dy); free(z);
    }
  }
  if (!err) {
    /* weight gradients: for every output element the terms are added in
     * ascending i, exactly as a loop over i would add them; the units are
     * independent, so they are spread over threads after the per-row active
     * lists are regrouped by unit (i ascending inside each unit's list). */
    int64_t* uptr = (int64_t*)calloc((size_t)(f + 1), sizeof(int64_t));
    int64_t tot = 0;
    for (int64_t i = 0; i < M; ++i) tot += nact[i];
    int64_t* urow = (int64_t*)malloc((size_t)(tot > 0 ? tot : 1) * sizeof(int64_t));
    double* uval = (double*)malloc((size_t)(tot > 0 ? 3 * tot : 1) * sizeof(double));
    double* dWdT = (double*)calloc((size_t)(f * d), sizeof(double));
    double* Xd = to_double(X, M * d);
    double* dYd = to_double(dY, M * d);
    if (!uptr || !urow || !uval || !dWdT || !Xd || !dYd) {
      err = 1;
    } else {
      for (int64_t i = 0; i < M; ++i)
        for (int64_t a = 0; a < nact[i]; ++a) uptr[act_j[i][a] + 1] += 1;
      for (int64_t j = 0; j < f; ++j) uptr[j + 1] += uptr[j];
      int64_t* fill = (int64_t*)malloc((size_t)(f > 0 ? f : 1) * sizeof(int64_t));
      if (!fill) {
        err = 1;
      } else {
        memcpy(fill, uptr, (size_t)f * sizeof(int64_t));
        for (int64_t i = 0; i < M; ++i)
          for (int64_t a = 0; a < nact[i]; ++a) {
            const int64_t p = fill[act_j[i][a]]++;
            urow[p] = i;
            uval[3 * p + 0] = act_v[i][3 * a + 0];
            uval[3 * p + 1] = act_v[i][3 * a + 1];
            uval[3 * p + 2] = act_v[i][3 * a + 2];
          }
        free(fill);
#pragma omp parallel for schedule(dynamic, 4)
        for (int64_t j = 0; j < f; ++j) {
          double* gu = dWu + j * d;
          double* gg = dWg + j * d;
          double* gd = dWdT + j * d;
          for (int64_t k = 0; k < d; ++k) { gu[k] = 0.0; gg[k] = 0.0; }
          double db = 0.0;
          for (int64_t p = uptr[j]; p < uptr[j + 1]; ++p) {
            const double* x = Xd + urow[p] * d;
            const double* dy = dYd + urow[p] * d;
            const double h = uval[3 * p + 0], du = uval[3 * p + 1], dz = uval[3 * p + 2];
            for (int64_t k = 0; k < d; ++k) {
              gu[k] += du * x[k];
              gg[k] += dz * x[k];
              gd[k] += h * dy[k];
            }
            db += dz;
          }
          if (dbg) dbg[j] = db;
        }
        for (int64_t j = 0; j < f; ++j)
          for (int64_t c = 0; c < d; ++c) dWd[c * f + j] = dWdT[j * d + c];
      }
    }
    free(uptr); free(urow); free(uval); free(dWdT); free(Xd); free(dYd);
  }
  if (act_j) for (int64_t i = 0; i < M; ++i) free(act_j[i]);
  if (act_v) for (int64_t i = 0; i < M; ++i) free(act_v[i]);
  free(act_j); free(act_v); free(nact);
  free(WgT); free(Wgd); free(Wud); free(WdT); free(b);
  return err;
}
