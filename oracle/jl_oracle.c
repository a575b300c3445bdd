/*
 * jl_oracle.c -- fp64 CPU oracle for Jet-Long dynamic bifocal RoPE attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the checker the CUDA library is compared
 * against.  Only the test-suite, the smoke entry point and the bench's CPU
 * baseline leg load it.  The library never calls it and never falls back to it,
 * and the two share no source, header, table or helper.
 *
 * What it computes is the plain per-pair definition of the method, in double
 * precision, with an explicit mask predicate and no blocking, fusion or
 * inclusion-exclusion:
 *
 *   G    = max(1, ceil(L / w_pretrained))
 *          -- Jet-Long (bittide paper summary) §3.1, group-size equation;
 *             techwalker explainer §二 (G from the current length, L=65536 with a
 *             32768 window gives G=2).
 *   f(x) = floor(x / G)
 *          -- bittide summary §3.1, position-map equation; G=1 makes f the
 *             identity, i.e. plain RoPE.
 *   pair (q, k), k <= q, is LOCAL iff q - k < w_local and then uses standard
 *   RoPE at positions (q, k); every other pair is REMOTE and uses RoPE at
 *   (f(q), f(k))
 *          -- techwalker explainer §二 (local window of 2048 with original
 *             positions, remote window remapped); bittide summary §3.2 (the
 *             merged result equals each query using standard RoPE for local keys
 *             and remapped RoPE for remote keys).
 *   score = scale * <R(pq) q, R(pk) k>,  O = softmax(score) V,  lse = ln sum exp
 *          -- bittide summary §3.2 / techwalker §四 (LogSumExp statistics).
 *
 * Decode (bittide summary §3.3; techwalker §三): the cache holds keys already
 * rotated at their original positions; the query is rotated at pos and then by
 * dq = f(pos) - pos; a remote cached key is rotated by dk = f(k) - k before the
 * dot product; local keys take no correction.
 *
 * RoPE convention (the pages do not state it): rotate-half pairs (i, i + D/2)
 * with frequency theta_i = base^(-2i/D), the convention of the Qwen3 models the
 * pages evaluate.  Angles are pos * theta_i in double precision.
 *
 * Inputs may be fp32, bf16 bit patterns (widened exactly) or fp64; every
 * computation is fp64.  Pinned by tests/test_oracle_pins.py (closed forms,
 * brute force with explicit rotation matrices and a materialised mask, the G=1
 * and w_local>=L reductions to library causal attention, the inclusion-exclusion
 * identity, rotation composition, the remote-distance bound, and the prefill /
 * decode agreement).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define JLO_F32 0
#define JLO_BF16 1
#define JLO_F64 2

/* Widen one stored element to double.  bf16 is the top half of an fp32. */
static double jlo_load(const void *base, int64_t idx, int dtype) {
  if (dtype == JLO_F32) return (double)((const float *)base)[idx];
  if (dtype == JLO_BF16) {
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return ((const double *)base)[idx];
}

/* G = max(1, ceil(L / w_pretrained)); returns -1 for non-positive inputs. */
long long jlo_group_size(long long L, long long w_pretrained) {
  if (L <= 0 || w_pretrained <= 0) return -1;
  long long g = (L + w_pretrained - 1) / w_pretrained;
  return g < 1 ? 1 : g;
}

/* f(x) = floor(x / G) for x >= 0. */
long long jlo_remap(long long x, long long G) { return x / G; }

/* theta_i = base^(-2i/D). */
double jlo_theta(int i, int D, double base) {
  return pow(base, -2.0 * (double)i / (double)D);
}

/* y = R(pos) x: pair (i, i + D/2) rotated by the angle pos * theta_i.
 * y may alias x. */
void jlo_rope(const double *x, double *y, int D, double pos, double base) {
  const int h = D / 2;
  for (int i = 0; i < h; ++i) {
    const double a = pos * jlo_theta(i, D, base);
    const double c = cos(a), s = sin(a);
    const double x1 = x[i], x2 = x[i + h];
    y[i] = x1 * c - x2 * s;
    y[i + h] = x1 * s + x2 * c;
  }
}

static double jlo_dot(const double *a, const double *b, int D) {
  double s = 0.0;
  for (int d = 0; d < D; ++d) s += a[d] * b[d];
  return s;
}

/* The local/remote predicate for a causal pair (k <= q). */
static int jlo_is_local(long long q, long long k, long long w_local) {
  return (q - k) < w_local;
}

/* Softmax of n scores against rows of V (row stride D): out = sum p_k V_k,
 * returns lse = ln sum exp(s_k). */
static double jlo_softmax_pv(const double *s, long long n, const double *V,
                             int D, double *out) {
  double M = -INFINITY;
  for (long long k = 0; k < n; ++k) M = s[k] > M ? s[k] : M;
  double Z = 0.0;
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (long long k = 0; k < n; ++k) {
    const double p = exp(s[k] - M);
    Z += p;
    const double *v = V + k * D;
    for (int d = 0; d < D; ++d) out[d] += p * v[d];
  }
  for (int d = 0; d < D; ++d) out[d] /= Z;
  return M + log(Z);
}

/*
 * Prefill rows.  q [B,L,Hq,D], k/v [B,L,Hkv,D], contiguous, element type
 * `dtype`.  The n_rows selected outputs are (row_b[r], row_q[r], row_h[r]);
 * out is [n_rows][D], lse [n_rows], both fp64.  scale <= 0 selects 1/sqrt(D).
 * Returns 0, or a negative code for invalid arguments.
 *
 * The rotated keys of one (batch, kv-head) are computed once and reused by all
 * selected rows of that head; this caches identical values and changes no
 * arithmetic of the per-pair definition.
 */
int jlo_bifocal_rows(const void *q, const void *k, const void *v, int dtype,
                     int B, int L, int Hq, int Hkv, int D, int w_local,
                     int w_pretrained, double rope_base, double scale,
                     int n_rows, const int *row_b, const int *row_q,
                     const int *row_h, double *out, double *lse) {
  if (!q || !k || !v || B < 1 || L < 1 || Hq < 1 || Hkv < 1 || D < 2 ||
      D > 1024 || (D % 2) || (Hq % Hkv) || w_local < 0 || w_pretrained < 1 ||
      n_rows < 0 || (n_rows && (!row_b || !row_q || !row_h || !out || !lse)))
    return -1;
  for (int r = 0; r < n_rows; ++r)
    if (row_b[r] < 0 || row_b[r] >= B || row_q[r] < 0 || row_q[r] >= L ||
        row_h[r] < 0 || row_h[r] >= Hq)
      return -2;
  if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
  const long long G = jlo_group_size(L, w_pretrained);
  const int group = Hq / Hkv;

  for (int b = 0; b < B; ++b) {
    for (int hk = 0; hk < Hkv; ++hk) {
      /* Rows of this (b, hk) and the largest query position among them. */
      int qmax = -1;
      for (int r = 0; r < n_rows; ++r)
        if (row_b[r] == b && row_h[r] / group == hk && row_q[r] > qmax)
          qmax = row_q[r];
      if (qmax < 0) continue;
      const long long nk = (long long)qmax + 1;
      double *kstd = (double *)malloc(sizeof(double) * nk * D);
      double *krem = (double *)malloc(sizeof(double) * nk * D);
      double *vd = (double *)malloc(sizeof(double) * nk * D);
      if (!kstd || !krem || !vd) {
        free(kstd); free(krem); free(vd);
        return -3;
      }
#pragma omp parallel for schedule(static)
      for (long long kk = 0; kk < nk; ++kk) {
        double raw[1024];
        const int64_t base = (((int64_t)b * L + kk) * Hkv + hk) * D;
        for (int d = 0; d < D; ++d) {
          raw[d] = jlo_load(k, base + d, dtype);
          vd[kk * D + d] = jlo_load(v, base + d, dtype);
        }
        jlo_rope(raw, kstd + kk * D, D, (double)kk, rope_base);
        jlo_rope(raw, krem + kk * D, D, (double)jlo_remap(kk, G), rope_base);
      }
      int err = 0;
#pragma omp parallel for schedule(dynamic, 1)
      for (int r = 0; r < n_rows; ++r) {
        if (row_b[r] != b || row_h[r] / group != hk) continue;
        const long long qp = row_q[r];
        double raw[1024], qs[1024], qr[1024];
        const int64_t qbase = (((int64_t)b * L + qp) * Hq + row_h[r]) * D;
        for (int d = 0; d < D; ++d) raw[d] = jlo_load(q, qbase + d, dtype);
        jlo_rope(raw, qs, D, (double)qp, rope_base);
        jlo_rope(raw, qr, D, (double)jlo_remap(qp, G), rope_base);
        double *s = (double *)malloc(sizeof(double) * (qp + 1));
        if (!s) {
#pragma omp atomic write
          err = 1;
          continue;
        }
        for (long long kk = 0; kk <= qp; ++kk) {
          if (jlo_is_local(qp, kk, w_local))
            s[kk] = scale * jlo_dot(qs, kstd + kk * D, D);
          else
            s[kk] = scale * jlo_dot(qr, krem + kk * D, D);
        }
        lse[r] = jlo_softmax_pv(s, qp + 1, vd, D, out + (int64_t)r * D);
        free(s);
      }
      free(kstd); free(krem); free(vd);
      if (err) return -3;
    }
  }
  return 0;
}

/*
 * Single-token decode.  q_new [B,Hq,D] is pre-RoPE at position pos; the caches
 * k_cache/v_cache are [B,cache_capacity,Hkv,D] with keys already rotated at
 * their original positions and slots 0..pos valid.  G follows from L = pos + 1.
 * out [B,Hq,D], lse [B,Hq] in fp64.  Returns 0 or a negative code.
 */
int jlo_bifocal_decode(const void *q_new, const void *k_cache,
                       const void *v_cache, int dtype, int B, int Hq, int Hkv,
                       int D, int pos, int cache_capacity, int w_local,
                       int w_pretrained, double rope_base, double scale,
                       double *out, double *lse) {
  if (!q_new || !k_cache || !v_cache || !out || !lse || B < 1 || Hq < 1 ||
      Hkv < 1 || D < 2 || D > 1024 || (D % 2) || (Hq % Hkv) || pos < 0 ||
      pos >= cache_capacity || w_local < 0 || w_pretrained < 1)
    return -1;
  if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
  const long long G = jlo_group_size((long long)pos + 1, w_pretrained);
  const int group = Hq / Hkv;
  const long long nk = (long long)pos + 1;
  const double dq = (double)(jlo_remap(pos, G) - pos);

  for (int b = 0; b < B; ++b) {
    for (int hk = 0; hk < Hkv; ++hk) {
      /* Corrected (remote) and uncorrected (local) cached keys of this head. */
      double *kc = (double *)malloc(sizeof(double) * nk * D);
      double *vd = (double *)malloc(sizeof(double) * nk * D);
      if (!kc || !vd) {
        free(kc); free(vd);
        return -3;
      }
#pragma omp parallel for schedule(static)
      for (long long kk = 0; kk < nk; ++kk) {
        const int64_t base = (((int64_t)b * cache_capacity + kk) * Hkv + hk) * D;
        double raw[1024];
        for (int d = 0; d < D; ++d) {
          raw[d] = jlo_load(k_cache, base + d, dtype);
          vd[kk * D + d] = jlo_load(v_cache, base + d, dtype);
        }
        if (jlo_is_local(pos, kk, w_local)) {
          for (int d = 0; d < D; ++d) kc[kk * D + d] = raw[d];
        } else {
          const double dk = (double)(jlo_remap(kk, G) - kk);
          jlo_rope(raw, kc + kk * D, D, dk, rope_base);
        }
      }
      for (int hh = 0; hh < group; ++hh) {
        const int h = hk * group + hh;
        double raw[1024], qs[1024], qr[1024];
        const int64_t qbase = ((int64_t)b * Hq + h) * D;
        for (int d = 0; d < D; ++d) raw[d] = jlo_load(q_new, qbase + d, dtype);
        jlo_rope(raw, qs, D, (double)pos, rope_base);
        jlo_rope(qs, qr, D, dq, rope_base);
        double *s = (double *)malloc(sizeof(double) * nk);
        if (!s) {
          free(kc); free(vd);
          return -3;
        }
#pragma omp parallel for schedule(static)
        for (long long kk = 0; kk < nk; ++kk)
          s[kk] = scale * jlo_dot(jlo_is_local(pos, kk, w_local) ? qs : qr,
                                  kc + kk * D, D);
        lse[(int64_t)b * Hq + h] =
            jlo_softmax_pv(s, nk, vd, D, out + ((int64_t)b * Hq + h) * D);
        free(s);
      }
      free(kc); free(vd);
    }
  }
  return 0;
}

/* Number of OpenMP threads the oracle runs with (1 without OpenMP). */
int jlo_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
