// jl_merge.cu -- the LogSumExp merge of the unfused three-call formulation of
// the bifocal prefill (bittide paper summary §3.2; techwalker explainer §四).
//
// The three calls are A = causal attention at remapped positions over every
// pair, B = the local window at original positions, C = the local window at
// remapped positions.  With unnormalised sums weighted by e^lse,
//   O = (e^lA O_A + e^lB O_B - e^lC O_C) / (e^lA + e^lB - e^lC),
//   lse = ln(e^lA + e^lB - e^lC),
// which equals attention with the per-pair rule.  Weights are taken relative
// to the largest of the three statistics; an empty window (lse = -inf) gives
// weight 0 and its output is not read.
#include "jl_internal.h"

namespace jl {
namespace {

constexpr int kD = 128;

// One warp per (batch, head, row); lane = 4 consecutive dims (8 bytes of bf16).
__global__ void __launch_bounds__(256)
    lse_merge_kernel(__nv_bfloat16 *__restrict__ out, float *__restrict__ lse,
                     const __nv_bfloat16 *__restrict__ ob, const float *__restrict__ lb,
                     const __nv_bfloat16 *__restrict__ oc, const float *__restrict__ lc,
                     int B, int L, int Hq) {
  const int64_t rows = static_cast<int64_t>(B) * Hq * L;
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const int l = static_cast<int>(r % L);
  const int h = static_cast<int>((r / L) % Hq);
  const int b = static_cast<int>(r / (static_cast<int64_t>(L) * Hq));
  const float la = lse[r], lbv = lb[r], lcv = lc[r];
  const float M = fmaxf(la, fmaxf(lbv, lcv));
  const float wa = expf(la - M);
  const float wb = lbv == -INFINITY ? 0.f : expf(lbv - M);
  const float wc = lcv == -INFINITY ? 0.f : expf(lcv - M);
  const float den = wa + wb - wc;
  const int64_t o = ((static_cast<int64_t>(b) * L + l) * Hq + h) * kD + 4 * lane;
  float acc[4];
  {
    const uint2 ua = *reinterpret_cast<const uint2 *>(out + o);
    const __nv_bfloat162 a0 = *reinterpret_cast<const __nv_bfloat162 *>(&ua.x);
    const __nv_bfloat162 a1 = *reinterpret_cast<const __nv_bfloat162 *>(&ua.y);
    acc[0] = wa * __low2float(a0);
    acc[1] = wa * __high2float(a0);
    acc[2] = wa * __low2float(a1);
    acc[3] = wa * __high2float(a1);
  }
  if (wb != 0.f) {
    const uint2 u = *reinterpret_cast<const uint2 *>(ob + o);
    const __nv_bfloat162 x0 = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
    const __nv_bfloat162 x1 = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
    acc[0] += wb * __low2float(x0);
    acc[1] += wb * __high2float(x0);
    acc[2] += wb * __low2float(x1);
    acc[3] += wb * __high2float(x1);
  }
  if (wc != 0.f) {
    const uint2 u = *reinterpret_cast<const uint2 *>(oc + o);
    const __nv_bfloat162 x0 = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
    const __nv_bfloat162 x1 = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
    acc[0] -= wc * __low2float(x0);
    acc[1] -= wc * __high2float(x0);
    acc[2] -= wc * __low2float(x1);
    acc[3] -= wc * __high2float(x1);
  }
  const float inv = 1.f / den;
  __nv_bfloat162 y0 = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
  __nv_bfloat162 y1 = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
  uint2 w;
  w.x = *reinterpret_cast<uint32_t *>(&y0);
  w.y = *reinterpret_cast<uint32_t *>(&y1);
  *reinterpret_cast<uint2 *>(out + o) = w;
  if (lane == 0) lse[r] = M + logf(den);
}

}  // namespace

cudaError_t launch_lse_merge(__nv_bfloat16 *out, float *lse, const __nv_bfloat16 *ob,
                             const float *lb, const __nv_bfloat16 *oc, const float *lc, int B,
                             int L, int Hq, cudaStream_t s) {
  const int64_t threads = static_cast<int64_t>(B) * Hq * L * 32;
  const int64_t blocks = (threads + 255) / 256;
  if (blocks >= (1LL << 31)) return cudaErrorInvalidValue;
  lse_merge_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(out, lse, ob, lb, oc, lc, B, L,
                                                                 Hq);
  return cudaGetLastError();
}

}  // namespace jl
