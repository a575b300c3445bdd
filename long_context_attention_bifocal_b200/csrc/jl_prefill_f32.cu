// jl_prefill_f32.cu -- bifocal prefill in full fp32 on the CUDA cores.
//
// Same definition as the tensor-core kernel (Jet-Long, techwalker explainer
// §二/§四; bittide paper summary §3.1-§3.2): a causal pair (q, k) with
// q - k < w_local scores <R(q)Q, R(k)K>, any farther pair <R(f(q))Q, R(f(k))K>
// with f(x) = floor(x/G); one online softmax over all keys of a row.  This path
// serves fp32 inputs, where TF32 tensor-core products would miss a 1e-4 error
// budget; it is a small-problem kernel, not a throughput path.
//
// One CTA per (batch, query head, 64-row query tile); thread r owns query row
// r.  Key tiles of 32 are rotated both ways into shared memory by the whole
// CTA; scores and the softmax use fp32 and expf.
#include <climits>

#include "jl_internal.h"

namespace jl {
namespace {

constexpr int kRows = 64;
constexpr int kKeys = 32;

template <int D>
__global__ void __launch_bounds__(kRows)
    bifocal_prefill_f32_kernel(const float *__restrict__ q, const float *__restrict__ k,
                               const float *__restrict__ v, float *__restrict__ out,
                               float *__restrict__ lse, const float2 *__restrict__ cs,
                               int L, int Hq, int Hkv, int G, int w, float scale) {
  constexpr int H2 = D / 2;
  extern __shared__ float sm[];
  float *qs = sm;                           // [kRows][D + 1]  R(q) Q
  float *qr = qs + kRows * (D + 1);         // [kRows][D + 1]  R(f(q)) Q
  float *ks = qr + kRows * (D + 1);         // [kKeys][D]      R(k) K
  float *kr = ks + kKeys * D;               // [kKeys][D]      R(f(k)) K
  float *vs = kr + kKeys * D;               // [kKeys][D]

  const int r = threadIdx.x;
  const int hq = blockIdx.y, b = blockIdx.z;
  const int hk = hq / (Hq / Hkv);
  const int q0 = blockIdx.x * kRows;
  const int qpos = q0 + r;
  const bool row_ok = qpos < L;

  {
    const float *src = q + ((static_cast<int64_t>(b) * L + (row_ok ? qpos : 0)) * Hq + hq) * D;
    const float2 *ts = cs + static_cast<int64_t>(row_ok ? qpos : 0) * H2;
    const float2 *tr = cs + static_cast<int64_t>(row_ok ? qpos / G : 0) * H2;
    for (int i = 0; i < H2; ++i) {
      const float x1 = row_ok ? src[i] : 0.f, x2 = row_ok ? src[i + H2] : 0.f;
      const float2 a = ts[i], c = tr[i];
      qs[r * (D + 1) + i] = x1 * a.x - x2 * a.y;
      qs[r * (D + 1) + i + H2] = x1 * a.y + x2 * a.x;
      qr[r * (D + 1) + i] = x1 * c.x - x2 * c.y;
      qr[r * (D + 1) + i + H2] = x1 * c.y + x2 * c.x;
    }
  }

  float o[D];
#pragma unroll
  for (int d = 0; d < D; ++d) o[d] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int last = min(L, q0 + kRows) - 1;  // largest valid query of the tile

  for (int k0 = 0; k0 <= last; k0 += kKeys) {
    __syncthreads();
    for (int idx = r; idx < kKeys * H2; idx += kRows) {
      const int kk = idx / H2, i = idx % H2;
      const int kp = k0 + kk;
      float x1 = 0.f, x2 = 0.f, v1 = 0.f, v2 = 0.f;
      float2 a = make_float2(1.f, 0.f), c = make_float2(1.f, 0.f);
      if (kp < L) {
        const int64_t base = ((static_cast<int64_t>(b) * L + kp) * Hkv + hk) * D;
        x1 = k[base + i];
        x2 = k[base + i + H2];
        v1 = v[base + i];
        v2 = v[base + i + H2];
        a = cs[static_cast<int64_t>(kp) * H2 + i];
        c = cs[static_cast<int64_t>(kp / G) * H2 + i];
      }
      ks[kk * D + i] = x1 * a.x - x2 * a.y;
      ks[kk * D + i + H2] = x1 * a.y + x2 * a.x;
      kr[kk * D + i] = x1 * c.x - x2 * c.y;
      kr[kk * D + i + H2] = x1 * c.y + x2 * c.x;
      vs[kk * D + i] = v1;
      vs[kk * D + i + H2] = v2;
    }
    __syncthreads();
    const int kend = min(kKeys, qpos - k0 + 1);  // causal: keys <= qpos
    for (int kk = 0; kk < kend; ++kk) {
      const int kp = k0 + kk;
      const bool local = (qpos - kp) < w;
      const float *qa = local ? qs + r * (D + 1) : qr + r * (D + 1);
      const float *kb = local ? ks + kk * D : kr + kk * D;
      float dot = 0.f;
#pragma unroll
      for (int d = 0; d < D; ++d) dot = fmaf(qa[d], kb[d], dot);
      const float s = dot * scale;
      if (s > m) {
        const float alpha = expf(m - s);
        l *= alpha;
#pragma unroll
        for (int d = 0; d < D; ++d) o[d] *= alpha;
        m = s;
      }
      const float pw = expf(s - m);
      l += pw;
#pragma unroll
      for (int d = 0; d < D; ++d) o[d] = fmaf(pw, vs[kk * D + d], o[d]);
    }
  }
  if (row_ok) {
    float *dst = out + ((static_cast<int64_t>(b) * L + qpos) * Hq + hq) * D;
    const float inv = 1.f / l;
#pragma unroll
    for (int d = 0; d < D; ++d) dst[d] = o[d] * inv;
    lse[(static_cast<int64_t>(b) * Hq + hq) * L + qpos] = m + logf(l);
  }
}

template <int D>
cudaError_t launch_d(const PrefillArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(float) * (2 * kRows * (D + 1) + 3 * kKeys * D);
  cudaError_t e = cudaFuncSetAttribute(bifocal_prefill_f32_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid((a.L + kRows - 1) / kRows, a.Hq, a.B);
  bifocal_prefill_f32_kernel<D><<<grid, kRows, smem, s>>>(
      static_cast<const float *>(a.q), static_cast<const float *>(a.k),
      static_cast<const float *>(a.v), static_cast<float *>(a.out), a.lse, a.table.cs, a.L,
      a.Hq, a.Hkv, a.G, a.w_eff, a.scale);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_f32(const PrefillArgs &a, cudaStream_t s) {
  if (a.D == 64) return launch_d<64>(a, s);
  if (a.D == 128) return launch_d<128>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace jl
