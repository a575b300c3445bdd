// jl_rope.cu -- the RoPE angle table, and the prefill's opt-in pass that
// rotates every key once per call.
//
// RoPE (rotate-half pairs (i, i + D/2), theta_i = base^(-2i/D)) is the position
// encoding both windows use; the remote window evaluates it at f(x) = floor(x/G)
// (Jet-Long, bittide paper summary §3.1).  Rotations compose, R(a)R(b) = R(a+b)
// (techwalker explainer §三), which is what lets every rotation of the library
// (queries and keys in the prefill kernels, the decode's corrections) come from
// one table of angles p * theta_i.
#include "jl_internal.h"

namespace jl {

namespace {

struct Thetas {
  double t[128];  // theta_i for i < D/2 (D <= 256)
};

// cs[p * half + i] = (cos(p theta_i), sin(p theta_i)): the angle and its sine
// and cosine in fp64, rounded once to fp32.
__global__ void rope_table_kernel(float2 *__restrict__ cs, int positions, int half,
                                  const Thetas th) {
  const int64_t n = static_cast<int64_t>(positions) * half;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int p = static_cast<int>(idx / half);
    const int i = static_cast<int>(idx - static_cast<int64_t>(p) * half);
    double s, c;
    sincos(static_cast<double>(p) * th.t[i], &s, &c);
    cs[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[2 * j] = __uint_as_float(w[j] << 16);
    x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// The opt-in "rotate the keys once" mode of the prefill: both rotated copies
// of every key, kstd = R(l) k and krem = R(floor(l / G)) k (either may be
// skipped), written once per call so that the attention kernel streams them
// instead of rotating each K tile per pass.  One thread per (key row, chunk
// of eight pairs): dims [8c, 8c + 8) and [half + 8c, half + 8c + 8).
__global__ void rotate_keys_kernel(const __nv_bfloat16 *__restrict__ k,
                                   __nv_bfloat16 *__restrict__ kstd,
                                   __nv_bfloat16 *__restrict__ krem,
                                   const float2 *__restrict__ cs, int64_t rows, int L,
                                   int Hkv, int D, int G) {
  const int half = D / 2;
  const int chunks = half / 8;
  const int64_t n = rows * chunks;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = idx / chunks;  // (b, l, h) flattened
    const int c = static_cast<int>(idx - row * chunks);
    const int l = static_cast<int>((row / Hkv) % L);
    const int64_t base = row * D + 8 * c;
    float x1[8], x2[8];
    unpack8(*reinterpret_cast<const uint4 *>(k + base), x1);
    unpack8(*reinterpret_cast<const uint4 *>(k + base + half), x2);
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      __nv_bfloat16 *dst = pass == 0 ? kstd : krem;
      if (dst == nullptr) continue;
      const int p = pass == 0 ? l : l / G;
      const float2 *t = cs + static_cast<int64_t>(p) * half + 8 * c;
      uint32_t o1[4], o2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 r0 = __ldg(t + 2 * e), r1 = __ldg(t + 2 * e + 1);
        o1[e] = pack2(x1[2 * e] * r0.x - x2[2 * e] * r0.y,
                      x1[2 * e + 1] * r1.x - x2[2 * e + 1] * r1.y);
        o2[e] = pack2(x1[2 * e] * r0.y + x2[2 * e] * r0.x,
                      x1[2 * e + 1] * r1.y + x2[2 * e + 1] * r1.x);
      }
      *reinterpret_cast<uint4 *>(dst + base) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
      *reinterpret_cast<uint4 *>(dst + base + half) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
    }
  }
}

}  // namespace

cudaError_t launch_rotate_keys(const __nv_bfloat16 *k, __nv_bfloat16 *kstd,
                               __nv_bfloat16 *krem, RopeTable t, int B, int L,
                               int Hkv, int D, int G, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(B) * L * Hkv;
  const int64_t n = rows * (D / 16);
  const int threads = 256;
  const int64_t want = (n + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  const int blocks = static_cast<int>(want < cap ? want : cap);
  rotate_keys_kernel<<<blocks, threads, 0, s>>>(k, kstd, krem, t.cs, rows, L, Hkv, D, G);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float2 *cs, int positions, int D, double base, cudaStream_t s) {
  Thetas th;
  const int half = D / 2;
  for (int i = 0; i < half; ++i) th.t[i] = pow(base, -2.0 * i / D);
  const int64_t n = static_cast<int64_t>(positions) * half;
  const int threads = 256;
  const int64_t blocks64 = (n + threads - 1) / threads;
  const int blocks = static_cast<int>(blocks64 < 65536 ? blocks64 : 65536);
  rope_table_kernel<<<blocks, threads, 0, s>>>(cs, positions, half, th);
  return cudaGetLastError();
}

}  // namespace jl
