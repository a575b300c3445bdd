// jl_rope.cu -- the RoPE angle table.
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

}  // namespace

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
