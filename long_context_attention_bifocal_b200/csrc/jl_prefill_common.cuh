// jl_prefill_common.cuh -- pieces shared by the two tensor-core prefill
// kernels: tile sizes, the pass schedule (the fused inclusion-exclusion merge
// of Jet-Long, techwalker explainer §四 / bittide paper summary §3.2), the
// 128-byte swizzle address, bounded waits and bf16 unpacking.
#pragma once

#include <climits>
#include <cstdint>

#include "jl_internal.h"
#include "jl_sm100.cuh"

namespace jl {
namespace prefill {

using namespace sm100;

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
constexpr int kHD = 128;  // head dim
constexpr uint32_t kTileBytes = kBM * kHD * 2;  // one 128x128 bf16 tile
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // 64 columns (128 B rows)
constexpr uint64_t kTimeoutNs = 1000000000ull;

enum : int { kStd = 0, kRem = 1 };
// Pass selection: the bifocal rule (every pair in its class), or only the
// local window with one RoPE class for every pair in it (the B and C calls of
// the unfused three-call formulation).
enum : int { kBandNone = 0, kBandStd = 1, kBandRem = 2 };
enum : int { kMaskNone = 0, kMaskFarOnly = 1, kMaskLocalOnly = 2 };

// The pass schedule of query tile i.  Kv tile j <= i is at tile distance
// d = i - j and spans pair distances [128d - 127, 128d + 127] (clipped at 0).
// It holds a remote pair iff 128d + 127 >= w and a local pair iff
// max(0, 128d - 127) < w.  The schedule runs two phases:
//   remote phase: tiles 0..a (those holding a remote pair), K_rem and Q_rem,
//                 masked to remote pairs where the tile also holds local ones;
//   local phase:  tiles b..i (those holding a local pair), K_std and Q_std,
//                 masked to local pairs where the tile also holds remote ones.
// A tile straddling the window edge is visited once in each phase under
// complementary masks; the diagonal tile also takes the causal mask.  The
// online softmax does not depend on the order, and putting every remote pass
// first lets a CTA keep one Q variant at a time.
struct PassIter {
  int i, w;      // query tile, local window (INT_MAX: every pair local)
  int a, b;      // last tile with a remote pair (-1: none), first with a local pair
  int phase;     // kRem, then kStd
  int j;         // current kv tile
  int band;      // kBandNone, or only the local passes with one class

  __device__ void begin(int qi, int wl, int band_mode = kBandNone) {
    band = band_mode;
    i = qi;
    w = wl;
    // smallest d with 128d + 127 >= w
    const long long dmin = wl <= 127 ? 0 : (static_cast<long long>(wl) - 127 + kBN - 1) / kBN;
    a = dmin > qi ? -1 : qi - static_cast<int>(dmin);
    // largest d with 128d - 127 < w (none if w == 0)
    if (wl <= 0) {
      b = qi + 1;
    } else {
      const long long dmax = (static_cast<long long>(wl) + 126) / kBN;
      b = dmax >= qi ? 0 : qi - static_cast<int>(dmax);
    }
    if (a >= 0 && band == kBandNone) {
      phase = kRem;
      j = 0;
    } else {
      phase = kStd;
      j = b;
    }
  }
  __device__ bool done() const { return phase == kStd && j > i; }
  __device__ int kind() const {
    return band == kBandNone ? phase : (band == kBandStd ? kStd : kRem);
  }
  __device__ int mask() const {
    if (phase == kRem) return j >= b ? kMaskFarOnly : kMaskNone;
    return j <= a ? kMaskLocalOnly : kMaskNone;
  }
  __device__ void next() {
    ++j;
    if (phase == kRem && j > a) {
      phase = kStd;
      j = b;
    }
  }
};

// byte offset of 16-byte chunk `chunk` of row `row` in a 128-byte-swizzled
// [rows][128 B] tile (TMA SWIZZLE_128B and the UMMA descriptors agree on it)
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void raise_abort(volatile int *abort_s, unsigned *status) {
  *abort_s = 1;
  atomicOr(status, kStatusTimeout);
}

// Wait used while draining: only the time limit ends it.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kTimeoutNs) break;
  }
}

// mbar_wait for the softmax warps: the result is made uniform across the warp,
// because the tcgen05.ld/st that follow a wait are warp-collective
// (.sync.aligned) and must never run with part of the warp.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity,
                                          const volatile int *abort_s,
                                          const volatile unsigned *abort_g) {
  const bool ok = mbar_wait(bar, parity, abort_s, abort_g, kTimeoutNs);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void unpack8(const uint4 &u, float (&x)[8]) {
  const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[2 * j] = __uint_as_float(w4[j] << 16);
    x[2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
  }
}

// Where the keys come from: raw (pre-RoPE) keys, rotated here to R(k) for the
// local passes and to R(f(k)) for the remote ones; or a cache whose keys are
// already rotated at their original positions, used as they are by the local
// passes and moved to f(k) by R(f(k) - k) for the remote ones (techwalker
// explainer §三: rotations compose, R(a) R(b) = R(a + b)).
enum : int { kKeysRaw = 0, kKeysCached = 1 };

// Rotates a 128-key tile in shared memory, in place, for a pass of class
// `kind` (kStd / kRem) over keys k0 .. k0 + 127, bf16 in the 128-byte-swizzled
// K-major layout the TMA wrote: dims 0-63 in the first 16 KB half, 64-127 in
// the second, pair (i, i + 64) at the same offset of the two halves.  The
// `nthr` threads calling it (thread index `tid`) split the 128 x 8 chunks of
// eight pairs between them; a thread's lanes of one warp take four rows of
// eight chunks, so table reads and shared-memory accesses stay contiguous.
// Rows at or past n_keys (zero fill beyond the sequence) are left alone.
// Arithmetic: fp32 with the fp32 table value of (cos, sin)(p theta_i), one
// rounding to bf16 at the end.
__device__ __forceinline__ void rotate_k_tile(uint8_t *tile, int k0, int kind, int key_mode,
                                              int G, int n_keys, const float2 *cs, int tid,
                                              int nthr) {
  if (key_mode == kKeysCached && kind == kStd) return;  // already at original positions
#pragma unroll 1
  for (int item = tid; item < kBN * 8; item += nthr) {
    const int r = item >> 3, c = item & 7;
    const int k = k0 + r;
    if (k >= n_keys) continue;
    int p;
    float sgn = 1.f;
    if (key_mode == kKeysRaw) {
      p = kind == kStd ? k : k / G;
    } else {
      p = k - k / G;  // R(f(k) - k) = R(-u): the table row u with the sine negated
      sgn = -1.f;
    }
    uint4 *a1 = reinterpret_cast<uint4 *>(tile + swz(r, c));
    uint4 *a2 = reinterpret_cast<uint4 *>(tile + kHalfBytes + swz(r, c));
    float x1[8], x2[8];
    unpack8(*a1, x1);
    unpack8(*a2, x2);
    const float4 *t = reinterpret_cast<const float4 *>(cs + static_cast<int64_t>(p) * 64 + 8 * c);
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float4 r2 = __ldg(t + e);  // (cos, sin) of pairs 2e and 2e + 1
      const float s0 = sgn * r2.y, s1 = sgn * r2.w;
      lo[e] = pack_bf16x2(x1[2 * e] * r2.x - x2[2 * e] * s0,
                          x1[2 * e + 1] * r2.z - x2[2 * e + 1] * s1);
      hi[e] = pack_bf16x2(x1[2 * e] * s0 + x2[2 * e] * r2.x,
                          x1[2 * e + 1] * s1 + x2[2 * e + 1] * r2.z);
    }
    *a1 = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    *a2 = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  }
}

// 2^x on the FMA/ALU pipes instead of the MUFU unit, for x <= 8:
// 2^floor(x) * p(x - floor(x)) with a cubic p fitted by weighted least squares
// on Chebyshev nodes with p(0) = 1 and p(1) = 2 (derive_exp2_poly.py; maximum
// relative error 1.1e-4, below the bf16 rounding of P that follows).
// floor(x) comes from one round-down add of 1.5 * 2^23, after which the low
// mantissa bits hold floor(x) as an integer -- no float-to-int conversion.
// Inputs below -127 are clamped (the result is then below 2^-126).
__device__ __forceinline__ float exp2_poly(float x) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  x = fmaxf(x, -127.f);
  const float t = __fadd_rd(x, kMagic);  // kMagic + floor(x), exact
  const float f = x - (t - kMagic);      // fraction in [0, 1)
  const int e = __float_as_int(t) - __float_as_int(kMagic);  // floor(x)
  float p = fmaf(0.07816384732723236f, f, 0.22644174098968506f);
  p = fmaf(p, f, 0.6953943967819214f);
  p = fmaf(p, f, 1.0f);
  return __int_as_float(__float_as_int(p) + static_cast<int>(static_cast<unsigned>(e) << 23));
}

// The same 2^x on a pair of fp32 values with packed fp32 arithmetic: clamp,
// one round-down add for floor, the cubic in three packed FMAs, and the
// exponent added to the bits of each result.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  const uint64_t kMagic2 = 0x4B4000004B400000ull;  // (1.5 * 2^23, 1.5 * 2^23)
  float x0, x1;
  sm100::f2_unpack(x2, x0, x1);
  x2 = sm100::f2_pack(fmaxf(x0, -127.f), fmaxf(x1, -127.f));
  const uint64_t t2 = sm100::f2_add_rd(x2, kMagic2);  // magic + floor(x), exact
  const uint64_t f2 = sm100::f2_sub(x2, sm100::f2_sub(t2, kMagic2));
  // the cubic's coefficients as fp32 bit patterns, one copy per half
  uint64_t p2 = sm100::f2_fma(0x3DA0145E3DA0145Eull, f2, 0x3E67E0583E67E058ull);
  p2 = sm100::f2_fma(p2, f2, 0x3F32055E3F32055Eull);
  p2 = sm100::f2_fma(p2, f2, 0x3F8000003F800000ull);
  // magic's low bits are zero, so (t << 23) is floor(x) << 23 modulo 2^32
  const uint32_t t_lo = static_cast<uint32_t>(t2), t_hi = static_cast<uint32_t>(t2 >> 32);
  const uint32_t p_lo = static_cast<uint32_t>(p2), p_hi = static_cast<uint32_t>(p2 >> 32);
  return (static_cast<uint64_t>(p_hi + (t_hi << 23)) << 32) | (p_lo + (t_lo << 23));
}

}  // namespace prefill
}  // namespace jl
