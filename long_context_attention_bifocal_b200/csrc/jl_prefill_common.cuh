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
// The third mode, kKeysRotated, takes both rotated copies from memory (the
// opt-in pass that rotates every key once per call): the kernels rotate
// nothing and read the copy of the pass's class.
enum : int { kKeysRaw = 0, kKeysCached = 1, kKeysRotated = 2 };

// In-place rotation of part of a 128-key tile in shared memory (bf16, the
// 128-byte-swizzled K-major layout the TMA wrote: dims 0-63 in the first
// 16 KB half, 64-127 in the second, so pair (i, i + 64) sits at the same
// offset of the two halves) to the positions of a pass.
//
// One thread's slice: the eight pairs 8c .. 8c + 7 (one 16-byte chunk of each
// half) of four consecutive keys kl .. kl + 3 of the tile.  Their positions p
// advance by 0 or 1 per key (k, floor(k / G), or k - floor(k / G) for a cache
// at original positions), so the table is read once, at the first key, and
// the factors then move on by R(p + 1) = R(p) R(1) (a complex multiplication
// with row 1 of the table, kept in shared memory as `step`: 32 float4, entry
// 8 e2 + c holding (cos, sin) of theta for pairs 8c + 2 e2 and 8c + 2 e2 + 1)
// where p advances.
// All four keys' words are loaded before any is rotated, so one shared-memory
// latency covers the slice.  Arithmetic in fp32, one rounding to bf16.
struct KeySlice {
  int c;   // chunk of pairs
  int kl;  // first key of the slice within the tile

  // position of key k in a pass of class `kind`; -1 when the keys are used as
  // they are (cached keys in a local pass)
  static __device__ __forceinline__ int position(int k, int kind, int key_mode, int G) {
    if (key_mode == kKeysRaw) return kind == kStd ? k : k / G;
    if (key_mode == kKeysRotated) return -1;
    return kind == kStd ? -1 : k - k / G;
  }

  // pulls the slice's table entries into L1 ahead of rotate()
  __device__ void prefetch(const float2 *cs, int k0, int kind, int key_mode, int G,
                           int n_keys) const {
    const int k = k0 + kl;
    if (k >= n_keys) return;
    const int p = position(k, kind, key_mode, G);
    if (p < 0) return;
    asm volatile("prefetch.global.L1 [%0];" ::"l"(cs + static_cast<int64_t>(p) * 64 + 8 * c));
  }

  __device__ void rotate(uint8_t *tile, const float2 *cs, const float2 *step, int k0, int kind,
                         int key_mode, int G, int n_keys) const {
    const int k = k0 + kl;
    const int rows = min(4, n_keys - k);
    if (rows <= 0) return;
    const int p = position(k, kind, key_mode, G);
    if (p < 0) return;
    const bool cached = key_mode == kKeysCached;
    const bool every = key_mode == kKeysRaw && kind == kStd;  // p = k: a step per key
    const float sg = cached ? -1.f : 1.f;  // R(-u) for the cached keys' correction
    uint4 w1[4], w2[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (u < rows) {
        const uint32_t off = swz(kl + u, c);
        w1[u] = *reinterpret_cast<const uint4 *>(tile + off);
        w2[u] = *reinterpret_cast<const uint4 *>(tile + kHalfBytes + off);
      }
    }
    float cf[8], sf[8];
    {
      const float4 *t = reinterpret_cast<const float4 *>(cs + static_cast<int64_t>(p) * 64 + 8 * c);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 v = __ldg(t + e);
        cf[2 * e] = v.x;
        sf[2 * e] = sg * v.y;
        cf[2 * e + 1] = v.z;
        sf[2 * e + 1] = sg * v.w;
      }
    }
    int m = k % G;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (u < rows) {
        const uint32_t a1[4] = {w1[u].x, w1[u].y, w1[u].z, w1[u].w};
        const uint32_t a2[4] = {w2[u].x, w2[u].y, w2[u].z, w2[u].w};
        uint32_t o1[4], o2[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float x1a = __uint_as_float(a1[q] << 16), x1b = __uint_as_float(a1[q] & 0xFFFF0000u);
          const float x2a = __uint_as_float(a2[q] << 16), x2b = __uint_as_float(a2[q] & 0xFFFF0000u);
          const int e = 2 * q;
          o1[q] = sm100::pack_bf16x2(fmaf(x1a, cf[e], -x2a * sf[e]),
                                     fmaf(x1b, cf[e + 1], -x2b * sf[e + 1]));
          o2[q] = sm100::pack_bf16x2(fmaf(x1a, sf[e], x2a * cf[e]),
                                     fmaf(x1b, sf[e + 1], x2b * cf[e + 1]));
        }
        const uint32_t off = swz(kl + u, c);
        *reinterpret_cast<uint4 *>(tile + off) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
        *reinterpret_cast<uint4 *>(tile + kHalfBytes + off) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
        // next key: k mod G, and whether its position moves on (f grows at
        // multiples of G; u = k - f everywhere else)
        m = (m + 1 == G) ? 0 : m + 1;
        if (u + 1 < rows && (every || (cached ? (m != 0) : (m == 0)))) {
          const float4 *st4 = reinterpret_cast<const float4 *>(step);
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            // (cos, sin)(theta) of pairs 8c + 2 e2, 8c + 2 e2 + 1; the table is
            // stored e2-major, so the eight chunks of one e2 are 128
            // contiguous bytes (one conflict-free wavefront for a warp)
            const float4 v = st4[8 * e2 + c];
            const float c1[2] = {v.x, v.z}, s1[2] = {sg * v.y, sg * v.w};
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int e = 2 * e2 + h;
              const float cn = fmaf(cf[e], c1[h], -sf[e] * s1[h]);
              sf[e] = fmaf(cf[e], s1[h], sf[e] * c1[h]);
              cf[e] = cn;
            }
          }
        }
      }
    }
  }
};

// The same rotation by NTHR dedicated threads (a multiple of 16) over a whole
// tile: thread t owns four pairs i0 .. i0 + 3 (i0 = 4 * (t % 16)), one 8-byte
// word of each half, of kRows = 128 * 16 / NTHR consecutive keys, moving its
// factors on by the step table as KeySlice does and loading the next key's
// words before rotating the current one.
template <int NTHR>
struct KeyRotator {
  static constexpr int kRows = kBN * 16 / NTHR;
  // (cos, sin)(theta_i) of the thread's pairs, two per float4: the step table
  // holds 32 float4, entry q = pairs 4q, 4q + 1 and entry 16 + q = pairs
  // 4q + 2, 4q + 3, so that sixteen threads' first (or second) halves are 256
  // contiguous bytes (conflict-free)
  const float4 *step;
  int i0;              // first pair of this thread
  int kb;              // first key of the thread's block within a tile

  __device__ void init(const float2 *step_smem, int tid) {
    i0 = 4 * (tid & 15);
    kb = kRows * (tid >> 4);
    step = reinterpret_cast<const float4 *>(step_smem) + (tid & 15);
  }

  struct Start {
    float4 a, b;
    int m;      // k mod G of the first key
    int rows;   // keys of the block to rotate (0: none)
  };
  // the block's first position and its table entries, read ahead of the wait
  // for the tile
  __device__ Start start(const float2 *cs, int k0, int kind, int key_mode, int G,
                         int n_keys) const {
    Start st;
    const int k = k0 + kb;
    const int p = k < n_keys ? KeySlice::position(k, kind, key_mode, G) : -1;
    st.rows = p < 0 ? 0 : min(kRows, n_keys - k);
    st.m = k % G;
    const float4 *t =
        reinterpret_cast<const float4 *>(cs + static_cast<int64_t>(p < 0 ? 0 : p) * 64 + i0);
    st.a = __ldg(t);
    st.b = __ldg(t + 1);
    return st;
  }

  __device__ void rotate(uint8_t *tile, const Start &st, int kind, int key_mode, int G) const {
    if (st.rows <= 0) return;
    const bool cached = key_mode == kKeysCached;
    const bool every = key_mode == kKeysRaw && kind == kStd;
    const float sg = cached ? -1.f : 1.f;
    float c[4] = {st.a.x, st.a.z, st.b.x, st.b.z};
    float s[4] = {sg * st.a.y, sg * st.a.w, sg * st.b.y, sg * st.b.w};
    const int c_off = i0 >> 3, h_off = (i0 & 4) * 2;  // 16-byte chunk, 8-byte half
    int m = st.m;
    uint32_t off = swz(kb, c_off) + h_off;
    uint2 w1 = *reinterpret_cast<const uint2 *>(tile + off);
    uint2 w2 = *reinterpret_cast<const uint2 *>(tile + kHalfBytes + off);
#pragma unroll 1
    for (int n = 0; n < st.rows; ++n) {
      const uint32_t noff = swz(kb + n + 1, c_off) + h_off;
      uint2 n1 = w1, n2 = w2;
      if (n + 1 < st.rows) {
        n1 = *reinterpret_cast<const uint2 *>(tile + noff);
        n2 = *reinterpret_cast<const uint2 *>(tile + kHalfBytes + noff);
      }
      const float x1[4] = {__uint_as_float(w1.x << 16), __uint_as_float(w1.x & 0xFFFF0000u),
                           __uint_as_float(w1.y << 16), __uint_as_float(w1.y & 0xFFFF0000u)};
      const float x2[4] = {__uint_as_float(w2.x << 16), __uint_as_float(w2.x & 0xFFFF0000u),
                           __uint_as_float(w2.y << 16), __uint_as_float(w2.y & 0xFFFF0000u)};
      float y1[4], y2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        y1[e] = fmaf(x1[e], c[e], -x2[e] * s[e]);
        y2[e] = fmaf(x1[e], s[e], x2[e] * c[e]);
      }
      *reinterpret_cast<uint2 *>(tile + off) =
          make_uint2(sm100::pack_bf16x2(y1[0], y1[1]), sm100::pack_bf16x2(y1[2], y1[3]));
      *reinterpret_cast<uint2 *>(tile + kHalfBytes + off) =
          make_uint2(sm100::pack_bf16x2(y2[0], y2[1]), sm100::pack_bf16x2(y2[2], y2[3]));
      m = (m + 1 == G) ? 0 : m + 1;
      if (every || (cached ? (m != 0) : (m == 0))) {
        const float4 t01 = step[0], t23 = step[16];
        const float c1[4] = {t01.x, t01.z, t23.x, t23.z};
        const float s1[4] = {t01.y, t01.w, t23.y, t23.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float sd = sg * s1[e];
          const float cn = fmaf(c[e], c1[e], -s[e] * sd);
          s[e] = fmaf(c[e], sd, s[e] * c1[e]);
          c[e] = cn;
        }
      }
      off = noff;
      w1 = n1;
      w2 = n2;
    }
  }
};

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
