// jl_decode_mma.cu -- single-token bifocal decode, TMA-staged and on the
// tensor cores (Jet-Long, techwalker explainer §三; bittide paper summary §3.3).
//
// What it computes is the decode of jl_decode.cu: q_std = R(pos) q and
// q_rem = R(dq) q_std (dq = f(pos) - pos, f(x) = floor(x/G), G from L = pos+1);
// a cached key k_c = R(k) K with pos - k < w_local is scored as is against
// q_std; a farther key is corrected in registers to R(dk) k_c (dk = f(k) - k)
// and scored against q_rem.  Softmax over all keys of the cache.
//
// B200 layout.  A CTA owns one chunk of keys (wholly remote or wholly local)
// of one batch entry and ALL kv heads; one consumer warp per kv head, one
// producer warp.  The producer streams 16-key blocks through a 3-stage ring in
// shared memory with TMA: per block and head, K and V as two 64-column boxes
// with the 128-byte swizzle (so ldmatrix reads are conflict-free).  For a
// remote chunk the producer warp also writes the 16 rows of correction factors
// (cos, sin)(u theta_i) that the block needs, u = k - f(k) growing by at most
// one per key: row u0 + r is the complex product of the fp32 table row u0 (one
// 512-byte read per block) and the step row r < 16 (held in registers), rounded
// to fp16 (the rotated key is rounded to bf16 anyway, so the 2^-11 factor
// rounding does not show).  So the corrections read no per-key data from HBM.
// The tensor maps end at key pos, so slots past pos read as zeros and are never
// touched.
//
// Consumer warp (kv head h, its group of g <= 16 query heads as the 16 rows of
// an m16n8k16 bf16 MMA):
//   S^T[head][key] = Q . K^T      8 k-steps x 2 key tiles, Q fragments held
//                                 in registers (pre-rotated, pre-scaled)
//   K fragments (ldmatrix) of a remote key are rotated by -u*theta_i in fp32:
//   pair (i, i+64) lives in k-steps ks and ks+4 of the same thread, the factor
//   (cos, sin)(u theta_i) is read from the staged table row.
//   online softmax per query row (fp32, base 2, rescale only when the running
//   max grows by more than 2^8), P packed straight from the S accumulators
//   into the A fragments of O += P . V (V fragments by ldmatrix.trans).
// Each warp writes (o, m, l) of its heads for the chunk; the combine kernel of
// jl_decode.cu merges the chunks.  Waits are bounded; a timeout raises the
// device status word and the kernel returns.
#include <cudaTypedefs.h>

#include <climits>
#include <mutex>

#include "jl_internal.h"
#include "jl_sm100.cuh"

namespace jl {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kHalf = 64;
constexpr int kBlock = 16;            // keys per stage
constexpr int kStages = 3;
constexpr int kMaxHeads = 8;          // kv heads per CTA (one consumer warp each)
constexpr int kMaxGroup = 16;         // query heads per kv head (MMA rows)
constexpr int kThreads = (kMaxHeads + 2) * 32;
constexpr int kProducerWarp = kMaxHeads;
constexpr int kFactorWarp = kMaxHeads + 1;
constexpr uint32_t kHalfTile = kBlock * 128;          // one 64-column box: 2 KiB
constexpr uint32_t kHeadBytes = 2 * kHalfTile;        // K (or V) of one head: 4 KiB
constexpr uint32_t kKBytes = kMaxHeads * kHeadBytes;  // 32 KiB
constexpr uint32_t kTabBox = kBlock * 128;            // 16 rows x 32 fp16 pairs: 2 KiB
constexpr uint32_t kTabBytes = 2 * kTabBox;           // pairs 0-31 | 32-63: 4 KiB
constexpr uint32_t kStageBytes = 2 * kKBytes + kTabBytes;
constexpr uint32_t kOffBar = kStages * kStageBytes;
constexpr uint32_t kSmemAlloc = kOffBar + 64 + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr int kCtaTarget = 148;  // one wave of CTAs on a B200 per batch entry

struct Params {
  const __nv_bfloat16 *q;
  const float2 *cs;  // cos/sin table: query rotation, correction factors
  float *ws;
  unsigned *status;
  int Hq, Hkv, group, pos, G, far_end, chunk, n_far, n_chunks;
  float scale_log2;
  int skip_first_arrival;  // test-only: withhold the first block (bounded-wait check)
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                        uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1,
                                          uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma16816(float *d, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// byte offset of 16-byte chunk `ch` (0..15 over the 128 dims) of key row `row`
// in a head's [2 halves][16 keys][128 B] swizzled tile
__device__ __forceinline__ uint32_t tile_off(int row, int ch) {
  return static_cast<uint32_t>((ch >> 3) * kHalfTile + row * 128 + (((ch & 7) ^ (row & 7)) << 4));
}

__device__ __forceinline__ bool warp_wait_u(uint32_t bar, uint32_t parity,
                                            const volatile int *abort_s,
                                            const volatile unsigned *abort_g) {
  const bool ok = mbar_wait(bar, parity, abort_s, abort_g, kTimeoutNs);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(kThreads, 1)
    bifocal_decode_mma_kernel(const __grid_constant__ CUtensorMap tm_k,
                              const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = blockIdx.x, b = blockIdx.y;
  const bool far = c < p.n_far;
  int k_begin, k_end;
  if (far) {
    k_begin = c * p.chunk;
    k_end = min(p.far_end, k_begin + p.chunk);
  } else {
    k_begin = p.far_end + (c - p.n_far) * p.chunk;
    k_end = min(p.pos + 1, k_begin + p.chunk);
  }
  const int nblk = (k_end - k_begin + kBlock - 1) / kBlock;

  auto bar = [&](int i) { return sb + kOffBar + 8u * static_cast<uint32_t>(i); };
  // barriers: full[kStages] (the producer's arrival with the TMA bytes, plus,
  // in a remote chunk, the 32 lanes of the factor warp), empty[kStages] (one
  // arrival per consumer warp); then the abort flag
  volatile int *abort_s = reinterpret_cast<volatile int *>(smem + kOffBar + 8 * 2 * kStages);
  volatile unsigned *abort_g = p.status;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(s), far ? 33 : 1);
      mbar_init(bar(kStages + s), p.Hkv);
    }
    *abort_s = (*abort_g != 0u) ? 1 : 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (*abort_s) return;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const uint32_t bytes = static_cast<uint32_t>(p.Hkv) * 2 * kHeadBytes;
      int issued = 0;
      // test-only: no block is loaded, so the consumers' first wait expires
      for (int blk = p.skip_first_arrival ? nblk : 0; blk < nblk; ++blk) {
        const int s = blk % kStages;
        const uint32_t ph = (blk / kStages) & 1;
        if (!mbar_wait(bar(kStages + s), ph ^ 1u, abort_s, abort_g, kTimeoutNs)) {
          *abort_s = 1;
          atomicOr(p.status, kStatusTimeout);
          break;
        }
        const int k0 = k_begin + blk * kBlock;
        const uint32_t st = sb + s * kStageBytes;
        mbar_arrive_expect_tx(bar(s), bytes);
        for (int h = 0; h < p.Hkv; ++h) {
          tma_load_4d(st + h * kHeadBytes, &tm_k, bar(s), 0, h, k0, b);
          tma_load_4d(st + h * kHeadBytes + kHalfTile, &tm_k, bar(s), kHalf, h, k0, b);
          tma_load_4d(st + kKBytes + h * kHeadBytes, &tm_v, bar(s), 0, h, k0, b);
          tma_load_4d(st + kKBytes + h * kHeadBytes + kHalfTile, &tm_v, bar(s), kHalf, h, k0, b);
        }
        ++issued;
      }
      // never leave with a copy in flight into this CTA's shared memory
      for (int d = (issued > kStages ? issued - kStages : 0); d < issued; ++d) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(bar(d % kStages), (d / kStages) & 1))
          if (globaltimer_ns() - t0 > kTimeoutNs) break;
      }
    }
    return;
  }
  if (warp == kFactorWarp) {
    if (!far) return;
    // Correction factors of pairs i = lane (box 0) and i = lane + 32 (box 1).
    // step[r] = (cos, sin)(r theta_i) for r < 16; the block base row u0 is read
    // one block ahead so its latency overlaps the previous block.
    float2 step[kBlock][2];
#pragma unroll
    for (int r = 0; r < kBlock; ++r) {
      step[r][0] = p.cs[r * kHalf + lane];
      step[r][1] = p.cs[r * kHalf + lane + 32];
    }
    int u0 = k_begin - k_begin / p.G;
    float2 base0 = p.cs[static_cast<int64_t>(u0) * kHalf + lane];
    float2 base1 = p.cs[static_cast<int64_t>(u0) * kHalf + lane + 32];
    for (int blk = 0; blk < nblk; ++blk) {
      const int s = blk % kStages;
      const uint32_t ph = (blk / kStages) & 1;
      if (!warp_wait_u(bar(kStages + s), ph ^ 1u, abort_s, abort_g)) {
        if (lane == 0) {
          *abort_s = 1;
          atomicOr(p.status, kStatusTimeout);
        }
        break;
      }
      const float2 c0 = base0, c1 = base1;
      if (blk + 1 < nblk) {
        const int kn = k_begin + (blk + 1) * kBlock;
        u0 = kn - kn / p.G;
        base0 = p.cs[static_cast<int64_t>(u0) * kHalf + lane];
        base1 = p.cs[static_cast<int64_t>(u0) * kHalf + lane + 32];
      }
      // line r of each box: pair (i % 32) in 16-byte chunk ((i % 32) / 4) ^ (r % 8)
      uint8_t *tab = smem + s * kStageBytes + 2 * kKBytes;
#pragma unroll
      for (int r = 0; r < kBlock; ++r) {
        const uint32_t off = r * 128 + ((((lane >> 2) ^ (r & 7)) << 4) | ((lane & 3) * 4));
        const float2 a = step[r][0], d = step[r][1];
        *reinterpret_cast<__half2 *>(tab + off) =
            __floats2half2_rn(c0.x * a.x - c0.y * a.y, c0.y * a.x + c0.x * a.y);
        *reinterpret_cast<__half2 *>(tab + kTabBox + off) =
            __floats2half2_rn(c1.x * d.x - c1.y * d.y, c1.y * d.x + c1.x * d.y);
      }
      mbar_arrive(bar(s));  // release: this lane's factor writes
    }
    return;
  }
  if (warp >= p.Hkv) return;

  // ------------------------------------------------------------ consumers --
  const int hk = warp;
  const int g = lane >> 2, cq = lane & 3;  // MMA fragment coordinates
  const int rows = p.group;                // real query rows of the MMA
  // Q fragments: a[ks][0..3] = rows (g, g+8) x dims 16ks + 2cq + {0,1} / +8
  uint32_t qa[8][4];
  {
    const int udq = p.pos - p.pos / p.G;
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int row = g + 8 * rr;
      const bool real = row < rows;
      const __nv_bfloat16 *src =
          p.q + (static_cast<int64_t>(b) * p.Hq + hk * p.group + (real ? row : 0)) * kD;
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {  // dims 16ks + 2cq + 8hh + {0,1}
          const int d0 = 16 * ks + 2 * cq + 8 * hh;
          float y1[2], y2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int i = d0 + e;  // rotation pair (i, i + 64)
            const float x1 = real ? __bfloat162float(src[i]) : 0.f;
            const float x2 = real ? __bfloat162float(src[i + kHalf]) : 0.f;
            const float2 a = p.cs[static_cast<int64_t>(p.pos) * kHalf + i];
            float z1 = x1 * a.x - x2 * a.y;
            float z2 = x1 * a.y + x2 * a.x;
            if (far) {  // by dq = -udq
              const float2 r = p.cs[static_cast<int64_t>(udq) * kHalf + i];
              const float w1 = z1 * r.x + z2 * r.y;
              const float w2 = z2 * r.x - z1 * r.y;
              z1 = w1;
              z2 = w2;
            }
            y1[e] = z1 * p.scale_log2;
            y2[e] = z2 * p.scale_log2;
          }
          // A fragment regs: [0] row g lo cols, [1] row g+8 lo, [2] row g hi, [3] row g+8 hi
          qa[ks][2 * hh + rr] = pack_bf16x2(y1[0], y1[1]);
          qa[ks + 4][2 * hh + rr] = pack_bf16x2(y2[0], y2[1]);
        }
      }
    }
  }

  float o[16][4];
#pragma unroll
  for (int nd = 0; nd < 16; ++nd)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nd][e] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  bool ok = true;

  for (int blk = 0; blk < nblk; ++blk) {
    const int s = blk % kStages;
    const uint32_t ph = (blk / kStages) & 1;
    if (!warp_wait_u(bar(s), ph, abort_s, abort_g)) {
      ok = false;
      break;
    }
    const int k0 = k_begin + blk * kBlock;
    const uint32_t kt = sb + s * kStageBytes + hk * kHeadBytes;
    const uint32_t vt = kt + kKBytes;
    const uint8_t *tab = smem + s * kStageBytes + 2 * kKBytes;
    const int u0 = k0 - k0 / p.G;

    // S^T = Q K^T for key tiles nt = 0, 1 (keys k0 + 8nt + [0, 8))
    float sacc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] = 0.f;
      // K fragments: kb[ks][0..1]; ldmatrix row = key 8nt + (lane & 7),
      // matrix (lane >> 3) -> 16-byte chunk 2*ks2 + (lane >> 3)
      uint32_t kb[8][2];
      const int krow = 8 * nt + (lane & 7);
#pragma unroll
      for (int ks2 = 0; ks2 < 8; ks2 += 2) {
        const int ch = 2 * ks2 + (lane >> 3);
        ldsm_x4(kt + tile_off(krow, ch), kb[ks2][0], kb[ks2][1], kb[ks2 + 1][0],
                kb[ks2 + 1][1]);
      }
      if (far) {
        // this thread's key k0 + 8nt + g: rotate by -u theta_i
        const int kk = k0 + 8 * nt + g;
        const int urow = (kk - kk / p.G) - u0;  // 0..15
        // row urow of the two swizzled boxes: pair i sits in box i / 32, line
        // urow, 16-byte chunk ((i % 32) / 4) ^ (urow & 7), offset (i % 4) * 4
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int i0 = 16 * ks + 2 * cq + 8 * hh;  // pairs i0, i0+1
            const int ib = i0 & 31;
            const uint2 hf = *reinterpret_cast<const uint2 *>(
                tab + (i0 >> 5) * kTabBox + urow * 128 + (((ib >> 2) ^ (urow & 7)) << 4) +
                (ib & 3) * 4);
            const float2 f01 = __half22float2(*reinterpret_cast<const __half2 *>(&hf.x));
            const float2 f23 = __half22float2(*reinterpret_cast<const __half2 *>(&hf.y));
            const float4 f = make_float4(f01.x, f01.y, f23.x, f23.y);
            const uint32_t lo = kb[ks][hh], hi = kb[ks + 4][hh];
            const float a0 = bf_lo(lo), a1 = bf_hi(lo), b0 = bf_lo(hi), b1 = bf_hi(hi);
            // (x1, x2) -> (x1 c + x2 s, x2 c - x1 s)
            kb[ks][hh] = pack_bf16x2(a0 * f.x + b0 * f.y, a1 * f.z + b1 * f.w);
            kb[ks + 4][hh] = pack_bf16x2(b0 * f.x - a0 * f.y, b1 * f.z - a1 * f.w);
          }
        }
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma16816(sacc[nt], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], kb[ks][0], kb[ks][1]);
    }
    // sacc[nt][0..1]: row g, keys 8nt + 2cq + {0,1}; [2..3]: row g+8
    if (k0 < k_begin || k0 + kBlock > k_end) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kk = k0 + 8 * nt + 2 * cq + (e & 1);
          if (kk >= k_end) sacc[nt][e] = -INFINITY;
        }
    }
    float alpha[2];
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      float mx = fmaxf(fmaxf(sacc[0][2 * rr], sacc[0][2 * rr + 1]),
                       fmaxf(sacc[1][2 * rr], sacc[1][2 * rr + 1]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      alpha[rr] = 1.f;
      if (mx > m[rr] + 8.f) {
        alpha[rr] = ex2_approx(m[rr] - mx);
        m[rr] = mx;
      }
    }
    if (alpha[0] != 1.f || alpha[1] != 1.f) {
#pragma unroll
      for (int nd = 0; nd < 16; ++nd) {
        o[nd][0] *= alpha[0];
        o[nd][1] *= alpha[0];
        o[nd][2] *= alpha[1];
        o[nd][3] *= alpha[1];
      }
      l[0] *= alpha[0];
      l[1] *= alpha[1];
    }
    uint32_t pa[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const float mu = (m[rr] == -INFINITY) ? 0.f : m[rr];
        const float p0 = ex2_approx(sacc[nt][2 * rr] - mu);
        const float p1 = ex2_approx(sacc[nt][2 * rr + 1] - mu);
        l[rr] += p0 + p1;
        pa[2 * nt + rr] = pack_bf16x2(p0, p1);
      }
    }
    // O += P V over 16 dim tiles; V fragments by ldmatrix.trans:
    // matrix (lane >> 3): keys 8*((lane>>3)&1) + (lane&7), dim chunk nd + (lane >> 4)
    const int vrow = 8 * ((lane >> 3) & 1) + (lane & 7);
#pragma unroll
    for (int nd = 0; nd < 16; nd += 2) {
      uint32_t v0, v1, v2, v3;
      ldsm_x4_t(vt + tile_off(vrow, nd + (lane >> 4)), v0, v1, v2, v3);
      mma16816(o[nd], pa[0], pa[1], pa[2], pa[3], v0, v1);
      mma16816(o[nd + 1], pa[0], pa[1], pa[2], pa[3], v2, v3);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(kStages + s));
  }
  if (!ok) {
    *abort_s = 1;
    atomicOr(p.status, kStatusTimeout);
    return;
  }
  // row sums across the 4 threads of a row group
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], 1);
    l[rr] += __shfl_xor_sync(0xffffffffu, l[rr], 2);
  }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int row = g + 8 * rr;
    if (row >= rows) continue;
    float *dst = p.ws + ((static_cast<int64_t>(b) * p.Hq + hk * p.group + row) * p.n_chunks + c) *
                            kDecodePartialFloats;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      dst[8 * nd + 2 * cq] = o[nd][2 * rr];
      dst[8 * nd + 2 * cq + 1] = o[nd][2 * rr + 1];
    }
    if (cq == 0) {
      dst[kD] = m[rr];
      dst[kD + 1] = l[rr];
    }
  }
  // the combine kernel (a programmatic dependent) may be scheduled once every
  // CTA got here; it waits for this grid's completion before reading
  asm volatile("griddepcontrol.launch_dependents;");
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// cache [B, cap, Hkv, 128] bf16 seen as a 4-D tensor ending at key `keys - 1`
bool make_cache_map(CUtensorMap *m, const void *base, int B, int cap, int keys, int Hkv) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(Hkv),
                              static_cast<cuuint64_t>(keys), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kD) * 2,
                                 static_cast<cuuint64_t>(Hkv) * kD * 2,
                                 static_cast<cuuint64_t>(cap) * Hkv * kD * 2};
  const cuuint32_t box[4] = {kHalf, 1, kBlock, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool decode_mma_supported(int Hq, int Hkv, int D) {
  return D == kD && Hkv <= kMaxHeads && Hq / Hkv <= kMaxGroup;
}

// Keys per CTA: about one wave of CTAs per batch entry, a multiple of the
// 16-key block; the remote range [0, far_end) and the local range are
// chunked separately.
void decode_mma_plan(int B, int pos, int far_end, int *chunk, int *n_far, int *n_chunks) {
  const long long keys = static_cast<long long>(pos) + 1;
  long long cch = (keys + kCtaTarget - 1) / kCtaTarget;
  cch = ((cch + kBlock - 1) / kBlock) * kBlock;
  if (cch < kBlock) cch = kBlock;
  *chunk = static_cast<int>(cch);
  *n_far = static_cast<int>((far_end + cch - 1) / cch);
  *n_chunks = *n_far + static_cast<int>((keys - far_end + cch - 1) / cch);
}

cudaError_t launch_decode_mma(const DecodeArgs &a, unsigned *status, cudaStream_t s) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(bifocal_decode_mma_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  });
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap mk, mv;
  if (!make_cache_map(&mk, a.kc, a.B, a.cap, a.pos + 1, a.Hkv) ||
      !make_cache_map(&mv, a.vc, a.B, a.cap, a.pos + 1, a.Hkv))
    return cudaErrorInvalidValue;
  Params p;
  p.q = a.q;
  p.cs = a.table.cs;
  p.ws = a.ws;
  p.status = status;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.group = a.Hq / a.Hkv;
  p.pos = a.pos;
  p.G = a.G;
  p.far_end = a.far_end;
  p.chunk = a.chunk;
  p.n_far = a.n_far_chunks;
  p.n_chunks = a.n_chunks;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.skip_first_arrival = a.debug_skip_arrival ? 1 : 0;
  dim3 grid(a.n_chunks, a.B);
  bifocal_decode_mma_kernel<<<grid, kThreads, kSmemAlloc, s>>>(mk, mv, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_decode_combine(a, s);
}

}  // namespace jl
