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
// of one batch entry and ALL kv heads: one consumer warp per kv head, a TMA
// producer warp and, in a remote chunk, a factor warp.  The producer streams
// 16-key blocks through a 3-stage ring in shared memory: per block and head, K
// and V as two 64-column boxes with the 128-byte swizzle (so ldmatrix reads
// are conflict-free), one box per producer lane.  The tensor maps end at key pos, so slots past pos read
// as zeros and are never touched.  Blocks start on multiples of 16 keys (keys
// of the first block before the chunk's first are masked like those past its
// end), so that with a paged cache (fixed-size pages of a shared pool, a block
// table per sequence) no block straddles two pages: there the maps cover the
// whole pool and the producer translates each block's first key through the
// block table, and a paged call computes bit for bit what a contiguous one
// does.  The factor warp writes, per block, the 16
// rows of correction factors (cos, sin)(u theta_i) the block needs (u = k -
// f(k) grows by at most one per key): row u0 + r is the complex product of the
// fp32 table row u0 (one 512-byte read per block) and the step row r < 16
// (held in registers), rounded to bf16, so the corrections read no per-key
// data from HBM.
//
// Consumer warp (kv head h, its group of <= 8 query heads): m16n8k16 bf16 MMAs
// with the block's 16 keys as rows and the query heads as columns, so that no
// MMA row is padding:
//   S = K . Q^T          8 k-steps, Q^T fragments held in registers
//                        (pre-rotated, pre-scaled by log2(e)/sqrt(D))
//   K fragments (ldmatrix) of a remote key are rotated by -u theta_i with
//   packed bf16x2 multiply-adds: pair (i, i+64) lies in k-steps ks and ks+4 of
//   the same thread.  (fp32 arithmetic here costs about 11 instructions per
//   two pairs instead of 5 and, on a B200, 8% of decode time at n = 131072;
//   the rotated key is rounded to bf16 for the MMA either way, and the extra
//   roundings leave the error against the fp64 reference within 1.5x.)
//   online softmax per head column (fp32, base 2, rescale only when the
//   running max grows by more than 2^8); P is transposed into the B fragments
//   of O^T += V^T . P^T with movmatrix (V^T fragments by ldmatrix.trans).
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
constexpr int kMaxGroup = 8;          // query heads per kv head (MMA columns)
constexpr int kThreads = (kMaxHeads + 2) * 32;
constexpr int kProducerWarp = kMaxHeads;
constexpr int kFactorWarp = kMaxHeads + 1;
constexpr uint32_t kHalfTile = kBlock * 128;          // 64 dims of one head: 2 KiB
constexpr uint32_t kHeadBytes = 2 * kHalfTile;        // K (or V) of one head: 4 KiB
constexpr uint32_t kHalfBytes = kMaxHeads * kHalfTile;  // one 64-dim half, all heads
constexpr uint32_t kKBytes = kMaxHeads * kHeadBytes;  // 32 KiB
constexpr uint32_t kTabRow = 32 * 8;                  // 32 x (cos, cos | sin, sin) bf16x2
constexpr uint32_t kTabBytes = kBlock * kTabRow;      // 16 rows: 4 KiB
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
  unsigned long long g_magic;  // ceil(2^64 / G): floor(k / G) = umulhi(k, g_magic), G >= 2
  int skip_first_arrival;  // test-only: withhold the first block (bounded-wait check)
  const DecodeWork *work;  // batched decode: this CTA's entry (nullptr: one position for all)
  // paged cache (block_table != nullptr): sequence b's key k lives in row
  // k % page_size of page block_table[b * max_pages + k / page_size] of the pool
  const int *block_table;
  int page_size, max_pages, num_pages;
  const int *n_work_dev;  // plan made on the device: CTAs at or past *n_work_dev exit
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
// floor(k / G) for 0 <= k < 2^31 and G >= 2, with magic = ceil(2^64 / G):
// k * magic / 2^64 exceeds k / G by less than k * G / (G 2^64) < 1 / G, so the
// floor is exact.
__device__ __forceinline__ int div_g(int k, unsigned long long magic) {
  return static_cast<int>(__umul64hi(static_cast<unsigned long long>(k), magic));
}

// 8x8 b16 matrix transpose across the warp
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Rotates two pairs: lo holds x1 of pairs (j, j+1) and hi their x2, as
// bf16x2; c2 = (c_j, c_j+1), s2 = (s_j, s_j+1) as bf16x2.
// (x1, x2) -> (x1 c + x2 s, x2 c - x1 s): one product rounded to bf16, then a
// fused multiply-add rounded once.
__device__ __forceinline__ void rotate_pairs_bf(uint32_t &lo, uint32_t &hi, uint32_t c2,
                                                uint32_t s2) {
  uint32_t t, u, nl, nh;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(t) : "r"(hi), "r"(s2));
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(nl) : "r"(lo), "r"(c2), "r"(t));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(u) : "r"(lo), "r"(s2));
  asm("neg.bf16x2 %0, %0;" : "+r"(u));
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(nh) : "r"(hi), "r"(c2), "r"(u));
  lo = nl;
  hi = nh;
}

// byte offset of 16-byte chunk `ch` (0..15 over the 128 dims) of key row `row`
// in a stage's K (or V) laid out [2 halves][heads][16 keys][128 B], swizzled,
// relative to the head's first row of half 0
__device__ __forceinline__ uint32_t tile_off(int row, int ch) {
  return static_cast<uint32_t>((ch >> 3) * kHalfBytes + row * 128 + (((ch & 7) ^ (row & 7)) << 4));
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
  // launched as a programmatic dependent of whatever precedes it on the
  // stream: its CTAs may be scheduled while that kernel finishes, and read
  // nothing before it has completed
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (p.n_work_dev != nullptr && static_cast<int>(blockIdx.x) >= *p.n_work_dev) return;
  // this CTA's keys [k_begin, k_end) of sequence b, and where its partials go:
  // query head h of the chunk at (pbase + h * pstride) * kDecodePartialFloats
  int b, k_begin, k_end, pos, G;
  bool far;
  unsigned long long g_magic;
  int64_t pbase, pstride;
  if (p.work != nullptr) {  // batched: one entry of the host-planned work table
    const DecodeWork w = p.work[blockIdx.x];
    b = w.b;
    k_begin = w.k_begin;
    k_end = w.k_end;
    far = w.far != 0;
    pos = w.pos;
    G = w.G;
    g_magic = w.g_magic;
    pbase = w.part;
    pstride = 1;
  } else {
    const int c = blockIdx.x;
    b = blockIdx.y;
    far = c < p.n_far;
    if (far) {
      k_begin = c * p.chunk;
      k_end = min(p.far_end, k_begin + p.chunk);
    } else {
      k_begin = p.far_end + (c - p.n_far) * p.chunk;
      k_end = min(p.pos + 1, k_begin + p.chunk);
    }
    pos = p.pos;
    G = p.G;
    g_magic = p.g_magic;
    pbase = static_cast<int64_t>(b) * p.Hq * p.n_chunks + c;
    pstride = p.n_chunks;
  }
  // first key of the first block: blocks start on multiples of 16 keys (a
  // page holds whole blocks)
  const bool paged = p.block_table != nullptr;
  const int kb0 = k_begin & ~(kBlock - 1);
  const int nblk = (k_end - kb0 + kBlock - 1) / kBlock;

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
    // Four boxes per block, one per lane 0-3: K or V (lane & 2), dims 0-63
    // or 64-127 (lane & 1), all kv heads and 16 keys in one box (the maps
    // order the dimensions dims, keys, heads, so a box lands as [heads][16
    // keys][128 B]).  Each copy costs the TMA unit tens of cycles to issue
    // whatever its size, so a few large copies keep the producer off the
    // critical path.
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
    }
    const bool is_v = (lane & 2) != 0;
    const int x = (lane & 1) * kHalf;
    const CUtensorMap *map = is_v ? &tm_v : &tm_k;
    const uint32_t dst_off = (is_v ? kKBytes : 0u) + ((lane & 1) ? kHalfBytes : 0u);
    const uint32_t bytes = static_cast<uint32_t>(p.Hkv) * 2 * kHeadBytes;
    // paged: the logical page and offset of the block advance by 16 keys a
    // block; a page's entry is read one block before it is needed, so that its
    // latency overlaps the wait for a free stage
    const int *bt = paged ? p.block_table + static_cast<int64_t>(b) * p.max_pages : nullptr;
    int lp = paged ? kb0 / p.page_size : 0;
    int off = paged ? kb0 - lp * p.page_size : 0;
    int page_next = (paged && nblk > 0) ? __ldg(bt + lp) : 0;
    int issued = 0;
    // test-only: no block is loaded, so the consumers' first wait expires
    for (int blk = p.skip_first_arrival ? nblk : 0; blk < nblk; ++blk) {
      const int s = blk % kStages;
      const uint32_t ph = (blk / kStages) & 1;
      int row = kb0 + blk * kBlock, bc = b;
      if (paged) {
        int page = page_next;
        if (page < 0 || page >= p.num_pages) {  // refused: read page 0, flag the call
          if (lane == 0) atomicOr(p.status, kStatusBounds);
          page = 0;
        }
        row = page * p.page_size + off;
        bc = 0;
        off += kBlock;
        if (off == p.page_size) {
          off = 0;
          ++lp;
          if (blk + 1 < nblk) page_next = __ldg(bt + lp);
        }
      }
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(bar(kStages + s), ph ^ 1u, abort_s, abort_g, kTimeoutNs);
        if (ok) mbar_arrive_expect_tx(bar(s), bytes);
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) {
        if (lane == 0) {
          *abort_s = 1;
          atomicOr(p.status, kStatusTimeout);
        }
        break;
      }
      if (lane < 4) tma_load_4d(sb + s * kStageBytes + dst_off, map, bar(s), x, row, 0, bc);
      ++issued;
    }
    // never leave with a copy in flight into this CTA's shared memory
    if (lane == 0) {
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
    // Correction factors of pairs 2 lane and 2 lane + 1: step[r] = (cos, sin)
    // (r theta) of both, r < 16; the block's base row u0 is read one block
    // ahead so its latency overlaps the previous block.
    const float4 *cs4 = reinterpret_cast<const float4 *>(p.cs);
    float4 step[kBlock];
#pragma unroll
    for (int r = 0; r < kBlock; ++r) step[r] = cs4[r * (kHalf / 2) + lane];
    int u0 = kb0 - div_g(kb0, g_magic);
    float4 base = cs4[static_cast<int64_t>(u0) * (kHalf / 2) + lane];
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
      const float4 cb = base;
      if (blk + 1 < nblk) {
        const int kn = kb0 + (blk + 1) * kBlock;
        u0 = kn - div_g(kn, g_magic);
        base = cs4[static_cast<int64_t>(u0) * (kHalf / 2) + lane];
      }
      // row r, 8-byte word lane ^ (4 (r % 4)): (c0, c1 | s0, s1) as bf16x2
      // of pairs 2 lane, 2 lane + 1 at angle (u0 + r) theta
      uint8_t *tab = smem + s * kStageBytes + 2 * kKBytes;
#pragma unroll
      for (int r = 0; r < kBlock; ++r) {
        const float4 a = step[r];
        const uint2 v = make_uint2(pack_bf16x2(cb.x * a.x - cb.y * a.y, cb.z * a.z - cb.w * a.w),
                                   pack_bf16x2(cb.y * a.x + cb.x * a.y, cb.w * a.z + cb.z * a.w));
        *reinterpret_cast<uint2 *>(tab + r * kTabRow + ((lane ^ ((r & 3) << 2)) << 3)) = v;
      }
      mbar_arrive(bar(s));  // release: this lane's factor writes
    }
    return;
  }
  if (warp >= p.Hkv) return;

  // ------------------------------------------------------------ consumers --
  // Warp = kv head hk.  m16n8k16 MMAs with the 16 keys of a block as the rows
  // and the group's query heads (<= 8) as the columns:
  //   S[key][head] = K . Q^T        A = K (ldmatrix), B = Q^T held in registers
  //   O^T[dim][head] += V^T . P^T   A = V^T (ldmatrix.trans), B = P^T
  // P moves from the accumulator layout of S to the B layout of P^T with two
  // 8x8 transposes (movmatrix).
  const int hk = warp;
  const int g = lane >> 2, cq = lane & 3;  // MMA fragment coordinates
  const int heads = p.group;               // real columns of the MMAs
  // Q^T fragments: qb[ks][hh] = head g, dims 16ks + 2cq + 8hh + {0,1}
  uint32_t qb[8][2];
  {
    const int udq = pos - pos / G;
    const bool real = g < heads;
    const __nv_bfloat16 *src =
        p.q + (static_cast<int64_t>(b) * p.Hq + hk * p.group + (real ? g : 0)) * kD;
#pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int d0 = 16 * ks + 2 * cq + 8 * hh;
        float y1[2], y2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = d0 + e;  // rotation pair (i, i + 64)
          const float x1 = real ? __bfloat162float(src[i]) : 0.f;
          const float x2 = real ? __bfloat162float(src[i + kHalf]) : 0.f;
          const float2 a = p.cs[static_cast<int64_t>(pos) * kHalf + i];
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
        qb[ks][hh] = pack_bf16x2(y1[0], y1[1]);
        qb[ks + 4][hh] = pack_bf16x2(y2[0], y2[1]);
      }
    }
  }

  // O^T accumulators of dim tile mt: [0] (dim 16mt+g, head 2cq), [1] (head
  // 2cq+1), [2] (dim 16mt+g+8, head 2cq), [3] (head 2cq+1)
  float o[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[mt][e] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};  // heads 2cq, 2cq+1
  bool ok = true;
  // ldmatrix row supplied by this lane: K (A, matrices keys 0-7 | 8-15 x
  // chunk 2ks | 2ks+1) and V^T (A by .trans, matrices chunk 2mt | 2mt+1 x keys
  // 0-7 | 8-15)
  const int krow = (lane & 7) + 8 * ((lane >> 3) & 1);
  const int vrow = (lane & 7) + 8 * (lane >> 4);

  for (int blk = 0; blk < nblk; ++blk) {
    const int s = blk % kStages;
    const uint32_t ph = (blk / kStages) & 1;
    if (!warp_wait_u(bar(s), ph, abort_s, abort_g)) {
      ok = false;
      break;
    }
    const int k0 = kb0 + blk * kBlock;
    const uint32_t kt = sb + s * kStageBytes + hk * kHalfTile;
    const uint32_t vt = kt + kKBytes;

    // K fragments kf[ks]: [0] key g, [1] key g+8 (dims 16ks + 2cq + {0,1}),
    // [2], [3] the same keys at dims + 8
    uint32_t kf[8][4];
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
      ldsm_x4(kt + tile_off(krow, 2 * ks + (lane >> 4)), kf[ks][0], kf[ks][1], kf[ks][2],
              kf[ks][3]);
    if (far) {
      // a remote key is rotated by -u theta_i, u = k - f(k): pair (i, i+64)
      // lies in k-steps ks and ks+4 of this thread; row u - u0 of the staged
      // factors holds (cos, sin) of pairs (2pp, 2pp+1) in 8-byte word
      // pp ^ (4 (row % 4)) as (c0, c1 | s0, s1), bf16x2 (conflict-free: the
      // keys of a half-warp fall on at most 4 consecutive rows)
      const uint8_t *tab = smem + s * kStageBytes + 2 * kKBytes;
      const int u0 = k0 - div_g(k0, g_magic);
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int kk = k0 + g + 8 * r;
        const int urow = (kk - div_g(kk, g_magic)) - u0;  // 0..15
        const uint8_t *trow = tab + urow * kTabRow;
        const int sw = (urow & 3) << 2;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int pp = 8 * ks + cq + 4 * hh;  // pairs 2pp, 2pp + 1
            const uint2 f = *reinterpret_cast<const uint2 *>(trow + ((pp ^ sw) << 3));
            rotate_pairs_bf(kf[ks][2 * hh + r], kf[ks + 4][2 * hh + r], f.x, f.y);
          }
        }
      }
    }
    // V^T fragments of the 8 dim tiles, then the stage goes back to the
    // producer: the rest of the block works from registers
    uint32_t vf[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
      ldsm_x4_t(vt + tile_off(vrow, 2 * mt + ((lane >> 3) & 1)), vf[mt][0], vf[mt][1], vf[mt][2],
                vf[mt][3]);
    // a block reaching past the chunk's end or starting before its first key
    const bool edge = k0 + kBlock > k_end || k0 < k_begin;
    auto in_chunk = [&](int k) { return k >= k_begin && k < k_end; };
    if (edge) {
      // keys outside the chunk: their P is 0, and their V (possibly past a
      // sequence's last key, so any value) must not reach O as 0 * inf or NaN
      const uint32_t m0 = (in_chunk(k0 + 2 * cq) ? 0x0000FFFFu : 0u) |
                          (in_chunk(k0 + 2 * cq + 1) ? 0xFFFF0000u : 0u);
      const uint32_t m1 = (in_chunk(k0 + 8 + 2 * cq) ? 0x0000FFFFu : 0u) |
                          (in_chunk(k0 + 9 + 2 * cq) ? 0xFFFF0000u : 0u);
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        vf[mt][0] &= m0;
        vf[mt][1] &= m0;
        vf[mt][2] &= m1;
        vf[mt][3] &= m1;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(kStages + s));
    // S = K . Q^T, two accumulation chains
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < 8; ks += 2) {
      mma16816(sa, kf[ks][0], kf[ks][1], kf[ks][2], kf[ks][3], qb[ks][0], qb[ks][1]);
      mma16816(sc, kf[ks + 1][0], kf[ks + 1][1], kf[ks + 1][2], kf[ks + 1][3], qb[ks + 1][0],
               qb[ks + 1][1]);
    }
    // sv[0..1]: key g, heads 2cq, 2cq+1; sv[2..3]: key g+8
    float sv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) sv[e] = sa[e] + sc[e];
    if (edge) {
      if (!in_chunk(k0 + g)) sv[0] = sv[1] = -INFINITY;
      if (!in_chunk(k0 + g + 8)) sv[2] = sv[3] = -INFINITY;
    }
    float alpha[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float mx = fmaxf(sv[e], sv[2 + e]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      alpha[e] = 1.f;
      if (mx > m[e] + 8.f) {  // lazy rescale: only when the max grows by > 2^8
        alpha[e] = ex2_approx(m[e] - mx);
        m[e] = mx;
      }
    }
    if (alpha[0] != 1.f || alpha[1] != 1.f) {
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        o[mt][0] *= alpha[0];
        o[mt][1] *= alpha[1];
        o[mt][2] *= alpha[0];
        o[mt][3] *= alpha[1];
      }
      l[0] *= alpha[0];
      l[1] *= alpha[1];
    }
    float pv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float mu = (m[e & 1] == -INFINITY) ? 0.f : m[e & 1];
      pv[e] = ex2_approx(sv[e] - mu);
    }
    l[0] += pv[0] + pv[2];
    l[1] += pv[1] + pv[3];
    // P^T B fragments: [0] keys 2cq, 2cq+1 of head g, [1] keys 8 + 2cq, 8 + 2cq + 1
    const uint32_t pb0 = movmatrix_t(pack_bf16x2(pv[0], pv[1]));
    const uint32_t pb1 = movmatrix_t(pack_bf16x2(pv[2], pv[3]));
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
      mma16816(o[mt], vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3], pb0, pb1);
  }
  if (!ok) {
    *abort_s = 1;
    atomicOr(p.status, kStatusTimeout);
    return;
  }
  // column sums across the 8 row groups
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 4);
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 8);
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 16);
  }
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int h = 2 * cq + e;
    if (h >= heads) continue;
    float *dst = p.ws + (pbase + static_cast<int64_t>(hk * p.group + h) * pstride) *
                            kDecodePartialFloats;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      dst[16 * mt + g] = o[mt][e];
      dst[16 * mt + g + 8] = o[mt][2 + e];
    }
    if (g == 0) {
      dst[kD] = m[e];
      dst[kD + 1] = l[e];
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

// cache [B, cap, Hkv, 128] bf16 seen as a 4-D tensor (dims, keys, heads,
// batch) ending at key `keys - 1`; a box is 64 dims x 16 keys x all heads
bool make_cache_map(CUtensorMap *m, const void *base, int B, int cap, int keys, int Hkv) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(keys),
                              static_cast<cuuint64_t>(Hkv), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(Hkv) * kD * 2,
                                 static_cast<cuuint64_t>(kD) * 2,
                                 static_cast<cuuint64_t>(cap) * Hkv * kD * 2};
  const cuuint32_t box[4] = {kHalf, kBlock, static_cast<cuuint32_t>(Hkv), 1};
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

// Keys per CTA: one wave of CTAs per batch entry, a multiple of the 16-key
// block; the remote range [0, far_end) and the local range are chunked
// separately, and the chunk grows until both together fit in the wave (a
// 149th CTA would run after the first ones finish, doubling the tail).
void decode_mma_plan(int B, int pos, int far_end, int *chunk, int *n_far, int *n_chunks) {
  const long long keys = static_cast<long long>(pos) + 1;
  long long cch = (keys + kCtaTarget - 1) / kCtaTarget;
  cch = ((cch + kBlock - 1) / kBlock) * kBlock;
  if (cch < kBlock) cch = kBlock;
  auto count = [&](long long c) {
    return (far_end + c - 1) / c + (keys - far_end + c - 1) / c;
  };
  while (count(cch) > kCtaTarget) cch += kBlock;
  *chunk = static_cast<int>(cch);
  *n_far = static_cast<int>((far_end + cch - 1) / cch);
  *n_chunks = static_cast<int>(count(cch));
}

cudaError_t launch_decode_mma(const DecodeArgs &a, unsigned *status, cudaStream_t s) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(bifocal_decode_mma_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  });
  if (attr_err != cudaSuccess) return attr_err;
  // the maps end at the last valid key (of the longest sequence when
  // batched); a paged pool is one sequence of num_pages * page_size rows
  CUtensorMap mk, mv;
  if (a.block_table != nullptr) {
    const int rows = a.num_pages * a.page_size;
    if (!make_cache_map(&mk, a.kc, 1, rows, rows, a.Hkv) ||
        !make_cache_map(&mv, a.vc, 1, rows, rows, a.Hkv))
      return cudaErrorInvalidValue;
  } else {
    const int keys = a.work != nullptr ? a.max_keys : a.pos + 1;
    if (!make_cache_map(&mk, a.kc, a.B, a.cap, keys, a.Hkv) ||
        !make_cache_map(&mv, a.vc, a.B, a.cap, keys, a.Hkv))
      return cudaErrorInvalidValue;
  }
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
  p.g_magic = a.G >= 2 ? (~0ull / static_cast<unsigned long long>(a.G)) + 1ull : 0ull;
  p.work = a.work;
  p.block_table = a.block_table;
  p.page_size = a.page_size;
  p.max_pages = a.max_pages;
  p.num_pages = a.num_pages;
  p.n_work_dev = a.n_work_dev;
  const dim3 grid = a.work != nullptr ? dim3(a.n_work) : dim3(a.n_chunks, a.B);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemAlloc;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, bifocal_decode_mma_kernel, mk, mv, p);
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_decode_combine(a, s);
}

}  // namespace jl
