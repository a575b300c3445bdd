// jl_prefill_sm100_x2.cu -- bifocal prefill, two query heads per CTA.
//
// Same computation as jl_prefill_sm100.cu (Jet-Long, techwalker explainer
// §二/§四, bittide paper summary §3.1-§3.2: local pairs at original positions,
// remote pairs at f(x) = floor(x/G), merged by per-tile complementary-mask
// passes inside one online softmax).  This kernel is the B200 throughput path
// for grouped-query attention with an even group size: a CTA takes one
// 128-row query tile of TWO query heads of the same kv head, so every K/V tile
// it loads feeds two S = Q K^T and two O += P V products, and the tensor core
// alternates between the two heads while each head's softmax runs.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax of head 0: thread r = query row r = TMEM lane r of S0/O0
//   warps 4-7  softmax of head 1: the same on S1/O1
//              Between passes, while its next S is being computed, each
//              softmax thread also rotates its slice (4 keys x 8 pairs) of the
//              K tile two passes ahead in shared memory, in place, to that
//              pass's positions (R(k) or R(f(k)) from the cos/sin table): RoPE
//              applied on the fly, with no rotated copy of the keys in global
//              memory.  Head 0's warps take keys 0-63, head 1's keys 64-127.
//   warp 8     TMA producer of the raw K tiles (3-stage ring)
//   warp 9     TMEM allocation and every tcgen05.mma, from one thread
//   warp 10    TMA producer of the V tiles (2-stage ring)
//   warp 11    idle (it completes the third warpgroup)
// Registers: launched at 168 a thread; the third warpgroup drops to 72 and the
// softmax warpgroups rise to 216 (setmaxnreg: 2 x 128 x 216 + 128 x 72 =
// 384 x 168), so a softmax thread holds its whole S row and reads S from TMEM
// once per pass.
// TMEM (512 columns): S0 | S1 | O0 | O1, 128 fp32 columns each.  After the
// softmax has read S_t into registers it writes P_t (bf16, two per column) into
// the first 64 columns of S_t, and O_t += P_t V takes P_t straight from TMEM,
// in two parts, each multiplied as soon as the softmax has written it (so half
// of PV_t runs while the softmax is still on the later keys).
// Issue order PV_0(j), S_0(j+1), PV_1(j), S_1(j+1): the next S_t follows the
// product that reads P_t from the same thread, and the tensor core runs one
// thread's MMAs in order, so no completion wait sits between them.
//
// Shared memory holds one Q variant per head: the remote passes of a query
// tile all come before its local passes, so Q_rem is used first and is then
// overwritten in place by Q_std (one switch per tile, signalled through the
// q_ready barrier).  Q rotation runs in the softmax warps from the cos/sin
// table, K rotation in the softmax warps between passes.
//
// Exponentials: MUFU ex2.approx.  A compile-time option (JL_X2_POLY_PAIRS)
// moves some column pairs of each unmasked row to 2^floor(x) * p(x - floor(x))
// on the FMA pipe (cubic fitted by least squares, derive_exp2_poly.py, max
// relative error 1.1e-4).  Measured on a B200 at L = 131072: 4 pairs of 64
// gained 4% while P went to the PV product in one piece, and lose 2-3% since
// P is released in two parts; it is off.
//
// Every mbarrier wait is bounded; an abandoned wait raises the CTA abort flag
// and the device status word, all roles drain their in-flight copies and MMAs,
// TMEM is freed and the kernel returns.
#include <cudaTypedefs.h>

#include <climits>
#include <mutex>
#include <type_traits>

#include "jl_prefill_common.cuh"

namespace jl {
namespace {

using namespace sm100;
using namespace prefill;

constexpr int kKStages = 3;  // K ring: a tile is loaded, then rotated, then read by S
constexpr int kVStages = 2;
constexpr int kThreads = 384;  // softmax 0, softmax 1, producers + MMA
constexpr int kProducerWarp = 8;   // K tiles
constexpr int kVProducerWarp = 10;  // V tiles
constexpr int kMmaWarp = 9;
constexpr int kRotThreads = 256;  // the softmax threads rotate the K tiles
// register budgets after setmaxnreg (2 x 216 + 72 = 3 x 168)
constexpr int kRegsSoftmax = 216;
constexpr int kRegsWg2 = 72;

constexpr uint32_t kOffQ0 = 0;
constexpr uint32_t kOffQ1 = kOffQ0 + kTileBytes;
constexpr uint32_t kOffK = kOffQ1 + kTileBytes;
constexpr uint32_t kOffV = kOffK + kKStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kVStages * kTileBytes;

enum : int {
  kBarQReady = 0,                  // [2] per head, 128 arrivals
  kBarKFull = kBarQReady + 2,      // [kKStages]
  kBarKEmpty = kBarKFull + kKStages,
  kBarKRot = kBarKEmpty + kKStages,  // [kKStages] K tile rotated, one arrival per softmax thread
  kBarVFull = kBarKRot + kKStages,   // [kVStages]
  kBarVEmpty = kBarVFull + kVStages,
  kBarSFull = kBarVEmpty + kVStages, // [2] per head, tcgen05.commit
  // [2][2] per head and part of P, 128 arrivals each; head t's pair at
  // kBarPFull + 4t (the two heads' barriers in different 32-byte sectors)
  kBarPFull = kBarSFull + 2,
  kBarODone = kBarPFull + 8,         // [2] per head, tcgen05.commit
  kBarDrain = kBarODone + 2,
  kNumBars = kBarDrain + 1
};

constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kOffSkip = kOffAbort + 4;
constexpr uint32_t kOffStep = (kOffSkip + 4 + 15) & ~15u;  // R(1) per pair (32 float4)
constexpr uint32_t kSmemUsed = kOffStep + 64 * 8;
constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;

// kv heads whose CTAs are scheduled together (see the CTA order in the
// kernel).  Measured on a B200 at L = 131072 (DRAM bytes read per launch, ms
// per call): all 8 kv heads interleaved 80-177 GB, 132 ms; 4 at a time 17 GB,
// 128.6 ms; 2: 9.2 GB, 128.4 ms; 1: 5.0 GB, 128.1 ms.
#ifndef JL_X2_KV_PER_GROUP
#define JL_X2_KV_PER_GROUP 1
#endif
constexpr int kKvPerGroup = JL_X2_KV_PER_GROUP;

// Of the 64 column pairs of an unmasked row, kPolyPairs (spread evenly) take
// 2^x on the FMA pipe instead of the MUFU unit; 0 keeps every exponential on
// the MUFU unit.
#ifndef JL_X2_POLY_PAIRS
#define JL_X2_POLY_PAIRS 0
#endif
constexpr int kPolyPairs = JL_X2_POLY_PAIRS;
// P is released to the PV product in two parts: the first kPSplit of the four
// 16-column stores (32 keys each), then the rest.  Measured on a B200 at
// L = 131072 (ms per call): P in one piece 135, split after 1 store 131, after
// 2 stores 135, four parts 138.
#ifndef JL_X2_P_SPLIT
#define JL_X2_P_SPLIT 1
#endif
constexpr int kPSplit = JL_X2_P_SPLIT;
static_assert(kPSplit >= 1 && kPSplit <= 3, "P split");
static_assert(kPolyPairs >= 0 && kPolyPairs <= 64, "pairs of a row");
// pair q in [0, 64) is one of the kPolyPairs (a compile-time constant for the
// unrolled loop)
__host__ __device__ constexpr bool poly_pair(int q) {
  return (q + 1) * kPolyPairs / 64 > q * kPolyPairs / 64;
}
__host__ __device__ constexpr uint32_t tm_s(int t) { return 128u * t; }
__host__ __device__ constexpr uint32_t tm_o(int t) { return 256u + 128u * t; }


struct KParams {
  const __nv_bfloat16 *q;
  __nv_bfloat16 *out;
  float *lse;
  const float2 *cs;
  unsigned *status;
  int B, L, Hq, Hkv, G, w, n_qtiles;
  int pair_group;  // head pairs whose CTAs are scheduled together (divides Hq / 2)
  int band;   // kBandNone, kBandStd or kBandRem
  int q_off;  // position of query row 0 (a multiple of 128; keys start at 0)
  int key_mode;  // kKeysRaw or kKeysCached
  int n_keys;    // keys [0, n_keys) exist (q_off + L)
  float scale_log2;
};

// Rotates this thread's query row with the table at `pos` and writes it,
// bf16 and swizzled, into the 128x128 tile at `dst`.
__device__ __forceinline__ void rotate_q_row(uint8_t *dst, int r, const __nv_bfloat16 *qrow,
                                             bool row_ok, const float2 *cs, int pos) {
#pragma unroll 1
  for (int c = 0; c < 8; ++c) {
    float x1[8], x2[8];
    if (row_ok) {
      unpack8(*reinterpret_cast<const uint4 *>(qrow + 8 * c), x1);
      unpack8(*reinterpret_cast<const uint4 *>(qrow + 64 + 8 * c), x2);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x1[e] = x2[e] = 0.f;
    }
    const float2 *t = cs + static_cast<int64_t>(pos) * 64 + 8 * c;
    uint32_t lo[4], hi[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 r0 = __ldg(t + 2 * e), r1 = __ldg(t + 2 * e + 1);
      lo[e] = pack_bf16x2(x1[2 * e] * r0.x - x2[2 * e] * r0.y,
                          x1[2 * e + 1] * r1.x - x2[2 * e + 1] * r1.y);
      hi[e] = pack_bf16x2(x1[2 * e] * r0.y + x2[2 * e] * r0.x,
                          x1[2 * e + 1] * r1.y + x2[2 * e + 1] * r1.x);
    }
    *reinterpret_cast<uint4 *>(dst + swz(r, c)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    *reinterpret_cast<uint4 *>(dst + kHalfBytes + swz(r, c)) =
        make_uint4(hi[0], hi[1], hi[2], hi[3]);
  }
}

// kGeneral: band passes or a query offset (the unfused three-call path and
// chunked prefill); the default prefill runs the instantiation without them.
// kRotate: the softmax threads rotate the K tiles (raw or cached keys); false
// when the keys were rotated once per call beforehand, so that the copy of the
// loop that reads them carries no rotation code.
template <bool kGeneral, bool kRotate>
__global__ void __launch_bounds__(kThreads, 1)
    bifocal_prefill_sm100_x2_kernel(const __grid_constant__ CUtensorMap tm_k,
                                    const __grid_constant__ CUtensorMap tm_krem,
                                    const __grid_constant__ CUtensorMap tm_v,
                                    const KParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int band = kGeneral ? p.band : kBandNone;
  const int q_off = kGeneral ? p.q_off : 0;

  // CTA order: groups of pair_group head pairs (whole kv heads) of one batch
  // entry in turn; within a group the heaviest query tiles first, the pairs
  // of one tile next to each other.  The CTAs that run together then share
  // one kv head and start their walks over its K/V tiles at nearly the same
  // time, so each tile comes from DRAM about once per wave of CTAs.
  const int pairs = p.Hq / 2;
  const int pg = p.pair_group;
  const int per_group = p.n_qtiles * pg;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int r_in = static_cast<int>(blockIdx.x) % per_group;
  const int qt = p.n_qtiles - 1 - r_in / pg;
  const int hq0 = 2 * ((grp % (pairs / pg)) * pg + r_in % pg);
  const int b = grp / (pairs / pg);
  const int hk = hq0 / (p.Hq / p.Hkv);

  volatile int *abort_s = reinterpret_cast<volatile int *>(smem + kOffAbort);
  volatile unsigned *abort_g = p.status;
  auto bar = [&](int i) { return sb + kOffBar + 8u * static_cast<uint32_t>(i); };

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(kBarQReady + t), 128);
      mbar_init(bar(kBarSFull + t), 1);
      for (int c = 0; c < 2; ++c) mbar_init(bar(kBarPFull + 4 * t + c), 128);
      mbar_init(bar(kBarODone + t), 1);
    }
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarKRot + s), kRotThreads);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_s = 0;
    *reinterpret_cast<volatile int *>(smem + kOffSkip) = (*abort_g != 0u) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(sb + kOffTmemSlot, kTmemCols);
    tmem_relinquish();
  }
  // the key rotation's step factors: table row 1, (cos, sin)(theta_i), as
  // float4 entry 8 e2 + c = pairs 8c + 2 e2 and 8c + 2 e2 + 1
  if (threadIdx.x < 32) {
    const int i0 = 8 * (threadIdx.x & 7) + 2 * (threadIdx.x >> 3);
    const float2 a = p.cs[64 + i0], b2 = p.cs[64 + i0 + 1];
    reinterpret_cast<float4 *>(smem + kOffStep)[threadIdx.x] = make_float4(a.x, a.y, b2.x, b2.y);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + kOffTmemSlot);
  const bool skip = *reinterpret_cast<volatile int *>(smem + kOffSkip) != 0;

  if (!skip) {
    // Registers are launched at 168 a thread; the producer/MMA warpgroup gives
    // 96 back per thread so that each softmax thread may hold a whole S row
    // (2 x 128 x 216 + 128 x 72 = 384 x 168).  Each warpgroup changes its
    // budget inside its own branch, so that the compiler allocates each role's
    // code within that role's budget.
    if (warp < 8) {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
      // --------------------------------------------- softmax warpgroups --
      const int t = warp >> 2;           // head of this warpgroup
      const int r = threadIdx.x & 127;   // query row == TMEM lane
      const int hq = hq0 + t;
      const int row_i = kBM * qt + r;    // row of the q / out / lse tensors
      const int qpos = q_off + row_i;  // its position
      const bool row_ok = row_i < p.L;
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
      const uint32_t s_col = lane_base + tm_s(t);
      const uint32_t o_col = lane_base + tm_o(t);
      uint8_t *qdst = smem + (t == 0 ? kOffQ0 : kOffQ1);
      const __nv_bfloat16 *qrow =
          p.q + ((static_cast<int64_t>(b) * p.L + (row_ok ? row_i : 0)) * p.Hq + hq) * kHD;
      const int pos_std = row_ok ? qpos : 0;
      const int pos_rem = row_ok ? qpos / p.G : 0;

      PassIter it;
      it.begin(qt + q_off / kBM, p.w, band);
      // first Q variant = the class of the first pass
      rotate_q_row(qdst, r, qrow, row_ok, p.cs, it.kind() == kRem ? pos_rem : pos_std);
      fence_proxy_async_smem();
      mbar_arrive(bar(kBarQReady + t));

      // K rotation: this thread's slice of every K tile of the walk, tile n
      // (stage n % kKStages) two passes ahead of the softmax
      KeySlice ks;
      ks.c = r & 7;
      ks.kl = 64 * t + 4 * (r >> 3);
      const float2 *step = reinterpret_cast<const float2 *>(smem + kOffStep);
      PassIter rit;
      rit.begin(qt + q_off / kBM, p.w, band);
      int rot_n = 0;
      // with the keys rotated beforehand there is nothing to do: the MMA warp
      // then waits for the K tiles themselves
      auto rotate_next = [&]() -> bool {
        if (!kRotate || rit.done()) return true;
        const int s = rot_n % kKStages;
        // uniform across the warp, like every wait of the softmax warps
        if (!warp_wait(bar(kBarKFull + s), (rot_n / kKStages) & 1, abort_s, abort_g))
          return false;
        ks.rotate(smem + kOffK + s * kTileBytes, p.cs, step, kBN * rit.j, rit.kind(), p.key_mode,
                  p.G, p.n_keys);
        fence_proxy_async_smem();  // the tensor core reads the tile through the async proxy
        mbar_arrive(bar(kBarKRot + s));
        ++rot_n;
        rit.next();
        return true;
      };
      bool ok = rotate_next() && rotate_next();

      float m = -INFINITY, l = 0.f;
      int j = 0;
      while (ok && !it.done()) {
        if (kRotate && !rit.done())  // the next slice's table entries, into L1 during the wait
          ks.prefetch(p.cs, kBN * rit.j, rit.kind(), p.key_mode, p.G, p.n_keys);
        if (!warp_wait(bar(kBarSFull + t), j & 1, abort_s, abort_g)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int kind = it.kind();
        const int mk = it.mask();
        const int kj = it.j;
        it.next();
        if (kind == kRem && !it.done() && it.kind() == kStd) {
          // last remote pass of this tile: its S is complete, so Q may now be
          // overwritten with the standard-position rotation
          rotate_q_row(qdst, r, qrow, row_ok, p.cs, pos_std);
          fence_proxy_async_smem();
          mbar_arrive(bar(kBarQReady + t));
        }

        const bool causal = (kj == qt + q_off / kBM);
        const bool plain = !causal && mk == kMaskNone;
        const int k0 = kBN * kj;
        // validity of column e for this row (only asked on masked tiles)
        auto valid = [&](int e) {
          const int dd = qpos - (k0 + e);
          bool v = !causal || dd >= 0;
          if (mk == kMaskFarOnly) v = v && dd >= p.w;
          if (mk == kMaskLocalOnly) v = v && dd < p.w;
          return v;
        };
        // S once: all 128 columns in registers (masked entries -> -inf)
        float sv[128];
        tmem_ld128(s_col, sv);
        if (!plain) {
#pragma unroll
          for (int e = 0; e < 128; ++e) sv[e] = valid(e) ? sv[e] : -INFINITY;
        }
        float mt;
        {
          float mx[8];
#pragma unroll
          for (int a = 0; a < 8; ++a) mx[a] = -INFINITY;
#pragma unroll
          for (int e = 0; e < 128; e += 2) mx[(e >> 1) & 7] = fmax3(mx[(e >> 1) & 7], sv[e], sv[e + 1]);
          mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
               p.scale_log2;  // scale > 0 keeps the order
        }
        const float m_new = fmaxf(m, mt);
        float alpha = 1.f;
        bool resc = false;
        if (m_new > m + 8.f) {  // lazy rescale: only when the max grows by > 2^8
          alpha = ex2_approx(m - m_new);
          m = m_new;
          resc = true;
        }
        // P = 2^(s * scale * log2(e) - m), written as bf16 into the first 64
        // columns of S (every S value is already in registers)
        const float neg_mu = (m == -INFINITY) ? 0.f : -m;
        const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
        const uint64_t nm2 = f2_pack(neg_mu, neg_mu);
        uint64_t rsum2[4] = {0ull, 0ull, 0ull, 0ull};
        // The exponent pass, in four stores of 32 keys.  P goes to the PV
        // product in two parts: the first kPSplit stores are released once
        // they have landed in TMEM (checked after the next store's
        // exponentials, so the store latency hides under them), and PV_t(j)
        // starts on them while the softmax is still on the later keys.  kPoly: unmasked tile, where the FMA-pipe 2^x may take
        // part.  kStream false: a warp that must first rescale O (the lazy
        // rule moved m) writes all of P, rescales O, then releases the chunks,
        // so that no part of PV_t(j) reaches O before the rescale.  Both are
        // compile-time choices per copy, so the unrolled loop has no branch.
        auto exp_pass = [&](auto poly_tag, auto stream_tag) {
          constexpr bool kPoly = decltype(poly_tag)::value;
          constexpr bool kStream = decltype(stream_tag)::value;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int i0 = 32 * c + 2 * e;
              float p0, p1;
              const uint64_t x2 = f2_fma(f2_pack(sv[i0], sv[i0 + 1]), sc2, nm2);
              if constexpr (kPoly) {
                if (poly_pair(16 * c + e)) {
                  f2_unpack(exp2_poly2(x2), p0, p1);
                } else {
                  float x0, x1;
                  f2_unpack(x2, x0, x1);
                  p0 = ex2_approx(x0);
                  p1 = ex2_approx(x1);
                }
              } else {
                float x0, x1;
                f2_unpack(x2, x0, x1);
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              rsum2[e & 3] = f2_add(rsum2[e & 3], f2_pack(p0, p1));
              pk[e] = pack_bf16x2(p0, p1);
            }
            if constexpr (kStream) {
              if (c == kPSplit) {  // the first part has landed: release it
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(kBarPFull + 4 * t));
              }
            }
            // every S value is in registers, so P may overwrite any S column
            tmem_st16_nowait(s_col + 16 * c, pk);
          }
          tmem_wait_st();
        };
        // O_t is stable during this pass: its last product was issued before
        // this S, and this S's completion covers it.  The TMEM access is
        // warp-collective, so the choice is made per warp.
        const bool rescale_o = j > 0 && __any_sync(0xffffffffu, resc && l > 0.f);
        if (!rescale_o) {
          if (kPolyPairs > 0 && plain)
            exp_pass(std::true_type{}, std::true_type{});
          else
            exp_pass(std::false_type{}, std::true_type{});
          tc_fence_before();
          mbar_arrive(bar(kBarPFull + 4 * t + 1));
        } else {
          exp_pass(std::false_type{}, std::false_type{});
          // (after P, so that S is no longer live)
          const float a = (resc && l > 0.f) ? alpha : 1.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(o_col + 32 * c, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= a;
            tmem_st32(o_col + 32 * c, o);
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(bar(kBarPFull + 4 * t));
          mbar_arrive(bar(kBarPFull + 4 * t + 1));
        }
        float rs;
        {
          float r0, r1;
          f2_unpack(f2_add(f2_add(rsum2[0], rsum2[1]), f2_add(rsum2[2], rsum2[3])), r0, r1);
          rs = r0 + r1;
        }
        l = l * alpha + rs;
        ++j;
        // the tile two passes ahead, while this head's next S is computed
        if (!rotate_next()) {
          ok = false;
          break;
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (ok && !warp_wait(bar(kBarODone + t), (j - 1) & 1, abort_s, abort_g)) ok = false;
      if (!ok) {
        raise_abort(abort_s, p.status);
      } else {
        tc_fence_after();
        const float inv = 1.f / l;
        __nv_bfloat16 *orow =
            p.out + ((static_cast<int64_t>(b) * p.L + (row_ok ? row_i : 0)) * p.Hq + hq) * kHD;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(o_col + 32 * c, o);
          if (row_ok) {
#pragma unroll
            for (int g = 0; g < 4; ++g) {
              uint4 w4;
              w4.x = pack_bf16x2(o[8 * g + 0] * inv, o[8 * g + 1] * inv);
              w4.y = pack_bf16x2(o[8 * g + 2] * inv, o[8 * g + 3] * inv);
              w4.z = pack_bf16x2(o[8 * g + 4] * inv, o[8 * g + 5] * inv);
              w4.w = pack_bf16x2(o[8 * g + 6] * inv, o[8 * g + 7] * inv);
              *reinterpret_cast<uint4 *>(orow + 32 * c + 8 * g) = w4;
            }
          }
        }
        if (row_ok)
          p.lse[(static_cast<int64_t>(b) * p.Hq + hq) * p.L + row_i] =
              (m + __log2f(l)) * 0.69314718055994530942f;
      }
    } else {
     asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsWg2));
     if (warp == kProducerWarp || warp == kVProducerWarp) {
      // ------------------------------------------- TMA producers (K and V) --
      // Warp 8 loads the raw K tiles of the walk into a kKStages ring, warp 10
      // the V tiles into a kVStages ring; pass n's tiles sit in stage
      // n % stages of each.
      if (lane == 0) {
        const bool is_k = warp == kProducerWarp;
        const CUtensorMap *vmap = &tm_v;
        const int stages = is_k ? kKStages : kVStages;
        const uint32_t base = sb + (is_k ? kOffK : kOffV);
        const int full = is_k ? kBarKFull : kBarVFull, empty = is_k ? kBarKEmpty : kBarVEmpty;
        prefetch_tmap(is_k ? &tm_k : vmap);
        if (is_k && p.key_mode == kKeysRotated) prefetch_tmap(&tm_krem);
        PassIter it;
        it.begin(qt + q_off / kBM, p.w, band);
        int n = 0;
        while (!it.done()) {
          const int s = n % stages;
          if (!mbar_wait(bar(empty + s), ((n / stages) & 1) ^ 1u, abort_s, abort_g, kTimeoutNs)) {
            raise_abort(abort_s, p.status);
            break;
          }
          // K: the raw tile, or with the keys rotated once per call, the copy
          // of this pass's class
          const CUtensorMap *map =
              !is_k ? vmap : (p.key_mode == kKeysRotated && it.kind() == kRem ? &tm_krem : &tm_k);
          mbar_arrive_expect_tx(bar(full + s), kTileBytes);
          tma_load_4d(base + s * kTileBytes, map, bar(full + s), 0, hk, kBN * it.j, b);
          tma_load_4d(base + s * kTileBytes + kHalfBytes, map, bar(full + s), 64, hk, kBN * it.j,
                      b);
          ++n;
          it.next();
        }
        // never leave with a copy in flight into this CTA's shared memory
        for (int d = (n > stages ? n - stages : 0); d < n; ++d)
          drain_wait(bar(full + d % stages), (d / stages) & 1);
      }
      __syncwarp();
    } else if (warp == kMmaWarp) {
      // ------------------------------------------------------- MMA issuer --
      if (lane == 0) {
        const uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, 0, 0);
        const uint32_t idesc_pv = idesc_bf16_f32(kBM, kHD, 0, 1);
        auto wait = [&](int i, uint32_t parity) {
          return mbar_wait(bar(i), parity, abort_s, abort_g, kTimeoutNs);
        };
        // Issue order (one thread, so the tensor core runs it in order):
        //   S_0(0) S_1(0) | PV_0(0) S_0(1) PV_1(0) S_1(1) | PV_0(1) S_0(2) ...
        // S_t(j+1) overwrites the columns P_t(j) lives in; it is issued after
        // PV_t(j), which has read them.  While head t's softmax runs on S_t(j),
        // the tensor core works on head 1-t.
        PassIter it;
        it.begin(qt + q_off / kBM, p.w, band);
        bool ok = true;
        int qphase[2] = {0, 0};
        auto issue_s = [&](int t, int jj, int kind_changed) -> bool {
          const int s = jj % kKStages;
          if (kind_changed) {
            if (!wait(kBarQReady + t, qphase[t] & 1)) return false;
            ++qphase[t];
          }
          // the tile rotated by the softmax threads, or as loaded when the
          // keys were rotated beforehand
          if (t == 0 && !wait((kRotate ? kBarKRot : kBarKFull) + s, (jj / kKStages) & 1))
            return false;
          tc_fence_after();
          const uint32_t a0 = sb + (t == 0 ? kOffQ0 : kOffQ1);
          const uint32_t b0 = sb + kOffK + s * kTileBytes;
          auto score_steps = [&](int kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            umma_bf16(tmem + tm_s(t), sdesc_sw128(a0 + off, 16, 1024),
                      sdesc_sw128(b0 + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
          };
          // Measured on a B200 at L = 131072 (same box, ms per call): issuing
          // the eight steps as a rolled loop is faster while the softmax
          // threads rotate the keys (172.5 against 180), the unrolled
          // sequence when the keys were rotated beforehand (135 against 145).
          if constexpr (!kRotate) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) score_steps(kk);
          } else {
#pragma unroll 1
            for (int kk = 0; kk < 8; ++kk) score_steps(kk);
          }
          umma_commit(bar(kBarSFull + t));
          if (t == 1) umma_commit(bar(kBarKEmpty + s));  // both heads' S issued
          return true;
        };
        auto issue_pv = [&](int t, int jj) -> bool {
          const int s = jj % kVStages;
          if (t == 0 && !wait(kBarVFull + s, (jj / kVStages) & 1)) return false;
          const uint32_t vb = sb + kOffV + s * kTileBytes;
          // P_t arrives in two parts; each is multiplied as soon as it is
          // released.  Each part's steps are a loop with compile-time bounds
          // and no exit, so it unrolls into a branch-free issue sequence (one
          // loop with the second wait inside it measured 4-8% slower).
          auto steps = [&](auto k0_tag, auto k1_tag) {
#pragma unroll
            for (int kk = decltype(k0_tag)::value; kk < decltype(k1_tag)::value; ++kk)
              umma_bf16_ts(tmem + tm_o(t), tmem + tm_s(t) + 8 * kk,
                           sdesc_sw128(vb + kk * 2048, kHalfBytes, 1024), idesc_pv,
                           (jj > 0 || kk > 0) ? 1u : 0u);
          };
          if (!wait(kBarPFull + 4 * t, jj & 1)) return false;
          tc_fence_after();
          steps(std::integral_constant<int, 0>{}, std::integral_constant<int, 2 * kPSplit>{});
          if (!wait(kBarPFull + 4 * t + 1, jj & 1)) return false;
          tc_fence_after();
          steps(std::integral_constant<int, 2 * kPSplit>{}, std::integral_constant<int, 8>{});
          umma_commit(bar(kBarODone + t));
          if (t == 1) umma_commit(bar(kBarVEmpty + s));
          return true;
        };
        int j = 0;
        int kind = it.kind();
        ok = issue_s(0, 0, 1) && issue_s(1, 0, 1);
        while (ok && !it.done()) {
          it.next();
          const bool more = !it.done();
          const int next_kind = more ? it.kind() : kind;
          const int changed = more && next_kind != kind;
          ok = issue_pv(0, j) && (!more || issue_s(0, j + 1, changed)) && issue_pv(1, j) &&
               (!more || issue_s(1, j + 1, changed));
          kind = next_kind;
          ++j;
        }
        if (!ok) raise_abort(abort_s, p.status);
        umma_commit(bar(kBarDrain));
        drain_wait(bar(kBarDrain), 0);
      }
      __syncwarp();
     }
    }
  }
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
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

bool make_map(CUtensorMap *m, const void *base, int B, int L, int H, int64_t stride_L = 0) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHD), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHD) * 2,
                                 static_cast<cuuint64_t>(H) * kHD * 2,
                                 static_cast<cuuint64_t>(stride_L > 0 ? stride_L : L) * H * kHD * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(kBN), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool prefill_x2_supported(const PrefillArgs &a) { return (a.Hq / a.Hkv) % 2 == 0; }

cudaError_t launch_prefill_sm100_x2(const PrefillArgs &a, cudaStream_t s) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    const void *fns[3] = {reinterpret_cast<const void *>(bifocal_prefill_sm100_x2_kernel<false, true>),
                          reinterpret_cast<const void *>(bifocal_prefill_sm100_x2_kernel<true, true>),
                          reinterpret_cast<const void *>(bifocal_prefill_sm100_x2_kernel<false, false>)};
    for (const void *fn : fns) {
      if (attr_err == cudaSuccess)
        attr_err = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    }
  });
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap mk, mkr, mv;
  // keys [0, q_off + L); a cache may be longer per batch entry than that
  // (kv_stride keys)
  const int keys = a.q_off + a.L;
  const int64_t kvs = a.kv_stride > 0 ? a.kv_stride : keys;
  if (!make_map(&mk, a.k, a.B, keys, a.Hkv, kvs) ||
      !make_map(&mkr, a.k_rem ? a.k_rem : a.k, a.B, keys, a.Hkv, kvs) ||
      !make_map(&mv, a.v, a.B, keys, a.Hkv, kvs))
    return cudaErrorInvalidValue;
  KParams p;
  p.q = static_cast<const __nv_bfloat16 *>(a.q);
  p.out = static_cast<__nv_bfloat16 *>(a.out);
  p.lse = a.lse;
  p.cs = a.table.cs;
  p.status = a.status;
  p.B = a.B;
  p.L = a.L;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.G;
  p.w = a.w_eff;
  p.band = a.band;
  p.q_off = a.q_off;
  p.key_mode = a.key_mode;
  p.n_keys = keys;
  p.n_qtiles = (a.L + kBM - 1) / kBM;
  {
    // whole kv heads per group: kKvPerGroup of them (all when fewer)
    const int pairs = a.Hq / 2, per_kv = (a.Hq / a.Hkv) / 2;
    int pg = per_kv * kKvPerGroup;
    if (pg > pairs || pairs % pg != 0) pg = pairs;
    p.pair_group = pg;
  }
  p.scale_log2 = a.scale * 1.4426950408889634f;
  const int64_t grid = static_cast<int64_t>(p.n_qtiles) * a.B * (a.Hq / 2);
  const unsigned g = static_cast<unsigned>(grid);
  const bool general = a.band != 0 || a.q_off != 0;
  if (a.key_mode != kKeysRotated) {
    if (general)
      bifocal_prefill_sm100_x2_kernel<true, true><<<g, kThreads, kSmemAlloc, s>>>(mk, mkr, mv, p);
    else
      bifocal_prefill_sm100_x2_kernel<false, true><<<g, kThreads, kSmemAlloc, s>>>(mk, mkr, mv, p);
  } else {
    // keys rotated once per call: only the plain prefill call (no band, no
    // query offset) takes that mode
    if (general) return cudaErrorInvalidValue;
    bifocal_prefill_sm100_x2_kernel<false, false><<<g, kThreads, kSmemAlloc, s>>>(mk, mkr, mv, p);
  }
  return cudaGetLastError();
}

}  // namespace jl
