// jl_prefill_sm100.cu -- bifocal prefill attention on the sm_100a tensor cores.
//
// What it computes (Jet-Long; techwalker explainer §二/§四, bittide paper
// summary §3.1-§3.2): causal attention in which a pair (q, k) with
// q - k < w_local scores <R(q)Q, R(k)K> and every farther pair scores
// <R(f(q))Q, R(f(k))K>, f(x) = floor(x/G).  The pages reach this with three
// flash-attention calls merged by LogSumExp weights (B: full causal at
// remapped positions, A: local band at original positions, C: local band at
// remapped positions; final = B - C + A).  Here the merge is done per tile
// instead, with complementary masks, so no subtraction (and no cancellation)
// happens:
//   * a kv tile whose pairs are all remote is one pass with remapped RoPE;
//   * a kv tile whose pairs are all local is one pass with standard RoPE;
//   * a tile straddling the window edge is two passes over the same keys, one
//     per class under complementary masks.
// All passes feed one online softmax (fp32 running max and sum, base 2), so the
// epilogue's O = acc / l and lse = m + ln l are exactly the LogSumExp-weighted
// combination of the per-class partial sums.
//
// B200 design: one CTA per (batch, query head, 128-row query tile), heaviest
// tiles first.  Warp roles:
//   warps 0-3  rotate the Q tile into swizzled shared memory (remapped
//              positions for the remote passes, then, once they are done,
//              standard positions for the local passes), and run the online
//              softmax: thread r owns query row r = TMEM lane r, reads S from
//              TMEM, writes P (bf16) into one of two shared-memory buffers,
//              rescales O in TMEM when the running max grows by more than 2^8
//              (lazy rescale), and finally normalises O and stores it.  Part of
//              each row's exponentials run on the FMA pipe (exp2_poly).
//              With P double-buffered the softmax of pass j+1 overlaps the
//              product O += P V of pass j.
//   warp 4     TMA producer: raw K tile and V tile per pass into a 3-stage ring.
//   warp 5     allocates TMEM and issues every tcgen05.mma from one thread:
//              S = Q K^T (M=N=128, K=128: 8 x K16 steps) into one of two TMEM
//              S buffers, and O += P V into the TMEM O accumulator.
//   warps 6-7  idle (they complete the second warpgroup)
//   warps 8-11 rotate each K tile in shared memory, in place, to the pass's
//              positions (R(k) or R(f(k)) from the cos/sin table) before the
//              score product reads it: RoPE applied on the fly.  Four warps,
//              one per SM sub-partition.
// Registers: launched at 168 a thread (sm_100 allocates them per four warps);
// the producer/MMA warpgroup gives 96 back per thread and the softmax
// warpgroup takes 48 of them, so a softmax thread holds its whole S row
// (128 x 216 + 128 x 72 + 128 x 168 <= 384 x 168).
// Every mbarrier wait is bounded (1 s); a thread that gives up raises the
// CTA's abort flag and the device status word, after which all CTAs drain and
// return without touching their outputs further.
#include <cudaTypedefs.h>

#include <climits>
#include <mutex>
#include <type_traits>

#include "jl_prefill_common.cuh"

namespace jl {
namespace {

using namespace sm100;
using namespace prefill;

// shared-memory layout (bytes from the 1 KiB-aligned base), barriers, TMEM
constexpr int kStages = 3;
constexpr int kThreads = 384;
constexpr int kRotWarp0 = 8;  // warps 8-11 rotate the K tiles
constexpr int kRotThreads = 128;

constexpr uint32_t kOffQ = 0;  // the Q variant of the current phase
constexpr uint32_t kOffK = kOffQ + kTileBytes;
constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;

enum : int {
  kBarQFull = 0,  // phase 0: first Q variant; phase 1: Q_std after the remote passes
  kBarKFull = 1,
  kBarKEmpty = kBarKFull + kStages,
  kBarVFull = kBarKEmpty + kStages,
  kBarVEmpty = kBarVFull + kStages,
  kBarKRot = kBarVEmpty + kStages,  // [kStages] K tile rotated, kRotThreads arrivals
  kBarSFull = kBarKRot + kStages,
  kBarSFree = kBarSFull + 2,
  kBarPFull = kBarSFree + 2,  // [2] per P buffer
  kBarODone = kBarPFull + 2,  // [2] per P buffer: O += P V of that buffer done
  kBarDrain = kBarODone + 2,
  kNumBars = kBarDrain + 1
};

constexpr uint32_t kOffTmemSlot = kOffBar + kNumBars * 8;
constexpr uint32_t kOffAbort = kOffTmemSlot + 4;
constexpr uint32_t kOffSkip = kOffAbort + 4;
constexpr uint32_t kOffStep = (kOffSkip + 4 + 15) & ~15u;  // R(1) per pair (32 float4)
constexpr uint32_t kSmemUsed = kOffStep + 64 * 8;
constexpr uint32_t kSmemAlloc = kSmemUsed + 1024;  // room to align the base to 1 KiB
static_assert(kSmemAlloc <= 232448, "shared memory budget");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmS0 = 0, kTmS1 = 128, kTmO = 256;
constexpr uint32_t kTmP = 384;  // [2] P buffers, 64 columns each (bf16 pairs)

// one column pair in kPolyEvery takes 2^x on the FMA pipe (unmasked tiles);
// a value above 16 keeps every exponential on the MUFU unit.  Off by default:
// on a B200 at L = 131072 one pair in 8 costs 2% and one in 2 costs 9%.
#ifndef JL_POLY_EVERY
#define JL_POLY_EVERY 1000
#endif
constexpr int kPolyEvery = JL_POLY_EVERY;

struct KParams {
  const __nv_bfloat16 *q;
  __nv_bfloat16 *out;
  float *lse;
  const float2 *cs;
  unsigned *status;
  int B, L, Hq, Hkv, G, w, n_qtiles;
  int band;   // kBandNone, kBandStd or kBandRem
  int q_off;  // position of query row 0 (a multiple of 128; keys start at 0)
  int key_mode;  // kKeysRaw or kKeysCached
  int n_keys;    // keys [0, n_keys) exist (q_off + L)
  float scale_log2;  // softmax scale * log2(e)
};

// kGeneral: band passes or a query offset (the unfused three-call path and
// chunked prefill); the default prefill runs the instantiation without them.
template <bool kGeneral>
__global__ void __launch_bounds__(kThreads, 1)
    bifocal_prefill_sm100_kernel(const __grid_constant__ CUtensorMap tm_k,
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

  // CTA order: the query heads of one kv head of one batch entry in turn;
  // within them the heaviest query tiles first, the heads of a tile next to
  // each other.  The CTAs that run together then share one kv head and walk
  // its K/V tiles at nearly the same time, so each tile comes from DRAM about
  // once per wave of CTAs.
  const int heads = p.Hq / p.Hkv;
  const int per_group = p.n_qtiles * heads;
  const int grp = static_cast<int>(blockIdx.x) / per_group;
  const int r_in = static_cast<int>(blockIdx.x) % per_group;
  const int qt = p.n_qtiles - 1 - r_in / heads;
  const int hk = grp % p.Hkv;
  const int hq = hk * heads + r_in % heads;
  const int b = grp / p.Hkv;

  volatile int *abort_s = reinterpret_cast<volatile int *>(smem + kOffAbort);
  volatile unsigned *abort_g = p.status;
  auto bar = [&](int i) { return sb + kOffBar + 8u * static_cast<uint32_t>(i); };

  if (threadIdx.x == 0) {
    mbar_init(bar(kBarQFull), 128);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
      mbar_init(bar(kBarKRot + s), kRotThreads);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(kBarSFull + s), 1);
      mbar_init(bar(kBarSFree + s), 128);
      mbar_init(bar(kBarPFull + s), 128);
      mbar_init(bar(kBarODone + s), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_s = 0;
    *reinterpret_cast<volatile int *>(smem + kOffSkip) = (*abort_g != 0u) ? 1 : 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(sb + kOffTmemSlot, kTmemCols);
    tmem_relinquish();
  }
  // the key rotation's step factors: table row 1, (cos, sin)(theta_i), as
  // float4 entry q = pairs 4q, 4q + 1 and entry 16 + q = pairs 4q + 2, 4q + 3
  if (threadIdx.x < 32) {
    const int i0 = 4 * (threadIdx.x & 15) + 2 * (threadIdx.x >> 4);
    const float2 a = p.cs[64 + i0], b2 = p.cs[64 + i0 + 1];
    reinterpret_cast<float4 *>(smem + kOffStep)[threadIdx.x] = make_float4(a.x, a.y, b2.x, b2.y);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + kOffTmemSlot);
  const bool skip = *reinterpret_cast<volatile int *>(smem + kOffSkip) != 0;

  if (!skip) {
    if (warp < 4) {
      asm volatile("setmaxnreg.inc.sync.aligned.u32 216;");
      // ------------------------------------------------ softmax warpgroup --
      const int r = threadIdx.x;  // query row within the tile == TMEM lane
      const int row_i = kBM * qt + r;    // row of the q / out / lse tensors
      const int qpos = q_off + row_i;  // its position
      const bool row_ok = row_i < p.L;
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * warp) << 16);
      const __nv_bfloat16 *qrow =
          p.q + ((static_cast<int64_t>(b) * p.L + (row_ok ? row_i : 0)) * p.Hq + hq) * kHD;
      const int pos_std = row_ok ? qpos : 0;
      const int pos_rem = row_ok ? qpos / p.G : 0;
      // Q rotated at `pos`, bf16, in the swizzled K-major layout the UMMA
      // descriptors expect (two 64-column halves)
      auto rotate_q = [&](int pos) {
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
          const float2 *tb = p.cs + static_cast<int64_t>(pos) * 64 + 8 * c;
          uint32_t lo[4], hi[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 r0 = __ldg(tb + 2 * e), r1 = __ldg(tb + 2 * e + 1);
            lo[e] = pack_bf16x2(x1[2 * e] * r0.x - x2[2 * e] * r0.y,
                                x1[2 * e + 1] * r1.x - x2[2 * e + 1] * r1.y);
            hi[e] = pack_bf16x2(x1[2 * e] * r0.y + x2[2 * e] * r0.x,
                                x1[2 * e + 1] * r1.y + x2[2 * e + 1] * r1.x);
          }
          uint8_t *dst = smem + kOffQ;
          *reinterpret_cast<uint4 *>(dst + swz(r, c)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          *reinterpret_cast<uint4 *>(dst + kHalfBytes + swz(r, c)) =
              make_uint4(hi[0], hi[1], hi[2], hi[3]);
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(kBarQFull));
      };
      {
        PassIter t0;
        t0.begin(qt + q_off / kBM, p.w, band);
        rotate_q(t0.kind() == kRem ? pos_rem : pos_std);
      }

      float m = -INFINITY, l = 0.f;
      PassIter t;
      t.begin(qt + q_off / kBM, p.w, band);
      int it = 0;
      bool ok = true;
      while (!t.done()) {
        const int sbuf = it & 1;
        const uint32_t sph = (it >> 1) & 1;
        if (!warp_wait(bar(kBarSFull + sbuf), sph, abort_s, abort_g)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float s[128];
        tmem_ld128(lane_base + (sbuf ? kTmS1 : kTmS0), s);
        tc_fence_before();
        mbar_arrive(bar(kBarSFree + sbuf));

        const int k0 = kBN * t.j;
        const int mk = t.mask();
        const bool causal = (t.j == qt + q_off / kBM);
        const int kind = t.kind();
        t.next();
        if (kind == kRem && !t.done() && t.kind() == kStd)
          rotate_q(pos_std);  // last remote pass: its S is complete, Q may change
        // masked entries -> -inf; row max of the raw scores, 8 independent chains
        if (causal || mk != kMaskNone) {
#pragma unroll
          for (int e = 0; e < 128; ++e) {
            const int dd = qpos - (k0 + e);
            bool valid = !causal || dd >= 0;
            if (mk == kMaskFarOnly) valid = valid && dd >= p.w;
            if (mk == kMaskLocalOnly) valid = valid && dd < p.w;
            s[e] = valid ? s[e] : -INFINITY;
          }
        }
        float mx[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) mx[a] = -INFINITY;
#pragma unroll
        for (int e = 0; e < 128; e += 2) mx[(e >> 1) & 7] = fmax3(mx[(e >> 1) & 7], s[e], s[e + 1]);
        const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                         p.scale_log2;  // scale > 0 keeps the order
        const float m_new = fmaxf(m, mt);
        float alpha = 1.f;
        bool resc = false;
        if (m_new > m + 8.f) {  // lazy rescale: only when the max grows by > 2^8
          alpha = ex2_approx(m - m_new);
          m = m_new;
          resc = true;
        }
        const int pbuf = it & 1;
        // O rescale (rare) needs the product of pass it-1 complete.  Waits on a
        // per-buffer barrier are unambiguous: the product of pass it-3 is done
        // (this pass's S completed after it) and pass it+1's cannot start.
        // The TMEM access is warp-collective.
        if (it > 0 && __any_sync(0xffffffffu, resc && l > 0.f)) {
          if (!warp_wait(bar(kBarODone + ((it - 1) & 1)), ((it - 1) >> 1) & 1, abort_s,
                         abort_g)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float a = (resc && l > 0.f) ? alpha : 1.f;
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(lane_base + kTmO + 32 * c, o);
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= a;
            tmem_st32(lane_base + kTmO + 32 * c, o);
          }
        }
        // P = 2^(s * scale * log2(e) - m) on pairs of columns with packed fp32
        // arithmetic (-inf gives 0); in unmasked tiles one pair in kPolyEvery
        // takes the FMA-pipe polynomial instead of two MUFU exponentials, so
        // the MUFU unit is not the only bound.  Column j of the P buffer (TMEM,
        // bf16) holds keys (2j, 2j+1); that buffer was last read by the
        // product of pass it-2, complete before this S.
        const bool plain = !causal && mk == kMaskNone;
        const float neg_mu = (m == -INFINITY) ? 0.f : -m;
        const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
        const uint64_t nm2 = f2_pack(neg_mu, neg_mu);
        uint64_t rsum2[4] = {0ull, 0ull, 0ull, 0ull};
        const uint32_t pcol = lane_base + kTmP + 64 * pbuf;
        // two copies of the loop so that neither has a branch inside
        auto exp_row = [&](auto with_poly) {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t pk[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int j = 16 * c4 + q;
              const uint64_t x2 = f2_fma(f2_pack(s[2 * j], s[2 * j + 1]), sc2, nm2);
              uint64_t p2;
              if (decltype(with_poly)::value && (q % kPolyEvery) == kPolyEvery - 1) {
                p2 = exp2_poly2(x2);
              } else {
                float a, b;
                f2_unpack(x2, a, b);
                p2 = f2_pack(ex2_approx(a), ex2_approx(b));
              }
              rsum2[q & 3] = f2_add(rsum2[q & 3], p2);
              float p0, p1;
              f2_unpack(p2, p0, p1);
              pk[q] = pack_bf16x2(p0, p1);
            }
            tmem_st16_nowait(pcol + 16 * c4, pk);
          }
        };
        if (plain)
          exp_row(std::true_type{});
        else
          exp_row(std::false_type{});
        tmem_wait_st();
        float rs;
        {
          const uint64_t r2 = f2_add(f2_add(rsum2[0], rsum2[1]), f2_add(rsum2[2], rsum2[3]));
          float r0, r1;
          f2_unpack(r2, r0, r1);
          rs = r0 + r1;
        }
        l = l * alpha + rs;
        tc_fence_before();
        mbar_arrive(bar(kBarPFull + pbuf));
        ++it;
      }
      ok = __all_sync(0xffffffffu, ok);
      // the last product (in-order completion: every earlier one is done too)
      if (ok && !warp_wait(bar(kBarODone + ((it - 1) & 1)), ((it - 1) >> 1) & 1, abort_s,
                           abort_g))
        ok = false;
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
          tmem_ld32(lane_base + kTmO + 32 * c, o);
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
    } else if (warp < kRotWarp0) {
     asm volatile("setmaxnreg.dec.sync.aligned.u32 72;");
     if (warp == 4) {
      // ------------------------------------------------------ TMA producer --
      if (lane == 0) {
        prefetch_tmap(&tm_k);
        if (p.key_mode == kKeysRotated) prefetch_tmap(&tm_krem);
        prefetch_tmap(&tm_v);
        PassIter t;
        t.begin(qt + q_off / kBM, p.w, band);
        int kiss = 0, viss = 0;  // loads issued
        while (!t.done()) {
          const int s = kiss % kStages;
          const uint32_t ph = (kiss / kStages) & 1;
          if (!mbar_wait(bar(kBarKEmpty + s), ph ^ 1u, abort_s, abort_g, kTimeoutNs)) {
            raise_abort(abort_s, p.status);
            break;
          }
          // the raw tile, or with the keys rotated once per call, the copy of
          // this pass's class
          const CUtensorMap *km = p.key_mode == kKeysRotated && t.kind() == kRem ? &tm_krem : &tm_k;
          mbar_arrive_expect_tx(bar(kBarKFull + s), kTileBytes);
          tma_load_4d(sb + kOffK + s * kTileBytes, km, bar(kBarKFull + s), 0, hk, kBN * t.j, b);
          tma_load_4d(sb + kOffK + s * kTileBytes + kHalfBytes, km, bar(kBarKFull + s), 64, hk,
                      kBN * t.j, b);
          ++kiss;
          if (!mbar_wait(bar(kBarVEmpty + s), ph ^ 1u, abort_s, abort_g, kTimeoutNs)) {
            raise_abort(abort_s, p.status);
            break;
          }
          mbar_arrive_expect_tx(bar(kBarVFull + s), kTileBytes);
          tma_load_4d(sb + kOffV + s * kTileBytes, &tm_v, bar(kBarVFull + s), 0, hk, kBN * t.j, b);
          tma_load_4d(sb + kOffV + s * kTileBytes + kHalfBytes, &tm_v, bar(kBarVFull + s), 64,
                      hk, kBN * t.j, b);
          ++viss;
          t.next();
        }
        // never leave with a copy in flight into this CTA's shared memory
        for (int d = (kiss > kStages ? kiss - kStages : 0); d < kiss; ++d)
          drain_wait(bar(kBarKFull + d % kStages), (d / kStages) & 1);
        for (int d = (viss > kStages ? viss - kStages : 0); d < viss; ++d)
          drain_wait(bar(kBarVFull + d % kStages), (d / kStages) & 1);
      }
      __syncwarp();
    } else if (warp == 5) {
      // ------------------------------------------------------- MMA issuer --
      if (lane == 0) {
        const uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, 0, 0);
        const uint32_t idesc_pv = idesc_bf16_f32(kBM, kHD, 0, 1);
        bool ok = true;
        auto pv = [&](int tt) -> bool {
          const int s = tt % kStages;
          const uint32_t ph = (tt / kStages) & 1;
          const int pbuf = tt & 1;
          if (!mbar_wait(bar(kBarPFull + pbuf), (tt >> 1) & 1, abort_s, abort_g, kTimeoutNs))
            return false;
          if (!mbar_wait(bar(kBarVFull + s), ph, abort_s, abort_g, kTimeoutNs)) return false;
          tc_fence_after();
          const uint32_t pa = tmem + kTmP + 64 * pbuf;  // P from TMEM, 8 columns per step
          const uint32_t vb = sb + kOffV + s * kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {  // 16 keys per step
            const uint32_t b_off = kk * 2048;  // 16 key rows of 128 B
            umma_bf16_ts(tmem + kTmO, pa + 8 * kk, sdesc_sw128(vb + b_off, kHalfBytes, 1024),
                         idesc_pv, (tt > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(bar(kBarODone + pbuf));
          umma_commit(bar(kBarVEmpty + s));
          return true;
        };
        PassIter t;
        t.begin(qt + q_off / kBM, p.w, band);
        int it = 0, qphase = 0, prev_kind = t.kind();
        while (ok && !t.done()) {
          const int kind = t.kind();
          if (it == 0 || kind != prev_kind) {
            // the Q variant this pass needs is in shared memory
            ok = mbar_wait(bar(kBarQFull), qphase & 1, abort_s, abort_g, kTimeoutNs);
            ++qphase;
            if (!ok) break;
          }
          prev_kind = kind;
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1;
          const int sbuf = it & 1;
          const uint32_t sph = (it >> 1) & 1;
          // the tile rotated by warps 8-11, or as loaded when the keys were
          // rotated beforehand
          if (!mbar_wait(bar((p.key_mode == kKeysRotated ? kBarKFull : kBarKRot) + s), ph, abort_s,
                         abort_g, kTimeoutNs) ||
              !mbar_wait(bar(kBarSFree + sbuf), sph ^ 1u, abort_s, abort_g, kTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = sb + kOffQ;
          const uint32_t b0 = sb + kOffK + s * kTileBytes;
          const uint32_t d = tmem + (sbuf ? kTmS1 : kTmS0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {  // 16 head dims per step
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            umma_bf16(d, sdesc_sw128(a0 + off, 16, 1024), sdesc_sw128(b0 + off, 16, 1024),
                      idesc_qk, kk > 0 ? 1u : 0u);
          }
          umma_commit(bar(kBarSFull + sbuf));
          umma_commit(bar(kBarKEmpty + s));
          if (it > 0 && !pv(it - 1)) {
            ok = false;
            break;
          }
          t.next();
          ++it;
        }
        if (ok && it > 0) ok = pv(it - 1);
        if (!ok) raise_abort(abort_s, p.status);
        // every issued MMA retired before TMEM is released
        umma_commit(bar(kBarDrain));
        drain_wait(bar(kBarDrain), 0);
      }
      __syncwarp();
     }
    } else {
      // -------------------------------------------------- K rotation (8-11) --
      // Pass n's K tile sits in stage n % kStages; once the TMA has landed it,
      // it is rotated in place to its pass's positions and handed to the MMA
      // warp (kBarKRot).  The producer refills a stage only after the score
      // product has read it.
      KeyRotator<kRotThreads> rot;
      rot.init(reinterpret_cast<const float2 *>(smem + kOffStep),
               static_cast<int>(threadIdx.x) - 32 * kRotWarp0);
      PassIter t;
      t.begin(qt + q_off / kBM, p.w, band);
      int n = 0;
      // with the keys rotated beforehand there is nothing to do (and nothing
      // waits for these warps: the MMA warp takes the tiles as loaded)
      while (p.key_mode != kKeysRotated && !t.done()) {
        const int s = n % kStages;
        const int k0 = kBN * t.j, kind = t.kind();
        // the table read for this tile goes out before the wait for its keys
        const auto st = rot.start(p.cs, k0, kind, p.key_mode, p.G, p.n_keys);
        if (!mbar_wait(bar(kBarKFull + s), (n / kStages) & 1, abort_s, abort_g, kTimeoutNs)) {
          raise_abort(abort_s, p.status);
          break;
        }
        rot.rotate(smem + kOffK + s * kTileBytes, st, kind, p.key_mode, p.G);
        fence_proxy_async_smem();  // the tensor core reads the tile through the async proxy
        mbar_arrive(bar(kBarKRot + s));
        ++n;
        t.next();
      }
    }
  }
  __syncthreads();
  if (warp == 5) {
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

// [B, L, H, 128] bf16 -> 4-D map (dims innermost first: D, H, L, B), box of
// 64 dims x 1 head x 128 rows, 128-byte swizzle, zero fill out of bounds.
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

cudaError_t launch_prefill_sm100(const PrefillArgs &a, cudaStream_t s) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(bifocal_prefill_sm100_kernel<false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
    if (attr_err == cudaSuccess)
      attr_err = cudaFuncSetAttribute(bifocal_prefill_sm100_kernel<true>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
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
  p.scale_log2 = a.scale * 1.4426950408889634f;
  const int64_t grid = static_cast<int64_t>(p.n_qtiles) * a.B * a.Hq;
  if (a.band != 0 || a.q_off != 0)
    bifocal_prefill_sm100_kernel<true><<<static_cast<unsigned>(grid), kThreads, kSmemAlloc, s>>>(mk, mkr, mv, p);
  else
    bifocal_prefill_sm100_kernel<false><<<static_cast<unsigned>(grid), kThreads, kSmemAlloc, s>>>(mk, mkr, mv, p);
  return cudaGetLastError();
}

}  // namespace jl
