// jl_plan.cu -- the batched decode's plan, made on the device.
//
// The same plan as the host planner of jl_bifocal_decode_batched (one wave of
// CTAs over all sequences' keys; each sequence's remote range [0, far_end) and
// local range [far_end, pos] cut into chunks of at most `chunk` keys, a
// multiple of 16, aiming at max(16, 148 - 2B) chunks), computed by one CTA from
// a DEVICE array of positions, so that a decode step reads no host data and
// can be captured in a CUDA graph.  A position outside [0, cap) raises the
// device status word and is planned as position 0 (no key outside the cache
// is ever read).  The entries are written in the host planner's order
// (sequence by sequence, remote chunks first), so a call planned here computes
// bit for bit what a host-planned call does.
#include "jl_internal.h"

namespace jl {
namespace {

constexpr int kPlanThreads = 1024;

__device__ __forceinline__ long long group_size_dev(long long L, long long w) {
  const long long g = (L + w - 1) / w;
  return g < 1 ? 1 : g;
}

// exclusive prefix sum over the CTA (1024 threads); returns this thread's
// offset and writes the CTA total to *total
__device__ int block_exclusive_scan(int v, int *total) {
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += y;
    }
    warp_sums[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int warp_base = warp > 0 ? warp_sums[warp - 1] : 0;
  *total = warp_sums[31];
  __syncthreads();
  return warp_base + incl - v;
}

__global__ void __launch_bounds__(kPlanThreads)
    decode_plan_kernel(const int *__restrict__ pos_in, int B, int cap, int w_local,
                       int w_pretrained, int plain_flag, int Hq, int n_max,
                       DecodeWork *__restrict__ work, DecodeSeq *__restrict__ seqs,
                       int *__restrict__ n_work, unsigned *__restrict__ status) {
  __shared__ unsigned long long s_total;
  __shared__ long long s_chunk;
  __shared__ int s_base;
  // total keys over the batch
  unsigned long long mine = 0;
  for (int b = threadIdx.x; b < B; b += kPlanThreads) {
    int p = pos_in[b];
    if (p < 0 || p >= cap) p = 0;
    mine += static_cast<unsigned long long>(p) + 1;
  }
  if (threadIdx.x == 0) s_total = 0;
  __syncthreads();
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, off);
  if ((threadIdx.x & 31) == 0) atomicAdd(&s_total, mine);
  __syncthreads();
  if (threadIdx.x == 0) {
    const long long total = static_cast<long long>(s_total);
    const long long target = kDecodeBatchCtas - 2LL * B > 16 ? kDecodeBatchCtas - 2LL * B : 16;
    long long chunk = (total + target - 1) / target;
    chunk = ((chunk + 15) / 16) * 16;
    if (chunk < 16) chunk = 16;
    s_chunk = chunk;
    s_base = 0;
  }
  __syncthreads();
  const long long chunk = s_chunk;
  // sequences in rounds of 1024: counts, offsets, entries
  for (int b0 = 0; b0 < B; b0 += kPlanThreads) {
    const int b = b0 + static_cast<int>(threadIdx.x);
    int p = 0, far_end = 0, n_rem = 0, n_loc = 0;
    long long G = 1;
    if (b < B) {
      p = pos_in[b];
      if (p < 0 || p >= cap) {
        atomicOr(status, kStatusBounds);
        p = 0;
      }
      G = group_size_dev(static_cast<long long>(p) + 1, w_pretrained);
      const bool plain = plain_flag || G == 1;
      const long long fe = static_cast<long long>(p) + 1 - w_local;
      far_end = plain ? 0 : static_cast<int>(fe < 0 ? 0 : fe);
      n_rem = static_cast<int>((far_end + chunk - 1) / chunk);
      n_loc = static_cast<int>((static_cast<long long>(p) + 1 - far_end + chunk - 1) / chunk);
    }
    int round_total = 0;
    const int off = block_exclusive_scan(n_rem + n_loc, &round_total);
    const int first = s_base + off;
    if (b < B) {
      seqs[b].first = first;
      seqs[b].n = n_rem + n_loc;
      const unsigned long long magic =
          G >= 2 ? (~0ull / static_cast<unsigned long long>(G)) + 1ull : 0ull;
      int idx = first;
      auto cut = [&](int lo, int hi, int far) {
        for (long long k0 = lo; k0 < hi; k0 += chunk, ++idx) {
          if (idx >= n_max) {  // cannot happen with the rule above; refuse, do not overrun
            atomicOr(status, kStatusBounds);
            return;
          }
          DecodeWork w;
          w.b = b;
          w.k_begin = static_cast<int>(k0);
          w.k_end = static_cast<int>(k0 + chunk < hi ? k0 + chunk : hi);
          w.far = far;
          w.pos = p;
          w.G = static_cast<int>(G);
          w.part = idx * Hq;
          w.pad = 0;
          w.g_magic = magic;
          work[idx] = w;
        }
      };
      cut(0, far_end, 1);
      cut(far_end, p + 1, 0);
    }
    __syncthreads();
    if (threadIdx.x == 0) s_base += round_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const int n = s_base;
    *n_work = n <= n_max ? n : 0;
    if (n > n_max) atomicOr(status, kStatusBounds);
  }
}

}  // namespace

cudaError_t launch_decode_plan(const int *pos, int B, int cap, int w_local, int w_pretrained,
                               bool plain, int Hq, int n_max, DecodeWork *work,
                               DecodeSeq *seqs, int *n_work, unsigned *status,
                               cudaStream_t s) {
  decode_plan_kernel<<<1, kPlanThreads, 0, s>>>(pos, B, cap, w_local, w_pretrained,
                                                plain ? 1 : 0, Hq, n_max, work, seqs, n_work,
                                                status);
  return cudaGetLastError();
}

}  // namespace jl
