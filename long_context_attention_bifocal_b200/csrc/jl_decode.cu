// jl_decode.cu -- single-token bifocal decode over a KV cache kept at the
// original RoPE positions (Jet-Long, techwalker explainer §三; bittide paper
// summary §3.3).
//
// The query q (pre-RoPE, position pos) becomes q_std = R(pos) q and
// q_rem = R(dq) q_std with dq = f(pos) - pos, f(x) = floor(x / G), G from
// L = pos + 1.  A cached key k_c = R(k) K with pos - k < w_local is used as is
// against q_std; a farther key is corrected in registers to R(dk) k_c,
// dk = f(k) - k (so it equals R(f(k)) K), and scored against q_rem.  Local keys
// take no correction (bittide §3.3: the mask selects which keys are rotated).
//
// B200 layout: split-KV.  A CTA owns (batch, kv head, up to 4 of its query
// heads, one chunk of keys); each chunk is wholly remote or wholly local, so
// a CTA holds one query variant.  A warp streams 4 keys per step: 8 lanes per
// key, lane s owning the rotation pairs 8s..8s+7, i.e. dims [8s, 8s+8) and
// [64+8s, 64+8s+8) -- two coalesced 16-byte loads per lane for K and two for V,
// and whole RoPE pairs in registers.  The correction angle -u*theta_i with
// u = k - f(k) >= 0 comes from two rows of the shared cos/sin table,
// u = 64*hi + lo: the row 64*hi (per lane, cached in registers) times the row
// lo (staged in shared memory), one complex product.  Scores are reduced over
// the 8 lanes with shuffles; the online softmax keeps an fp32 running max
// (base 2, rescaled only when it grows by more than 2^8) and sum per head.
// Each CTA writes (o, m, l) for its chunk; a second kernel merges the chunks
// with the same LogSumExp algebra the prefill uses and writes out and lse.
#include <climits>
#include <cmath>
#include <mutex>

#include "jl_internal.h"

namespace jl {
namespace {

constexpr int kD = 128;
constexpr int kHalf = 64;
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kTargetCtas = 4 * 148;  // about four CTAs per B200 SM

__device__ __forceinline__ void unpack8(const uint4 &u, float (&x)[8]) {
  const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[2 * j] = __uint_as_float(w4[j] << 16);
    x[2 * j + 1] = __uint_as_float(w4[j] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct SplitParams {
  const __nv_bfloat16 *q, *kc, *vc;
  float *ws;
  const float2 *cs;
  int Hq, Hkv, group, pos, cap, G, far_end, chunk, n_far, n_chunks;
  float scale_log2;
};

// theta_i = base^(-2i/D), computed on the host in fp64, for the variant that
// evaluates its angles itself
struct Thetas {
  double t[kHalf];
};

// (cos, sin)(row * theta_pair) as fp32: read from the library's table, or, in
// the table-free variant, evaluated here the same way the table was built
// (fp64 sincos of the fp64 angle, rounded once).
template <bool kSelfAngles>
__device__ __forceinline__ float2 angle(const SplitParams &p, const double *theta, int64_t row,
                                        int pair) {
  if constexpr (kSelfAngles) {
    double s, c;
    sincos(static_cast<double>(row) * theta[pair], &s, &c);
    return make_float2(static_cast<float>(c), static_cast<float>(s));
  } else {
    return p.cs[row * kHalf + pair];
  }
}

template <int NH, bool kSelfAngles>
__device__ __forceinline__ void decode_split_body(const SplitParams &p, const double *theta) {
  // cos/sin rows 0..63 as float4 [row][pair-pair e2][lane slot sl]:
  // (cos, sin) of pairs 8*sl + 2*e2 and 8*sl + 2*e2 + 1 -- 8 lanes of a key
  // read 128 contiguous bytes per load (32 KiB total)
  __shared__ float4 tlo[64 * 4 * 8];
  __shared__ float red[kWarps][NH][kD + 2];

  const int c = blockIdx.x;
  const int ngroups = p.group / NH;
  const int hk = blockIdx.y / ngroups;
  const int h0 = hk * p.group + (blockIdx.y % ngroups) * NH;
  const int b = blockIdx.z;
  const bool far = c < p.n_far;
  int k_begin, k_end;
  if (far) {
    k_begin = c * p.chunk;
    k_end = min(p.far_end, k_begin + p.chunk);
  } else {
    k_begin = p.far_end + (c - p.n_far) * p.chunk;
    k_end = min(p.pos + 1, k_begin + p.chunk);
  }

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 3;   // key slot within the warp's 4
  const int sl = lane & 7;   // rotation pairs 8*sl .. 8*sl+7

  if (far) {
    for (int i = threadIdx.x; i < 64 * 4 * 8; i += kThreads) {
      const int row = i >> 5, e2 = (i >> 3) & 3, s8 = i & 7;
      const float2 a = angle<kSelfAngles>(p, theta, row, 8 * s8 + 2 * e2);
      const float2 bq = angle<kSelfAngles>(p, theta, row, 8 * s8 + 2 * e2 + 1);
      tlo[i] = make_float4(a.x, a.y, bq.x, bq.y);
    }
  }

  // q for this lane's pairs, rotated (q_std, then q_rem = R(dq) q_std for a
  // remote chunk) and pre-scaled by scale * log2(e).
  float q1[NH][8], q2[NH][8];
  {
    const int udq = p.pos - p.pos / p.G;  // -dq >= 0
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const __nv_bfloat16 *src = p.q + (static_cast<int64_t>(b) * p.Hq + h0 + h) * kD;
      float x1[8], x2[8];
      unpack8(*reinterpret_cast<const uint4 *>(src + 8 * sl), x1);
      unpack8(*reinterpret_cast<const uint4 *>(src + kHalf + 8 * sl), x2);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float2 a = angle<kSelfAngles>(p, theta, p.pos, 8 * sl + e);
        float y1 = x1[e] * a.x - x2[e] * a.y;
        float y2 = x1[e] * a.y + x2[e] * a.x;
        if (far) {  // rotate by dq = -udq: angle -udq*theta
          const float2 r = angle<kSelfAngles>(p, theta, udq, 8 * sl + e);
          const float z1 = y1 * r.x + y2 * r.y;
          const float z2 = y2 * r.x - y1 * r.y;
          y1 = z1;
          y2 = z2;
        }
        q1[h][e] = y1 * p.scale_log2;
        q2[h][e] = y2 * p.scale_log2;
      }
    }
  }
  __syncthreads();

  float o1[NH][8], o2[NH][8], m[NH], l[NH];
#pragma unroll
  for (int h = 0; h < NH; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o1[h][e] = o2[h][e] = 0.f;
  }
  int hi_cached = -1;
  float2 thi[8];

  const int64_t row_stride = static_cast<int64_t>(p.Hkv) * kD;
  const __nv_bfloat16 *kbase = p.kc + (static_cast<int64_t>(b) * p.cap * p.Hkv + hk) * kD;
  const __nv_bfloat16 *vbase = p.vc + (static_cast<int64_t>(b) * p.cap * p.Hkv + hk) * kD;

  // Every lane runs every step (the shuffles need the full warp); a slot past
  // the chunk end loads nothing and skips the softmax update.
  for (int k0 = k_begin; k0 < k_end; k0 += 4 * kWarps) {
    const int kq = k0 + warp * 4 + g;
    const bool valid = kq < k_end;
    const int kk = valid ? kq : k_begin;
    const __nv_bfloat16 *kr = kbase + kk * row_stride;
    const __nv_bfloat16 *vr = vbase + kk * row_stride;
    uint4 ku1 = make_uint4(0, 0, 0, 0), ku2 = ku1, vu1 = ku1, vu2 = ku1;
    if (valid) {
      ku1 = *reinterpret_cast<const uint4 *>(kr + 8 * sl);
      ku2 = *reinterpret_cast<const uint4 *>(kr + kHalf + 8 * sl);
      vu1 = *reinterpret_cast<const uint4 *>(vr + 8 * sl);
      vu2 = *reinterpret_cast<const uint4 *>(vr + kHalf + 8 * sl);
    }
    float k1[8], k2[8];
    unpack8(ku1, k1);
    unpack8(ku2, k2);
    if (far) {
      // rotate by dk = f(k) - k = -u
      const int u = kk - kk / p.G;
      const int hi = u >> 6, lo = u & 63;
      if (hi != hi_cached) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          thi[e] = angle<kSelfAngles>(p, theta, static_cast<int64_t>(hi) * 64, 8 * sl + e);
        hi_cached = hi;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float4 t4 = tlo[(lo * 4 + (e >> 1)) * 8 + sl];
        const float2 tl = (e & 1) ? make_float2(t4.z, t4.w) : make_float2(t4.x, t4.y);
        const float cu = thi[e].x * tl.x - thi[e].y * tl.y;  // cos(u theta)
        const float su = thi[e].y * tl.x + thi[e].x * tl.y;  // sin(u theta)
        const float a = k1[e] * cu + k2[e] * su;
        const float bb = k2[e] * cu - k1[e] * su;
        k1[e] = a;
        k2[e] = bb;
      }
    }
    float s[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        acc = fmaf(q1[h][e], k1[e], acc);
        acc = fmaf(q2[h][e], k2[e], acc);
      }
      s[h] = acc;
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
#pragma unroll
      for (int h = 0; h < NH; ++h) s[h] += __shfl_xor_sync(0xffffffffu, s[h], off);
    }
    float v1[8], v2[8];
    unpack8(vu1, v1);
    unpack8(vu2, v2);
    if (!valid) continue;
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      if (s[h] > m[h] + 8.f) {
        const float alpha = ex2(m[h] - s[h]);
        l[h] *= alpha;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          o1[h][e] *= alpha;
          o2[h][e] *= alpha;
        }
        m[h] = s[h];
      }
      const float pw = ex2(s[h] - m[h]);
      l[h] += pw;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        o1[h][e] = fmaf(pw, v1[e], o1[h][e]);
        o2[h][e] = fmaf(pw, v2[e], o2[h][e]);
      }
    }
  }

  // merge the 4 key slots of the warp (lanes sl, sl+8, sl+16, sl+24)
#pragma unroll
  for (int off = 8; off < 32; off <<= 1) {
#pragma unroll
    for (int h = 0; h < NH; ++h) {
      const float mo = __shfl_xor_sync(0xffffffffu, m[h], off);
      const float lo_ = __shfl_xor_sync(0xffffffffu, l[h], off);
      const float mn = fmaxf(m[h], mo);
      const float a = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - mn);
      const float bo = (mo == -INFINITY) ? 0.f : ex2(mo - mn);
      l[h] = l[h] * a + lo_ * bo;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float x1 = __shfl_xor_sync(0xffffffffu, o1[h][e], off);
        const float x2 = __shfl_xor_sync(0xffffffffu, o2[h][e], off);
        o1[h][e] = o1[h][e] * a + x1 * bo;
        o2[h][e] = o2[h][e] * a + x2 * bo;
      }
      m[h] = mn;
    }
  }
  if (g == 0) {
#pragma unroll
    for (int h = 0; h < NH; ++h) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        red[warp][h][8 * sl + e] = o1[h][e];
        red[warp][h][kHalf + 8 * sl + e] = o2[h][e];
      }
      if (sl == 0) {
        red[warp][h][kD] = m[h];
        red[warp][h][kD + 1] = l[h];
      }
    }
  }
  __syncthreads();
  // merge the warps; thread t handles (head t / kD, dim t % kD)
  for (int idx = threadIdx.x; idx < NH * kD; idx += kThreads) {
    const int h = idx / kD, d = idx % kD;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, red[w][h][kD]);
    float acc = 0.f, lsum = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = red[w][h][kD];
      const float f = (mw == -INFINITY) ? 0.f : ex2(mw - mx);
      acc += red[w][h][d] * f;
      lsum += red[w][h][kD + 1] * f;
    }
    float *dst = p.ws + ((static_cast<int64_t>(b) * p.Hq + h0 + h) * p.n_chunks + c) *
                            kDecodePartialFloats;
    dst[d] = acc;
    if (d == 0) {
      dst[kD] = mx;
      dst[kD + 1] = lsum;
    }
  }
  // the combine kernel (a programmatic dependent) may be scheduled once every
  // CTA got here; it waits for this grid's completion before reading
  asm volatile("griddepcontrol.launch_dependents;");
}

template <int NH>
__global__ void __launch_bounds__(kThreads) bifocal_decode_split_kernel(const SplitParams p) {
  decode_split_body<NH, false>(p, nullptr);
}

// The same split kernel with its angles evaluated in-kernel instead of read
// from the library-owned table (used by the entry point that allocates nothing).
template <int NH>
__global__ void __launch_bounds__(kThreads)
    bifocal_decode_split_selfangle_kernel(const SplitParams p, const Thetas th) {
  decode_split_body<NH, true>(p, th.t);
}

// Merges the chunk partials: M = max_c m_c, weights 2^(m_c - M),
// O = sum_c w_c o_c / sum_c w_c l_c, lse = (M + log2 sum_c w_c l_c) * ln 2.
// One CTA of 8 warps per (batch, query head, 32-dim slice): warp w takes the
// chunks c = w, w + 8, ..., one dim per lane (128-byte loads).  A warp first
// issues the loads of all its chunks (up to kCombinePerWarp at a time), so the
// partials cost one memory latency, not one per chunk; it merges them against
// its own maximum, and the warps' results are merged once more in shared
// memory with the same rescaling.  The kernel is launched as a programmatic
// dependent of the split kernel: it may start while that kernel runs and
// waits (griddepcontrol.wait) until the partials are complete and visible.
constexpr int kCombineThreads = 256;
constexpr int kCombineSlice = 32;
constexpr int kCombineSlices = kD / kCombineSlice;
constexpr int kCombineWarps = kCombineThreads / 32;
constexpr int kCombinePerWarp = 24;  // chunks per warp and round (192 per round)
__global__ void __launch_bounds__(kCombineThreads)
    bifocal_decode_combine_kernel(const float *__restrict__ ws, __nv_bfloat16 *__restrict__ out,
                                  float *__restrict__ lse, int n_chunks, int Hq,
                                  const DecodeSeq *__restrict__ seqs) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float part[kCombineWarps][kCombineSlice];
  __shared__ float wmax[kCombineWarps], wsum[kCombineWarps];
  const int bh = blockIdx.x / kCombineSlices, sl = blockIdx.x % kCombineSlices;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  // chunk c of (batch, head) bh at src + c * stride; one position for every
  // sequence: [bh][chunk] layout; batched: [chunk][head] from the sequence table
  const float *src;
  int64_t stride;
  if (seqs != nullptr) {
    const DecodeSeq q = seqs[bh / Hq];
    n_chunks = q.n;
    src = ws + (static_cast<int64_t>(q.first) * Hq + bh % Hq) * kDecodePartialFloats;
    stride = static_cast<int64_t>(Hq) * kDecodePartialFloats;
  } else {
    src = ws + static_cast<int64_t>(bh) * n_chunks * kDecodePartialFloats;
    stride = kDecodePartialFloats;
  }
  // this warp's running merge: maximum, weighted sum of o (this lane's dim)
  // and of l
  float M = -INFINITY, acc = 0.f, lsum = 0.f;
  for (int base = 0; base < n_chunks; base += kCombineWarps * kCombinePerWarp) {
    float mc[kCombinePerWarp], lc[kCombinePerWarp], oc[kCombinePerWarp];
#pragma unroll
    for (int i = 0; i < kCombinePerWarp; ++i) {
      const int c = base + warp + kCombineWarps * i;
      mc[i] = -INFINITY;
      lc[i] = 0.f;
      oc[i] = 0.f;
      if (c < n_chunks) {
        const float *pc = src + static_cast<int64_t>(c) * stride;
        mc[i] = pc[kD];
        lc[i] = pc[kD + 1];
        oc[i] = pc[kCombineSlice * sl + lane];
      }
    }
    float mr = M;
#pragma unroll
    for (int i = 0; i < kCombinePerWarp; ++i) mr = fmaxf(mr, mc[i]);
    if (mr != -INFINITY) {
      const float r = (M == -INFINITY) ? 0.f : ex2(M - mr);
      acc *= r;
      lsum *= r;
#pragma unroll
      for (int i = 0; i < kCombinePerWarp; ++i) {
        const float f = (mc[i] == -INFINITY) ? 0.f : ex2(mc[i] - mr);
        acc = fmaf(f, oc[i], acc);
        lsum = fmaf(f, lc[i], lsum);
      }
      M = mr;
    }
  }
  part[warp][lane] = acc;
  if (lane == 0) {
    wmax[warp] = M;
    wsum[warp] = lsum;
  }
  __syncthreads();
  if (t < kCombineSlice) {
    float Mx = wmax[0];
#pragma unroll
    for (int w = 1; w < kCombineWarps; ++w) Mx = fmaxf(Mx, wmax[w]);
    float o = 0.f, L = 0.f;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) {
      const float f = (wmax[w] == -INFINITY) ? 0.f : ex2(wmax[w] - Mx);
      o = fmaf(f, part[w][t], o);
      L = fmaf(f, wsum[w], L);
    }
    out[static_cast<int64_t>(bh) * kD + kCombineSlice * sl + t] = __float2bfloat16_rn(o / L);
    if (sl == 0 && t == 0) lse[bh] = (Mx + __log2f(L)) * 0.69314718055994530942f;
  }
}

template <int NH>
cudaError_t launch_nh(const DecodeArgs &a, const SplitParams &sp, cudaStream_t s) {
  dim3 grid(a.n_chunks, a.Hkv * ((a.Hq / a.Hkv) / NH), a.B);
  bifocal_decode_split_kernel<NH><<<grid, kThreads, 0, s>>>(sp);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_decode_combine(a, s);
}

template <int NH>
cudaError_t launch_nh_selfangle(const DecodeArgs &a, const SplitParams &sp, const Thetas &th,
                                cudaStream_t s) {
  dim3 grid(a.n_chunks, a.Hkv * ((a.Hq / a.Hkv) / NH), a.B);
  bifocal_decode_split_selfangle_kernel<NH><<<grid, kThreads, 0, s>>>(sp, th);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_decode_combine(a, s);
}

// Split partials of the entry point that allocates nothing: a fixed array in
// the library's device image, present on every device that loads the library
// until the process exits.  All such calls share it (the last call's partials
// stay in it); every entry a call reads was written earlier by the same call.
static __device__ __align__(256) float g_decode_noalloc_scratch[kDecodeNoAllocFloats];

constexpr int kMaxScratchDevices = 64;

std::mutex g_noalloc_mu;
float *g_noalloc_addr[kMaxScratchDevices] = {};

}  // namespace

// Device address of the fixed scratch array on the current device, resolved
// once per device (with that device current) and cached until
// decode_noalloc_forget().
cudaError_t decode_noalloc_scratch(float **out) {
  std::mutex &mu = g_noalloc_mu;
  float **addr = g_noalloc_addr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxScratchDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void *ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<float *>(ptr);
  }
  *out = addr[dev];
  return cudaSuccess;
}

// Drops the cached addresses (a device reset unloads the module, after which
// the array may sit elsewhere); the next call on each device resolves it again.
void decode_noalloc_forget() {
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  for (int i = 0; i < kMaxScratchDevices; ++i) g_noalloc_addr[i] = nullptr;
}

cudaError_t launch_decode_noalloc(const DecodeArgs &a_in, double rope_base, cudaStream_t s) {
  DecodeArgs a = a_in;
  cudaError_t e = decode_noalloc_scratch(&a.ws);
  if (e != cudaSuccess) return e;
  Thetas th;
  for (int i = 0; i < kHalf; ++i) th.t[i] = pow(rope_base, -2.0 * i / kD);
  SplitParams sp;
  sp.q = a.q;
  sp.kc = a.kc;
  sp.vc = a.vc;
  sp.ws = a.ws;
  sp.cs = nullptr;
  sp.Hq = a.Hq;
  sp.Hkv = a.Hkv;
  sp.group = a.Hq / a.Hkv;
  sp.pos = a.pos;
  sp.cap = a.cap;
  sp.G = a.G;
  sp.far_end = a.far_end;
  sp.chunk = a.chunk;
  sp.n_far = a.n_far_chunks;
  sp.n_chunks = a.n_chunks;
  sp.scale_log2 = a.scale * 1.4426950408889634f;
  if (sp.group % 4 == 0) return launch_nh_selfangle<4>(a, sp, th, s);
  if (sp.group % 2 == 0) return launch_nh_selfangle<2>(a, sp, th, s);
  return launch_nh_selfangle<1>(a, sp, th, s);
}

cudaError_t launch_decode_combine(const DecodeArgs &a, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(a.B * a.Hq * kCombineSlices));
  cfg.blockDim = dim3(kCombineThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, bifocal_decode_combine_kernel, static_cast<const float *>(a.ws),
                            a.out, a.lse, a.n_chunks, a.Hq, a.seqs);
}

size_t decode_ws_floats(int B, int Hq, int D, int n_chunks) {
  return static_cast<size_t>(B) * Hq * n_chunks * kDecodePartialFloats;
}

// Keys per chunk: enough chunks for about kTargetCtas CTAs, a multiple of 64,
// between 64 and 4096.  The remote range [0, far_end) and the local range
// [far_end, pos] are chunked separately.
void decode_plan(int B, int Hq, int Hkv, int pos, int far_end, int *chunk,
                 int *n_far_chunks, int *n_chunks) {
  const int group = Hq / Hkv;
  const int nh = (group % 4 == 0) ? 4 : (group % 2 == 0) ? 2 : 1;
  const int64_t ctas_per_chunk = static_cast<int64_t>(B) * Hkv * (group / nh);
  const int64_t keys = static_cast<int64_t>(pos) + 1;
  int64_t c = (keys * ctas_per_chunk + kTargetCtas - 1) / kTargetCtas;
  c = ((c + 63) / 64) * 64;
  if (c < 64) c = 64;
  if (c > 4096) c = 4096;
  *chunk = static_cast<int>(c);
  *n_far_chunks = static_cast<int>((far_end + c - 1) / c);
  *n_chunks = *n_far_chunks + static_cast<int>((keys - far_end + c - 1) / c);
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
  SplitParams sp;
  sp.q = a.q;
  sp.kc = a.kc;
  sp.vc = a.vc;
  sp.ws = a.ws;
  sp.cs = a.table.cs;
  sp.Hq = a.Hq;
  sp.Hkv = a.Hkv;
  sp.group = a.Hq / a.Hkv;
  sp.pos = a.pos;
  sp.cap = a.cap;
  sp.G = a.G;
  sp.far_end = a.far_end;
  sp.chunk = a.chunk;
  sp.n_far = a.n_far_chunks;
  sp.n_chunks = a.n_chunks;
  sp.scale_log2 = a.scale * 1.4426950408889634f;
  if (sp.group % 4 == 0) return launch_nh<4>(a, sp, s);
  if (sp.group % 2 == 0) return launch_nh<2>(a, sp, s);
  return launch_nh<1>(a, sp, s);
}

}  // namespace jl
