// jl_api.cu -- the C ABI of libjetlong: argument validation, the method's
// scalar parameters, library-owned per-device state, and kernel dispatch.
//
// Scalar parameters (Jet-Long, bittide paper summary §3.1; techwalker
// explainer §二):  G = max(1, ceil(L / w_pretrained)), recomputed from the
// current length (prefill: the prompt length; decode: pos + 1).  With G = 1
// the remap f(x) = floor(x/G) is the identity and both windows use the same
// RoPE, so the call takes exactly the non-bifocal path (every pair "local");
// the same holds when the local window covers every pair.
#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "jl_internal.h"

namespace jl {

namespace {

thread_local std::string g_last_error;

constexpr int kMaxDevices = 64;

struct DeviceState {
  std::mutex mu;
  bool init = false;
  int sms = 0;
  float2 *table = nullptr;
  int table_positions = 0;
  int table_D = 0;
  double table_base = 0.0;
  unsigned *status = nullptr;
  // tables replaced by larger ones: another host thread may hold a pointer
  // to one between taking it and launching, so they live until jl_finalize
  std::vector<void *> retired;
};

DeviceState g_dev[kMaxDevices];

jl_status current(DeviceState **out, int *dev_out = nullptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(JL_ERR_UNSUPPORTED, "device %d out of range", dev);
  DeviceState &d = g_dev[dev];
  std::lock_guard<std::mutex> lock(d.mu);
  if (!d.init) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    if (prop.major != 10 || prop.minor != 0)
      return fail(JL_ERR_UNSUPPORTED,
                  "libjetlong is built for sm_100a (B200); device %d is sm_%d%d", dev,
                  prop.major, prop.minor);
    d.sms = prop.multiProcessorCount;
    e = cudaMalloc(&d.status, 256);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(status)");
    e = cudaMemset(d.status, 0, 256);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(status)");
    d.init = true;
  }
  *out = &d;
  if (dev_out) *dev_out = dev;
  return JL_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

long long group_size_ll(long long L, long long w) {
  if (L < 1 || w < 1) return -1;
  // ceil(L / w) without forming L + w - 1, which overflows near LLONG_MAX
  const long long g = L / w + (L % w != 0 ? 1 : 0);
  return g < 1 ? 1 : g;
}

}  // namespace

jl_status fail(jl_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

jl_status cuda_fail(cudaError_t e, const char *what) {
  return fail(JL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int sm_count() {
  DeviceState *d = nullptr;
  if (current(&d) != JL_OK) return 148;
  return d->sms;
}

jl_status rope_table(int D, double base, int min_positions, cudaStream_t s, RopeTable *out) {
  DeviceState *d = nullptr;
  jl_status st = current(&d);
  if (st != JL_OK) return st;
  std::lock_guard<std::mutex> lock(d->mu);
  if (d->table == nullptr || d->table_D != D || d->table_base != base ||
      d->table_positions < min_positions) {
    int want = min_positions < 4096 ? 4096 : min_positions;
    if (d->table && d->table_D == D && d->table_base == base && want < 2 * d->table_positions)
      want = 2 * d->table_positions;
    want = ((want + 4095) / 4096) * 4096;
    if (d->table) {  // kept alive: launches in flight or about to start may read it
      d->retired.push_back(d->table);
      d->table = nullptr;
      d->table_positions = 0;
    }
    float2 *t = nullptr;
    const size_t n = static_cast<size_t>(want) * (D / 2);
    cudaError_t e = cudaMalloc(&t, sizeof(float2) * n);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(rope table)");
    e = launch_rope_table(t, want, D, base, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);  // usable from any stream after this
    if (e != cudaSuccess) {
      cudaFree(t);
      return cuda_fail(e, "rope table build");
    }
    d->table = t;
    d->table_positions = want;
    d->table_D = D;
    d->table_base = base;
  }
  out->cs = d->table;
  out->positions = d->table_positions;
  out->half = D / 2;
  return JL_OK;
}

jl_status status_word(unsigned **out) {
  DeviceState *d = nullptr;
  jl_status st = current(&d);
  if (st != JL_OK) return st;
  *out = d->status;
  return JL_OK;
}

}  // namespace jl

using namespace jl;

namespace {

jl_status check_common(int B, int L, int Hq, int Hkv, int D, int w_local, int w_pretrained,
                       double rope_base) {
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1)
    return fail(JL_ERR_INVALID_ARG, "sizes must be >= 1 (B=%d L=%d Hq=%d Hkv=%d)", B, L, Hq, Hkv);
  if (Hq % Hkv != 0)
    return fail(JL_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (D < 2 || D % 2 != 0) return fail(JL_ERR_INVALID_ARG, "head dim %d must be even", D);
  if (w_local < 0) return fail(JL_ERR_INVALID_ARG, "w_local must be >= 0 (got %d)", w_local);
  if (w_pretrained < 1)
    return fail(JL_ERR_INVALID_ARG, "w_pretrained must be >= 1 (got %d)", w_pretrained);
  if (!(rope_base > 1.0) || !std::isfinite(rope_base))
    return fail(JL_ERR_INVALID_ARG, "rope_base must be a finite number > 1");
  return JL_OK;
}

// Two query heads of one kv head per CTA where the group size is even (the
// faster kernel); JL_PREFILL_KERNEL=one selects the one-tile kernel, read on
// every call so that tests can cover both.
cudaError_t launch_attention(const jl::PrefillArgs &a, cudaStream_t s) {
  const char *kv = std::getenv("JL_PREFILL_KERNEL");
  const bool one_tile = kv != nullptr && std::strcmp(kv, "one") == 0;
  return (!one_tile && jl::prefill_x2_supported(a)) ? jl::launch_prefill_sm100_x2(a, s)
                                                    : jl::launch_prefill_sm100(a, s);
}

}  // namespace

extern "C" {

long long jl_group_size(long long L, long long w_pretrained) {
  return group_size_ll(L, w_pretrained);
}

const char *jl_last_error(void) { return g_last_error.c_str(); }

size_t jl_bifocal_prefill_rotated_keys_bytes(int B, int L, int Hkv, int D) {
  if (B < 1 || L < 1 || Hkv < 1 || D < 1) return 0;
  const size_t one = static_cast<size_t>(B) * L * Hkv * D * sizeof(__nv_bfloat16);
  return 2 * ((one + 255) & ~static_cast<size_t>(255));
}

size_t jl_bifocal_prefill_workspace_size(int B, int L, int Hkv, int D, jl_dtype dtype) {
  // keys are rotated inside the prefill kernels: no workspace for any size
  (void)B, (void)L, (void)Hkv, (void)D, (void)dtype;
  return 0;
}

jl_status jl_bifocal_prefill_ex(const void *q, const void *k, const void *v, void *out,
                                float *lse, int B, int L, int Hq, int Hkv, int D,
                                int w_local, int w_pretrained, double rope_base,
                                jl_dtype dtype, float softmax_scale, unsigned flags,
                                void *workspace, size_t workspace_bytes,
                                jl_stream_t stream) {
  g_last_error.clear();
  jl_status st = check_common(B, L, Hq, Hkv, D, w_local, w_pretrained, rope_base);
  if (st != JL_OK) return st;
  if (!q || !k || !v || !out || !lse)
    return fail(JL_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(JL_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if ((flags & ~static_cast<unsigned>(JL_FLAG_NO_BIFOCAL | JL_FLAG_ROTATE_KEYS_ONCE)) != 0)
    return fail(JL_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if (dtype != JL_BF16 && dtype != JL_F32)
    return fail(JL_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(dtype));
  if (dtype == JL_BF16 && D != 128)
    return fail(JL_ERR_UNSUPPORTED, "bf16 prefill supports head dim 128 (got %d)", D);
  if (dtype == JL_F32 && D != 64 && D != 128)
    return fail(JL_ERR_UNSUPPORTED, "fp32 prefill supports head dim 64 or 128 (got %d)", D);
  if (static_cast<long long>((L + 127) / 128) * B * Hq >= (1LL << 31))
    return fail(JL_ERR_UNSUPPORTED, "problem too large for one launch");
  if (!(softmax_scale >= 0.f) && !(softmax_scale < 0.f))
    return fail(JL_ERR_INVALID_ARG, "softmax_scale is NaN");
  const bool once = dtype == JL_BF16 && (flags & JL_FLAG_ROTATE_KEYS_ONCE);
  const size_t need_ws = once ? jl_bifocal_prefill_rotated_keys_bytes(B, L, Hkv, D) : 0;
  if (once) {
    if (workspace == nullptr)
      return fail(JL_ERR_INVALID_ARG, "JL_FLAG_ROTATE_KEYS_ONCE needs a workspace");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
      return fail(JL_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    if (workspace_bytes < need_ws)
      return fail(JL_ERR_INVALID_ARG, "workspace too small: %zu bytes, need %zu",
                  workspace_bytes, need_ws);
  }

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long G = group_size_ll(L, w_pretrained);
  const bool plain = (flags & JL_FLAG_NO_BIFOCAL) || G == 1 || w_local >= L;
  PrefillArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.lse = lse;
  a.B = B;
  a.L = L;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.D = D;
  a.G = static_cast<int>(G);
  a.w_eff = plain ? INT_MAX : w_local;
  a.scale = softmax_scale > 0.f ? softmax_scale : static_cast<float>(1.0 / std::sqrt(D));
  a.key_mode = 0;  // raw keys, rotated in the kernel
  st = rope_table(D, rope_base, L, s, &a.table);
  if (st != JL_OK) return st;
  st = status_word(&a.status);
  if (st != JL_OK) return st;

  if (dtype == JL_F32) {
    cudaError_t e = launch_prefill_f32(a, s);
    return e == cudaSuccess ? JL_OK : cuda_fail(e, "fp32 prefill launch");
  }

  if (once) {
    // both rotated copies, once, into the workspace; the kernel reads them
    __nv_bfloat16 *kstd = static_cast<__nv_bfloat16 *>(workspace);
    __nv_bfloat16 *krem =
        reinterpret_cast<__nv_bfloat16 *>(static_cast<char *>(workspace) + need_ws / 2);
    const bool need_std = a.w_eff > 0;
    const bool need_rem = !plain;  // some pair is remote
    cudaError_t e = launch_rotate_keys(static_cast<const __nv_bfloat16 *>(k),
                                       need_std ? kstd : nullptr, need_rem ? krem : nullptr,
                                       a.table, B, L, Hkv, D, a.G, s);
    if (e != cudaSuccess) return cuda_fail(e, "key rotation launch");
    a.k = need_std ? kstd : krem;
    a.k_rem = need_rem ? krem : kstd;
    a.key_mode = 2;
  }
  cudaError_t e = launch_attention(a, s);
  return e == cudaSuccess ? JL_OK : cuda_fail(e, "prefill launch");
}

jl_status jl_bifocal_prefill(const void *q, const void *k, const void *v, void *out,
                             float *lse, int B, int L, int Hq, int Hkv, int D, int w_local,
                             int w_pretrained, double rope_base, jl_stream_t stream) {
  return jl_bifocal_prefill_ex(q, k, v, out, lse, B, L, Hq, Hkv, D, w_local, w_pretrained,
                               rope_base, JL_BF16, 0.f, 0u, nullptr, 0, stream);
}

size_t jl_bifocal_prefill_chunk_workspace_size(int B, int q_offset, int Lq, int Hkv, int D) {
  // the remote passes correct the cached keys inside the kernels: no workspace
  (void)B, (void)q_offset, (void)Lq, (void)Hkv, (void)D;
  return 0;
}

jl_status jl_bifocal_prefill_chunk(const void *q, const void *k_cache_roped, const void *v_cache,
                                   int q_offset, int cache_capacity, void *out, float *lse, int B,
                                   int Lq, int Hq, int Hkv, int D, int w_local, int w_pretrained,
                                   double rope_base, unsigned flags, void *workspace,
                                   size_t workspace_bytes, jl_stream_t stream) {
  g_last_error.clear();
  jl_status st = check_common(B, Lq, Hq, Hkv, D, w_local, w_pretrained, rope_base);
  if (st != JL_OK) return st;
  if (!q || !k_cache_roped || !v_cache || !out || !lse)
    return fail(JL_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k_cache_roped) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned16(lse))
    return fail(JL_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if ((flags & ~static_cast<unsigned>(JL_FLAG_NO_BIFOCAL)) != 0)
    return fail(JL_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if (D != 128) return fail(JL_ERR_UNSUPPORTED, "chunked prefill supports head dim 128 (got %d)", D);
  if (q_offset < 0 || q_offset % 128 != 0)
    return fail(JL_ERR_UNSUPPORTED, "q_offset (%d) must be a non-negative multiple of 128",
                q_offset);
  const long long Lk = static_cast<long long>(q_offset) + Lq;
  if (Lk > cache_capacity)
    return fail(JL_ERR_INVALID_ARG, "q_offset + Lq (%lld) exceeds cache_capacity (%d)", Lk,
                cache_capacity);
  if (Lk >= (1LL << 31) - 256) return fail(JL_ERR_UNSUPPORTED, "sequence too long");
  if (static_cast<long long>((Lq + 127) / 128) * B * Hq >= (1LL << 31))
    return fail(JL_ERR_UNSUPPORTED, "problem too large for one launch");
  (void)workspace, (void)workspace_bytes;  // unused: keys are corrected in the kernels

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long G = group_size_ll(Lk, w_pretrained);
  const bool plain = (flags & JL_FLAG_NO_BIFOCAL) || G == 1 || w_local >= Lk;
  PrefillArgs a;
  a.q = q;
  a.v = v_cache;
  a.out = out;
  a.lse = lse;
  a.B = B;
  a.L = Lq;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.D = D;
  a.G = static_cast<int>(G);
  a.w_eff = plain ? INT_MAX : w_local;
  a.scale = static_cast<float>(1.0 / std::sqrt(D));
  a.q_off = q_offset;
  a.kv_stride = cache_capacity;
  st = rope_table(D, rope_base, static_cast<int>(Lk), s, &a.table);
  if (st != JL_OK) return st;
  st = status_word(&a.status);
  if (st != JL_OK) return st;
  // keys at original positions: the cache as it is; at remapped positions:
  // R(f(k) - k) of the cached key, applied in the kernel
  a.k = k_cache_roped;
  a.key_mode = 1;
  cudaError_t e = launch_attention(a, s);
  return e == cudaSuccess ? JL_OK : cuda_fail(e, "chunked prefill launch");
}

size_t jl_bifocal_prefill_3pass_workspace_size(int B, int L, int Hq, int Hkv, int D) {
  if (B < 1 || L < 1 || Hq < 1 || Hkv < 1 || D < 2) return 0;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t o = up(static_cast<size_t>(B) * L * Hq * D * sizeof(__nv_bfloat16));
  const size_t l = up(static_cast<size_t>(B) * Hq * L * sizeof(float));
  return 2 * o + 2 * l;
}

jl_status jl_bifocal_prefill_3pass(const void *q, const void *k, const void *v, void *out,
                                   float *lse, int B, int L, int Hq, int Hkv, int D,
                                   int w_local, int w_pretrained, double rope_base,
                                   unsigned flags, void *workspace, size_t workspace_bytes,
                                   jl_stream_t stream) {
  g_last_error.clear();
  jl_status st = check_common(B, L, Hq, Hkv, D, w_local, w_pretrained, rope_base);
  if (st != JL_OK) return st;
  if (!q || !k || !v || !out || !lse || !workspace)
    return fail(JL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(JL_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(JL_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if ((flags & ~static_cast<unsigned>(JL_FLAG_NO_BIFOCAL)) != 0)
    return fail(JL_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if (D != 128) return fail(JL_ERR_UNSUPPORTED, "the three-call path supports head dim 128 (got %d)", D);
  if (static_cast<long long>((L + 127) / 128) * B * Hq >= (1LL << 31))
    return fail(JL_ERR_UNSUPPORTED, "problem too large for one launch");
  const size_t need = jl_bifocal_prefill_3pass_workspace_size(B, L, Hq, Hkv, D);
  if (workspace_bytes < need)
    return fail(JL_ERR_INVALID_ARG, "workspace too small: %zu bytes, need %zu", workspace_bytes,
                need);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long G = (flags & JL_FLAG_NO_BIFOCAL) ? 1 : group_size_ll(L, w_pretrained);
  PrefillArgs a;
  a.q = q;
  a.v = v;
  a.B = B;
  a.L = L;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.D = D;
  a.G = static_cast<int>(G);
  a.scale = static_cast<float>(1.0 / std::sqrt(D));
  st = rope_table(D, rope_base, L, s, &a.table);
  if (st != JL_OK) return st;
  st = status_word(&a.status);
  if (st != JL_OK) return st;

  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  char *ws = static_cast<char *>(workspace);
  const size_t kb = 0;
  const size_t ob = up(static_cast<size_t>(B) * L * Hq * D * sizeof(__nv_bfloat16));
  const size_t lb = up(static_cast<size_t>(B) * Hq * L * sizeof(float));
  __nv_bfloat16 *o_b = reinterpret_cast<__nv_bfloat16 *>(ws + kb);
  __nv_bfloat16 *o_c = reinterpret_cast<__nv_bfloat16 *>(ws + kb + ob);
  float *l_b = reinterpret_cast<float *>(ws + kb + 2 * ob);
  float *l_c = reinterpret_cast<float *>(ws + kb + 2 * ob + lb);

  // A: every pair at remapped positions, into out / lse
  a.k = k;
  a.key_mode = 0;
  a.out = out;
  a.lse = lse;
  a.w_eff = 0;
  a.band = 0;
  cudaError_t e = launch_attention(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch (A)");
  if (w_local == 0) return JL_OK;  // empty window: B and C have no pairs
  // B: the local window at original positions; C: the same window remapped
  a.w_eff = w_local;
  a.band = 1;
  a.out = o_b;
  a.lse = l_b;
  e = launch_attention(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch (B)");
  a.band = 2;
  a.out = o_c;
  a.lse = l_c;
  e = launch_attention(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch (C)");
  e = launch_lse_merge(static_cast<__nv_bfloat16 *>(out), lse, o_b, l_b, o_c, l_c, B, L, Hq, s);
  return e == cudaSuccess ? JL_OK : cuda_fail(e, "merge launch");
}

size_t jl_bifocal_decode_workspace_size(int B, int Hq, int Hkv, int D, int pos) {
  if (B < 1 || Hq < 1 || Hkv < 1 || D < 1 || pos < 0 || Hq % Hkv != 0) return 0;
  // the remote/local split adds at most one chunk to either plan
  int chunk = 0, n_far = 0, n_chunks = 0;
  decode_plan(B, Hq, Hkv, pos, 0, &chunk, &n_far, &n_chunks);
  int chunk2 = 0, n_far2 = 0, n_chunks2 = 0;
  decode_mma_plan(B, pos, 0, &chunk2, &n_far2, &n_chunks2);
  const int most = n_chunks > n_chunks2 ? n_chunks : n_chunks2;
  return decode_ws_floats(B, Hq, D, most + 1) * sizeof(float);
}

jl_status jl_bifocal_decode(const void *q_new, const void *k_cache_roped, const void *v_cache,
                            int pos, int cache_capacity, void *out, float *lse,
                            void *workspace, size_t workspace_bytes, int B, int Hq, int Hkv,
                            int D, int w_local, int w_pretrained, double rope_base,
                            unsigned flags, jl_stream_t stream) {
  g_last_error.clear();
  jl_status st = check_common(B, 1, Hq, Hkv, D, w_local, w_pretrained, rope_base);
  if (st != JL_OK) return st;
  if (!q_new || !k_cache_roped || !v_cache || !out || !lse || !workspace)
    return fail(JL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q_new) || !aligned16(k_cache_roped) || !aligned16(v_cache) ||
      !aligned16(out) || !aligned16(lse) || !aligned16(workspace))
    return fail(JL_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if ((flags & ~static_cast<unsigned>(JL_FLAG_NO_BIFOCAL | JL_FLAG_DEBUG_SKIP_ARRIVE)) != 0)
    return fail(JL_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if (D != 128) return fail(JL_ERR_UNSUPPORTED, "decode supports head dim 128 (got %d)", D);
  if ((flags & JL_FLAG_DEBUG_SKIP_ARRIVE) && !decode_mma_supported(Hq, Hkv, D))
    return fail(JL_ERR_UNSUPPORTED,
                "JL_FLAG_DEBUG_SKIP_ARRIVE needs the tensor-core decode kernel "
                "(Hkv <= 8, Hq / Hkv <= 8)");
  if (cache_capacity < 1 || pos < 0 || pos >= cache_capacity)
    return fail(JL_ERR_INVALID_ARG, "need 0 <= pos (%d) < cache_capacity (%d)", pos,
                cache_capacity);
  const size_t need = jl_bifocal_decode_workspace_size(B, Hq, Hkv, D, pos);
  if (workspace_bytes < need)
    return fail(JL_ERR_INVALID_ARG, "workspace too small: %zu bytes, need %zu",
                workspace_bytes, need);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const long long G = group_size_ll(static_cast<long long>(pos) + 1, w_pretrained);
  const bool plain = (flags & JL_FLAG_NO_BIFOCAL) || G == 1;
  DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16 *>(q_new);
  a.kc = static_cast<const __nv_bfloat16 *>(k_cache_roped);
  a.vc = static_cast<const __nv_bfloat16 *>(v_cache);
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.lse = lse;
  a.ws = static_cast<float *>(workspace);
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.D = D;
  a.pos = pos;
  a.cap = cache_capacity;
  a.G = static_cast<int>(G);
  // keys k <= pos - w_local are remote
  const long long fe = static_cast<long long>(pos) + 1 - w_local;
  a.far_end = plain ? 0 : static_cast<int>(fe < 0 ? 0 : fe);
  a.scale = static_cast<float>(1.0 / std::sqrt(D));
  a.debug_skip_arrival = (flags & JL_FLAG_DEBUG_SKIP_ARRIVE) != 0;
  st = rope_table(D, rope_base, pos + 1 < 64 ? 64 : pos + 1, s, &a.table);
  if (st != JL_OK) return st;
  cudaError_t e;
  if (decode_mma_supported(Hq, Hkv, D)) {
    unsigned *status = nullptr;
    st = status_word(&status);
    if (st != JL_OK) return st;
    decode_mma_plan(B, pos, a.far_end, &a.chunk, &a.n_far_chunks, &a.n_chunks);
    e = launch_decode_mma(a, status, s);
  } else {
    decode_plan(B, Hq, Hkv, pos, a.far_end, &a.chunk, &a.n_far_chunks, &a.n_chunks);
    e = launch_decode(a, s);
  }
  return e == cudaSuccess ? JL_OK : cuda_fail(e, "decode launch");
}

size_t jl_bifocal_decode_batched_workspace_size(int B, int Hq, int Hkv, int D) {
  if (B < 1 || Hq < 1 || Hkv < 1 || D != 128) return 0;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t n_max = static_cast<size_t>(kDecodeBatchCtas) + 2 * static_cast<size_t>(B);
  return up(n_max * sizeof(DecodeWork)) + up(static_cast<size_t>(B) * sizeof(DecodeSeq)) +
         up(sizeof(int)) + n_max * Hq * kDecodePartialFloats * sizeof(float);
}

namespace {

// Paged cache of jl_bifocal_decode_paged (null block_table: contiguous caches).
struct PagedCache {
  const int *block_table = nullptr;
  int page_size = 0, max_pages = 0, num_pages = 0;
};

// Batched decode over host positions `pos` (already validated): plans one wave
// of CTAs, copies the plan into the workspace and launches.
jl_status run_decode_batched(const void *q_new, const void *k_cache, const void *v_cache,
                             const int *pos, int cache_capacity, const PagedCache &pc,
                             void *out, float *lse, void *workspace, int B, int Hq, int Hkv,
                             int D, int w_local, int w_pretrained, double rope_base,
                             unsigned flags, cudaStream_t s) {
  const bool pos_on_device = (flags & JL_FLAG_DEVICE_POS) != 0;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t n_max = static_cast<size_t>(kDecodeBatchCtas) + 2 * static_cast<size_t>(B);
  const size_t work_bytes = up(n_max * sizeof(DecodeWork));
  const size_t seq_bytes = up(B * sizeof(DecodeSeq));
  char *ws = static_cast<char *>(workspace);
  DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16 *>(q_new);
  a.kc = static_cast<const __nv_bfloat16 *>(k_cache);
  a.vc = static_cast<const __nv_bfloat16 *>(v_cache);
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.lse = lse;
  a.work = reinterpret_cast<const DecodeWork *>(ws);
  a.seqs = reinterpret_cast<const DecodeSeq *>(ws + work_bytes);
  int *n_work_dev = reinterpret_cast<int *>(ws + work_bytes + seq_bytes);
  a.ws = reinterpret_cast<float *>(ws + work_bytes + seq_bytes + up(sizeof(int)));
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.D = D;
  a.cap = cache_capacity;
  a.G = 1;
  a.far_end = 0;
  a.n_far_chunks = 0;
  a.scale = static_cast<float>(1.0 / std::sqrt(D));
  a.block_table = pc.block_table;
  a.page_size = pc.page_size;
  a.max_pages = pc.max_pages;
  a.num_pages = pc.num_pages;
  unsigned *status = nullptr;
  jl_status st = status_word(&status);
  if (st != JL_OK) return st;
  cudaError_t e = cudaSuccess;
  std::vector<unsigned char> tables;
  if (pos_on_device) {
    // the plan is made on the device: every CTA the plan can hold is launched
    // and the surplus exit; the maps and the table cover the whole cache
    a.max_keys = cache_capacity;
    a.pos = cache_capacity - 1;
    a.chunk = 16;
    a.n_work = static_cast<int>(n_max);
    a.n_chunks = a.n_work;
    a.n_work_dev = n_work_dev;
    st = rope_table(D, rope_base, cache_capacity < 64 ? 64 : cache_capacity, s, &a.table);
    if (st != JL_OK) return st;
    e = launch_decode_plan(pos, B, cache_capacity, w_local, w_pretrained,
                           (flags & JL_FLAG_NO_BIFOCAL) != 0, Hq, static_cast<int>(n_max),
                           reinterpret_cast<DecodeWork *>(ws),
                           reinterpret_cast<DecodeSeq *>(ws + work_bytes), n_work_dev, status, s);
    if (e != cudaSuccess) return cuda_fail(e, "decode plan launch");
  } else {
    long long total = 0;
    int max_keys = 0;
    for (int b = 0; b < B; ++b) {
      total += static_cast<long long>(pos[b]) + 1;
      max_keys = pos[b] + 1 > max_keys ? pos[b] + 1 : max_keys;
    }
    // Plan: one wave of CTAs over all keys; each sequence's remote range
    // [0, far_end) and local range [far_end, pos] are cut into chunks of at
    // most `chunk` keys (a multiple of 16).  Each range adds at most one
    // partial chunk, so aiming at kDecodeBatchCtas - 2B chunks keeps the plan
    // within one wave (up to 66 sequences) and always within
    // kDecodeBatchCtas + 2B.  (jl_plan.cu makes the same plan on the device.)
    const long long target =
        kDecodeBatchCtas - 2LL * B > 16 ? kDecodeBatchCtas - 2LL * B : 16;
    long long chunk = (total + target - 1) / target;
    chunk = ((chunk + 15) / 16) * 16;
    if (chunk < 16) chunk = 16;
    std::vector<DecodeWork> work;
    std::vector<DecodeSeq> seqs(B);
    for (int b = 0; b < B; ++b) {
      const int p = pos[b];
      const long long G = group_size_ll(static_cast<long long>(p) + 1, w_pretrained);
      const bool plain = (flags & JL_FLAG_NO_BIFOCAL) || G == 1;
      const long long fe = static_cast<long long>(p) + 1 - w_local;
      const int far_end = plain ? 0 : static_cast<int>(fe < 0 ? 0 : fe);
      const unsigned long long magic =
          G >= 2 ? (~0ull / static_cast<unsigned long long>(G)) + 1ull : 0ull;
      seqs[b].first = static_cast<int>(work.size());
      auto cut = [&](int lo, int hi, int far) {
        for (long long k0 = lo; k0 < hi; k0 += chunk) {
          DecodeWork w;
          w.b = b;
          w.k_begin = static_cast<int>(k0);
          w.k_end = static_cast<int>(k0 + chunk < hi ? k0 + chunk : hi);
          w.far = far;
          w.pos = p;
          w.G = static_cast<int>(G);
          w.part = static_cast<int>(work.size()) * Hq;
          w.pad = 0;
          w.g_magic = magic;
          work.push_back(w);
        }
      };
      cut(0, far_end, 1);
      cut(far_end, p + 1, 0);
      seqs[b].n = static_cast<int>(work.size()) - seqs[b].first;
    }
    if (work.size() > n_max) return fail(JL_ERR_CUDA, "internal: decode plan too large");
    tables.resize(work_bytes + B * sizeof(DecodeSeq));
    std::memcpy(tables.data(), work.data(), work.size() * sizeof(DecodeWork));
    std::memcpy(tables.data() + work_bytes, seqs.data(), B * sizeof(DecodeSeq));
    a.max_keys = max_keys;
    a.pos = max_keys - 1;
    a.chunk = static_cast<int>(chunk);
    a.n_work = static_cast<int>(work.size());
    a.n_chunks = a.n_work;
    st = rope_table(D, rope_base, max_keys < 64 ? 64 : max_keys, s, &a.table);
    if (st != JL_OK) return st;
    // pageable source: the copy is staged before the call returns
    e = cudaMemcpyAsync(ws, tables.data(), tables.size(), cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "decode table copy");
  }
  e = launch_decode_mma(a, status, s);
  return e == cudaSuccess ? JL_OK : cuda_fail(e, "batched decode launch");
}

// Checks shared by the two batched entry points (everything but the caches).
jl_status check_batched(const void *q_new, const void *k_cache, const void *v_cache,
                        const int *pos, void *out, float *lse, void *workspace,
                        size_t workspace_bytes, int B, int Hq, int Hkv, int D, int w_local,
                        int w_pretrained, double rope_base, unsigned flags) {
  jl_status st = check_common(B, 1, Hq, Hkv, D, w_local, w_pretrained, rope_base);
  if (st != JL_OK) return st;
  if (!q_new || !k_cache || !v_cache || !out || !lse || !workspace || !pos)
    return fail(JL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q_new) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      !aligned16(lse))
    return fail(JL_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(JL_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  if ((flags & ~static_cast<unsigned>(JL_FLAG_NO_BIFOCAL | JL_FLAG_DEVICE_POS)) != 0)
    return fail(JL_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if ((flags & JL_FLAG_DEVICE_POS) && (reinterpret_cast<uintptr_t>(pos) & 3u) != 0)
    return fail(JL_ERR_INVALID_ARG, "device positions must be 4-byte aligned");
  if (D != 128) return fail(JL_ERR_UNSUPPORTED, "decode supports head dim 128 (got %d)", D);
  if (!decode_mma_supported(Hq, Hkv, D))
    return fail(JL_ERR_UNSUPPORTED,
                "batched decode needs the tensor-core kernel (Hkv <= 8, Hq / Hkv <= 8)");
  const size_t need = jl_bifocal_decode_batched_workspace_size(B, Hq, Hkv, D);
  if (workspace_bytes < need)
    return fail(JL_ERR_INVALID_ARG, "workspace too small: %zu bytes, need %zu", workspace_bytes,
                need);
  return JL_OK;
}

}  // namespace

jl_status jl_bifocal_decode_batched(const void *q_new, const void *k_cache_roped,
                                    const void *v_cache, const int *pos, int cache_capacity,
                                    void *out, float *lse, void *workspace,
                                    size_t workspace_bytes, int B, int Hq, int Hkv, int D,
                                    int w_local, int w_pretrained, double rope_base,
                                    unsigned flags, jl_stream_t stream) {
  g_last_error.clear();
  jl_status st = check_batched(q_new, k_cache_roped, v_cache, pos, out, lse, workspace,
                               workspace_bytes, B, Hq, Hkv, D, w_local, w_pretrained,
                               rope_base, flags);
  if (st != JL_OK) return st;
  if (cache_capacity < 1) return fail(JL_ERR_INVALID_ARG, "cache_capacity must be >= 1");
  for (int b = 0; b < B && !(flags & JL_FLAG_DEVICE_POS); ++b)
    if (pos[b] < 0 || pos[b] >= cache_capacity)
      return fail(JL_ERR_INVALID_ARG, "need 0 <= pos[%d] (%d) < cache_capacity (%d)", b, pos[b],
                  cache_capacity);
  return run_decode_batched(q_new, k_cache_roped, v_cache, pos, cache_capacity, PagedCache{},
                            out, lse, workspace, B, Hq, Hkv, D, w_local, w_pretrained, rope_base,
                            flags, reinterpret_cast<cudaStream_t>(stream));
}

jl_status jl_bifocal_decode_paged(const void *q_new, const void *k_pages, const void *v_pages,
                                  int num_pages, int page_size, const int *block_table,
                                  int max_pages_per_seq, const int *pos, void *out, float *lse,
                                  void *workspace, size_t workspace_bytes, int B, int Hq,
                                  int Hkv, int D, int w_local, int w_pretrained,
                                  double rope_base, unsigned flags, jl_stream_t stream) {
  g_last_error.clear();
  jl_status st = check_batched(q_new, k_pages, v_pages, pos, out, lse, workspace,
                               workspace_bytes, B, Hq, Hkv, D, w_local, w_pretrained,
                               rope_base, flags);
  if (st != JL_OK) return st;
  if (!block_table) return fail(JL_ERR_INVALID_ARG, "null pointer");
  if ((reinterpret_cast<uintptr_t>(block_table) & 3u) != 0)
    return fail(JL_ERR_INVALID_ARG, "block_table must be 4-byte aligned");
  if (page_size < 16 || page_size % 16 != 0)
    return fail(JL_ERR_INVALID_ARG, "page_size must be a positive multiple of 16 (got %d)",
                page_size);
  if (num_pages < 1 || max_pages_per_seq < 1)
    return fail(JL_ERR_INVALID_ARG, "need num_pages >= 1 and max_pages_per_seq >= 1");
  if (static_cast<long long>(num_pages) * page_size > INT_MAX)
    return fail(JL_ERR_INVALID_ARG, "the pool holds more than 2^31 - 1 rows");
  const long long span = static_cast<long long>(max_pages_per_seq) * page_size;
  for (int b = 0; b < B && !(flags & JL_FLAG_DEVICE_POS); ++b)
    if (pos[b] < 0 || pos[b] >= span)
      return fail(JL_ERR_INVALID_ARG,
                  "need 0 <= pos[%d] (%d) < max_pages_per_seq * page_size (%lld)", b, pos[b],
                  span);
  PagedCache pc;
  pc.block_table = block_table;
  pc.page_size = page_size;
  pc.max_pages = max_pages_per_seq;
  pc.num_pages = num_pages;
  const int cap = span > INT_MAX ? INT_MAX : static_cast<int>(span);
  return run_decode_batched(q_new, k_pages, v_pages, pos, cap, pc, out, lse, workspace, B, Hq,
                            Hkv, D, w_local, w_pretrained, rope_base, flags,
                            reinterpret_cast<cudaStream_t>(stream));
}

jl_status jl_bifocal_decode_noalloc(const void *q_new, const void *k_cache_roped,
                                    const void *v_cache, int pos, int cache_capacity,
                                    void *out, float *lse, int B, int Hq, int Hkv, int D,
                                    int w_local, int w_pretrained, double rope_base,
                                    unsigned flags, jl_stream_t stream) {
  g_last_error.clear();
  jl_status st = check_common(B, 1, Hq, Hkv, D, w_local, w_pretrained, rope_base);
  if (st != JL_OK) return st;
  if (!q_new || !k_cache_roped || !v_cache || !out || !lse)
    return fail(JL_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q_new) || !aligned16(k_cache_roped) || !aligned16(v_cache) ||
      !aligned16(out) || !aligned16(lse))
    return fail(JL_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if ((flags & ~static_cast<unsigned>(JL_FLAG_NO_BIFOCAL)) != 0)
    return fail(JL_ERR_INVALID_ARG, "unknown flag bits 0x%x", flags);
  if (D != 128) return fail(JL_ERR_UNSUPPORTED, "decode supports head dim 128 (got %d)", D);
  if (cache_capacity < 1 || pos < 0 || pos >= cache_capacity)
    return fail(JL_ERR_INVALID_ARG, "need 0 <= pos (%d) < cache_capacity (%d)", pos,
                cache_capacity);
  const long long G = group_size_ll(static_cast<long long>(pos) + 1, w_pretrained);
  const bool plain = (flags & JL_FLAG_NO_BIFOCAL) || G == 1;
  DecodeArgs a;
  a.q = static_cast<const __nv_bfloat16 *>(q_new);
  a.kc = static_cast<const __nv_bfloat16 *>(k_cache_roped);
  a.vc = static_cast<const __nv_bfloat16 *>(v_cache);
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.lse = lse;
  a.ws = nullptr;
  a.B = B;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.D = D;
  a.pos = pos;
  a.cap = cache_capacity;
  a.G = static_cast<int>(G);
  const long long fe = static_cast<long long>(pos) + 1 - w_local;
  a.far_end = plain ? 0 : static_cast<int>(fe < 0 ? 0 : fe);
  a.scale = static_cast<float>(1.0 / std::sqrt(D));
  a.table = RopeTable{nullptr, 0, D / 2};
  decode_plan(B, Hq, Hkv, pos, a.far_end, &a.chunk, &a.n_far_chunks, &a.n_chunks);
  const size_t need = decode_ws_floats(B, Hq, D, a.n_chunks);
  if (need > kDecodeNoAllocFloats)
    return fail(JL_ERR_UNSUPPORTED,
                "jl_bifocal_decode_noalloc: these sizes need %zu floats of scratch; its fixed "
                "array holds %zu (use jl_bifocal_decode with a workspace)",
                need, kDecodeNoAllocFloats);
  cudaError_t e = launch_decode_noalloc(a, rope_base, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? JL_OK : cuda_fail(e, "no-alloc decode launch");
}

jl_status jl_check_device_status(jl_stream_t stream) {
  g_last_error.clear();
  DeviceState *d = nullptr;
  jl_status st = current(&d);
  if (st != JL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned word = 0;
  e = cudaMemcpy(&word, d->status, sizeof word, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  if (word != 0) {
    cudaMemset(d->status, 0, sizeof word);
    if (word & kStatusTimeout)
      return fail(JL_ERR_TIMEOUT, "a kernel abandoned a bounded wait (status 0x%x)", word);
    return fail(JL_ERR_INVALID_ARG, "a kernel refused an out-of-range index (status 0x%x)",
                word);
  }
  return JL_OK;
}

void jl_finalize(void) {
  int prev = 0;
  const bool have_prev = cudaGetDevice(&prev) == cudaSuccess;
  for (int i = 0; i < kMaxDevices; ++i) {
    DeviceState &d = g_dev[i];
    std::lock_guard<std::mutex> lock(d.mu);
    if (!d.init) continue;
    if (cudaSetDevice(i) != cudaSuccess) continue;
    cudaDeviceSynchronize();
    if (d.table) cudaFree(d.table);
    if (d.status) cudaFree(d.status);
    for (void *r : d.retired) cudaFree(r);
    d.retired.clear();
    d.table = nullptr;
    d.status = nullptr;
    d.table_positions = 0;
    d.init = false;
  }
  decode_noalloc_forget();
  if (have_prev) cudaSetDevice(prev);
}

}  // extern "C"
