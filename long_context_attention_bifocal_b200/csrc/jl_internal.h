// jl_internal.h -- declarations shared by the translation units of libjetlong.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstddef>
#include <cstdint>

#include "jetlong.h"

namespace jl {

// Status-word bits written by kernels (never a trap).
enum : unsigned {
  kStatusTimeout = 1u << 0,  // a bounded mbarrier wait expired
  kStatusBounds = 1u << 1,   // an index check refused an access
};

// Angle table: cs[p * half + i] = (cos(p * theta_i), sin(p * theta_i)),
// computed with fp64 sincos and rounded to fp32.
struct RopeTable {
  const float2 *cs;
  int positions;  // valid p in [0, positions)
  int half;       // D / 2
};

// Records a message for jl_last_error() and returns st.
jl_status fail(jl_status st, const char *fmt, ...);
jl_status cuda_fail(cudaError_t e, const char *what);

// Per-device library state (current device).
jl_status rope_table(int D, double base, int min_positions, cudaStream_t s,
                     RopeTable *out);
jl_status status_word(unsigned **out);
int sm_count();

// ---- launchers (each returns the launch's cudaError_t) ----
cudaError_t launch_rope_table(float2 *cs, int positions, int D, double base, cudaStream_t s);
// Rotated copies of the keys of a [B,L,Hkv,D] bf16 tensor (the prefill's
// "rotate the keys once" mode): kstd = R(l) k (if kstd), krem = R(floor(l/G)) k
// (if krem), same layout.
cudaError_t launch_rotate_keys(const __nv_bfloat16 *k, __nv_bfloat16 *kstd,
                               __nv_bfloat16 *krem, RopeTable t, int B, int L,
                               int Hkv, int D, int G, cudaStream_t s);

struct PrefillArgs {
  const void *q;      // [B,L,Hq,D] pre-RoPE
  const void *k;      // [B,L,Hkv,D] keys: raw (key_mode 0), a cache rotated at
                      // original positions (key_mode 1, batch stride kv_stride), or
                      // rotated at original positions by the library (key_mode 2)
  const void *k_rem = nullptr;  // key_mode 2: the keys rotated at floor(l / G)
  const void *v;      // [B,L,Hkv,D]
  void *out;          // [B,L,Hq,D]
  float *lse;         // [B,Hq,L]
  int B, L, Hq, Hkv, D;
  int G;
  int w_eff;          // local iff q - k < w_eff (INT_MAX: every pair local)
  float scale;        // softmax scale
  RopeTable table;
  unsigned *status;
  int band = 0;       // 0: bifocal rule; 1 / 2: only the local window, standard / remapped
  int q_off = 0;      // position of query row 0 (multiple of 128); keys are [0, q_off + L)
  int64_t kv_stride = 0;  // keys per batch entry in k and v; 0: q_off + L
  int key_mode = 0;   // 0: raw keys (R(k) / R(f(k)) in the kernel); 1: cached keys at
                      // original positions (as they are / R(f(k) - k) in the kernel);
                      // 2: both rotations done beforehand (k, k_rem read as they are)
};

cudaError_t launch_prefill_sm100(const PrefillArgs &a, cudaStream_t s);
// two query heads of one kv head per CTA; needs an even Hq / Hkv
bool prefill_x2_supported(const PrefillArgs &a);
cudaError_t launch_prefill_sm100_x2(const PrefillArgs &a, cudaStream_t s);
cudaError_t launch_prefill_f32(const PrefillArgs &a, cudaStream_t s);

// Batched decode with one position per sequence: the host plans one wave of
// CTAs over all sequences' keys and copies these tables into the workspace.
struct DecodeWork {              // one CTA: a key range of one sequence
  int b;                         // sequence
  int k_begin, k_end;            // keys [k_begin, k_end), all remote or all local
  int far;                       // 1: remote keys (corrected)
  int pos, G;                    // the sequence's position and group size
  int part;                      // partials of query head h at (part + h) * kDecodePartialFloats
  int pad;
  unsigned long long g_magic;    // ceil(2^64 / G) when G >= 2
};
struct DecodeSeq {               // one sequence's partials: chunks first .. first + n - 1
  int first, n;
};
constexpr int kDecodeBatchCtas = 148;  // CTAs the batched plan aims for (one B200 wave)

struct DecodeArgs {
  const __nv_bfloat16 *q;   // [B,Hq,D] pre-RoPE
  const __nv_bfloat16 *kc;  // [B,cap,Hkv,D] rotated at original positions
  const __nv_bfloat16 *vc;  // [B,cap,Hkv,D]
  __nv_bfloat16 *out;       // [B,Hq,D]
  float *lse;               // [B,Hq]
  float *ws;                // split partials
  int B, Hq, Hkv, D, pos, cap;
  int G;
  int far_end;              // keys [0, far_end) take the dk correction
  float scale;
  RopeTable table;
  int chunk;                // keys per split
  int n_far_chunks, n_chunks;
  bool debug_skip_arrival = false;  // JL_FLAG_DEBUG_SKIP_ARRIVE (tensor-core kernel)
  // batched decode (tensor-core kernel): work table, sequence table, their
  // sizes, and the largest number of valid keys of any sequence
  const DecodeWork *work = nullptr;
  const DecodeSeq *seqs = nullptr;
  int n_work = 0, max_keys = 0;
  // paged cache (batched decode only): kc / vc are pools of num_pages pages of
  // page_size rows [page_size, Hkv, D]; block_table [B, max_pages] on the device
  const int *block_table = nullptr;
  int page_size = 0, max_pages = 0, num_pages = 0;
  // plan made on the device: the number of work entries lives here and the
  // grid has n_work (the most the plan can hold) CTAs; the surplus ones exit
  const int *n_work_dev = nullptr;
};

// The batched decode's plan from a device array of positions (one CTA):
// fills work[0 .. *n_work) and seqs[0 .. B), at most n_max entries.
cudaError_t launch_decode_plan(const int *pos, int B, int cap, int w_local, int w_pretrained,
                               bool plain, int Hq, int n_max, DecodeWork *work,
                               DecodeSeq *seqs, int *n_work, unsigned *status,
                               cudaStream_t s);


// One split partial in the decode workspace: o[128], m (log2 units), l, and
// two floats of padding so every partial starts on a 16-byte boundary.
constexpr int kDecodePartialFloats = 132;

// Workspace floats for the given split layout.
size_t decode_ws_floats(int B, int Hq, int D, int n_chunks);
void decode_plan(int B, int Hq, int Hkv, int pos, int far_end, int *chunk,
                 int *n_far_chunks, int *n_chunks);
cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s);
// merges a.n_chunks split partials of a.ws into a.out and a.lse
cudaError_t launch_decode_combine(const DecodeArgs &a, cudaStream_t s);

// In place: out/lse hold call A; returns the LSE merge of A + B - C.
cudaError_t launch_lse_merge(__nv_bfloat16 *out, float *lse, const __nv_bfloat16 *ob,
                             const float *lb, const __nv_bfloat16 *oc, const float *lc, int B,
                             int L, int Hq, cudaStream_t s);

// TMA-staged tensor-core decode (all kv heads of a key chunk per CTA):
// needs D == 128, Hkv <= 8 and Hq / Hkv <= 16.
bool decode_mma_supported(int Hq, int Hkv, int D);
void decode_mma_plan(int B, int pos, int far_end, int *chunk, int *n_far, int *n_chunks);
cudaError_t launch_decode_mma(const DecodeArgs &a, unsigned *status, cudaStream_t s);

// Fixed-size scratch of jl_bifocal_decode_noalloc, in floats (4 MiB).
constexpr size_t kDecodeNoAllocFloats = static_cast<size_t>(1) << 20;
// Same decode, split partials in the library's fixed scratch array and angles
// evaluated in-kernel; a.ws is ignored.  Allocates nothing.
cudaError_t launch_decode_noalloc(const DecodeArgs &a, double rope_base, cudaStream_t s);
void decode_noalloc_forget();

}  // namespace jl
