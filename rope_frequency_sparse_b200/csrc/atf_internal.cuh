// atf_internal.cuh -- kernel parameter blocks and launchers shared by the
// library's translation units (not part of the public C ABI).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/atf.h"

namespace atf {

constexpr int kMaxPairs = 64;      // d <= 128
constexpr int kMaxDecodeBatch = 64;  // sequences per decode launch

// Window table in the kernels' integer domain: W_i clamped to INT32_MAX (every
// distance the kernels can see is below 2^31, so clamping changes nothing).
struct Windows {
  int w[kMaxPairs];
};

struct RopeParams {
  const void* x;
  void* x_rot;      // nullable
  void* x_chunked;  // nullable, bf16 only: [B][H][d/16][S][16]
  int batch, seq, heads, d;
  long long pos_offset;
  int rotate;  // 0: copy, 1: RoPE, 2: rotate-half RoPE, 3: rotate-half copy (2, 3 write pairs interleaved)
  int fp32;    // 1: fp32 elements, 0: bf16
  double omega[kMaxPairs];
};

struct PrefillParams {
  const void* q;    // rotated queries  [B][q_len][Hq][d]
  const void* k;    // rotated keys     [B][kv_len][Hkv][d]
  const void* v;    // values           [B][kv_len][Hkv][d]
  void* out;        // [B][q_len][Hq][d]
  int batch, q_len, kv_len, hq, hkv, d;
  long long q_offset;
  unsigned long long* skipped;  // nullable
  unsigned int* err;            // device error word
  Windows win;
};

struct DecodeParams {
  const void* q;         // raw queries [B][Hq][d]
  const void* kc;        // rotated key cache, chunk-major [B][Hkv][d/16][n_cache][16]
  const void* v;         // value cache [B][n_cache][Hkv][d]
  void* out;             // [B][Hq][d]
  float* partials;       // [B][Hq][n_split][d + 2]
  int batch, hq, hkv, d, n_split;
  int pairing;           // atf_pairing of the raw queries
  long long n_cache;
  long long kv_len[kMaxDecodeBatch];    // keys in this cache: slots 0 .. kv_len-1
  long long q_pos[kMaxDecodeBatch];     // query position (its RoPE angle)
  long long key_pos0[kMaxDecodeBatch];  // position of slot 0 (a key range of a longer sequence)
  float* partial_out;           // nullable: [B][Hq][d + 2] merged (sum, max, row sum) instead of out
  unsigned long long* skipped;  // nullable
  unsigned int* err;
  Windows win;
  double omega[kMaxPairs];
};

struct AppendParams {
  const void* k_new;  // [total_new][hkv][d] bf16, sequences one after the other
  const void* v_new;  // same layout
  void* kc;           // rotated key cache, chunk-major [B][Hkv][d/16][n_cache][16]
  void* vc;           // value cache [B][n_cache][Hkv][d]
  int batch, hkv, d, pairing;
  long long n_cache;
  long long cu[kMaxDecodeBatch + 1];  // first row of sequence b in k_new / v_new
  long long pos[kMaxDecodeBatch];     // position (cache slot) of sequence b's first new token
  double omega[kMaxPairs];
};

// Launchers (return cudaGetLastError() of the launch).
cudaError_t launch_rope(const RopeParams& p, cudaStream_t s);
cudaError_t launch_kv_append(const AppendParams& p, cudaStream_t s);
cudaError_t launch_prefill_simt(const PrefillParams& p, cudaStream_t s);
cudaError_t launch_prefill_tc(const PrefillParams& p, const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                              const CUtensorMap& tm_v, bool dense, cudaStream_t s);
cudaError_t launch_decode_merge(const float* parts, int n_parts, long long rows, int d, void* out, cudaStream_t s);
cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tm_v, const CUtensorMap& tm_k,
                          cudaStream_t s);

// Device address of the library's error word on the current device (bounded
// waits record their code there), or NULL without a usable device.
unsigned int* device_error_word();

// Records a printf-style message as this thread's atf_last_error() and returns st.
atf_status report_error(atf_status st, const char* fmt, ...);

// Number of key-range splits per (sequence, kv head) for a decode launch.
int decode_num_splits(long long max_kv_len, int batch, int hkv);

}  // namespace atf
