// atf_api.cu -- the C ABI (include/atf.h): argument checks, the window table,
// scratch carving, TMA descriptors and kernel launches.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/atf.h"
#include "atf_internal.cuh"
#include "ptx.cuh"

using namespace atf;

// Device error word: kernels record the code of a bounded wait that expired.
__device__ unsigned int g_atf_device_error;

namespace {

thread_local std::string g_last_error;

atf_status fail(atf_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

atf_status cuda_fail(cudaError_t e, const char* what) {
  return fail(ATF_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxDevices = 64;

}  // namespace

unsigned int* atf::device_error_word() {
  static unsigned int* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_atf_device_error) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<unsigned int*>(p);
  }
  return addr[dev];
}

namespace {

// W_i = ceil(alpha * lambda_i), lambda_i = 2 pi / omega_i, omega_i = theta^(-2i/d), fp64.
void window_table(int d, double theta, double alpha, long long* W, double* omega) {
  const double two_pi = 6.283185307179586476925286766559;
  for (int i = 0; i < d / 2; ++i) {
    const double om = std::pow(theta, -2.0 * static_cast<double>(i) / static_cast<double>(d));
    if (omega) omega[i] = om;
    if (std::isinf(alpha)) {
      W[i] = INT64_MAX;
    } else {
      const double w = std::ceil(alpha * (two_pi / om));
      W[i] = w >= 9.2e18 ? INT64_MAX : static_cast<long long>(w);
    }
  }
}

void kernel_windows(int d, double theta, double alpha, Windows* out, double* omega) {
  long long W[kMaxPairs];
  window_table(d, theta, alpha, W, omega);
  for (int i = 0; i < kMaxPairs; ++i) out->w[i] = 0x7fffffff;
  for (int i = 0; i < d / 2; ++i) out->w[i] = W[i] > 0x7fffffffLL ? 0x7fffffff : static_cast<int>(W[i]);
}

atf_status check_params(int d, double theta, double alpha) {
  if (d != 64 && d != 128) return fail(ATF_ERR_UNSUPPORTED, "head dim d=%d not supported (64 or 128)", d);
  if (!(theta > 1.0) || std::isinf(theta)) return fail(ATF_ERR_INVALID_ARG, "theta must be finite and > 1");
  if (!(alpha > 0.0)) return fail(ATF_ERR_INVALID_ARG, "alpha must be > 0 (or +inf)");
  return ATF_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// A [batch][tokens][heads][d] bf16 tensor (queries, keys or values) as a 4-D
// tensor (d, head, token, batch); one box = 64 dims x 1 head x 128 tokens,
// 128-byte swizzle; tokens past the end read as zero.
atf_status kv_tensor_map(CUtensorMap* map, const void* base, int batch, int kv_len, int hkv, int d) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(ATF_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(hkv), static_cast<cuuint64_t>(kv_len),
                        static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(hkv) * d * 2,
                           static_cast<cuuint64_t>(kv_len) * hkv * d * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ATF_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return ATF_OK;
}

// Chunk-major rotated key cache [batch][kv_heads][d/16][n_cache][16] bf16 as a
// 5-D tensor (16 elements, token, chunk, head, batch); one box = 16 elements x
// 128 tokens of one chunk (32-byte rows, 32-byte swizzle); tokens past n_cache
// read as zero.
atf_status kc_tensor_map(CUtensorMap* map, const void* base, int batch, int hkv, int d, long long n_cache) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(ATF_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  const cuuint64_t nc = static_cast<cuuint64_t>(d / 16);
  const cuuint64_t n = static_cast<cuuint64_t>(n_cache);
  cuuint64_t dims[5] = {16, n, nc, static_cast<cuuint64_t>(hkv), static_cast<cuuint64_t>(batch)};
  cuuint64_t strides[4] = {32, n * 32, nc * n * 32, static_cast<cuuint64_t>(hkv) * nc * n * 32};
  cuuint32_t box[5] = {16, 128, 1, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ATF_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return ATF_OK;
}

// Self-test kernel: one warp waits on a barrier nobody completes, gives up after
// `limit` cycles, records the expiry in the device error word.
__global__ void timeout_selftest_kernel(long long limit, unsigned int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const long long t0 = clock64();
    bool done = false;
    while (!(done = mbar_try_wait(&bar, 0)) && clock64() - t0 < limit) {
    }
    if (!done) atomicCAS(err, 0u, 0x7E57u);
    mbar_arrive(&bar);  // complete the phase so the barrier is not left pending
  }
}

}  // namespace

atf_status atf::report_error(atf_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

extern "C" {

const char* atf_last_error(void) { return g_last_error.c_str(); }

atf_status atf_windows(int d, double theta, double alpha, long long* W_out) {
  if (!W_out) return fail(ATF_ERR_INVALID_ARG, "W_out is NULL");
  if (atf_status st = check_params(d, theta, alpha)) return st;
  window_table(d, theta, alpha, W_out, nullptr);
  return ATF_OK;
}

atf_status atf_rope_layout(const void* x, void* x_rot, void* x_chunked, int batch, int seq, int heads, int d,
                           long long pos_offset, double theta, int rotate, int dtype, void* stream) {
  if (atf_status st = check_params(d, theta, 1.0)) return st;
  if (batch < 0 || seq < 0 || heads < 1 || pos_offset < 0)
    return fail(ATF_ERR_INVALID_ARG, "rope_layout: bad sizes");
  if (dtype != ATF_BF16 && dtype != ATF_FP32) return fail(ATF_ERR_INVALID_ARG, "bad dtype %d", dtype);
  if (rotate < 0 || rotate > 3) return fail(ATF_ERR_INVALID_ARG, "rope_layout: rotate %d", rotate);
  if (x_chunked && dtype != ATF_BF16) return fail(ATF_ERR_UNSUPPORTED, "chunk-major layout is bf16 only");
  if (static_cast<long long>(batch) * seq == 0) return ATF_OK;
  if (!x || (!x_rot && !x_chunked)) return fail(ATF_ERR_INVALID_ARG, "rope_layout: null pointer");
  if (!aligned16(x) || (x_rot && !aligned16(x_rot)) || (x_chunked && !aligned16(x_chunked)))
    return fail(ATF_ERR_INVALID_ARG, "rope_layout: pointers must be 16-byte aligned");
  RopeParams p{};
  p.x = x;
  p.x_rot = x_rot;
  p.x_chunked = x_chunked;
  p.batch = batch;
  p.seq = seq;
  p.heads = heads;
  p.d = d;
  p.pos_offset = pos_offset;
  p.rotate = rotate;
  p.fp32 = dtype == ATF_FP32;
  Windows w;
  kernel_windows(d, theta, INFINITY, &w, p.omega);
  cudaError_t e = launch_rope(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rope kernel launch");
  return ATF_OK;
}

size_t atf_prefill_workspace_bytes(int batch, int q_len, int kv_len, int heads, int kv_heads, int d, int dtype,
                                   int rotated) {
  if (rotated || batch <= 0 || d <= 0) return 0;
  const size_t esz = dtype == ATF_FP32 ? 4 : 2;
  const size_t qb = round_up(static_cast<size_t>(batch) * q_len * heads * d * esz, 256);
  const size_t kb = round_up(static_cast<size_t>(batch) * kv_len * kv_heads * d * esz, 256);
  return qb + kb;
}

atf_status atf_prefill_ex(const atf_prefill_args* a, void* stream) {
  if (!a) return fail(ATF_ERR_INVALID_ARG, "args is NULL");
  if (atf_status st = check_params(a->d, a->theta, a->alpha)) return st;
  if (a->dtype != ATF_BF16 && a->dtype != ATF_FP32) return fail(ATF_ERR_INVALID_ARG, "bad dtype %d", a->dtype);
  if (a->batch < 0 || a->q_len < 0 || a->kv_len < 0 || a->q_offset < 0 || a->heads < 1 || a->kv_heads < 1)
    return fail(ATF_ERR_INVALID_ARG, "prefill: negative or zero sizes");
  if (a->pairing != ATF_PAIRS_INTERLEAVED && a->pairing != ATF_PAIRS_ROTATE_HALF)
    return fail(ATF_ERR_INVALID_ARG, "prefill: pairing %d", a->pairing);
  if (a->heads % a->kv_heads) return fail(ATF_ERR_INVALID_ARG, "heads %% kv_heads != 0");
  if (static_cast<long long>(a->kv_len) < a->q_offset + a->q_len)
    return fail(ATF_ERR_INVALID_ARG, "prefill: kv_len (%d) < q_offset + q_len (%lld)", a->kv_len,
                a->q_offset + a->q_len);
  if (a->q_offset + a->q_len > 0x7fffffffLL) return fail(ATF_ERR_UNSUPPORTED, "positions must stay below 2^31");
  if (static_cast<long long>(a->batch) * a->q_len == 0) return ATF_OK;
  if (!a->q || !a->k || !a->v || !a->out) return fail(ATF_ERR_INVALID_ARG, "prefill: null tensor pointer");
  if (!aligned16(a->q) || !aligned16(a->k) || !aligned16(a->v) || !aligned16(a->out))
    return fail(ATF_ERR_INVALID_ARG, "prefill: pointers must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!a->rotated) {
    const size_t need =
        atf_prefill_workspace_bytes(a->batch, a->q_len, a->kv_len, a->heads, a->kv_heads, a->d, a->dtype, 0);
    if (!a->workspace || a->workspace_bytes < need)
      return fail(ATF_ERR_INVALID_ARG, "prefill: workspace of %zu bytes needed", need);
    if (!aligned16(a->workspace)) return fail(ATF_ERR_INVALID_ARG, "prefill: workspace must be 16-byte aligned");
  }
  unsigned int* err = device_error_word();
  if (!err) return fail(ATF_ERR_CUDA, "no CUDA device / device error word unavailable");

  const void* q = a->q;
  const void* k = a->k;
  if (!a->rotated) {
    const size_t esz = a->dtype == ATF_FP32 ? 4 : 2;
    char* ws = static_cast<char*>(a->workspace);
    void* q_rot = ws;
    void* k_rot = ws + round_up(static_cast<size_t>(a->batch) * a->q_len * a->heads * a->d * esz, 256);
    // queries at positions q_offset + t, keys at positions n (every batch entry alike)
    const int mode = a->pairing == ATF_PAIRS_ROTATE_HALF ? 2 : 1;  // rotate-half pairs end up interleaved
    atf_status st = atf_rope_layout(a->q, q_rot, nullptr, a->batch, a->q_len, a->heads, a->d, a->q_offset,
                                    a->theta, mode, a->dtype, stream);
    if (st) return st;
    st = atf_rope_layout(a->k, k_rot, nullptr, a->batch, a->kv_len, a->kv_heads, a->d, 0, a->theta, mode,
                         a->dtype, stream);
    if (st) return st;
    q = q_rot;
    k = k_rot;
  }

  PrefillParams p{};
  p.q = q;
  p.k = k;
  p.v = a->v;
  p.out = a->out;
  p.batch = a->batch;
  p.q_len = a->q_len;
  p.kv_len = a->kv_len;
  p.hq = a->heads;
  p.hkv = a->kv_heads;
  p.d = a->d;
  p.q_offset = a->q_offset;
  p.skipped = a->skipped_pairs;
  p.err = err;
  kernel_windows(a->d, a->theta, a->alpha, &p.win, nullptr);

  cudaError_t e;
  if (a->dtype == ATF_FP32) {
    e = launch_prefill_simt(p, s);
  } else {
    CUtensorMap tq, tk, tv;
    if (atf_status st = kv_tensor_map(&tq, q, a->batch, a->q_len, a->heads, a->d)) return st;
    if (atf_status st = kv_tensor_map(&tk, k, a->batch, a->kv_len, a->kv_heads, a->d)) return st;
    if (atf_status st = kv_tensor_map(&tv, a->v, a->batch, a->kv_len, a->kv_heads, a->d)) return st;
    e = launch_prefill_tc(p, tq, tk, tv, std::isinf(a->alpha), s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "prefill kernel launch");
  return ATF_OK;
}

atf_status atf_prefill(const void* q, const void* k, const void* v, void* out, int seq, int heads, int kv_heads,
                       int d, double theta, double alpha, void* stream) {
  atf_prefill_args a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.out = out;
  a.batch = 1;
  a.q_len = seq;
  a.kv_len = seq;
  a.heads = heads;
  a.kv_heads = kv_heads;
  a.d = d;
  a.q_offset = 0;
  a.dtype = ATF_BF16;
  a.rotated = 0;
  a.theta = theta;
  a.alpha = alpha;
  if (seq < 0 || heads < 1 || kv_heads < 1) return fail(ATF_ERR_INVALID_ARG, "prefill: bad sizes");
  const size_t need = atf_prefill_workspace_bytes(1, seq, seq, heads, kv_heads, d, ATF_BF16, 0);
  if (need == 0 || seq == 0) return atf_prefill_ex(&a, stream);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  cudaError_t e = cudaMallocAsync(&ws, need, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(prefill scratch)");
  a.workspace = ws;
  a.workspace_bytes = need;
  atf_status st = atf_prefill_ex(&a, stream);
  e = cudaFreeAsync(ws, s);
  if (st) return st;
  if (e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync(prefill scratch)");
  return ATF_OK;
}

size_t atf_decode_workspace_bytes(int batch, int heads, int kv_heads, long long max_kv_len, int d) {
  if (batch <= 0 || heads <= 0 || kv_heads <= 0 || d <= 0) return 0;
  const int per = batch < kMaxDecodeBatch ? batch : kMaxDecodeBatch;
  const int ns = decode_num_splits(max_kv_len, per, kv_heads);
  return static_cast<size_t>(batch) * heads * ns * (d + 2) * sizeof(float);
}

}  // extern "C"

namespace {

// The decode of atf_decode and atf_decode_partial.  Sequence b's cache holds
// n_keys[b] keys in slots 0.., slot 0 at position key_pos0[b] (0 when NULL); its
// query sits at q_pos[b] (n_keys[b] - 1 + key_pos0[b] when NULL).  Writes the
// bf16 output, or with partial_out the merged partial of these keys.
atf_status decode_impl(const void* q, const void* k_chunked, const void* v, void* out, float* partial_out,
                       int batch, const long long* n_keys, const long long* key_pos0, const long long* q_pos,
                       long long n_cache, int heads, int kv_heads, int d, double theta, double alpha, int pairing,
                       void* workspace, size_t workspace_bytes, unsigned long long* skipped_pairs, void* stream) {
  const bool partial = partial_out != nullptr;
  if (atf_status st = check_params(d, theta, alpha)) return st;
  if (pairing != ATF_PAIRS_INTERLEAVED && pairing != ATF_PAIRS_ROTATE_HALF)
    return fail(ATF_ERR_INVALID_ARG, "decode: pairing %d", pairing);
  if (batch < 0 || heads < 1 || kv_heads < 1 || n_cache < 1) return fail(ATF_ERR_INVALID_ARG, "decode: bad sizes");
  if (heads % kv_heads) return fail(ATF_ERR_INVALID_ARG, "heads %% kv_heads != 0");
  if (heads / kv_heads > 8) return fail(ATF_ERR_UNSUPPORTED, "decode: at most 8 query heads per kv head");
  if (n_cache > 0x7fffffffLL) return fail(ATF_ERR_UNSUPPORTED, "decode: cache longer than 2^31-1");
  if (batch == 0) return ATF_OK;
  if (!q || !k_chunked || !v || !(out || partial_out) || !n_keys) return fail(ATF_ERR_INVALID_ARG, "decode: null pointer");
  if (!aligned16(q) || !aligned16(k_chunked) || !aligned16(v) || (out && !aligned16(out)) ||
      (partial_out && !aligned16(partial_out)) || !aligned16(workspace))
    return fail(ATF_ERR_INVALID_ARG, "decode: pointers must be 16-byte aligned");
  long long max_len = 0;
  for (int b = 0; b < batch; ++b) {
    const long long lo = partial ? 0 : 1;  // a key range may be empty; a whole sequence holds its query's key
    if (n_keys[b] < lo || n_keys[b] > n_cache)
      return fail(ATF_ERR_INVALID_ARG, "decode: kv_len[%d]=%lld outside [%lld, n_cache]", b, n_keys[b], lo);
    const long long p0 = key_pos0 ? key_pos0[b] : 0;
    const long long qp = q_pos ? q_pos[b] : p0 + n_keys[b] - 1;
    if (p0 < 0 || qp < 0 || qp < p0 + n_keys[b] - 1 || qp > (1LL << 40))
      return fail(ATF_ERR_INVALID_ARG, "decode: sequence %d: the query (position %lld) must not precede its keys "
                  "(positions %lld ..%lld)", b, qp, p0, p0 + n_keys[b] - 1);
    // the kernels hold windows and distances in 32 bits (W_i clamped to 2^31-1):
    // every query-key distance must stay below 2^31 for that clamp to be exact
    if (qp - p0 > 0x7fffffffLL)
      return fail(ATF_ERR_UNSUPPORTED, "decode: sequence %d: the query (position %lld) is 2^31 or more positions "
                  "after its first key (position %lld)", b, qp, p0);
    if (n_keys[b] > max_len) max_len = n_keys[b];
  }
  const size_t need = atf_decode_workspace_bytes(batch, heads, kv_heads, max_len, d);
  if (!workspace || workspace_bytes < need)
    return fail(ATF_ERR_INVALID_ARG, "decode: workspace of %zu bytes needed", need);
  unsigned int* err = device_error_word();
  if (!err) return fail(ATF_ERR_CUDA, "no CUDA device / device error word unavailable");
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const int per = batch < kMaxDecodeBatch ? batch : kMaxDecodeBatch;
  const int ns = decode_num_splits(max_len, per, kv_heads);
  Windows w;
  DecodeParams p{};
  kernel_windows(d, theta, alpha, &w, p.omega);
  p.win = w;
  p.hq = heads;
  p.hkv = kv_heads;
  p.d = d;
  p.n_split = ns;
  p.pairing = pairing;
  p.n_cache = n_cache;
  p.skipped = skipped_pairs;
  p.err = err;
  const size_t esz = 2;
  for (int b0 = 0; b0 < batch; b0 += kMaxDecodeBatch) {
    const int nb = batch - b0 < kMaxDecodeBatch ? batch - b0 : kMaxDecodeBatch;
    p.batch = nb;
    for (int i = 0; i < nb; ++i) {
      p.kv_len[i] = n_keys[b0 + i];
      p.key_pos0[i] = key_pos0 ? key_pos0[b0 + i] : 0;
      p.q_pos[i] = q_pos ? q_pos[b0 + i] : p.key_pos0[i] + p.kv_len[i] - 1;
    }
    p.q = static_cast<const char*>(q) + static_cast<size_t>(b0) * heads * d * esz;
    p.kc = static_cast<const char*>(k_chunked) + static_cast<size_t>(b0) * kv_heads * n_cache * d * esz;
    p.v = static_cast<const char*>(v) + static_cast<size_t>(b0) * n_cache * kv_heads * d * esz;
    p.out = out ? static_cast<char*>(out) + static_cast<size_t>(b0) * heads * d * esz : nullptr;
    p.partial_out = partial_out ? partial_out + static_cast<size_t>(b0) * heads * (d + 2) : nullptr;
    p.partials = static_cast<float*>(workspace) + static_cast<size_t>(b0) * heads * ns * (d + 2);
    CUtensorMap tv, tk;
    if (atf_status st = kv_tensor_map(&tv, p.v, nb, static_cast<int>(n_cache), kv_heads, d)) return st;
    if (atf_status st = kc_tensor_map(&tk, p.kc, nb, kv_heads, d, n_cache)) return st;
    cudaError_t e = launch_decode(p, tv, tk, s);
    if (e != cudaSuccess) return cuda_fail(e, "decode kernel launch");
  }
  return ATF_OK;
}

}  // namespace

extern "C" {

atf_status atf_decode(const void* q, const void* k_chunked, const void* v, void* out, int batch,
                      const long long* kv_len, long long n_cache, int heads, int kv_heads, int d, double theta,
                      double alpha, int pairing, void* workspace, size_t workspace_bytes,
                      unsigned long long* skipped_pairs, void* stream) {
  if (batch > 0 && !out) return fail(ATF_ERR_INVALID_ARG, "decode: null pointer");
  return decode_impl(q, k_chunked, v, out, nullptr, batch, kv_len, nullptr, nullptr, n_cache, heads, kv_heads, d,
                     theta, alpha, pairing, workspace, workspace_bytes, skipped_pairs, stream);
}

atf_status atf_decode_partial(const void* q, const void* k_chunked, const void* v, float* partial, int batch,
                              const long long* n_keys, const long long* key_pos0, const long long* q_pos,
                              long long n_cache, int heads, int kv_heads, int d, double theta, double alpha,
                              int pairing, void* workspace, size_t workspace_bytes,
                              unsigned long long* skipped_pairs, void* stream) {
  if (batch > 0 && (!partial || !key_pos0 || !q_pos)) return fail(ATF_ERR_INVALID_ARG, "decode_partial: null pointer");
  return decode_impl(q, k_chunked, v, nullptr, partial, batch, n_keys, key_pos0, q_pos, n_cache, heads, kv_heads, d,
                     theta, alpha, pairing, workspace, workspace_bytes, skipped_pairs, stream);
}

atf_status atf_decode_merge(const float* partials, int n_parts, int batch, int heads, int d, void* out,
                            void* stream) {
  if (d != 64 && d != 128) return fail(ATF_ERR_UNSUPPORTED, "head dim d=%d not supported (64 or 128)", d);
  if (n_parts < 1 || batch < 0 || heads < 1) return fail(ATF_ERR_INVALID_ARG, "decode_merge: bad sizes");
  if (batch == 0) return ATF_OK;
  if (!partials || !out) return fail(ATF_ERR_INVALID_ARG, "decode_merge: null pointer");
  if (!aligned16(partials) || !aligned16(out))
    return fail(ATF_ERR_INVALID_ARG, "decode_merge: pointers must be 16-byte aligned");
  cudaError_t e = launch_decode_merge(partials, n_parts, static_cast<long long>(batch) * heads, d, out,
                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "decode merge launch");
  return ATF_OK;
}

atf_status atf_kv_append(const void* k_new, const void* v_new, void* k_cache_chunked, void* v_cache, int batch,
                         const int* n_new, const long long* pos, long long n_cache, int kv_heads, int d,
                         double theta, int pairing, void* stream) {
  if (atf_status st = check_params(d, theta, 1.0)) return st;
  if (batch < 0 || kv_heads < 1 || n_cache < 1) return fail(ATF_ERR_INVALID_ARG, "kv_append: bad sizes");
  if (n_cache > 0x7fffffffLL) return fail(ATF_ERR_UNSUPPORTED, "kv_append: cache longer than 2^31-1");
  if (pairing != ATF_PAIRS_INTERLEAVED && pairing != ATF_PAIRS_ROTATE_HALF)
    return fail(ATF_ERR_INVALID_ARG, "kv_append: pairing %d", pairing);
  if (batch == 0) return ATF_OK;
  if (!n_new || !pos) return fail(ATF_ERR_INVALID_ARG, "kv_append: null n_new / pos");
  long long total = 0;
  for (int b = 0; b < batch; ++b) {
    if (n_new[b] < 0 || pos[b] < 0 || pos[b] + n_new[b] > n_cache)
      return fail(ATF_ERR_INVALID_ARG, "kv_append: sequence %d: %d tokens at %lld do not fit %lld slots", b,
                  n_new[b], pos[b], n_cache);
    total += n_new[b];
  }
  if (total == 0) return ATF_OK;
  if (!k_new || !v_new || !k_cache_chunked || !v_cache) return fail(ATF_ERR_INVALID_ARG, "kv_append: null pointer");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache_chunked) || !aligned16(v_cache))
    return fail(ATF_ERR_INVALID_ARG, "kv_append: pointers must be 16-byte aligned");
  AppendParams p{};
  Windows w;
  kernel_windows(d, theta, INFINITY, &w, p.omega);
  p.hkv = kv_heads;
  p.d = d;
  p.pairing = pairing;
  p.n_cache = n_cache;
  const size_t row_bytes = static_cast<size_t>(kv_heads) * d * 2;  // one token of k_new / v_new
  long long row0 = 0;                                                // first row of the group
  for (int b0 = 0; b0 < batch; b0 += kMaxDecodeBatch) {
    const int nb = batch - b0 < kMaxDecodeBatch ? batch - b0 : kMaxDecodeBatch;
    p.batch = nb;
    p.cu[0] = 0;
    for (int i = 0; i < nb; ++i) {
      p.cu[i + 1] = p.cu[i] + n_new[b0 + i];
      p.pos[i] = pos[b0 + i];
    }
    p.k_new = static_cast<const char*>(k_new) + static_cast<size_t>(row0) * row_bytes;
    p.v_new = static_cast<const char*>(v_new) + static_cast<size_t>(row0) * row_bytes;
    p.kc = static_cast<char*>(k_cache_chunked) + static_cast<size_t>(b0) * n_cache * row_bytes;
    p.vc = static_cast<char*>(v_cache) + static_cast<size_t>(b0) * n_cache * row_bytes;
    cudaError_t e = launch_kv_append(p, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "kv_append kernel launch");
    row0 += p.cu[nb];
  }
  return ATF_OK;
}

atf_status atf_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  unsigned int code = 0;
  e = cudaMemcpyFromSymbol(&code, g_atf_device_error, sizeof code);
  if (e != cudaSuccess) return cuda_fail(e, "read device error word");
  if (code) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_atf_device_error, &zero, sizeof zero);
    return fail(ATF_ERR_TIMEOUT, "a kernel gave up a bounded wait (code 0x%x)", code);
  }
  return ATF_OK;
}

atf_status atf_selftest_timeout(long long limit_cycles, void* stream) {
  if (limit_cycles < 0) return fail(ATF_ERR_INVALID_ARG, "limit_cycles < 0");
  unsigned int* err = device_error_word();
  if (!err) return fail(ATF_ERR_CUDA, "no CUDA device / device error word unavailable");
  timeout_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_cycles, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return ATF_OK;
}

}  // extern "C"
