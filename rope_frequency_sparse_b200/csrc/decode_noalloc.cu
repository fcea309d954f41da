// decode_noalloc.cu -- atf_decode for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc (or any allocating routine) on the decode
// path: a host application whose own memory manager owns all device memory and
// forbids allocations behind its back, or a latency-critical serving loop where
// an allocation may synchronise the device.  They also cannot easily provide a
// workspace.  For them the decode's split-softmax partials live in a fixed
// file-scope device array instead of a caller workspace.
//
// The array is kDecodeScratchBytes (8 MiB) and is held on every GPU that loads
// the library until the process exits.  All calls on a device share it, and it
// keeps the previous call's contents; the decode overwrites every partial it
// later reads, so nothing needs clearing.  Two calls whose kernels overlap on the
// GPU (different streams, no ordering between them) race on it.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/atf.h"
#include "atf_internal.cuh"

namespace {

constexpr size_t kDecodeScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kDecodeScratchBytes];

// Device address of g_decode_scratch on the current device.  In host code the
// symbol is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached.
void* scratch_address(atf_status* st) {
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *st = atf::report_error(ATF_ERR_CUDA, "decode_noalloc: no current CUDA device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
      *st = atf::report_error(ATF_ERR_CUDA, "decode_noalloc: cudaGetSymbolAddress of the scratch array failed");
      return nullptr;
    }
    addr[dev] = p;
  }
  *st = ATF_OK;
  return addr[dev];
}

}  // namespace

extern "C" size_t atf_decode_noalloc_scratch_bytes(void) { return kDecodeScratchBytes; }

extern "C" atf_status atf_decode_noalloc(const void* q, const void* k_chunked, const void* v, void* out, int batch,
                                         const long long* kv_len, long long n_cache, int heads, int kv_heads, int d,
                                         double theta, double alpha, int pairing,
                                         unsigned long long* skipped_pairs, void* stream) {
  if (batch > 0 && !kv_len) return atf::report_error(ATF_ERR_INVALID_ARG, "decode_noalloc: kv_len is NULL");
  long long max_len = 1;
  for (int b = 0; b < batch; ++b)
    if (kv_len[b] > max_len) max_len = kv_len[b];
  const size_t need = atf_decode_workspace_bytes(batch, heads, kv_heads, max_len, d);
  if (need > kDecodeScratchBytes)
    return atf::report_error(ATF_ERR_UNSUPPORTED,
                             "decode_noalloc: this call needs %zu bytes of scratch, more than the fixed %zu; "
                             "use atf_decode with a workspace",
                             need, kDecodeScratchBytes);
  atf_status st = ATF_OK;
  void* scratch = batch > 0 ? scratch_address(&st) : nullptr;
  if (st != ATF_OK) return st;
  return atf_decode(q, k_chunked, v, out, batch, kv_len, n_cache, heads, kv_heads, d, theta, alpha, pairing,
                    scratch, kDecodeScratchBytes, skipped_pairs, stream);
}
