// prefill_host.cu -- atf_prefill_host: the prefill path from host buffers, with
// the host<->device copies overlapped with each other and with the kernels.
//
// A prefill whose inputs start in host memory is bound by the PCIe copies, not by
// the kernels: the inputs (q, k, v) and the output cross the bus once each, and the
// kernels take a fraction of that time.  Done one after the other the call costs
// copy-in + kernels + copy-out.  Here the query rows are cut into chunks, and
//
//   upload stream:    k | v | q chunk n-1 | q chunk n-2 | q chunk n-3 | ...
//   compute stream A:      rope(k) | rope+attn(n-1)   | rope+attn(n-3) ...
//   compute stream B:                    | rope+attn(n-2)   | ...
//   download stream:                          out n-1 | out n-2 | ...
//
// so the copies in the two directions (separate copy engines) run at the same
// time, and each chunk's kernels run while later chunks are being uploaded.  A
// chunk holds a run of query rows of every batch entry and is attended as a
// chunked prefill at offset q_offset + its first row against all kv_len keys:
// the result is the same as one prefill over all rows.  The chunks go from the
// last rows to the first because the last rows are the costliest (they see the
// most keys), so their kernels overlap the most remaining copy work and the call
// ends on the cheapest chunk.  One chunk's grid (its rows x heads / 256 CTAs)
// may not fill the GPU; the chunks alternate between the caller's stream and a
// second compute stream so that two chunks' kernels can share the SMs.
//
// The copy streams, the second compute stream and the events are created once
// per device and host thread and kept for the life of the process.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <vector>

#include "../../include/atf.h"
#include "atf_internal.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kAlign = 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct CopyStreams {
  bool ready = false;
  cudaStream_t up = nullptr;     // host -> device
  cudaStream_t down = nullptr;   // device -> host
  cudaStream_t aux = nullptr;    // second compute stream (every other chunk)
  cudaEvent_t start = nullptr;      // caller stream: everything before the call
  cudaEvent_t in_ready = nullptr;   // upload stream: the latest upload
  cudaEvent_t kv_ready = nullptr;   // caller stream: rotated keys and values in place
  cudaEvent_t out_ready = nullptr;  // a compute stream: the latest chunk's output
  cudaEvent_t aux_done = nullptr;   // second compute stream: its last chunk
  cudaEvent_t done = nullptr;       // download stream: the last download
};

atf_status copy_streams(CopyStreams** out) {
  static thread_local CopyStreams per_device[kMaxDevices];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return atf::report_error(ATF_ERR_CUDA, "prefill_host: no current CUDA device");
  CopyStreams& cs = per_device[dev];
  if (!cs.ready) {
    cudaError_t e = cudaStreamCreateWithFlags(&cs.up, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&cs.down, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&cs.aux, cudaStreamNonBlocking);
    cudaEvent_t* evs[6] = {&cs.start, &cs.in_ready, &cs.kv_ready, &cs.out_ready, &cs.aux_done, &cs.done};
    for (int i = 0; i < 6 && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(evs[i], cudaEventDisableTiming);
    if (e != cudaSuccess)
      return atf::report_error(ATF_ERR_CUDA, "prefill_host: creating copy streams: %s", cudaGetErrorString(e));
    cs.ready = true;
  }
  *out = &cs;
  return ATF_OK;
}

// Device scratch layout: k (raw), k (rotated), v, q (raw), q (rotated), out; each
// region 256-byte aligned.  With rotated inputs the raw regions are empty and the
// uploads land directly in the rotated ones.
struct Layout {
  size_t k_raw, k_rot, v, q_raw, q_rot, out, total;
};

Layout layout(int batch, int q_len, int kv_len, int heads, int kv_heads, int d, int rotated) {
  const size_t kvb = round_up(static_cast<size_t>(batch) * kv_len * kv_heads * d * 2, kAlign);
  const size_t qb = round_up(static_cast<size_t>(batch) * q_len * heads * d * 2, kAlign);
  Layout L{};
  size_t off = 0;
  L.k_raw = off;
  off += rotated ? 0 : kvb;
  L.k_rot = off;
  off += kvb;
  L.v = off;
  off += kvb;
  L.q_raw = off;
  off += rotated ? 0 : qb;
  L.q_rot = off;
  off += qb;
  L.out = off;
  off += qb;
  L.total = off;
  return L;
}

// Copies `rows` bytes-wide rows: row b from src + b * src_pitch to dst + b * dst_pitch.
// One 2-D copy when the pitches fit the 2-D copy's limit, else one copy per row.
cudaError_t copy_rows(void* dst, size_t dst_pitch, const void* src, size_t src_pitch, size_t width, int rows,
                      cudaStream_t s) {
  constexpr size_t kMaxPitch = 0x7fffffff;
  if (rows > 1 && dst_pitch <= kMaxPitch && src_pitch <= kMaxPitch)
    return cudaMemcpy2DAsync(dst, dst_pitch, src, src_pitch, width, rows, cudaMemcpyDefault, s);
  for (int b = 0; b < rows; ++b) {
    cudaError_t e = cudaMemcpyAsync(static_cast<char*>(dst) + b * dst_pitch,
                                    static_cast<const char*>(src) + b * src_pitch, width, cudaMemcpyDefault, s);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

struct Chunk {
  int first, rows;
};

// Chunks of query rows in processing order, last rows first.  chunk_rows > 0:
// [c*R, c*R + R) for c = n-1 .. 0.  chunk_rows = 0: R = q_len/8 rounded up to a
// multiple of 256, and the chunks taken from the end grow R/4 (at least 256),
// R/2, then R: the first chunk's kernel sees every key and takes the longest,
// and the downloads wait for it, so it is kept small.  Every boundary is a
// multiple of 256 rows, where the one-shot prefill's query tiles start too.
std::vector<Chunk> chunk_schedule(int q_len, int chunk_rows) {
  std::vector<Chunk> out;
  if (chunk_rows > 0) {
    for (int r0 = (q_len - 1) / chunk_rows * chunk_rows; r0 >= 0; r0 -= chunk_rows)
      out.push_back({r0, q_len - r0 < chunk_rows ? q_len - r0 : chunk_rows});
    return out;
  }
  const int R = static_cast<int>(round_up((static_cast<size_t>(q_len) + 7) / 8, 256));
  int size = R / 4 > 256 ? R / 4 : 256;
  for (int top = q_len; top > 0;) {
    int lo = top - size;
    lo = lo <= 0 ? 0 : lo / 256 * 256;
    out.push_back({lo, top - lo});
    top = lo;
    size = 2 * size < R ? 2 * size : R;
  }
  return out;
}

}  // namespace

extern "C" size_t atf_prefill_host_workspace_bytes(int batch, int q_len, int kv_len, int heads, int kv_heads, int d,
                                                   int rotated) {
  if (batch <= 0 || q_len <= 0 || kv_len <= 0 || heads <= 0 || kv_heads <= 0 || d <= 0) return 0;
  return layout(batch, q_len, kv_len, heads, kv_heads, d, rotated).total;
}

extern "C" atf_status atf_prefill_host(const atf_prefill_args* a, int chunk_rows, void* stream) {
  if (!a) return atf::report_error(ATF_ERR_INVALID_ARG, "args is NULL");
  if (a->dtype != ATF_BF16) return atf::report_error(ATF_ERR_UNSUPPORTED, "prefill_host: bf16 only");
  if (a->batch < 0 || a->q_len < 0 || a->kv_len < 0 || a->q_offset < 0 || a->heads < 1 || a->kv_heads < 1 ||
      chunk_rows < 0)
    return atf::report_error(ATF_ERR_INVALID_ARG, "prefill_host: negative or zero sizes");
  if (static_cast<long long>(a->kv_len) < a->q_offset + a->q_len)
    return atf::report_error(ATF_ERR_INVALID_ARG, "prefill_host: kv_len (%d) < q_offset + q_len (%lld)", a->kv_len,
                             a->q_offset + a->q_len);
  if (static_cast<long long>(a->batch) * a->q_len == 0) return ATF_OK;
  if (!a->q || !a->k || !a->v || !a->out) return atf::report_error(ATF_ERR_INVALID_ARG, "prefill_host: null pointer");
  if (a->d != 64 && a->d != 128)
    return atf::report_error(ATF_ERR_UNSUPPORTED, "head dim d=%d not supported (64 or 128)", a->d);
  // the remaining checks of atf_prefill_ex, made here before any copy is queued
  if (!(a->theta > 1.0) || !(a->theta < INFINITY) || !(a->alpha > 0.0))
    return atf::report_error(ATF_ERR_INVALID_ARG, "prefill_host: need finite theta > 1 and alpha > 0");
  if (a->pairing != ATF_PAIRS_INTERLEAVED && a->pairing != ATF_PAIRS_ROTATE_HALF)
    return atf::report_error(ATF_ERR_INVALID_ARG, "prefill_host: pairing %d", a->pairing);
  if (a->heads % a->kv_heads) return atf::report_error(ATF_ERR_INVALID_ARG, "heads %% kv_heads != 0");
  if (a->q_offset + a->q_len > 0x7fffffffLL)
    return atf::report_error(ATF_ERR_UNSUPPORTED, "positions must stay below 2^31");
  const Layout L = layout(a->batch, a->q_len, a->kv_len, a->heads, a->kv_heads, a->d, a->rotated);
  if (!a->workspace || a->workspace_bytes < L.total)
    return atf::report_error(ATF_ERR_INVALID_ARG, "prefill_host: device workspace of %zu bytes needed", L.total);
  if (!aligned16(a->workspace))
    return atf::report_error(ATF_ERR_INVALID_ARG, "prefill_host: workspace must be 16-byte aligned");

  CopyStreams* cs = nullptr;
  if (atf_status st = copy_streams(&cs)) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(a->workspace);
  const int B = a->batch, Hq = a->heads, Hkv = a->kv_heads, d = a->d;
  const size_t q_row = static_cast<size_t>(Hq) * d * 2;      // bytes of one token's queries
  const size_t kv_bytes = static_cast<size_t>(B) * a->kv_len * Hkv * d * 2;
  const std::vector<Chunk> chunks = chunk_schedule(a->q_len, chunk_rows);
  void* k_up = ws + (a->rotated ? L.k_rot : L.k_raw);
  char* q_up = ws + (a->rotated ? L.q_rot : L.q_raw);
  const int mode = a->pairing == ATF_PAIRS_ROTATE_HALF ? 2 : 1;
  cudaStream_t compute[2] = {s, cs->aux};

  atf_status st = ATF_OK;
  cudaError_t e = cudaEventRecord(cs->start, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs->up, cs->start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs->down, cs->start, 0);
  // k, then v; rope(k) overlaps the upload of v
  if (e == cudaSuccess) e = cudaMemcpyAsync(k_up, a->k, kv_bytes, cudaMemcpyDefault, cs->up);
  if (e == cudaSuccess) e = cudaEventRecord(cs->in_ready, cs->up);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, cs->in_ready, 0);
  if (e == cudaSuccess && !a->rotated)
    st = atf_rope_layout(k_up, ws + L.k_rot, nullptr, B, a->kv_len, Hkv, d, 0, a->theta, mode, ATF_BF16, s);
  if (e == cudaSuccess && !st) e = cudaMemcpyAsync(ws + L.v, a->v, kv_bytes, cudaMemcpyDefault, cs->up);
  if (e == cudaSuccess && !st) e = cudaEventRecord(cs->in_ready, cs->up);
  if (e == cudaSuccess && !st) e = cudaStreamWaitEvent(s, cs->in_ready, 0);
  // the second compute stream starts once the rotated keys and the values are in place
  if (e == cudaSuccess && !st) e = cudaEventRecord(cs->kv_ready, s);
  if (e == cudaSuccess && !st) e = cudaStreamWaitEvent(cs->aux, cs->kv_ready, 0);

  const size_t host_pitch = static_cast<size_t>(a->q_len) * q_row;
  for (size_t i = 0; i < chunks.size() && e == cudaSuccess && !st; ++i) {
    const int r0 = chunks[i].first, rows = chunks[i].rows;
    cudaStream_t cstr = compute[i & 1];
    // the chunk's rows of every batch entry, packed as a dense [B][rows][Hq][d]
    // tensor at the place the rows before it take in the packed buffer
    const size_t chunk_off = static_cast<size_t>(B) * r0 * q_row;
    const size_t width = static_cast<size_t>(rows) * q_row;
    e = copy_rows(q_up + chunk_off, width, static_cast<const char*>(a->q) + r0 * q_row, host_pitch, width, B,
                  cs->up);
    if (e == cudaSuccess) e = cudaEventRecord(cs->in_ready, cs->up);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cstr, cs->in_ready, 0);
    if (e != cudaSuccess) break;
    atf_prefill_args p = *a;
    p.q = q_up + chunk_off;
    if (!a->rotated) {
      st = atf_rope_layout(p.q, ws + L.q_rot + chunk_off, nullptr, B, rows, Hq, d, a->q_offset + r0, a->theta,
                           mode, ATF_BF16, cstr);
      if (st) break;
      p.q = ws + L.q_rot + chunk_off;
    }
    p.k = ws + L.k_rot;
    p.v = ws + L.v;
    p.out = ws + L.out + chunk_off;
    p.q_len = rows;
    p.q_offset = a->q_offset + r0;
    p.rotated = 1;
    p.workspace = nullptr;
    p.workspace_bytes = 0;
    st = atf_prefill_ex(&p, cstr);
    if (st) break;
    e = cudaEventRecord(cs->out_ready, cstr);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs->down, cs->out_ready, 0);
    if (e == cudaSuccess)
      e = copy_rows(static_cast<char*>(a->out) + r0 * q_row, host_pitch, ws + L.out + chunk_off, width, width, B,
                    cs->down);
  }
  // Join the upload, second compute and download streams back to the caller's
  // stream, on success and on error.
  cudaError_t ej = cudaEventRecord(cs->in_ready, cs->up);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, cs->in_ready, 0);
  if (ej == cudaSuccess) ej = cudaEventRecord(cs->aux_done, cs->aux);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, cs->aux_done, 0);
  if (ej == cudaSuccess) ej = cudaEventRecord(cs->done, cs->down);
  if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, cs->done, 0);
  if (st) return st;
  if (e != cudaSuccess) return atf::report_error(ATF_ERR_CUDA, "prefill_host: %s", cudaGetErrorString(e));
  if (ej != cudaSuccess) return atf::report_error(ATF_ERR_CUDA, "prefill_host: join: %s", cudaGetErrorString(ej));
  return ATF_OK;
}
