// fasa.cu -- FASA-style decode on the rotated, pair-chunk-major key cache:
// Token Importance Predictor (TIP) scores from dominant frequency pairs, top-k
// selection, then Focused Attention Computation (FAC) over the selected tokens.
// Page "FASA", section "Das FASA-Framework arbeitet in zwei Hauptphasen"; the
// dominant frequency chunks of section "Funktionale Sparsitaet auf
// Frequenz-Chunk-Ebene" are given here as a set of RoPE pairs.
//
// Kernels, per call:
//   1. fasa_score_kernel: one CTA per (4096 keys, kv head, sequence).  Streams
//      only the 8-pair chunks of the cache that hold a dominant pair (32 bytes
//      per key and chunk, coalesced) and scores every key for all query heads of
//      the kv head.  From +0, every dim of the dominant pairs (ascending) adds
//      its product with one fp32 fused multiply-add, s <- fl(q_j k_j + s), two
//      keys at a time as packed f32x2 pairs, so the top-k decision can be
//      reproduced bit for bit.  Each score's order-preserving bit pattern goes
//      to memory as its top 16 bits (the fp32 score itself only when the caller
//      asks for it), with a 4096-bin histogram per query head of the top 12
//      bits (sign, exponent and three mantissa bits: a bin spans an eighth of an
//      octave).
//   2. fasa_threshold_kernel (one CTA per row) finds from the histogram the bin
//      holding the budget-th largest score; fasa_scan_kernel, 32 CTAs per
//      (query head, sequence), then sweeps 1/32 of the 16-bit prefixes each:
//      keys above that bin are in (appended to an unsorted list), keys in it
//      are candidates.
//   3. fasa_finish_kernel: one CTA per (query head, sequence).  Recomputes the
//      candidates' exact scores from the cache in the same order of fused
//      multiply-adds (the same bits); radix passes over the candidates on the
//      rest of the 64-bit selection key (score bits, then ~index, so equal
//      scores go to the lower index) pick the remaining keys; the chosen
//      indices are sorted ascending.
//   4. fasa_attend_kernel: (split of 128 selected keys, query head, sequence);
//      four warps gather the keys' rows from the chunk-major cache and their
//      values and run an online softmax; partials as in the split decode.
//   5. fasa_combine_kernel: merges the splits (log-sum-exp) into bf16 output.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>

#include "../../include/atf.h"
#include "atf_internal.cuh"
#include "ptx.cuh"

namespace atf {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreKeysPerThread = 16;
constexpr int kScoreKeys = kScoreThreads * kScoreKeysPerThread;  // keys per score CTA
constexpr int kHistBits = 12;
constexpr int kHistBins = 1 << kHistBits;
constexpr int kScanCtas = 32;  // CTAs sweeping one (query head, sequence) row
constexpr int kScanThreads = 256;
constexpr int kScanUnroll4 = 4;  // 16-byte loads (8 prefixes each) in flight per thread
constexpr int kScanStage = 1024;  // per scan CTA, list entries staged in shared memory before the global append
constexpr int kFinishThreads = 1024;
constexpr int kAttendKeys = 128;  // selected keys per attention split
constexpr int kAttendWarps = 4;
constexpr int kBins = 256;  // radix digit of the refinement passes
constexpr int kMaxG = 8;
constexpr int kMaxFasaBudget = 4096;  // selected keys per query head (sorted in shared memory)

struct FasaParams {
  const __nv_bfloat16* q;  // rotated queries [B][Hq][d]
  const __nv_bfloat16* kc;  // rotated keys, chunk-major [B][Hkv][d/16][n_cache][16]
  const __nv_bfloat16* v;   // values [B][n_cache][Hkv][d]
  __nv_bfloat16* out;       // [B][Hq][d]
  float* scores;            // [B][Hq][n_cache] fp32 scores, or NULL (only written when asked for)
  uint16_t* pfx;            // [B][Hq][n_pad]: the top 16 bits of each score's order-preserving key
  uint32_t* cand;           // [B][Hq][n_cache] candidates of the threshold bin
  float* cand_score;        // [B][Hq][n_cache] their exact scores
  unsigned int* hist;       // [B][Hq][kHistBins]
  unsigned int* counts;     // [B][Hq][2]: keys above the threshold bin, candidates
  int* thr;                 // [B][Hq]: the threshold bin
  int* above;               // [B][Hq][budget]: keys above the threshold bin, unsorted
  int* sel;                 // [B][Hq][budget], ascending, -1 padded
  float* partials;          // [B][Hq][n_split][d + 2]
  int batch, hq, hkv, d, budget, n_split;
  long long n_cache, n_pad;  // n_pad: prefix row length, n_cache rounded up to 8
  unsigned long long mask;  // dominant pairs
  long long kv_len[kMaxDecodeBatch];
};

// Order-preserving map of a float's bits to an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int D, int G>
__global__ void __launch_bounds__(kScoreThreads, 3) fasa_score_kernel(FasaParams p) {  // 3 CTAs per SM
  constexpr int NC = D / 16;
  const int kvh = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const long long L = p.kv_len[b];
  const long long n0 = static_cast<long long>(blockIdx.x) * kScoreKeys;
  if (n0 >= L) return;
  __shared__ ulonglong2 sq[G][D / 2];  // ((q_2i, q_2i), (q_2i+1, q_2i+1)) per head and pair, as f32x2
  // per head, kHistBins 16-bit counts packed two to a word (a CTA scores at most
  // kScoreKeys < 2^16 keys)
  extern __shared__ unsigned int shist[];
  for (int i = tid; i < G * (D / 2); i += kScoreThreads) {
    const int g = i / (D / 2), pr = i % (D / 2);
    const __nv_bfloat16* qh = p.q + (static_cast<long long>(b) * p.hq + kvh * G + g) * D;
    const float qa = __bfloat162float(qh[2 * pr]), qb = __bfloat162float(qh[2 * pr + 1]);
    sq[g][pr] = make_ulonglong2(pack2(qa, qa), pack2(qb, qb));
  }
  for (int i = tid; i < G * (kHistBins / 2); i += kScoreThreads) shist[i] = 0u;
  __syncthreads();

  const uint4* kbase = reinterpret_cast<const uint4*>(p.kc) +
                       (static_cast<long long>(b) * p.hkv + kvh) * NC * p.n_cache * 2;
  // four keys per step, as two packed fp32 pairs (an f32x2 fused multiply-add
  // rounds each half exactly as the scalar one does); all four keys' loads are
  // issued before the arithmetic, and each query load serves the four keys
  auto word = [](const uint4& lo, const uint4& hi, int j) -> uint32_t {
    return j == 0 ? lo.x : j == 1 ? lo.y : j == 2 ? lo.z : j == 3 ? lo.w : j == 4 ? hi.x : j == 5 ? hi.y : j == 6 ? hi.z : hi.w;
  };
#pragma unroll 1
  for (int r = 0; r < kScoreKeysPerThread; r += 4) {
    long long nk[4];
    bool vk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      nk[k] = n0 + (r + k) * kScoreThreads + tid;
      vk[k] = nk[k] < L;
    }
    if (!vk[0]) break;
    uint64_t s2[2][G];
#pragma unroll
    for (int g = 0; g < G; ++g) s2[0][g] = s2[1][g] = 0ull;  // (+0, +0)
#pragma unroll 1
    for (int c = 0; c < NC; ++c) {
      const uint32_t bits = static_cast<uint32_t>((p.mask >> (8 * c)) & 0xFFu);
      if (!bits) continue;
      uint4 lo[4], hi[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        lo[k] = hi[k] = make_uint4(0, 0, 0, 0);
        if (vk[k]) {
          const uint4* row = kbase + (static_cast<long long>(c) * p.n_cache + nk[k]) * 2;
          lo[k] = __ldg(row);
          hi[k] = __ldg(row + 1);
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (!((bits >> j) & 1u)) continue;
        uint64_t k0[2], k1[2];  // dim 2i and dim 2i+1 of keys (0, 1) and (2, 3)
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const uint32_t w0 = word(lo[2 * h2], hi[2 * h2], j), w1 = word(lo[2 * h2 + 1], hi[2 * h2 + 1], j);
          k0[h2] = pack2(__uint_as_float(w0 << 16), __uint_as_float(w1 << 16));
          k1[h2] = pack2(__uint_as_float(w0 & 0xFFFF0000u), __uint_as_float(w1 & 0xFFFF0000u));
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const ulonglong2 qp = sq[g][8 * c + j];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            s2[h2][g] = ffma2(qp.x, k0[h2], s2[h2][g]);  // dim 2i
            s2[h2][g] = ffma2(qp.y, k1[h2], s2[h2][g]);  // dim 2i+1
          }
        }
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      {
        const long long hrow = static_cast<long long>(b) * p.hq + kvh * G + g;
        uint16_t* prow = p.pfx + hrow * p.n_pad;
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          float sc[2];
          unpack2(fadd2(s2[h2][g], 0ull), sc[0], sc[1]);  // -0 scores as +0
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            if (vk[2 * h2 + e]) {
              const uint32_t key = order_key(sc[e]);
              prow[nk[2 * h2 + e]] = static_cast<uint16_t>(key >> 16);
              if (p.scores) p.scores[hrow * p.n_cache + nk[2 * h2 + e]] = sc[e];
              const uint32_t bin = key >> (32 - kHistBits);
              atomicAdd(&shist[g * (kHistBins / 2) + (bin >> 1)], 1u << (16 * (bin & 1u)));
            }
          }
        }
      }
    }
  }
  __syncthreads();
  for (int i = tid; i < G * (kHistBins / 2); i += kScoreThreads) {
    const unsigned int w = shist[i];
    if (!w) continue;
    const int g = i / (kHistBins / 2), bin = 2 * (i % (kHistBins / 2));
    unsigned int* hg = p.hist + (static_cast<long long>(b) * p.hq + kvh * G + g) * kHistBins;
    if (w & 0xFFFFu) atomicAdd(&hg[bin], w & 0xFFFFu);
    if (w >> 16) atomicAdd(&hg[bin + 1], w >> 16);
  }
}

// Block-wide exclusive prefix count of `flag` over the kFinishThreads threads;
// returns this thread's rank and writes the block total to *total.
__device__ __forceinline__ int block_rank(bool flag, int* warp_counts, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t bal = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) warp_counts[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    const int c = lane < kFinishThreads / 32 ? warp_counts[lane] : 0;
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += t;
    }
    if (lane < kFinishThreads / 32) warp_counts[lane] = incl - c;
    if (lane == 31) *total = incl;
  }
  __syncthreads();
  const int r = warp_counts[warp] + __popc(bal & ((1u << lane) - 1u));
  __syncthreads();  // warp_counts is reused by the next call
  return r;
}

// Digit (bits shift .. shift+width-1) of the 64-bit selection key of key n.
__device__ __forceinline__ uint32_t sel_digit(float score, uint32_t n, int shift, int width) {
  const uint64_t key = (static_cast<uint64_t>(order_key(score)) << 32) | static_cast<uint64_t>(~n);
  return static_cast<uint32_t>(key >> shift) & ((1u << width) - 1u);
}

// Appends the lanes' values where `flag` holds to a shared-memory list of
// kScanStage entries, slots taken from *s_count with one atomic per warp; a lane
// whose slot lies past the list appends to the global list itself (slots at or past
// `capacity` are counted but not written).
__device__ __forceinline__ void warp_append_staged(bool flag, uint32_t value, unsigned int* s_count, uint32_t* s_list,
                                                   unsigned int* counter, uint32_t* list, unsigned int capacity) {
  const int lane = threadIdx.x & 31;
  const uint32_t bal = __ballot_sync(0xffffffffu, flag);
  if (!bal) return;
  unsigned int base = 0;
  if (lane == __ffs(bal) - 1) base = atomicAdd(s_count, static_cast<unsigned int>(__popc(bal)));
  base = __shfl_sync(0xffffffffu, base, __ffs(bal) - 1);
  const unsigned int slot = base + __popc(bal & ((1u << lane) - 1u));
  if (!flag) return;
  if (slot < static_cast<unsigned int>(kScanStage)) {
    s_list[slot] = value;
  } else {
    const unsigned int g = atomicAdd(counter, 1u);
    if (g < capacity) list[g] = value;
  }
}

// The exact score of key n for one query head (q: that head's rotated query as
// floats), in the scoring kernel's order: dominant dims ascending, one fp32 fused
// multiply-add each, -0 as +0.
__device__ __forceinline__ float exact_score(const FasaParams& p, const float* q, const uint4* kbase, long long n) {
  float s = 0.f;
  const int nc = p.d / 16;
  for (int c = 0; c < nc; ++c) {
    const uint32_t bits = static_cast<uint32_t>((p.mask >> (8 * c)) & 0xFFu);
    if (!bits) continue;
    const uint4* row = kbase + (static_cast<long long>(c) * p.n_cache + n) * 2;
    const uint4 lo = __ldg(row), hi = __ldg(row + 1);
    const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (!((bits >> j) & 1u)) continue;
      const int dim = 16 * c + 2 * j;
      s = __fmaf_rn(q[dim], __uint_as_float(w[j] << 16), s);
      s = __fmaf_rn(q[dim + 1], __uint_as_float(w[j] & 0xFFFF0000u), s);
    }
  }
  return __fadd_rn(s, 0.f);
}

// The threshold bin of every (query head, sequence) row: the histogram bin holding
// the need-th largest score (kHistBins when every key is selected: nothing to
// sweep).  Thread t holds the 16 bins [4096 - 16 (t + 1), 4096 - 16 t), scanned
// from the top.
__global__ void __launch_bounds__(kScanThreads) fasa_threshold_kernel(FasaParams p) {
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const long long row = static_cast<long long>(b) * p.hq + h;
  const int L = static_cast<int>(p.kv_len[b]);
  const int need = L < p.budget ? L : p.budget;
  __shared__ int s_scan[kScanThreads];
  if (need == L) {
    if (tid == 0) p.thr[row] = kHistBins;
    return;
  }
  constexpr int kPer = kHistBins / kScanThreads;
  const unsigned int* hg = p.hist + row * kHistBins;
  int mine = 0;
#pragma unroll
  for (int k = 0; k < kPer; ++k) mine += static_cast<int>(hg[kHistBins - kPer * tid - 1 - k]);
  s_scan[tid] = mine;
  if (tid == 0) p.thr[row] = kHistBins;  // no bin (emits nothing) unless the search below finds one
  __syncthreads();
  for (int off = 1; off < kScanThreads; off <<= 1) {  // inclusive scan (Hillis-Steele)
    const int t = tid >= off ? s_scan[tid - off] : 0;
    __syncthreads();
    s_scan[tid] += t;
    __syncthreads();
  }
  const int incl = s_scan[tid], excl = incl - mine;
  if (excl < need && need <= incl) {
    int acc = excl;
    for (int k = 0; k < kPer; ++k) {
      const int bin = kHistBins - kPer * tid - 1 - k;
      acc += static_cast<int>(hg[bin]);
      if (acc >= need) {
        p.thr[row] = bin;
        break;
      }
    }
  }
}

__global__ void __launch_bounds__(kScanThreads) fasa_scan_kernel(FasaParams p) {
  const int part = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const long long row = static_cast<long long>(b) * p.hq + h;
  const int L = static_cast<int>(p.kv_len[b]);
  const uint32_t thr = static_cast<uint32_t>(p.thr[row]);
  if (thr >= static_cast<uint32_t>(kHistBins)) return;  // every key is selected (or nothing to find)
  // this CTA's share of the keys: a multiple of 8 long, so that 16-byte loads of
  // 8 prefixes stay aligned (prefix rows are n_pad long, a multiple of 8)
  const int per = ((L + kScanCtas - 1) / kScanCtas + 7) & ~7;
  const int n_lo = part * per, n_hi = min(L, n_lo + per);
  const uint16_t* prow = p.pfx + row * p.n_pad;
  unsigned int* cnt = p.counts + row * 2;
  uint32_t* above = reinterpret_cast<uint32_t*>(p.above + row * p.budget);
  uint32_t* cand = p.cand + row * p.n_cache;
  // the CTA's entries of both lists gather in shared memory; one global atomic per
  // list reserves their slots at the end
  __shared__ uint32_t s_above[kScanStage], s_cand[kScanStage];
  __shared__ unsigned int s_na, s_nc, s_ga, s_gc;
  if (tid == 0) s_na = s_nc = 0u;
  __syncthreads();
  for (int base = n_lo; base < n_hi; base += 8 * kScanThreads * kScanUnroll4) {
    uint4 v[kScanUnroll4];
#pragma unroll
    for (int u = 0; u < kScanUnroll4; ++u) {
      const int idx = base + 8 * (u * kScanThreads + tid);
      v[u] = idx < n_hi ? __ldg(reinterpret_cast<const uint4*>(prow + idx)) : make_uint4(0, 0, 0, 0);
    }
    // almost every key lies below the threshold bin: each lane marks its keys
    // above it and in it (bit 8u + e for key 8 * (u * kScanThreads + tid) + e),
    // and the warp appends only at the positions some lane marked
    uint32_t am = 0u, cm = 0u;
#pragma unroll
    for (int u = 0; u < kScanUnroll4; ++u) {
      const int idx = base + 8 * (u * kScanThreads + tid);
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t bin = (e & 1 ? w[e >> 1] >> 16 : w[e >> 1] & 0xFFFFu) >> 4;
        const bool ok = idx + e < n_hi;
        am |= static_cast<uint32_t>(ok && bin > thr) << (8 * u + e);
        cm |= static_cast<uint32_t>(ok && bin == thr) << (8 * u + e);
      }
    }
    for (uint32_t rest = __reduce_or_sync(0xffffffffu, am | cm); rest; rest &= rest - 1u) {
      const int j = __ffs(rest) - 1;
      const uint32_t n = static_cast<uint32_t>(base + 8 * ((j >> 3) * kScanThreads + tid) + (j & 7));
      warp_append_staged((am >> j) & 1u, n, &s_na, s_above, &cnt[0], above, static_cast<unsigned int>(p.budget));
      warp_append_staged((cm >> j) & 1u, n, &s_nc, s_cand, &cnt[1], cand, static_cast<unsigned int>(L));
    }
  }
  __syncthreads();
  const unsigned int na = min(s_na, static_cast<unsigned int>(kScanStage));
  const unsigned int nc = min(s_nc, static_cast<unsigned int>(kScanStage));
  if (tid == 0) {
    s_ga = na ? atomicAdd(&cnt[0], na) : 0u;
    s_gc = nc ? atomicAdd(&cnt[1], nc) : 0u;
  }
  __syncthreads();
  for (unsigned int i = tid; i < na; i += kScanThreads)
    if (s_ga + i < static_cast<unsigned int>(p.budget)) above[s_ga + i] = s_above[i];
  for (unsigned int i = tid; i < nc; i += kScanThreads)
    if (s_gc + i < static_cast<unsigned int>(L)) cand[s_gc + i] = s_cand[i];
}

__global__ void __launch_bounds__(kFinishThreads) fasa_finish_kernel(FasaParams p) {
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const long long row = static_cast<long long>(b) * p.hq + h;
  uint32_t* cand = p.cand + row * p.n_cache;
  float* cand_score = p.cand_score + row * p.n_cache;
  int* out = p.sel + row * p.budget;
  const int L = static_cast<int>(p.kv_len[b]);
  const int need = L < p.budget ? L : p.budget;

  __shared__ int s_sel[kMaxFasaBudget];
  __shared__ unsigned int s_hist[kBins];
  __shared__ int s_warp[kFinishThreads / 32];
  __shared__ int s_nsel, s_total, s_thr, s_above;
  __shared__ float sq[128];

  if (need == L) {  // every key is selected, already in order
    for (int i = tid; i < p.budget; i += kFinishThreads) out[i] = i < L ? i : -1;
    return;
  }
  // (the counts can only exceed these bounds if the scores and the histogram
  // disagree; the lists were not written past them)
  const int n_above = static_cast<int>(min(p.counts[row * 2], static_cast<unsigned int>(need)));
  int m = static_cast<int>(min(p.counts[row * 2 + 1], static_cast<unsigned int>(L)));
  for (int i = tid; i < n_above; i += kFinishThreads) s_sel[i] = p.above[row * p.budget + i];
  if (tid == 0) s_nsel = n_above;
  __syncthreads();
  int left = need - n_above;  // still to choose among the candidates
  if (left > 0 && left < m) {
    // the candidates' exact scores, recomputed from the cache in the scoring
    // kernel's order (the same bits), all candidates in parallel
    for (int i = tid; i < p.d; i += kFinishThreads) sq[i] = __bfloat162float(p.q[row * p.d + i]);
    __syncthreads();
    const uint4* kbase = reinterpret_cast<const uint4*>(p.kc) +
                         (static_cast<long long>(b) * p.hkv + h / (p.hq / p.hkv)) * (p.d / 16) * p.n_cache * 2;
    for (int i = tid; i < m; i += kFinishThreads) cand_score[i] = exact_score(p, sq, kbase, cand[i]);
    __syncthreads();
  }
  // radix passes over the rest of the selection key: score bits 51..32 below the
  // histogram's 12, then the 32 bits of ~index
  for (int pass = 0; pass < 7 && left > 0 && left < m; ++pass) {
    const int shift = pass < 6 ? 44 - 8 * pass : 0, width = pass < 6 ? 8 : 4;
    for (int i = tid; i < kBins; i += kFinishThreads) s_hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < m; i += kFinishThreads) atomicAdd(&s_hist[sel_digit(cand_score[i], cand[i], shift, width)], 1u);
    __syncthreads();
    if (tid < 32) {
      // the threshold digit: the largest t with #(digits >= t) >= left (t = 0 at the
      // latest, since m > left), and the count above it; one warp, each lane a run
      // of consecutive digits, suffix sums across the lanes
      const int nb = 1 << width, per = (nb + 31) / 32, lo = tid * per;
      int lsum = 0;
      for (int u = lo; u < lo + per && u < nb; ++u) lsum += static_cast<int>(s_hist[u]);
      int suf = lsum;  // digits >= lo
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, suf, off);
        if (tid + off < 32) suf += y;
      }
      int t = -1, above = 0;
      int run = suf - lsum;  // digits past this lane's run
      for (int u = min(lo + per, nb) - 1; u >= lo; --u) {
        const int c = static_cast<int>(s_hist[u]);
        if (run + c >= left) {
          t = u;
          above = run;
          break;
        }
        run += c;
      }
      const int tmax = __reduce_max_sync(0xffffffffu, t);
      if (t == tmax && t >= 0) {  // one lane holds it
        s_thr = t;
        s_above = above;
      }
    }
    __syncthreads();
    const uint32_t thr = static_cast<uint32_t>(s_thr);
    // emit the digits above the threshold; compact the equal ones to the front
    int kept = 0;
    for (int base = 0; base < m; base += kFinishThreads) {
      const int i = base + tid;
      uint32_t n = 0, dg = 0;
      float sv = 0.f;
      if (i < m) {
        n = cand[i];
        sv = cand_score[i];
        dg = sel_digit(sv, n, shift, width);
        if (dg > thr) {
          const int slot = atomicAdd(&s_nsel, 1);
          if (slot < need) s_sel[slot] = static_cast<int>(n);
        }
      }
      const bool keep = i < m && dg == thr;
      const int rk = block_rank(keep, s_warp, &s_total);  // all reads of this block of cand are done
      if (keep) {
        cand[kept + rk] = n;
        cand_score[kept + rk] = sv;
      }
      kept += s_total;
      __syncthreads();
    }
    left -= s_above;
    m = kept;
  }
  __syncthreads();
  // the remaining candidates are all in (left == m), or none are needed
  for (int i = tid; i < m && left > 0; i += kFinishThreads) {
    const int slot = atomicAdd(&s_nsel, 1);
    if (slot < need) s_sel[slot] = static_cast<int>(cand[i]);
  }
  __syncthreads();
  for (int i = s_nsel + tid; i < need; i += kFinishThreads) s_sel[i] = -1;  // never with consistent inputs
  // bitonic sort of the need chosen indices (padded to a power of two)
  int P = 1;
  while (P < need) P <<= 1;
  for (int i = need + tid; i < P; i += kFinishThreads) s_sel[i] = 0x7fffffff;
  __syncthreads();
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += kFinishThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const int a = s_sel[i], c = s_sel[ixj];
          const bool up = (i & k) == 0;
          if ((a > c) == up) {
            s_sel[i] = c;
            s_sel[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < p.budget; i += kFinishThreads) out[i] = i < need ? s_sel[i] : -1;
}

template <int D>
__global__ void __launch_bounds__(kAttendWarps * 32) fasa_attend_kernel(FasaParams p) {
  constexpr int NC = D / 16;
  constexpr int DPL = D / 32;  // dims per lane: 4 (d = 128) or 2 (d = 64)
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.hq / p.hkv, kvh = h / G;
  const long long row = static_cast<long long>(b) * p.hq + h;
  const int L = static_cast<int>(p.kv_len[b]);
  const int need = L < p.budget ? L : p.budget;
  const int* sel = p.sel + row * p.budget;
  const int j0 = split * kAttendKeys, j1 = min(need, j0 + kAttendKeys);

  constexpr float kLog2e = 1.4426950408889634f;
  const float scale = kLog2e * rsqrtf(static_cast<float>(D));
  float q[DPL];
  {
    const __nv_bfloat16* qh = p.q + row * D + DPL * lane;
#pragma unroll
    for (int e = 0; e < DPL; ++e) q[e] = __bfloat162float(qh[e]) * scale;
  }
  __shared__ int s_idx[kAttendKeys];  // the split's key indices, loaded once
  for (int i = threadIdx.x; i < j1 - j0; i += kAttendWarps * 32) s_idx[i] = sel[j0 + i];
  __syncthreads();
  const int c = (DPL * lane) / 16, off = (DPL * lane) % 16;  // this lane's dims in the chunk-major row
  const __nv_bfloat16* kb = p.kc + ((static_cast<long long>(b) * p.hkv + kvh) * NC + c) * p.n_cache * 16 + off;
  const __nv_bfloat16* vb = p.v + static_cast<long long>(b) * p.n_cache * p.hkv * D + kvh * D + DPL * lane;

  float mrun = -INFINITY, lsum = 0.f, o[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) o[e] = 0.f;
  constexpr int U = 8;  // keys in flight per warp
  for (int j = j0 + warp * U; j < j1; j += kAttendWarps * U) {
    float kv[U][DPL], vv[U][DPL];
    bool kok[U];  // the slot holds a key index in range (always, with consistent inputs)
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int jj = j + u;
      kok[u] = false;
      if (jj < j1) {
        long long n = s_idx[jj - j0];
        kok[u] = n >= 0 && n < L;
        if (!kok[u]) n = 0;
        if constexpr (DPL == 4) {
          const uint2 kw = *reinterpret_cast<const uint2*>(kb + n * 16);
          const uint2 vw = *reinterpret_cast<const uint2*>(vb + n * p.hkv * D);
          kv[u][0] = bf16lo_to_f32(kw.x);
          kv[u][1] = bf16hi_to_f32(kw.x);
          kv[u][2] = bf16lo_to_f32(kw.y);
          kv[u][3] = bf16hi_to_f32(kw.y);
          vv[u][0] = bf16lo_to_f32(vw.x);
          vv[u][1] = bf16hi_to_f32(vw.x);
          vv[u][2] = bf16lo_to_f32(vw.y);
          vv[u][3] = bf16hi_to_f32(vw.y);
        } else {
          const uint32_t kw = *reinterpret_cast<const uint32_t*>(kb + n * 16);
          const uint32_t vw = *reinterpret_cast<const uint32_t*>(vb + n * p.hkv * D);
          kv[u][0] = bf16lo_to_f32(kw);
          kv[u][1] = bf16hi_to_f32(kw);
          vv[u][0] = bf16lo_to_f32(vw);
          vv[u][1] = bf16hi_to_f32(vw);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (j + u >= j1) break;
      if (!kok[u]) continue;  // warp-uniform
      float sdot = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) sdot = fmaf(q[e], kv[u][e], sdot);
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) sdot += __shfl_xor_sync(0xffffffffu, sdot, o2);
      const float mnew = fmaxf(mrun, sdot);
      const float corr = ex2_approx(mrun - mnew);  // 0 on the first key (mrun = -inf)
      const float pr = ex2_approx(sdot - mnew);
      lsum = lsum * corr + pr;
#pragma unroll
      for (int e = 0; e < DPL; ++e) o[e] = fmaf(o[e], corr, pr * vv[u][e]);
      mrun = mnew;
    }
  }
  // merge the warps
  __shared__ float sm[kAttendWarps], sl[kAttendWarps], so[kAttendWarps][D];
  if (lane == 0) {
    sm[warp] = mrun;
    sl[warp] = lsum;
  }
#pragma unroll
  for (int e = 0; e < DPL; ++e) so[warp][DPL * lane + e] = o[e];
  __syncthreads();
  float* part = p.partials + (row * p.n_split + split) * (D + 2);
  for (int e = threadIdx.x; e < D; e += kAttendWarps * 32) {
    float M = -INFINITY;
    for (int w = 0; w < kAttendWarps; ++w) M = fmaxf(M, sm[w]);
    float a = 0.f, l = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < kAttendWarps; ++w) {
        if (sm[w] == -INFINITY) continue;
        const float f = ex2_approx(sm[w] - M);
        a += so[w][e] * f;
        l += sl[w] * f;
      }
    }
    part[e] = a;
    if (e == 0) {
      part[D] = M;
      part[D + 1] = l;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(D) fasa_combine_kernel(FasaParams p) {
  const int h = blockIdx.x, b = blockIdx.y, e = threadIdx.x;
  const long long row = static_cast<long long>(b) * p.hq + h;
  const float* part = p.partials + row * p.n_split * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < p.n_split; ++s) M = fmaxf(M, part[s * (D + 2) + D]);
  float a = 0.f, l = 0.f;
  for (int s = 0; s < p.n_split; ++s) {
    const float ms = part[s * (D + 2) + D];
    if (ms == -INFINITY) continue;
    const float f = ex2_approx(ms - M);
    a += part[s * (D + 2) + e] * f;
    l += part[s * (D + 2) + D + 1] * f;
  }
  p.out[row * D + e] = __float2bfloat16(l > 0.f ? a / l : 0.f);
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

struct FasaLayout {
  size_t pfx, cand, cand_score, hist, counts, thr, above, sel, partials, total;
};

FasaLayout fasa_layout(int batch, int heads, long long n_cache, int budget, int d, bool own_sel) {
  const size_t rows = static_cast<size_t>(batch) * heads;
  const int n_split = (budget + kAttendKeys - 1) / kAttendKeys;
  FasaLayout L{};
  size_t off = 0;
  L.pfx = off;
  off += align256(rows * ((n_cache + 7) / 8 * 8) * sizeof(uint16_t));
  L.cand = off;
  off += align256(rows * n_cache * sizeof(uint32_t));
  L.cand_score = off;
  off += align256(rows * n_cache * sizeof(float));
  L.hist = off;  // histograms and counters are cleared together
  off += rows * kHistBins * sizeof(unsigned int);
  L.counts = off;
  off += align256(rows * 2 * sizeof(unsigned int));
  L.thr = off;
  off += align256(rows * sizeof(int));
  L.above = off;
  off += align256(rows * budget * sizeof(int));
  L.sel = off;
  off += own_sel ? 0 : align256(rows * budget * sizeof(int));
  L.partials = off;
  off += align256(rows * n_split * (d + 2) * sizeof(float));
  L.total = off;
  return L;
}

template <int D>
cudaError_t launch_fasa(const FasaParams& p, long long max_len, cudaStream_t s) {
  const int G = p.hq / p.hkv;
  const size_t hist_smem = static_cast<size_t>(G) * (kHistBins / 2) * sizeof(unsigned int);
  // one bit per device: the attribute is set once (racing first calls both set it, harmlessly)
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(configured.load(std::memory_order_acquire) & (1ull << dev))) {
    const int bytes = kMaxG * (kHistBins / 2) * static_cast<int>(sizeof(unsigned int));
    const void* fns[8] = {reinterpret_cast<const void*>(fasa_score_kernel<D, 1>),
                          reinterpret_cast<const void*>(fasa_score_kernel<D, 2>),
                          reinterpret_cast<const void*>(fasa_score_kernel<D, 3>),
                          reinterpret_cast<const void*>(fasa_score_kernel<D, 4>),
                          reinterpret_cast<const void*>(fasa_score_kernel<D, 5>),
                          reinterpret_cast<const void*>(fasa_score_kernel<D, 6>),
                          reinterpret_cast<const void*>(fasa_score_kernel<D, 7>),
                          reinterpret_cast<const void*>(fasa_score_kernel<D, 8>)};
    for (const void* f : fns) {
      e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e != cudaSuccess) return e;
    }
    if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_acq_rel);
  }
  const unsigned nblk = static_cast<unsigned>((max_len + kScoreKeys - 1) / kScoreKeys);
  const dim3 grid(nblk, p.hkv, p.batch);
  switch (G) {
    case 1: fasa_score_kernel<D, 1><<<grid, kScoreThreads, hist_smem, s>>>(p); break;
    case 2: fasa_score_kernel<D, 2><<<grid, kScoreThreads, hist_smem, s>>>(p); break;
    case 3: fasa_score_kernel<D, 3><<<grid, kScoreThreads, hist_smem, s>>>(p); break;
    case 4: fasa_score_kernel<D, 4><<<grid, kScoreThreads, hist_smem, s>>>(p); break;
    case 5: fasa_score_kernel<D, 5><<<grid, kScoreThreads, hist_smem, s>>>(p); break;
    case 6: fasa_score_kernel<D, 6><<<grid, kScoreThreads, hist_smem, s>>>(p); break;
    case 7: fasa_score_kernel<D, 7><<<grid, kScoreThreads, hist_smem, s>>>(p); break;
    default: fasa_score_kernel<D, 8><<<grid, kScoreThreads, hist_smem, s>>>(p); break;
  }
  fasa_threshold_kernel<<<dim3(p.hq, p.batch), kScanThreads, 0, s>>>(p);
  fasa_scan_kernel<<<dim3(kScanCtas, p.hq, p.batch), kScanThreads, 0, s>>>(p);
  fasa_finish_kernel<<<dim3(p.hq, p.batch), kFinishThreads, 0, s>>>(p);
  fasa_attend_kernel<D><<<dim3(p.n_split, p.hq, p.batch), kAttendWarps * 32, 0, s>>>(p);
  fasa_combine_kernel<D><<<dim3(p.hq, p.batch), D, 0, s>>>(p);
  return cudaGetLastError();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace atf

using namespace atf;

extern "C" size_t atf_fasa_workspace_bytes(int batch, int heads, long long n_cache, int budget, int d) {
  if (batch <= 0 || heads <= 0 || n_cache <= 0 || budget <= 0 || d <= 0) return 0;
  return fasa_layout(batch, heads, n_cache, budget, d, false).total;
}

extern "C" atf_status atf_fasa_decode(const void* q_rot, const void* k_chunked, const void* v, void* out, int batch,
                                      const long long* kv_len, long long n_cache, int heads, int kv_heads, int d,
                                      unsigned long long pair_mask, int budget, int* selected, float* scores,
                                      void* workspace, size_t workspace_bytes, void* stream) {
  if (d != 64 && d != 128) return report_error(ATF_ERR_UNSUPPORTED, "fasa: head dim d=%d not supported", d);
  if (batch < 0 || heads < 1 || kv_heads < 1 || n_cache < 1 || heads % kv_heads)
    return report_error(ATF_ERR_INVALID_ARG, "fasa: bad sizes");
  if (heads / kv_heads > kMaxG) return report_error(ATF_ERR_UNSUPPORTED, "fasa: more than 8 query heads per kv head");
  if (batch > kMaxDecodeBatch) return report_error(ATF_ERR_UNSUPPORTED, "fasa: batch above %d", kMaxDecodeBatch);
  if (budget < 1 || budget > kMaxFasaBudget)
    return report_error(ATF_ERR_UNSUPPORTED, "fasa: budget must be in [1, %d]", kMaxFasaBudget);
  if (n_cache > 0x7fffffffLL) return report_error(ATF_ERR_UNSUPPORTED, "fasa: cache longer than 2^31-1");
  const unsigned long long valid = d == 128 ? ~0ull : ((1ull << (d / 2)) - 1);
  if (!pair_mask || (pair_mask & ~valid))
    return report_error(ATF_ERR_INVALID_ARG, "fasa: pair mask must be non-empty and within the d/2 pairs");
  if (batch == 0) return ATF_OK;
  if (!kv_len) return report_error(ATF_ERR_INVALID_ARG, "fasa: kv_len is NULL");
  long long max_len = 0;
  for (int b = 0; b < batch; ++b) {
    if (kv_len[b] < 1 || kv_len[b] > n_cache)
      return report_error(ATF_ERR_INVALID_ARG, "fasa: kv_len[%d] = %lld outside [1, n_cache]", b, kv_len[b]);
    max_len = kv_len[b] > max_len ? kv_len[b] : max_len;
  }
  if (!q_rot || !k_chunked || !v || !out || !workspace) return report_error(ATF_ERR_INVALID_ARG, "fasa: null pointer");
  if (!aligned16(q_rot) || !aligned16(k_chunked) || !aligned16(v) || !aligned16(out) || !aligned16(workspace) ||
      (selected && !aligned16(selected)) || (scores && !aligned16(scores)))
    return report_error(ATF_ERR_INVALID_ARG, "fasa: pointers must be 16-byte aligned");
  const FasaLayout Lw = fasa_layout(batch, heads, n_cache, budget, d, selected != nullptr);
  if (workspace_bytes < Lw.total)
    return report_error(ATF_ERR_INVALID_ARG, "fasa: workspace of %zu bytes needed", Lw.total);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  FasaParams p{};
  p.q = static_cast<const __nv_bfloat16*>(q_rot);
  p.kc = static_cast<const __nv_bfloat16*>(k_chunked);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.scores = scores;
  p.pfx = reinterpret_cast<uint16_t*>(ws + Lw.pfx);
  p.cand_score = reinterpret_cast<float*>(ws + Lw.cand_score);
  p.cand = reinterpret_cast<uint32_t*>(ws + Lw.cand);
  p.hist = reinterpret_cast<unsigned int*>(ws + Lw.hist);
  p.counts = reinterpret_cast<unsigned int*>(ws + Lw.counts);
  p.thr = reinterpret_cast<int*>(ws + Lw.thr);
  p.above = reinterpret_cast<int*>(ws + Lw.above);
  p.sel = selected ? selected : reinterpret_cast<int*>(ws + Lw.sel);
  p.partials = reinterpret_cast<float*>(ws + Lw.partials);
  p.batch = batch;
  p.hq = heads;
  p.hkv = kv_heads;
  p.d = d;
  p.budget = budget;
  p.n_split = (budget + kAttendKeys - 1) / kAttendKeys;
  p.n_cache = n_cache;
  p.n_pad = (n_cache + 7) / 8 * 8;
  p.mask = pair_mask;
  for (int b = 0; b < batch; ++b) p.kv_len[b] = kv_len[b];
  cudaError_t e = cudaMemsetAsync(p.hist, 0, Lw.above - Lw.hist, s);  // histograms and counters
  if (e == cudaSuccess) e = d == 128 ? launch_fasa<128>(p, max_len, s) : launch_fasa<64>(p, max_len, s);
  if (e != cudaSuccess) return report_error(ATF_ERR_CUDA, "fasa: launch: %s", cudaGetErrorString(e));
  return ATF_OK;
}
