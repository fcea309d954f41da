// fasa.cu -- FASA-style decode on the rotated, pair-chunk-major key cache:
// Token Importance Predictor (TIP) scores from dominant frequency pairs, top-k
// selection, then Focused Attention Computation (FAC) over the selected tokens.
// Page "FASA", section "Das FASA-Framework arbeitet in zwei Hauptphasen"; the
// dominant frequency chunks of section "Funktionale Sparsitaet auf
// Frequenz-Chunk-Ebene" are given here as a set of RoPE pairs.
//
// Every TIP score is one fixed fp32 evaluation on the tensor cores: the 16 dims
// of each cache chunk that holds a dominant pair (the other pairs' query dims
// zeroed) are one mma.sync step of bf16 products accumulated into fp32, chunks
// in ascending order, in one fixed arrangement of dims and heads (score_tiles);
// -0 counts as +0.  The kept keys are the `budget` highest such scores, equal
// scores by lower index.  Kernels, per call:
//   1. fasa_sample_kernel: one CTA per (131072 keys, kv head, sequence) scores the
//      sampled keys -- the first 32 of every 1024 -- for all query heads of the
//      kv head into a 4096-bin histogram per query head (top 12 bits of the
//      score's order-preserving bit pattern: sign, exponent and three mantissa
//      bits).
//   2. fasa_threshold_kernel: per query head, the threshold T is the lower edge
//      of the bin that holds the sample's k-th largest score, k twice the
//      sample's share of the budget plus 8, so that about twice the budget of
//      all keys score at or above T.
//   3. fasa_score_kernel: one CTA per (8192 keys, kv head, sequence); each warp
//      owns a segment of 1024 consecutive keys, 128 at a time (8 tiles of 16
//      keys x all query heads of the kv head), the keys' chunk rows brought in
//      by a per-warp ring of bulk copies.  It reads only the 8-pair chunks that
//      hold a dominant pair and appends the keys scoring at or above T, with
//      their scores, to the segment's list of that head, each 128-key step's
//      candidates as one block after the earlier steps'.
//   4. fasa_select_kernel: one CTA per (query head, sequence) gathers the
//      segments' lists into shared memory; one 4096-bin histogram pass finds the
//      bin holding the budget-th largest score, whose keys are ranked exactly
//      (larger score, then lower index); every thread then writes its segment's
//      kept keys in index order, with their TIP scores.  A crowded boundary bin
//      or a list longer than shared memory takes radix passes instead; if fewer
//      than `budget` keys reached T (the sample was not representative), every
//      key's score is recomputed the same way and the selection runs over all.
//   5. fasa_attend_kernel: (split of 128 selected keys, query head, sequence);
//      each warp copies its 32 keys' K rows (chunk-major pieces) and V rows into
//      shared memory with asynchronous copies, all in flight at once, computes
//      their 32 dot products together and a softmax over them; partials as in
//      the split decode.  With the TIP scores, chunks whose pairs are all
//      dominant are not read (the TIP score is their part of q.k).
//   6. fasa_combine_kernel: merges the splits (log-sum-exp) into bf16 output.
// Kernels 1 and 2 run once over the batch; 3 to 6 run as one chain per sequence
// on library streams forked from and joined back to the caller's stream.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/atf.h"
#include "atf_internal.cuh"
#include "ptx.cuh"

namespace atf {
namespace {

constexpr int kSampleRun = 32;        // sampled keys: the first kSampleRun of every kSamplePeriod
constexpr int kSamplePeriod = 1024;
constexpr int kSampleCtaKeys = 131072;  // keys of a sequence per sample CTA (128 runs)
constexpr int kSampleThreads = 512;  // 16 warps, eight runs each
constexpr int kThresholdThreads = 256;
constexpr int kHistBits = 12;
constexpr int kHistBins = 1 << kHistBits;
constexpr int kScoreWarps = 8;
constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kSegShift = 10;
constexpr int kSegKeys = 1 << kSegShift;                  // keys per warp segment
constexpr int kScoreCtaKeys = kScoreWarps * kSegKeys;     // keys per score CTA
constexpr int kScoreStages = 3;  // bulk-copy stages per score warp
constexpr size_t kScoreSmem = static_cast<size_t>(kScoreWarps) * kScoreStages * 128 * 32;
constexpr int kSelectThreads = 1024;
constexpr int kSelectCap = 16384;  // candidates a select CTA holds in shared memory
constexpr int kBins = 256;         // radix digit of the select passes
constexpr int kAttendKeys = 128;   // selected keys per attention split
constexpr int kAttendWarps = 4;
constexpr int kMaxG = 8;
constexpr int kMaxFasaBudget = 4096;  // selected keys per query head

struct FasaParams {
  const __nv_bfloat16* q;  // rotated queries [B][Hq][d]
  const __nv_bfloat16* kc;  // rotated keys, chunk-major [B][Hkv][d/16][n_cache][16]
  const __nv_bfloat16* v;   // values [B][n_cache][Hkv][d]
  __nv_bfloat16* out;       // [B][Hq][d]
  float* scores;            // [B][Hq][n_cache] fp32 scores, or NULL (only written when asked for)
  uint32_t* cand;           // [B][Hq][seg_cap]: per warp segment, the candidate key indices
  float* cand_score;        // [B][Hq][seg_cap]: their scores (-0 as +0)
  unsigned int* seg_cnt;    // [B][Hq][n_seg]: candidates in each segment
  unsigned int* hist;       // [B][Hq][kHistBins] sample histograms
  uint32_t* thr;            // [B][Hq] threshold T as an order-preserving key
  int* sel;                 // [B][Hq][budget], ascending, -1 padded
  float* sel_score;         // [B][Hq][budget]: the kept keys' TIP scores (rows with sel_has_score)
  int* sel_has_score;       // [B][Hq]: 1 if the row's sel_score is written
  unsigned int* err;        // device error word (bounded waits)
  float* partials;          // [B][Hq][n_split][d + 2]
  int batch, hq, hkv, d, budget, n_split;
  int b_off;                // first sequence of a launch that covers part of the batch
  long long n_cache, n_seg, seg_cap;  // seg_cap = n_seg * kSegKeys >= n_cache
  unsigned long long mask;  // dominant pairs
  uint32_t chunk_mask;      // bit c: chunk c holds a dominant pair
  long long kv_len[kMaxDecodeBatch];
};

// Order-preserving map of a float's bits to an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float whose order_key is k.
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// Sampled keys of a sequence of L keys, and the sample rank whose score sets the
// threshold: twice the sample's share of `need`, plus 8.
__host__ __device__ __forceinline__ long long sample_count(long long L) {
  const long long rest = L % kSamplePeriod;
  return L / kSamplePeriod * kSampleRun + (rest < kSampleRun ? rest : kSampleRun);
}
__host__ __device__ __forceinline__ long long sample_rank(long long L, int need) {
  return (2LL * need * sample_count(L) + L - 1) / L + 8;
}

// TIP scores on the tensor cores.  One mma.sync m16n8k16 (bf16 in, fp32
// accumulate) takes a tile of 16 keys x the 16 dims of one cache chunk (A, row =
// key) against the same 16 dims of the kv head's query heads (B, column = query
// head g of the group, zero for g >= G and for non-dominant pairs).  The chunks
// holding a dominant pair are taken in ascending order, each accumulating into
// the same fp32 fragment.  Within a chunk, lane (g, t) = (lane / 4, lane % 4)
// supplies words 2t and 2t+1 of its keys' 32-byte chunk rows (dims 4t .. 4t+3)
// as k-slots (2t, 2t+1) and (2t+8, 2t+9), and the same dims of the query as B --
// a fixed arrangement, so every kernel that scores a key gets the same bits.
// Result fragment: c[0], c[1] = key g of the tile, heads 2t and 2t+1; c[2],
// c[3] = key g+8, heads 2t and 2t+1.
template <int NC>
struct QFrag {
  uint32_t b[NC][2];
};

// The B fragments of query heads row0 .. row0+G-1 for every chunk.
template <int D>
__device__ __forceinline__ QFrag<D / 16> load_qfrag(const __nv_bfloat16* q, long long row0, int G,
                                                    unsigned long long mask, int lane) {
  constexpr int NC = D / 16;
  QFrag<NC> f;
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    uint32_t lo = 0u, hi = 0u;
    if (g < G) {
      const uint32_t* qw = reinterpret_cast<const uint32_t*>(q + (row0 + g) * D + 16 * c + 4 * t);
      if ((mask >> (8 * c + 2 * t)) & 1ull) lo = __ldg(qw);
      if ((mask >> (8 * c + 2 * t + 1)) & 1ull) hi = __ldg(qw + 1);
    }
    f.b[c][0] = lo;
    f.b[c][1] = hi;
  }
  return f;
}

// Writes the B fragments of load_qfrag to sqf[c][lane] (one warp).
template <int D>
__device__ __forceinline__ void store_qfrag(uint2 (*sqf)[32], const __nv_bfloat16* q, long long row0, int G,
                                            unsigned long long mask, int lane) {
  const QFrag<D / 16> f = load_qfrag<D>(q, row0, G, mask, lane);
#pragma unroll
  for (int c = 0; c < D / 16; ++c) sqf[c][lane] = make_uint2(f.b[c][0], f.b[c][1]);
}

// Scores NT tiles of 16 keys in groups of P consecutive tiles (tile i: keys
// first + (i / P) * stride + 16 (i % P) .. + 15; keys at or past L read as zero
// unless `whole` says none is) for the kv head whose chunk-major planes start at
// kbase, with the B fragments in sqf.  The chunks holding a dominant pair
// (chunk_mask) are visited in ascending order.
template <int NT, int P>
__device__ __forceinline__ long long tile_first(long long first, long long stride, int i) {
  return first + (i / P) * stride + 16 * (i % P);
}
template <int NT, int P>
__device__ __forceinline__ void score_tiles(float (&acc)[NT][4], const uint2 (*sqf)[32], const __nv_bfloat16* kbase,
                                            long long n_cache, uint32_t chunk_mask, long long first, long long stride,
                                            bool whole, long long L, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
  for (uint32_t cm = chunk_mask; cm; cm &= cm - 1u) {
    const int c = __ffs(cm) - 1;
    const uint2 qb = sqf[c][lane];
    const __nv_bfloat16* row = kbase + (static_cast<long long>(c) * n_cache + first + g) * 16 + 4 * t;
    uint32_t a[NT][4];
    if (whole) {
#pragma unroll
      for (int i = 0; i < NT; ++i) {
        const long long off = (tile_first<NT, P>(0, stride, i)) * 16;
        const uint2 w0 = __ldg(reinterpret_cast<const uint2*>(row + off));
        const uint2 w1 = __ldg(reinterpret_cast<const uint2*>(row + off + 8 * 16));
        a[i][0] = w0.x;
        a[i][1] = w1.x;
        a[i][2] = w0.y;
        a[i][3] = w1.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < NT; ++i) {
        const long long off = tile_first<NT, P>(0, stride, i);
        const long long n0 = first + off + g;
        uint2 w0 = make_uint2(0u, 0u), w1 = w0;
        if (n0 < L) w0 = __ldg(reinterpret_cast<const uint2*>(row + off * 16));
        if (n0 + 8 < L) w1 = __ldg(reinterpret_cast<const uint2*>(row + off * 16 + 8 * 16));
        a[i][0] = w0.x;
        a[i][1] = w1.x;
        a[i][2] = w0.y;
        a[i][3] = w1.y;
      }
    }
#pragma unroll
    for (int i = 0; i < NT; ++i) mma_bf16_16816(acc[i], a[i], qb.x, qb.y);
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kSampleThreads) fasa_sample_kernel(FasaParams p) {
  constexpr int NC = D / 16;
  constexpr int kRuns = kSampleCtaKeys / kSamplePeriod;
  constexpr int kWarps = kSampleThreads / 32;
  constexpr int kRunsPerStep = 4;  // two tiles each
  static_assert(kRuns % (kWarps * kRunsPerStep) == 0 && kSampleRun == 32, "whole steps of four runs per warp");
  const int kvh = blockIdx.y, b = blockIdx.z, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long L = p.kv_len[b];
  const int need = L < p.budget ? static_cast<int>(L) : p.budget;
  const long long n0 = static_cast<long long>(blockIdx.x) * kSampleCtaKeys;
  if (need == L || n0 >= L) return;  // nothing to select, or no key of this CTA
  __shared__ uint2 s_qf[NC][32];
  __shared__ unsigned int s_lo[G], s_hi[G];  // the range of words any sampled key of this CTA touched
  // per head, kHistBins 16-bit counts packed two to a word (a CTA samples at most
  // 128 runs of 32 keys)
  extern __shared__ unsigned int shist[];
  const long long row0 = static_cast<long long>(b) * p.hq + kvh * G;
  for (int i = tid; i < G * (kHistBins / 2); i += kSampleThreads) shist[i] = 0u;
  if (tid < G) {
    s_lo[tid] = kHistBins / 2;
    s_hi[tid] = 0u;
  }
  if (warp == 0) store_qfrag<D>(s_qf, p.q, row0, G, p.mask, lane);
  __syncthreads();
  const __nv_bfloat16* kbase = p.kc + (static_cast<long long>(b) * p.hkv + kvh) * NC * p.n_cache * 16;
  const int g = lane >> 2, t = lane & 3;
  unsigned int lo_w[2] = {kHistBins / 2, kHistBins / 2}, hi_w[2] = {0u, 0u};
  // warp w, step s: runs (s kWarps + w) kRunsPerStep .. + kRunsPerStep - 1
#pragma unroll 1
  for (int st = 0; st < kRuns / (kWarps * kRunsPerStep); ++st) {
    const long long first = n0 + static_cast<long long>((st * kWarps + warp) * kRunsPerStep) * kSamplePeriod;
    if (first >= L) break;  // warp-uniform
    const bool whole = first + (kRunsPerStep - 1) * kSamplePeriod + kSampleRun <= L;
    float acc[2 * kRunsPerStep][4];
    score_tiles<2 * kRunsPerStep, 2>(acc, s_qf, kbase, p.n_cache, p.chunk_mask, first, kSamplePeriod, whole, L, lane);
#pragma unroll
    for (int i = 0; i < 2 * kRunsPerStep; ++i)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int h = 2 * t + (k & 1);
        const long long n = tile_first<2 * kRunsPerStep, 2>(first, kSamplePeriod, i) + g + 8 * (k >> 1);
        if (h < G && n < L) {
          const uint32_t bin = order_key(__fadd_rn(acc[i][k], 0.f)) >> (32 - kHistBits);
          atomicAdd(&shist[h * (kHistBins / 2) + (bin >> 1)], 1u << (16 * (bin & 1u)));
          lo_w[k & 1] = min(lo_w[k & 1], bin >> 1);
          hi_w[k & 1] = max(hi_w[k & 1], bin >> 1);
        }
      }
  }
  // per head, the touched range over the lanes that hold it (lanes with t = h / 2)
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    unsigned int lo = lo_w[e], hi = hi_w[e];
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    const int h = 2 * t + e;
    if (g == 0 && h < G && lo <= hi) {
      atomicMin(&s_lo[h], lo);
      atomicMax(&s_hi[h], hi);
    }
  }
  __syncthreads();
  // add the touched words' counts to the global histograms
#pragma unroll 1
  for (int h = 0; h < G; ++h) {
    const unsigned int lo = s_lo[h], hi = s_hi[h];
    unsigned int* hg = p.hist + (row0 + h) * kHistBins;
    for (unsigned int i = lo + tid; i <= hi; i += kSampleThreads) {
      const unsigned int w = shist[h * (kHistBins / 2) + i];
      if (w & 0xFFFFu) atomicAdd(&hg[2 * i], w & 0xFFFFu);
      if (w >> 16) atomicAdd(&hg[2 * i + 1], w >> 16);
    }
  }
}

// The threshold T of every (query head, sequence) row with a selection to make:
// the lower edge of the histogram bin that holds the sample's k-th largest score
// (0 -- every key a candidate -- when the sample holds fewer than k keys).
// Thread t holds the 16 bins [kHistBins - 16 (t + 1), kHistBins - 16 t).
__global__ void __launch_bounds__(kThresholdThreads) fasa_threshold_kernel(FasaParams p) {
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long row = static_cast<long long>(b) * p.hq + h;
  const long long L = p.kv_len[b];
  const int need = L < p.budget ? static_cast<int>(L) : p.budget;
  if (need == L) return;
  constexpr int kPer = kHistBins / kThresholdThreads;
  static_assert(kPer == 16, "four 16-byte loads per thread");
  __shared__ int s_warp[kThresholdThreads / 32];
  const uint4* hv = reinterpret_cast<const uint4*>(p.hist + row * kHistBins + kHistBins - kPer * (tid + 1));
  unsigned int c[kPer];
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint4 x = __ldcg(hv + v);
    c[4 * v] = x.x;
    c[4 * v + 1] = x.y;
    c[4 * v + 2] = x.z;
    c[4 * v + 3] = x.w;
  }
  int mine = 0;
#pragma unroll
  for (int k = 0; k < kPer; ++k) mine += static_cast<int>(c[k]);
  // inclusive count from the top bin through this thread's bins
  int incl = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  for (int w = 0; w < warp; ++w) incl += s_warp[w];
  const int ks = static_cast<int>(sample_rank(L, need));
  if (tid == kThresholdThreads - 1 && incl < ks) p.thr[row] = 0u;  // the sample is too small
  if (incl - mine < ks && ks <= incl) {
    int acc = incl - mine;
    for (int k = kPer - 1; k >= 0; --k) {  // c[k] is bin kHistBins - 16 (t + 1) + k
      acc += static_cast<int>(c[k]);
      if (acc >= ks) {
        p.thr[row] = static_cast<uint32_t>(kHistBins - kPer * (tid + 1) + k) << (32 - kHistBits);
        break;
      }
    }
  }
}

template <int D, int G>
__global__ void __launch_bounds__(kScoreThreads, 2) fasa_score_kernel(FasaParams p) {  // 2 CTAs per SM
  constexpr int NC = D / 16;
  constexpr int NT = 8;  // tiles of 16 keys per warp step
  constexpr int kStepKeys = 16 * NT;
  constexpr uint32_t kStageBytes = kStepKeys * 32;  // one chunk row of each key of a step
  static_assert(kSegKeys % kStepKeys == 0, "a segment is a whole number of steps");
  const int kvh = blockIdx.y, b = p.b_off + blockIdx.z, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long L = p.kv_len[b];
  const int need = L < p.budget ? static_cast<int>(L) : p.budget;
  const bool select = need < L;
  if ((!select && !p.scores) || static_cast<long long>(blockIdx.x) * kScoreCtaKeys >= L) return;
  extern __shared__ __align__(128) uint8_t s_ring[];  // per warp: kScoreStages stages of kStageBytes
  __shared__ uint64_t s_full[kScoreWarps][kScoreStages];
  __shared__ uint2 s_qf[NC][32];
  __shared__ float s_tf[8];  // the thresholds as floats
  __shared__ unsigned int s_cnt[kScoreWarps][8];
  __shared__ int s_abort;
  const long long row0 = static_cast<long long>(b) * p.hq + kvh * G;
  if (tid < 8) s_tf[tid] = select && tid < G ? key_float(p.thr[row0 + tid]) : 0.f;
  if (tid < kScoreWarps * 8) s_cnt[tid / 8][tid % 8] = 0u;
  if (tid < kScoreWarps * kScoreStages) mbar_init(&s_full[tid / kScoreStages][tid % kScoreStages], 1);
  if (tid == 0) s_abort = 0;
  if (warp == 0) store_qfrag<D>(s_qf, p.q, row0, G, p.mask, lane);
  fence_mbar_init();
  __syncthreads();
  const long long wseg = static_cast<long long>(blockIdx.x) * kScoreWarps + warp;
  const long long base = wseg * kSegKeys;
  if (base >= L) return;
  const int n_steps = static_cast<int>(min(static_cast<long long>(kSegKeys / kStepKeys),
                                           (L - base + kStepKeys - 1) / kStepKeys));
  const uint32_t cm = p.chunk_mask;
  const int n_chunks = __popc(cm);
  const int n_stages = n_steps * n_chunks;  // (step, chunk) pairs, chunk fastest
  const __nv_bfloat16* kbase = p.kc + (static_cast<long long>(b) * p.hkv + kvh) * NC * p.n_cache * 16;
  uint8_t* ring = s_ring + static_cast<size_t>(warp) * kScoreStages * kStageBytes;
  uint64_t* full = s_full[warp];
  // the c-th set bit of the chunk mask
  auto nth_chunk = [cm](int k) {
    uint32_t m = cm;
    for (int j = 0; j < k; ++j) m &= m - 1u;
    return __ffs(m) - 1;
  };
  auto issue = [&](int q) {  // lane 0: the bulk copy of stage q into slot q % kScoreStages
    const int it = q / n_chunks, c = nth_chunk(q - it * n_chunks);
    const long long s0 = base + static_cast<long long>(kStepKeys) * it;
    const uint32_t bytes = static_cast<uint32_t>(min(static_cast<long long>(kStepKeys), L - s0)) * 32u;
    uint64_t* bar = &full[q % kScoreStages];
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(ring + (q % kScoreStages) * kStageBytes, kbase + (static_cast<long long>(c) * p.n_cache + s0) * 16,
              bytes, bar);
  };
  int issued = 0;
  if (lane == 0)
    for (; issued < min(kScoreStages, n_stages); ++issued) issue(issued);
  issued = __shfl_sync(0xffffffffu, issued, 0);

  const int g = lane >> 2, t = lane & 3;
  const bool hv0 = 2 * t < G, hv1 = 2 * t + 1 < G;
  const float t0 = s_tf[2 * t], t1 = s_tf[2 * t + 1];
  unsigned int* err = p.err;
  int q = 0;
  bool ok = true;
  for (int it = 0; it < n_steps && ok; ++it) {
    const long long s0 = base + static_cast<long long>(kStepKeys) * it;
    const bool whole = s0 + kStepKeys <= L;
    float acc[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    for (int ci = 0; ci < n_chunks; ++ci, ++q) {
      if (!warp_wait(&full[q % kScoreStages], (q / kScoreStages) & 1, &s_abort, err, 0x501)) {
        ok = false;
        break;
      }
      const uint2 qb = s_qf[nth_chunk(ci)][lane];
      const uint8_t* st = ring + (q % kScoreStages) * kStageBytes + 32 * g + 8 * t;
      uint32_t a[NT][4];
#pragma unroll
      for (int i = 0; i < NT; ++i) {
        uint2 w0 = *reinterpret_cast<const uint2*>(st + 512 * i);
        uint2 w1 = *reinterpret_cast<const uint2*>(st + 512 * i + 256);
        if (!whole) {  // the copy stopped at key L - 1
          if (s0 + 16 * i + g >= L) w0 = make_uint2(0u, 0u);
          if (s0 + 16 * i + g + 8 >= L) w1 = make_uint2(0u, 0u);
        }
        a[i][0] = w0.x;
        a[i][1] = w1.x;
        a[i][2] = w0.y;
        a[i][3] = w1.y;
      }
      __syncwarp();  // every lane has read the slot: it may be refilled
      if (lane == 0 && issued < n_stages) issue(issued);
      ++issued;
#pragma unroll
      for (int i = 0; i < NT; ++i) mma_bf16_16816(acc[i], a[i], qb.x, qb.y);
    }
    if (!ok) break;
    // acc[i][k]: key s0 + 16 i + g + 8 (k >> 1), head 2t + (k & 1)
    if (p.scores) {
#pragma unroll
      for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int h = 2 * t + (k & 1);
          const long long n = s0 + 16 * i + g + 8 * (k >> 1);
          if (h < G && n < L) p.scores[(row0 + h) * p.n_cache + n] = __fadd_rn(acc[i][k], 0.f);
        }
    }
    if (!select) continue;
    // candidate bits: bit 4i + k for acc[i][k] at or above its head's threshold
    // (!(s < T) holds for s >= T; T is never -0, and a -0 score counts as +0)
    uint32_t m = 0u;
    if (whole) {
#pragma unroll
      for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          m |= static_cast<uint32_t>(!(acc[i][k] < ((k & 1) ? t1 : t0))) << (4 * i + k);
    } else {
#pragma unroll
      for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          m |= static_cast<uint32_t>(!(acc[i][k] < ((k & 1) ? t1 : t0)) && s0 + 16 * i + g + 8 * (k >> 1) < L)
               << (4 * i + k);
    }
    m &= (hv0 ? 0x55555555u : 0u) | (hv1 ? 0xAAAAAAAAu : 0u);
    if (!__any_sync(0xffffffffu, m != 0u)) continue;
    // slots: the lanes sharing this lane's two heads (lanes t, t + 4, .., t + 28)
    // take consecutive runs after the segment's count, so each step's candidates
    // of a head form one block of the list, after the blocks of earlier steps
    // (the selection orders keys within a block)
    const int c0 = __popc(m & 0x55555555u), c1 = __popc(m & 0xAAAAAAAAu);
    int p0 = c0, p1 = c1;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      const int y0 = __shfl_up_sync(0xffffffffu, p0, off), y1 = __shfl_up_sync(0xffffffffu, p1, off);
      if (lane >= off) {
        p0 += y0;
        p1 += y1;
      }
    }
    const int tot0 = __shfl_sync(0xffffffffu, p0, 28 + t), tot1 = __shfl_sync(0xffffffffu, p1, 28 + t);
    unsigned int pos0 = s_cnt[warp][2 * t] + static_cast<unsigned int>(p0 - c0);
    unsigned int pos1 = s_cnt[warp][2 * t + 1] + static_cast<unsigned int>(p1 - c1);
    __syncwarp();
    if (g == 0) {
      s_cnt[warp][2 * t] += static_cast<unsigned int>(tot0);
      s_cnt[warp][2 * t + 1] += static_cast<unsigned int>(tot1);
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      for (uint32_t mi = (m >> (4 * i)) & 15u; mi; mi &= mi - 1u) {
        const int k = __ffs(mi) - 1;
        const float v = k == 0 ? acc[i][0] : k == 1 ? acc[i][1] : k == 2 ? acc[i][2] : acc[i][3];
        const unsigned int pos = (k & 1) ? pos1++ : pos0++;
        const long long slot = (row0 + 2 * t + (k & 1)) * p.seg_cap + base + pos;
        p.cand[slot] = static_cast<uint32_t>(s0 + 16 * i + g + 8 * (k >> 1));
        p.cand_score[slot] = __fadd_rn(v, 0.f);
      }
    }
  }
  if (!ok) {  // a copy did not land in time: wait (bounded) for this warp's copies still in flight
    if (lane == 0)
      for (int r = q; r < min(issued, n_stages); ++r) {
        const long long w0 = clock64();
        while (!mbar_try_wait(&full[r % kScoreStages], (r / kScoreStages) & 1) && clock64() - w0 < kWaitLimitCycles) {
        }
      }
    return;
  }
  __syncwarp();
  if (select && lane < G) p.seg_cnt[(row0 + lane) * p.n_seg + wseg] = s_cnt[warp][lane];
}

// Exclusive prefix sum of v over the kSelectThreads threads; *total gets the sum.
// Every thread of the block must call it.
__device__ __forceinline__ int block_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int x = lane < kSelectThreads / 32 ? s_warp[lane] : 0;
    int xi = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, xi, off);
      if (lane >= off) xi += t;
    }
    if (lane < kSelectThreads / 32) s_warp[lane] = xi - x;
    if (lane == 31) *total = xi;
  }
  __syncthreads();
  const int r = s_warp[warp] + incl - v;
  __syncthreads();  // s_warp is reused by the next call
  return r;
}

// The candidates of one (query head, sequence), held in shared memory: order
// keys and key indices.
struct SmemList {
  const uint32_t* key;
  const uint32_t* idx;
  long long n;
  __device__ __forceinline__ bool get(long long i, uint32_t& k, uint32_t& x) const {
    k = key[i];
    x = idx[i];
    return true;
  }
};

// The same in global memory: slot i of the warp segments (valid below the
// segment's count), or with `dense` every slot below n (slot = key index).
struct SegmentList {
  const uint32_t* cand;
  const float* score;
  const unsigned int* cnt;
  long long n;
  bool dense;
  __device__ __forceinline__ bool get(long long i, uint32_t& k, uint32_t& x) const {
    if (!dense && static_cast<unsigned int>(i & (kSegKeys - 1)) >= cnt[i >> kSegShift]) return false;
    k = order_key(score[i]);
    x = cand[i];
    return true;
  }
};

struct SelectScratch {
  unsigned int* hist;  // kBins
  int* warp;           // 32
  int* total;
  int* digit;
  int* gt;
  int* out;            // kMaxFasaBudget
};

// Radix select over the 32-bit values val(i) of the entries i of `list` with
// in(i): returns the value v such that `rank` entries (1 <= rank <= count) lie
// at or above it in the order of `largest` (descending if true), and writes to
// *before the number strictly beyond it.  Every thread of the block calls it.
template <class List, class Val, class In>
__device__ uint32_t radix_select(const List& list, Val val, In in, int rank, bool largest, int* before, int* equal,
                                 const SelectScratch& sc) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0u, pmask = 0u;
  int left = rank, beyond = 0;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < kBins; i += kSelectThreads) sc.hist[i] = 0u;
    if (tid == 0) {
      *sc.digit = 0;
      *sc.gt = 0;
    }
    __syncthreads();
    // one atomic per distinct digit and warp: many entries share their top digits
    for (long long i0 = 0; i0 < list.n; i0 += kSelectThreads) {
      const long long i = i0 + tid;
      uint32_t k, x, d = 0xFFFFFFFFu;
      if (i < list.n && list.get(i, k, x) && in(k, x)) {
        const uint32_t v = val(k, x);
        if ((v & pmask) == prefix) d = (v >> shift) & (kBins - 1);
      }
      const unsigned int peers = __match_any_sync(0xffffffffu, d);
      if (d != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&sc.hist[d], static_cast<unsigned int>(__popc(peers)));
    }
    __syncthreads();
    if (warp == 0) {
      // the digit d: the first, in the selection order, whose cumulative count
      // reaches `left`; lane l holds 8 consecutive digits in that order
      int c8 = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) c8 += static_cast<int>(sc.hist[largest ? 255 - (8 * lane + u) : 8 * lane + u]);
      int incl = c8;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      if (incl - c8 < left && left <= incl) {
        int run = incl - c8;
        for (int u = 0; u < 8; ++u) {
          const int d = largest ? 255 - (8 * lane + u) : 8 * lane + u;
          const int cu = static_cast<int>(sc.hist[d]);
          if (run + cu >= left) {
            *sc.digit = d;
            *sc.gt = run;
            break;
          }
          run += cu;
        }
      }
    }
    __syncthreads();
    left -= *sc.gt;
    beyond += *sc.gt;
    prefix |= static_cast<uint32_t>(*sc.digit) << shift;
    pmask |= static_cast<uint32_t>(kBins - 1) << shift;
    if (pass == 3) *equal = static_cast<int>(sc.hist[*sc.digit]);  // entries equal to the whole value
    __syncthreads();  // digit, gt and the histogram are rewritten by the next pass
  }
  *before = beyond;
  return prefix;
}

// Writes to out[0 .. need) the indices of the `need` largest entries of `list`
// by order key (equal keys: lower index first), ascending, and -1 to out[need ..
// budget).  The list holds at least `need` entries, all with indices below L.
// `bitmap` (bitmap_words words of shared memory, free once the list has been
// read) orders the kept indices when L fits in it; otherwise they are sorted.

template <class List>
__device__ void select_emit(const List& list, int need, int budget, long long L, int* out, uint32_t* bitmap,
                            int bitmap_words, const SelectScratch& sc) {
  const int tid = threadIdx.x;
  auto by_key = [](uint32_t k, uint32_t) { return k; };
  auto all = [](uint32_t, uint32_t) { return true; };
  int above = 0, eq = 0;
  const uint32_t V = radix_select(list, by_key, all, need, true, &above, &eq, sc);
  const int left = need - above;  // entries equal to V to keep: the lowest indices
  uint32_t I = 0xFFFFFFFFu;
  if (eq > left) {  // the left-th smallest index among the entries equal to V decides
    auto by_idx = [](uint32_t, uint32_t x) { return x; };
    auto equal = [V](uint32_t k, uint32_t) { return k == V; };
    int below = 0, same = 0;
    I = radix_select(list, by_idx, equal, left, false, &below, &same, sc);
  }
  auto kept = [V, I](uint32_t k, uint32_t x) { return k > V || (k == V && x <= I); };
  if (tid == 0) *sc.total = 0;
  __syncthreads();
  const int lane = tid & 31, warp = tid >> 5;
  for (long long i0 = 0; i0 < list.n; i0 += kSelectThreads) {
    const long long i = i0 + tid;
    uint32_t k = 0u, x = 0u;
    const bool keep = i < list.n && list.get(i, k, x) && kept(k, x);
    const unsigned int bal = __ballot_sync(0xffffffffu, keep);
    const int leader = bal ? __ffs(bal) - 1 : 0;
    int base = 0;
    if (bal && lane == leader) base = atomicAdd(sc.total, __popc(bal));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (keep) {
      const int slot = base + __popc(bal & ((1u << lane) - 1u));
      if (slot < need) sc.out[slot] = static_cast<int>(x);
    }
  }
  __syncthreads();
  const int nw = static_cast<int>((L + 31) / 32);
  if (nw <= bitmap_words) {
    // one bit per key index; warp w then emits the set bits of its run of words,
    // 32 words at a time (lane l: word 32 j + l of the run), after the counts of
    // the runs before it
    for (int i = tid; i < nw; i += kSelectThreads) bitmap[i] = 0u;
    __syncthreads();
    for (int i = tid; i < need; i += kSelectThreads) {
      const int x = sc.out[i];
      if (x >= 0 && x < L) atomicOr(&bitmap[x >> 5], 1u << (x & 31));  // always, with consistent counts
    }
    __syncthreads();
    constexpr int kWarps = kSelectThreads / 32;
    const int per = (nw + kWarps - 1) / kWarps;
    const int r0 = min(nw, warp * per), r1 = min(nw, r0 + per);
    int cnt = 0;
    for (int w = r0 + lane; w < r1; w += 32) cnt += __popc(bitmap[w]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    int pos = block_scan(lane == 0 ? cnt : 0, sc.warp, sc.total);
    pos = __shfl_sync(0xffffffffu, pos, 0);  // this warp's first output slot
    for (int j = r0; j < r1; j += 32) {
      const int w = j + lane;
      const uint32_t bits = w < r1 ? bitmap[w] : 0u;
      const int c = __popc(bits);
      int incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      int q = pos + incl - c;
      for (uint32_t b = bits; b; b &= b - 1u)
        if (q < need) out[q++] = 32 * w + __ffs(b) - 1;
      pos += __shfl_sync(0xffffffffu, incl, 31);
    }
  } else {
    // bitonic sort of the kept indices (padded to a power of two)
    int P = 1;
    while (P < need) P <<= 1;
    for (int i = need + tid; i < P; i += kSelectThreads) sc.out[i] = 0x7fffffff;
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < P; i += kSelectThreads) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const int a = sc.out[i], c = sc.out[ixj];
            if ((a > c) == ((i & k) == 0)) {
              sc.out[i] = c;
              sc.out[ixj] = a;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int i = tid; i < need; i += kSelectThreads) out[i] = sc.out[i];
  }
  for (int i = need + tid; i < budget; i += kSelectThreads) out[i] = -1;
}

constexpr int kFineBits = 12;                 // bins of the single-pass selection
constexpr int kFineBins = 1 << kFineBits;
constexpr int kBoundaryMax = 256;             // keys of the boundary bin ranked exactly

// The shared-memory list as runs, one per thread in thread order (the warp
// segments: every key of a run is below every key of the next run): keeps the
// `need` largest keys (equal keys: lower index first) and writes them ascending
// to out[0 .. need), -1 to out[need .. budget).  One histogram pass of 4096 bins
// over the 12 bits below the prefix shared by every key (between T and the
// largest) finds the boundary bin; its keys are ranked exactly against each
// other, once each, and the kept ones marked in bit 31 of their list index
// (key indices are below 2^31).  Returns false, having written nothing and
// marked nothing, if the boundary bin holds more than kBoundaryMax keys.
// scratch: kFineBins + 3 kBoundaryMax words.
__device__ bool select_runs(const uint32_t* key, uint32_t* idx, int run_off, int run_len, uint32_t kmin,
                            uint32_t kmax, int need, int budget, int* out, float* out_score, uint32_t* scratch,
                            const SelectScratch& sc) {
  const int tid = threadIdx.x;
  // the bits below the common prefix of kmin and kmax (the whole key if they differ at the top)
  const uint32_t diff = kmin ^ kmax;
  const int top = diff ? 32 - __clz(diff) : 1;  // bits that vary: 0 .. top-1
  const int shift = top > kFineBits ? top - kFineBits : 0;
  auto bin_of = [kmin, shift](uint32_t k) { return static_cast<int>((k - (kmin >> shift << shift)) >> shift); };
  // (every key lies in [kmin, kmax]; bin_of is monotone in k and below kFineBins)
  unsigned int* hist = scratch;
  uint32_t* bkey = scratch + kFineBins;
  uint32_t* bidx = bkey + kBoundaryMax;
  uint32_t* bpos = bidx + kBoundaryMax;
  for (int i = tid; i < kFineBins; i += kSelectThreads) hist[i] = 0u;
  __syncthreads();
  for (int j = 0; j < run_len; ++j) atomicAdd(&hist[bin_of(key[run_off + j])], 1u);
  __syncthreads();
  // suffix counts from the top bin: thread t holds bins kFineBins - 4 (t + 1) .. kFineBins - 4 t - 1
  constexpr int kPer = kFineBins / kSelectThreads;
  int c[kPer], mine = 0;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    c[u] = static_cast<int>(hist[kFineBins - kPer * tid - 1 - u]);
    mine += c[u];
  }
  const int before = block_scan(mine, sc.warp, sc.total);  // keys in higher bins than this thread's
  if (tid == 0) {
    *sc.digit = -1;
    *sc.gt = 0;
  }
  __syncthreads();
  if (before < need && need <= before + mine) {
    int acc = before;
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (acc + c[u] >= need) {
        *sc.digit = kFineBins - kPer * tid - 1 - u;  // the boundary bin
        *sc.gt = acc;                                 // keys above it
        break;
      }
      acc += c[u];
    }
  }
  __syncthreads();
  const int B = *sc.digit, above = *sc.gt;
  const int nb = B >= 0 ? static_cast<int>(hist[B]) : 0;
  if (B < 0 || nb > kBoundaryMax) return false;  // uniform: every thread read the same
  // the boundary bin's keys, then each one's rank among them (larger key first,
  // equal keys by lower index): kept if fewer than need - above precede it
  if (tid == 0) *sc.total = 0;
  __syncthreads();
  for (int j = 0; j < run_len; ++j) {
    const uint32_t k = key[run_off + j];
    if (bin_of(k) == B) {
      const int slot = atomicAdd(sc.total, 1);
      bkey[slot] = k;
      bidx[slot] = idx[run_off + j];
      bpos[slot] = static_cast<uint32_t>(run_off + j);
    }
  }
  __syncthreads();
  for (int e = tid; e < nb; e += kSelectThreads) {
    const uint32_t k = bkey[e], x = bidx[e];
    int r = 0;
    for (int f = 0; f < nb; ++f) r += bkey[f] > k || (bkey[f] == k && bidx[f] < x);
    if (r < need - above) idx[bpos[e]] = x | 0x80000000u;
  }
  __syncthreads();
  auto kept = [&](int j) {
    const int bn = bin_of(key[run_off + j]);
    return bn > B || (bn == B && (idx[run_off + j] >> 31));
  };
  int nk = 0;
  for (int j = 0; j < run_len; ++j) nk += kept(j);
  int pos = block_scan(nk, sc.warp, sc.total);
  // this run's kept keys in ascending index order after those of the runs before.
  // A run lists the candidates of each 128-key step of its segment as one block,
  // steps in ascending order; only within a block are they unordered.
  for (int j = 0; j < run_len;) {
    const uint32_t blk = (idx[run_off + j] & 0x7FFFFFFFu) >> 7;
    int je = j + 1;
    while (je < run_len && ((idx[run_off + je] & 0x7FFFFFFFu) >> 7) == blk) ++je;
    int nb_kept = 0;
    for (int a = j; a < je; ++a) {
      if (!kept(a)) continue;
      const uint32_t x = idx[run_off + a] & 0x7FFFFFFFu;
      int rank = 0;
      for (int c2 = j; c2 < je; ++c2) rank += kept(c2) && (idx[run_off + c2] & 0x7FFFFFFFu) < x;
      if (pos + rank < need) {
        out[pos + rank] = static_cast<int>(x);
        out_score[pos + rank] = key_float(key[run_off + a]);
      }
      ++nb_kept;
    }
    pos += nb_kept;
    j = je;
  }
  for (int i = need + tid; i < budget; i += kSelectThreads) out[i] = -1;
  return true;
}

template <int D>
__global__ void __launch_bounds__(kSelectThreads) fasa_select_kernel(FasaParams p) {
  const int h = blockIdx.x, b = p.b_off + blockIdx.y, tid = threadIdx.x;
  const long long row = static_cast<long long>(b) * p.hq + h;
  const long long L = p.kv_len[b];
  const int need = L < p.budget ? static_cast<int>(L) : p.budget;
  int* out = p.sel + row * p.budget;
  if (tid == 0) p.sel_has_score[row] = 0;  // set to 1 by the path that writes the scores
  if (need == L) {  // every key is selected, already in order
    for (int i = tid; i < p.budget; i += kSelectThreads) out[i] = i < L ? i : -1;
    return;
  }
  extern __shared__ uint32_t s_list[];  // order keys [kSelectCap], then key indices [kSelectCap]
  __shared__ unsigned int s_hist[kBins];
  __shared__ int s_warp[32];
  __shared__ int s_total, s_digit, s_gt;
  __shared__ int s_out[kMaxFasaBudget];
  __shared__ uint32_t s_kmax;
  if (tid == 0) s_kmax = 0u;
  const SelectScratch scr{s_hist, s_warp, &s_total, &s_digit, &s_gt, s_out};
  const uint32_t T = p.thr[row];
  const long long nseg = (L + kSegKeys - 1) / kSegKeys;
  const unsigned int* cnt = p.seg_cnt + row * p.n_seg;
  uint32_t* cand = p.cand + row * p.seg_cap;
  float* cscore = p.cand_score + row * p.seg_cap;

  int mine = 0;
  for (long long w = tid; w < nseg; w += kSelectThreads) mine += static_cast<int>(cnt[w]);
  block_scan(mine, s_warp, &s_total);
  const long long m = s_total;
  int reached = 0;  // candidates at or above T
  if (m <= kSelectCap) {
    // gather the segments' lists in segment order: thread t copies segment t of
    // each group of kSelectThreads segments
    uint32_t* s_key = s_list;
    uint32_t* s_idx = s_list + kSelectCap;
    int carry = 0, run_off = 0, run_len = nseg <= kSelectThreads ? 0 : -1;
    uint32_t kmax = 0u;
    for (long long w0 = 0; w0 < nseg; w0 += kSelectThreads) {
      const long long w = w0 + tid;
      const int cw = w < nseg ? static_cast<int>(cnt[w]) : 0;
      const int off = carry + block_scan(cw, s_warp, &s_total);
      if (run_len >= 0) {  // one segment per thread: its run
        run_off = off;
        run_len = cw;
      }
      for (int j0 = 0; j0 < cw; j0 += 8) {  // eight entries' loads in flight at a time
        float sv[8];
        uint32_t xv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (j0 + u < cw) {
            sv[u] = cscore[w * kSegKeys + j0 + u];
            xv[u] = cand[w * kSegKeys + j0 + u];
          }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (j0 + u < cw) {
            const uint32_t k = order_key(sv[u]);
            s_key[off + j0 + u] = k;
            s_idx[off + j0 + u] = xv[u];
            reached += k >= T;
            kmax = max(kmax, k);
          }
      }
      carry += s_total;
    }
    block_scan(reached, s_warp, &s_total);
    if (s_total >= need) {
      // the fast path needs one run per thread, every key at or above T, and room
      // for its scratch after the key indices (s_idx[m ..])
      kmax = __reduce_max_sync(0xffffffffu, kmax);
      if ((tid & 31) == 0) atomicMax(&s_kmax, kmax);
      __syncthreads();
      const bool fast = run_len >= 0 && s_total == m && kSelectCap - m >= kFineBins + 3 * kBoundaryMax;
      if (fast && select_runs(s_key, s_idx, run_off, run_len, T, s_kmax, need, p.budget, out,
                              p.sel_score + row * p.budget, s_list + kSelectCap + m, scr)) {
        if (tid == 0) p.sel_has_score[row] = 1;
        return;
      }
      // (select_runs wrote nothing; its scratch lay after the list)
      select_emit(SmemList{s_key, s_idx, m}, need, p.budget, L, out, s_list, 2 * kSelectCap, scr);
      return;
    }
  } else {
    const SegmentList list{cand, cscore, cnt, nseg * kSegKeys, false};
    for (long long i = tid; i < list.n; i += kSelectThreads) {
      uint32_t k, x;
      reached += list.get(i, k, x) && k >= T;
    }
    block_scan(reached, s_warp, &s_total);
    if (s_total >= need) {
      select_emit(list, need, p.budget, L, out, s_list, 2 * kSelectCap, scr);
      return;
    }
  }
  // fewer than `need` keys reached T: every key's score, in the same arithmetic
  // and arrangement as the scoring kernel, into the (now unused) candidate
  // arrays, slot n = key n, then select over all
  {
    constexpr int NC = D / 16;
    __shared__ uint2 s_qf[NC][32];
    const int G = p.hq / p.hkv, kvh = h / G, hl = h - kvh * G;
    const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    if (warp == 0) store_qfrag<D>(s_qf, p.q, static_cast<long long>(b) * p.hq + kvh * G, G, p.mask, lane);
    __syncthreads();
    const __nv_bfloat16* kbase = p.kc + (static_cast<long long>(b) * p.hkv + kvh) * NC * p.n_cache * 16;
    for (long long tile = warp; tile * 16 < L; tile += kSelectThreads / 32) {
      float acc[1][4];
      score_tiles<1, 1>(acc, s_qf, kbase, p.n_cache, p.chunk_mask, tile * 16, 0, tile * 16 + 16 <= L, L, lane);
      if (t == hl / 2) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const long long n = tile * 16 + g + 8 * r;
          if (n < L) {
            cscore[n] = __fadd_rn(acc[0][2 * r + (hl & 1)], 0.f);
            cand[n] = static_cast<uint32_t>(n);
          }
        }
      }
    }
  }
  __syncthreads();
  select_emit(SegmentList{cand, cscore, cnt, L, true}, need, p.budget, L, out, s_list, 2 * kSelectCap, scr);
}

// 16-byte asynchronous copy global -> shared (completion per thread by
// cp.async.wait_group), L1 bypassed.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Focused attention over one split of 128 selected keys of one (query head,
// sequence): warp w takes 32 of them.  The warp copies its keys' K rows (from
// the chunk-major cache: d/16 pieces of 32 bytes) and V rows into shared memory
// with 16-byte asynchronous copies, all in flight together, then lane l sums q.k
// over its d/32 dims for all 32 keys, a transposing butterfly leaves key l's dot
// product in lane l, and the warp's softmax over its 32 keys weights the V rows.
template <int D>
__global__ void __launch_bounds__(kAttendWarps * 32) fasa_attend_kernel(FasaParams p) {
  constexpr int NC = D / 16;
  constexpr int DPL = D / 32;        // dims per lane: 4 (d = 128) or 2 (d = 64)
  constexpr int kGran = D / 8;       // 16-byte pieces of a K row, and of a V row
  const int split = blockIdx.x, h = blockIdx.y, b = p.b_off + blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.hq / p.hkv, kvh = h / G;
  const long long row = static_cast<long long>(b) * p.hq + h;
  const long long L = p.kv_len[b];
  const int need = L < p.budget ? static_cast<int>(L) : p.budget;
  const int j0 = split * kAttendKeys + 32 * warp;  // this warp's first selected key
  const int nk = max(0, min(32, need - j0));

  extern __shared__ __align__(16) __nv_bfloat16 s_rows[];  // per warp: K rows [32][D], then V rows [32][D]
  __nv_bfloat16* sk = s_rows + static_cast<size_t>(warp) * 64 * D;
  __nv_bfloat16* sv = sk + 32 * D;
  const int n_mine = lane < nk ? p.sel[row * p.budget + j0 + lane] : -1;
  const bool ok = n_mine >= 0 && n_mine < L;  // always, with consistent inputs
  // With the kept keys' TIP scores at hand (the partial dot products over the
  // dominant pairs), only the other pairs are summed here: the chunks whose
  // eight pairs are all dominant are not read at all.
  const bool tip = p.sel_has_score[row] != 0;
  const float s_tip = tip && lane < nk ? p.sel_score[row * p.budget + j0 + lane] : 0.f;
  uint32_t full_chunks = 0u;  // bit c: chunk c entirely dominant (skipped when tip)
  if (tip)
#pragma unroll
    for (int c = 0; c < NC; ++c) full_chunks |= static_cast<uint32_t>(((p.mask >> (8 * c)) & 0xFFu) == 0xFFu) << c;
  const __nv_bfloat16* kb = p.kc + (static_cast<long long>(b) * p.hkv + kvh) * NC * p.n_cache * 16;
  const __nv_bfloat16* vb = p.v + static_cast<long long>(b) * p.n_cache * p.hkv * D + kvh * D;
  // piece i of the warp's copy: key i / (2 kGran), then its K pieces, then its V pieces
  for (int i = lane; i < 32 * 2 * kGran; i += 32) {
    const int key = i / (2 * kGran), gi = i % (2 * kGran);
    const int n = __shfl_sync(0xffffffffu, n_mine, key);  // warp-uniform loop: every lane shuffles
    const bool kok = __shfl_sync(0xffffffffu, static_cast<int>(ok), key) != 0;
    if (!kok) continue;
    if (gi < kGran) {  // K: chunk gi / 2, half gi % 2
      if ((full_chunks >> (gi >> 1)) & 1u) continue;
      const __nv_bfloat16* src = kb + (static_cast<long long>(gi >> 1) * p.n_cache + n) * 16 + 8 * (gi & 1);
      cp_async16(sk + key * D + 8 * gi, src);
    } else {
      const int gv = gi - kGran;
      cp_async16(sv + key * D + 8 * gv, vb + static_cast<long long>(n) * p.hkv * D + 8 * gv);
    }
  }
  cp_async_wait_all();
  __syncwarp();

  constexpr float kLog2e = 1.4426950408889634f;
  const float scale = kLog2e * rsqrtf(static_cast<float>(D));
  float q[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) {
    q[e] = __bfloat162float(p.q[row * D + DPL * lane + e]) * scale;
    if (tip && ((p.mask >> ((DPL * lane + e) / 2)) & 1ull)) q[e] = 0.f;  // in the TIP score already
  }
  const bool lane_reads = !((full_chunks >> ((DPL * lane) / 16)) & 1u);  // this lane's K dims were copied
  // partial dot products of all 32 keys over this lane's dims
  float dp[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    float acc = 0.f;
    if (k < nk && lane_reads) {
      const __nv_bfloat16* kr = sk + k * D + DPL * lane;
      if constexpr (DPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(kr);
        acc = fmaf(q[0], bf16lo_to_f32(w.x), acc);
        acc = fmaf(q[1], bf16hi_to_f32(w.x), acc);
        acc = fmaf(q[2], bf16lo_to_f32(w.y), acc);
        acc = fmaf(q[3], bf16hi_to_f32(w.y), acc);
      } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(kr);
        acc = fmaf(q[0], bf16lo_to_f32(w), acc);
        acc = fmaf(q[1], bf16hi_to_f32(w), acc);
      }
    }
    dp[k] = acc;
  }
  // transposing butterfly: at each step a lane keeps the half of its array that
  // its bit selects and adds the partner's copy of that half; lane l ends with
  // key l's full dot product in dp[0]
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? dp[i] : dp[i + off];
      const float keep = upper ? dp[i + off] : dp[i];
      dp[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  const bool live = lane < nk && ok;
  const float sdot = live ? fmaf(s_tip, scale, dp[0]) : -INFINITY;
  float mrun = sdot;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mrun = fmaxf(mrun, __shfl_xor_sync(0xffffffffu, mrun, off));
  const float pr = live ? ex2_approx(sdot - mrun) : 0.f;
  float lsum = pr;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
  float o[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) o[e] = 0.f;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const float pk = __shfl_sync(0xffffffffu, pr, k);
    if (k < nk && pk != 0.f) {
      const __nv_bfloat16* vr = sv + k * D + DPL * lane;
      if constexpr (DPL == 4) {
        const uint2 w = *reinterpret_cast<const uint2*>(vr);
        o[0] = fmaf(pk, bf16lo_to_f32(w.x), o[0]);
        o[1] = fmaf(pk, bf16hi_to_f32(w.x), o[1]);
        o[2] = fmaf(pk, bf16lo_to_f32(w.y), o[2]);
        o[3] = fmaf(pk, bf16hi_to_f32(w.y), o[3]);
      } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(vr);
        o[0] = fmaf(pk, bf16lo_to_f32(w), o[0]);
        o[1] = fmaf(pk, bf16hi_to_f32(w), o[1]);
      }
    }
  }
  if (nk == 0) mrun = -INFINITY;  // an empty warp contributes nothing
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
  const int h = blockIdx.x, b = p.b_off + blockIdx.y, e = threadIdx.x;
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
  size_t cand, cand_score, seg_cnt, hist, thr, sel, sel_score, sel_has_score, partials, total;
};

FasaLayout fasa_layout(int batch, int heads, long long n_cache, int budget, int d, bool own_sel) {
  const size_t rows = static_cast<size_t>(batch) * heads;
  const size_t n_seg = static_cast<size_t>((n_cache + kSegKeys - 1) / kSegKeys);
  const int n_split = (budget + kAttendKeys - 1) / kAttendKeys;
  FasaLayout L{};
  size_t off = 0;
  L.cand = off;
  off += align256(rows * n_seg * kSegKeys * sizeof(uint32_t));
  L.cand_score = off;
  off += align256(rows * n_seg * kSegKeys * sizeof(float));
  L.seg_cnt = off;
  off += align256(rows * n_seg * sizeof(unsigned int));
  L.hist = off;
  off += align256(rows * kHistBins * sizeof(unsigned int));
  L.thr = off;
  off += align256(rows * sizeof(uint32_t));
  L.sel = off;
  off += own_sel ? 0 : align256(rows * budget * sizeof(int));
  L.sel_score = off;
  off += align256(rows * budget * sizeof(float));
  L.sel_has_score = off;
  off += align256(rows * sizeof(int));
  L.partials = off;
  off += align256(rows * n_split * (d + 2) * sizeof(float));
  L.total = off;
  return L;
}

template <int D, int G>
void launch_front(const FasaParams& p, long long max_len, cudaStream_t s) {
  const size_t hist_smem = static_cast<size_t>(G) * (kHistBins / 2) * sizeof(unsigned int);
  fasa_sample_kernel<D, G><<<dim3(static_cast<unsigned>((max_len + kSampleCtaKeys - 1) / kSampleCtaKeys), p.hkv,
                                  p.batch),
                             kSampleThreads, hist_smem, s>>>(p);
  fasa_threshold_kernel<<<dim3(p.hq, p.batch), kThresholdThreads, 0, s>>>(p);
}

template <int D, int G>
void launch_score(const FasaParams& p, int nb, long long max_len, cudaStream_t s) {
  fasa_score_kernel<D, G><<<dim3(static_cast<unsigned>((max_len + kScoreCtaKeys - 1) / kScoreCtaKeys), p.hkv, nb),
                            kScoreThreads, kScoreSmem, s>>>(p);
}

// Streams and events of the per-sequence chains, per device: created once,
// used under the mutex (the chains are forked from and joined back to the
// caller's stream, so two calls must not interleave their records).
constexpr int kChainStreams = 4;
struct ChainPool {
  cudaStream_t st[kChainStreams] = {};
  cudaEvent_t fork = nullptr, join[kChainStreams] = {};
  bool ready = false;
};
std::mutex g_chain_mu;
ChainPool g_chain[64];

template <int D>
cudaError_t launch_fasa(const FasaParams& p, long long max_len, cudaStream_t s) {
  const int G = p.hq / p.hkv;
  constexpr size_t kSelectSmem = 2 * kSelectCap * sizeof(uint32_t);
  constexpr size_t kAttendSmem = static_cast<size_t>(kAttendWarps) * 64 * D * sizeof(__nv_bfloat16);
  // one bit per device: the attributes are set once (racing first calls both set them, harmlessly)
  static std::atomic<unsigned long long> configured{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(configured.load(std::memory_order_acquire) & (1ull << dev))) {
    const int bytes = kMaxG * (kHistBins / 2) * static_cast<int>(sizeof(unsigned int));
    const void* fns[8] = {reinterpret_cast<const void*>(fasa_sample_kernel<D, 1>),
                          reinterpret_cast<const void*>(fasa_sample_kernel<D, 2>),
                          reinterpret_cast<const void*>(fasa_sample_kernel<D, 3>),
                          reinterpret_cast<const void*>(fasa_sample_kernel<D, 4>),
                          reinterpret_cast<const void*>(fasa_sample_kernel<D, 5>),
                          reinterpret_cast<const void*>(fasa_sample_kernel<D, 6>),
                          reinterpret_cast<const void*>(fasa_sample_kernel<D, 7>),
                          reinterpret_cast<const void*>(fasa_sample_kernel<D, 8>)};
    for (const void* f : fns) {
      e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e != cudaSuccess) return e;
    }
    const void* score_fns[8] = {reinterpret_cast<const void*>(fasa_score_kernel<D, 1>),
                                reinterpret_cast<const void*>(fasa_score_kernel<D, 2>),
                                reinterpret_cast<const void*>(fasa_score_kernel<D, 3>),
                                reinterpret_cast<const void*>(fasa_score_kernel<D, 4>),
                                reinterpret_cast<const void*>(fasa_score_kernel<D, 5>),
                                reinterpret_cast<const void*>(fasa_score_kernel<D, 6>),
                                reinterpret_cast<const void*>(fasa_score_kernel<D, 7>),
                                reinterpret_cast<const void*>(fasa_score_kernel<D, 8>)};
    for (const void* f : score_fns) {
      e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kScoreSmem));
      if (e != cudaSuccess) return e;
    }
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fasa_select_kernel<D>),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSelectSmem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fasa_attend_kernel<D>),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kAttendSmem));
    if (e != cudaSuccess) return e;
    if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_acq_rel);
  }
  auto score = [&](const FasaParams& q, int nb, long long len, cudaStream_t st) {
    switch (G) {
      case 1: launch_score<D, 1>(q, nb, len, st); break;
      case 2: launch_score<D, 2>(q, nb, len, st); break;
      case 3: launch_score<D, 3>(q, nb, len, st); break;
      case 4: launch_score<D, 4>(q, nb, len, st); break;
      case 5: launch_score<D, 5>(q, nb, len, st); break;
      case 6: launch_score<D, 6>(q, nb, len, st); break;
      case 7: launch_score<D, 7>(q, nb, len, st); break;
      default: launch_score<D, 8>(q, nb, len, st); break;
    }
  };
  // select -> attention -> combine for sequences b_off .. b_off + nb - 1
  auto finish = [&](const FasaParams& q, int nb, cudaStream_t st) {
    fasa_select_kernel<D><<<dim3(q.hq, nb), kSelectThreads, kSelectSmem, st>>>(q);
    fasa_attend_kernel<D><<<dim3(q.n_split, q.hq, nb), kAttendWarps * 32, kAttendSmem, st>>>(q);
    fasa_combine_kernel<D><<<dim3(q.hq, nb), D, 0, st>>>(q);
  };
  switch (G) {
    case 1: launch_front<D, 1>(p, max_len, s); break;
    case 2: launch_front<D, 2>(p, max_len, s); break;
    case 3: launch_front<D, 3>(p, max_len, s); break;
    case 4: launch_front<D, 4>(p, max_len, s); break;
    case 5: launch_front<D, 5>(p, max_len, s); break;
    case 6: launch_front<D, 6>(p, max_len, s); break;
    case 7: launch_front<D, 7>(p, max_len, s); break;
    default: launch_front<D, 8>(p, max_len, s); break;
  }
  if (p.batch == 1 || dev >= 64) {
    score(p, p.batch, max_len, s);
    finish(p, p.batch, s);
    return cudaGetLastError();
  }
  // one chain (score -> select -> attention -> combine) per sequence on the
  // library's streams: the chains' latency-bound selections and attention
  // overlap other chains' bandwidth-bound scoring
  std::lock_guard<std::mutex> lk(g_chain_mu);
  ChainPool& pool = g_chain[dev];
  if (!pool.ready) {
    for (int i = 0; i < kChainStreams && e == cudaSuccess; ++i) {
      e = cudaStreamCreateWithFlags(&pool.st[i], cudaStreamNonBlocking);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&pool.join[i], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&pool.fork, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
    pool.ready = true;
  }
  e = cudaEventRecord(pool.fork, s);
  const int used = p.batch < kChainStreams ? p.batch : kChainStreams;
  for (int i = 0; i < used && e == cudaSuccess; ++i) e = cudaStreamWaitEvent(pool.st[i], pool.fork, 0);
  if (e != cudaSuccess) return e;
  for (int b = 0; b < p.batch; ++b) {
    FasaParams q = p;
    q.b_off = b;
    cudaStream_t st = pool.st[b % kChainStreams];
    score(q, 1, p.kv_len[b], st);
    finish(q, 1, st);
  }
  for (int i = 0; i < used && e == cudaSuccess; ++i) {
    e = cudaEventRecord(pool.join[i], pool.st[i]);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, pool.join[i], 0);
  }
  if (e != cudaSuccess) return e;
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
  p.cand = reinterpret_cast<uint32_t*>(ws + Lw.cand);
  p.cand_score = reinterpret_cast<float*>(ws + Lw.cand_score);
  p.seg_cnt = reinterpret_cast<unsigned int*>(ws + Lw.seg_cnt);
  p.hist = reinterpret_cast<unsigned int*>(ws + Lw.hist);
  p.thr = reinterpret_cast<uint32_t*>(ws + Lw.thr);
  p.sel = selected ? selected : reinterpret_cast<int*>(ws + Lw.sel);
  p.err = device_error_word();
  if (!p.err) return report_error(ATF_ERR_CUDA, "fasa: no CUDA device / device error word unavailable");
  p.partials = reinterpret_cast<float*>(ws + Lw.partials);
  p.sel_score = reinterpret_cast<float*>(ws + Lw.sel_score);
  p.sel_has_score = reinterpret_cast<int*>(ws + Lw.sel_has_score);
  p.batch = batch;
  p.hq = heads;
  p.hkv = kv_heads;
  p.d = d;
  p.budget = budget;
  p.n_split = (budget + kAttendKeys - 1) / kAttendKeys;
  p.n_cache = n_cache;
  p.n_seg = (n_cache + kSegKeys - 1) / kSegKeys;
  p.seg_cap = p.n_seg * kSegKeys;
  p.mask = pair_mask;
  p.chunk_mask = 0u;
  for (int c = 0; c < d / 16; ++c)
    if ((pair_mask >> (8 * c)) & 0xFFull) p.chunk_mask |= 1u << c;
  for (int b = 0; b < batch; ++b) p.kv_len[b] = kv_len[b];
  cudaError_t e = cudaMemsetAsync(p.hist, 0, Lw.thr - Lw.hist, s);  // the sample histograms
  if (e == cudaSuccess) e = d == 128 ? launch_fasa<128>(p, max_len, s) : launch_fasa<64>(p, max_len, s);
  if (e != cudaSuccess) return report_error(ATF_ERR_CUDA, "fasa: launch: %s", cudaGetErrorString(e));
  return ATF_OK;
}
