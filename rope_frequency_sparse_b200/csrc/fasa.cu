// fasa.cu -- FASA-style decode on the rotated, pair-chunk-major key cache:
// Token Importance Predictor (TIP) scores from dominant frequency pairs, top-k
// selection, then Focused Attention Computation (FAC) over the selected tokens.
// Page "FASA", section "Das FASA-Framework arbeitet in zwei Hauptphasen"; the
// dominant frequency chunks of section "Funktionale Sparsitaet auf
// Frequenz-Chunk-Ebene" are given here as a set of RoPE pairs.
//
// Every TIP score is one fixed fp32 evaluation: from +0, each dim of the
// dominant pairs (ascending) adds its product with one fused multiply-add,
// s <- fl(q_j k_j + s), and -0 counts as +0.  The kept keys are the `budget`
// highest such scores, equal scores by lower index.  Kernels, per call:
//   1. fasa_sample_kernel: one CTA per (32768 keys, kv head, sequence) scores the
//      sampled keys -- the first 32 of every 512 -- for all query heads of the kv
//      head into a 4096-bin histogram per query head (top 12 bits of the score's
//      order-preserving bit pattern: sign, exponent and three mantissa bits).
//   2. fasa_threshold_kernel: per query head, the threshold T is the lower edge
//      of the bin that holds the sample's k-th largest score, k twice the
//      sample's share of the budget plus 8, so that about twice the budget of
//      all keys score at or above T.
//   3. fasa_score_kernel: one CTA per (8192 keys, kv head, sequence); each warp
//      owns a segment of 1024 consecutive keys, four per lane at a time (two
//      packed f32x2 fused multiply-adds: each half rounds as the scalar one
//      does).  It reads only the 8-pair chunks that hold a dominant pair (32
//      bytes per key and chunk, coalesced) and appends the keys scoring at or
//      above T, with their scores, to the segment's list in ascending key order.
//   4. fasa_select_kernel: one CTA per (query head, sequence) gathers the
//      segments' lists in order into shared memory and runs a radix select on the
//      scores' order-preserving bits for the budget-th largest; the keys above it
//      and the lowest-index ones equal to it are emitted in list order, which is
//      ascending.  If fewer than `budget` keys reached T (the sample was not
//      representative), it recomputes every key's score the same way and selects
//      over all of them; a list longer than shared memory is selected in place.
//   5. fasa_attend_kernel: (split of 128 selected keys, query head, sequence);
//      each warp copies its 32 keys' K rows (chunk-major pieces) and V rows into
//      shared memory with asynchronous copies, all in flight at once, computes
//      their 32 dot products together and a softmax over them; partials as in
//      the split decode.
//   6. fasa_combine_kernel: merges the splits (log-sum-exp) into bf16 output.
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

constexpr int kSampleRun = 32;        // sampled keys: the first kSampleRun of every kSamplePeriod
constexpr int kSamplePeriod = 512;
constexpr int kSampleCtaKeys = 32768;  // keys of a sequence per sample CTA (64 runs)
constexpr int kSampleThreads = 512;  // 16 warps, four runs each
constexpr int kThresholdThreads = 256;
constexpr int kHistBits = 12;
constexpr int kHistBins = 1 << kHistBits;
constexpr int kScoreWarps = 8;
constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kSegShift = 10;
constexpr int kSegKeys = 1 << kSegShift;                  // keys per warp segment
constexpr int kScoreCtaKeys = kScoreWarps * kSegKeys;     // keys per score CTA
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
  float* partials;          // [B][Hq][n_split][d + 2]
  int batch, hq, hkv, d, budget, n_split;
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

// One cache chunk of the TIP score for KP packed key pairs: for each dominant
// pair j of chunk c (bits), dims 2j and 2j+1 of the chunk add q_dim * k_dim with
// one fused multiply-add each, both keys of a pair in one f32x2 instruction
// (each half rounds as the scalar fused multiply-add does).  kv[2e] and kv[2e+1]
// hold the chunk's 32 bytes of the keys of pair e; sqf[g * qs + 2j] and
// sqf[g * qs + 2j + 1] hold q of head g at dims 16c + 2j and 16c + 2j + 1 (the
// query is read from shared memory as 8-byte broadcasts).
__device__ __forceinline__ uint32_t chunk_word(const uint4 (&kv)[2], int j) {
  return j == 0 ? kv[0].x : j == 1 ? kv[0].y : j == 2 ? kv[0].z : j == 3 ? kv[0].w
       : j == 4 ? kv[1].x : j == 5 ? kv[1].y : j == 6 ? kv[1].z : kv[1].w;
}
template <int G, int KP>
__device__ __forceinline__ void score_chunk(const uint4 (&kv)[2 * KP][2], uint32_t bits, const float* sqf, int qs,
                                            uint64_t (&s2)[KP][G]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (!((bits >> j) & 1u)) continue;
    uint64_t k0[KP], k1[KP];  // dim 2j and dim 2j+1 of the key pairs
#pragma unroll
    for (int e = 0; e < KP; ++e) {
      const uint32_t w0 = chunk_word(kv[2 * e], j), w1 = chunk_word(kv[2 * e + 1], j);
      k0[e] = pack2(bf16lo_to_f32(w0), bf16lo_to_f32(w1));
      k1[e] = pack2(bf16hi_to_f32(w0), bf16hi_to_f32(w1));
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float2 q2 = *reinterpret_cast<const float2*>(sqf + g * qs + 2 * j);
      const uint64_t qa = pack2(q2.x, q2.x), qb = pack2(q2.y, q2.y);
#pragma unroll
      for (int e = 0; e < KP; ++e) {
        s2[e][g] = ffma2(qa, k0[e], s2[e][g]);
        s2[e][g] = ffma2(qb, k1[e], s2[e][g]);
      }
    }
  }
}

// Loads the 32 bytes of chunk c of key n (zeros for n >= L).
__device__ __forceinline__ void load_key_chunk(uint4 (&kv)[2], const uint4* kbase, long long n_cache, int c,
                                               long long n, long long L) {
  if (n < L) {
    const uint4* row = kbase + (static_cast<long long>(c) * n_cache + n) * 2;
    kv[0] = __ldg(row);
    kv[1] = __ldg(row + 1);
  } else {
    kv[0] = kv[1] = make_uint4(0, 0, 0, 0);
  }
}

// Fills sqf[g][j] = q of query head row0 + g at dim j, as floats.
template <int D, int G>
__device__ __forceinline__ void load_q(float (&sqf)[G][D], const __nv_bfloat16* q, long long row0, int tid,
                                       int nthreads) {
  for (int i = tid; i < G * D; i += nthreads) sqf[i / D][i % D] = __bfloat162float(q[row0 * D + i]);
}

template <int D, int G>
__global__ void __launch_bounds__(kSampleThreads) fasa_sample_kernel(FasaParams p) {
  constexpr int NC = D / 16;
  constexpr int kRuns = kSampleCtaKeys / kSamplePeriod;
  constexpr int kWarps = kSampleThreads / 32;
  static_assert(kRuns == 4 * kWarps, "each warp scores four runs, two at a time");
  const int kvh = blockIdx.y, b = blockIdx.z, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long L = p.kv_len[b];
  const int need = L < p.budget ? static_cast<int>(L) : p.budget;
  const long long n0 = static_cast<long long>(blockIdx.x) * kSampleCtaKeys;
  if (need == L || n0 >= L) return;  // nothing to select, or no key of this CTA
  __shared__ __align__(16) float sqf[G][D];
  __shared__ unsigned int s_lo[G], s_hi[G];  // the range of words any sampled key of this CTA touched
  // per head, kHistBins 16-bit counts packed two to a word (a CTA samples at most
  // 64 runs of 32 keys)
  extern __shared__ unsigned int shist[];
  const long long row0 = static_cast<long long>(b) * p.hq + kvh * G;
  load_q<D, G>(sqf, p.q, row0, tid, kSampleThreads);
  for (int i = tid; i < G * (kHistBins / 2); i += kSampleThreads) shist[i] = 0u;
  if (tid < G) {
    s_lo[tid] = kHistBins / 2;
    s_hi[tid] = 0u;
  }
  __syncthreads();

  const uint4* kbase = reinterpret_cast<const uint4*>(p.kc) +
                       (static_cast<long long>(b) * p.hkv + kvh) * NC * p.n_cache * 2;
  unsigned int lo_w[G], hi_w[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    lo_w[g] = kHistBins / 2;
    hi_w[g] = 0u;
  }
  // warp w scores runs (w, w + kWarps), then (w + 2 kWarps, w + 3 kWarps): one
  // key of each run per lane, the two as a packed pair
#pragma unroll 1
  for (int h = 0; h < 2; ++h) {
    const long long na = n0 + static_cast<long long>(warp + 2 * kWarps * h) * kSamplePeriod + lane;
    const long long nb = na + static_cast<long long>(kWarps) * kSamplePeriod;
    if (na - lane >= L) break;  // warp-uniform
    uint64_t s2[1][G];
#pragma unroll
    for (int g = 0; g < G; ++g) s2[0][g] = 0ull;
#pragma unroll 1
    for (int c = 0; c < NC; ++c) {
      const uint32_t bits = static_cast<uint32_t>((p.mask >> (8 * c)) & 0xFFu);
      if (!bits) continue;
      uint4 kv[2][2];
      load_key_chunk(kv[0], kbase, p.n_cache, c, na, L);
      load_key_chunk(kv[1], kbase, p.n_cache, c, nb, L);
      score_chunk<G, 1>(kv, bits, &sqf[0][16 * c], D, s2);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float sc[2];
      unpack2(s2[0][g], sc[0], sc[1]);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if ((e ? nb : na) < L) {
          const uint32_t bin = order_key(__fadd_rn(sc[e], 0.f)) >> (32 - kHistBits);
          atomicAdd(&shist[g * (kHistBins / 2) + (bin >> 1)], 1u << (16 * (bin & 1u)));
          lo_w[g] = min(lo_w[g], bin >> 1);
          hi_w[g] = max(hi_w[g], bin >> 1);
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const unsigned int lo = __reduce_min_sync(0xffffffffu, lo_w[g]), hi = __reduce_max_sync(0xffffffffu, hi_w[g]);
    if (lane == 0 && lo <= hi) {
      atomicMin(&s_lo[g], lo);
      atomicMax(&s_hi[g], hi);
    }
  }
  __syncthreads();
  // add the touched words' counts to the global histograms
#pragma unroll 1
  for (int g = 0; g < G; ++g) {
    const unsigned int lo = s_lo[g], hi = s_hi[g];
    unsigned int* hg = p.hist + (row0 + g) * kHistBins;
    for (unsigned int i = lo + tid; i <= hi; i += kSampleThreads) {
      const unsigned int w = shist[g * (kHistBins / 2) + i];
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
__global__ void __launch_bounds__(kScoreThreads, 3) fasa_score_kernel(FasaParams p) {  // 3 CTAs per SM
  constexpr int NC = D / 16;
  constexpr int KP = 2;                 // packed key pairs per lane
  constexpr int KU = 2 * KP;            // keys per lane per step
  constexpr int kStepKeys = 32 * KU;    // keys per warp step
  static_assert(kSegKeys % kStepKeys == 0, "a segment is a whole number of steps");
  const int kvh = blockIdx.y, b = blockIdx.z, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long L = p.kv_len[b];
  const int need = L < p.budget ? static_cast<int>(L) : p.budget;
  const bool select = need < L;
  if ((!select && !p.scores) || static_cast<long long>(blockIdx.x) * kScoreCtaKeys >= L) return;
  __shared__ __align__(16) float sqf[G][D];
  const long long row0 = static_cast<long long>(b) * p.hq + kvh * G;
  load_q<D, G>(sqf, p.q, row0, tid, kScoreThreads);
  __shared__ float s_tf[G];            // the thresholds as floats
  __shared__ unsigned int s_cnt[kScoreWarps][G];
  if (tid < G) s_tf[tid] = select ? key_float(p.thr[row0 + tid]) : 0.f;
  if (tid < kScoreWarps * G) s_cnt[tid / G][tid % G] = 0u;
  __syncthreads();
  const long long wseg = static_cast<long long>(blockIdx.x) * kScoreWarps + warp;
  const long long base = wseg * kSegKeys;
  if (base >= L) return;
  const int n_steps = static_cast<int>(min(static_cast<long long>(kSegKeys / kStepKeys),
                                           (L - base + kStepKeys - 1) / kStepKeys));
  const uint4* kbase = reinterpret_cast<const uint4*>(p.kc) +
                       (static_cast<long long>(b) * p.hkv + kvh) * NC * p.n_cache * 2;
  const uint32_t cm = p.chunk_mask;
  const int c_first = __ffs(cm) - 1;
  auto next_chunk = [cm](int c) { return __ffs(cm & ~((2u << c) - 1u)) - 1; };

  // KU keys per lane per step: key u is base + kStepKeys * it + 32 u + lane;
  // keys (2e, 2e+1) are scored as packed pair e
  auto load = [&](uint4 (&buf)[KU][2], int it, int c) {
    const long long n0 = base + kStepKeys * it + lane;
#pragma unroll
    for (int u = 0; u < KU; ++u) load_key_chunk(buf[u], kbase, p.n_cache, c, n0 + 32 * u, L);
  };
  uint64_t s2[KP][G];
#pragma unroll
  for (int e = 0; e < KP; ++e)
#pragma unroll
    for (int g = 0; g < G; ++g) s2[e][g] = 0ull;  // (+0, +0)
  auto compute = [&](const uint4 (&buf)[KU][2], int c) {
    score_chunk<G, KP>(buf, static_cast<uint32_t>((p.mask >> (8 * c)) & 0xFFu), &sqf[0][16 * c], D, s2);
  };
  const unsigned int lt = (1u << lane) - 1u;
  auto finish_step = [&](int it) {
    float sc[G][KU];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < KP; ++e) {
        unpack2(s2[e][g], sc[g][2 * e], sc[g][2 * e + 1]);
        s2[e][g] = 0ull;
      }
    const long long n0 = base + kStepKeys * it + lane;
    bool vu[KU];
#pragma unroll
    for (int u = 0; u < KU; ++u) vu[u] = n0 + 32 * u < L;
    if (p.scores) {
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int u = 0; u < KU; ++u)
          if (vu[u]) p.scores[(row0 + g) * p.n_cache + n0 + 32 * u] = __fadd_rn(sc[g][u], 0.f);
    }
    if (!select) return;
    // !(s < T) holds for s >= T; T is never -0, and a -0 score counts as +0
    bool any = false;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float t = s_tf[g];
#pragma unroll
      for (int u = 0; u < KU; ++u) any |= vu[u] && !(sc[g][u] < t);
    }
    if (!__any_sync(0xffffffffu, any)) return;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float t = s_tf[g];
      unsigned int cnt = s_cnt[warp][g];
      const long long seg = (row0 + g) * p.seg_cap + base;
#pragma unroll
      for (int u = 0; u < KU; ++u) {  // ascending key order within the segment
        const bool c = vu[u] && !(sc[g][u] < t);
        const unsigned int bal = __ballot_sync(0xffffffffu, c);
        if (c) {
          const unsigned int pos = cnt + static_cast<unsigned int>(__popc(bal & lt));
          p.cand[seg + pos] = static_cast<uint32_t>(n0 + 32 * u);
          p.cand_score[seg + pos] = __fadd_rn(sc[g][u], 0.f);
        }
        cnt += static_cast<unsigned int>(__popc(bal));
      }
      __syncwarp();
      if (lane == 0) s_cnt[warp][g] = cnt;
      __syncwarp();
    }
  };

  // four keys per lane per step, one chunk at a time; three CTAs per SM keep
  // enough warps in flight to cover the loads (a second register stage for the
  // next chunk's loads costs more in occupancy than it hides)
  uint4 buf[KU][2];
  for (int it = 0; it < n_steps; ++it) {
    for (int c = c_first; c >= 0; c = next_chunk(c)) {
      load(buf, it, c);
      compute(buf, c);
    }
    finish_step(it);
  }
  if (select && lane < G) {
    unsigned int v = 0;
#pragma unroll
    for (int g = 0; g < G; ++g)
      if (lane == g) v = s_cnt[warp][g];
    p.seg_cnt[(row0 + lane) * p.n_seg + wseg] = v;
  }
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

// The candidates of one (query head, sequence) in ascending key order, held in
// shared memory: order keys and key indices.
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
};

// Writes to out[0 .. need) the indices of the `need` largest entries of `list`
// (by order key, equal keys by position, the list being in ascending key
// order), in list order, and -1 to out[need .. budget).  The list holds at
// least `need` entries.
template <class List>
__device__ void select_emit(const List& list, int need, int budget, int* out, const SelectScratch& sc) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0u, pmask = 0u;
  int left = need;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < kBins; i += kSelectThreads) sc.hist[i] = 0u;
    if (tid == 0) {
      *sc.digit = 0;
      *sc.gt = 0;
    }
    __syncthreads();
    for (long long i = tid; i < list.n; i += kSelectThreads) {
      uint32_t k, x;
      if (list.get(i, k, x) && (k & pmask) == prefix) atomicAdd(&sc.hist[(k >> shift) & (kBins - 1)], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // the digit d: the largest with #(digits >= d) >= left; lane l holds the
      // digits 8l .. 8l+7, suffix sums across the lanes
      int c8 = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) c8 += static_cast<int>(sc.hist[8 * lane + u]);
      int suf = c8;  // digits >= 8 lane
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, suf, off);
        if (lane + off < 32) suf += y;
      }
      const int above = suf - c8;  // digits >= 8 lane + 8
      if (above < left && left <= suf) {
        int run = above;
        for (int u = 8 * lane + 7; u >= 8 * lane; --u) {
          const int cu = static_cast<int>(sc.hist[u]);
          if (run + cu >= left) {
            *sc.digit = u;
            *sc.gt = run;
            break;
          }
          run += cu;
        }
      }
    }
    __syncthreads();
    left -= *sc.gt;
    prefix |= static_cast<uint32_t>(*sc.digit) << shift;
    pmask |= static_cast<uint32_t>(kBins - 1) << shift;
    __syncthreads();  // digit and gt are rewritten by the next pass
  }
  // prefix is the need-th largest key; all keys above it are kept, and the first
  // `left` equal to it in list order.  Thread t emits the contiguous block
  // [t * per, (t + 1) * per) of the list.
  const long long per = (list.n + kSelectThreads - 1) / kSelectThreads;
  const long long lo = tid * per, hi = min(list.n, lo + per);
  int eq = 0;
  for (long long i = lo; i < hi; ++i) {
    uint32_t k, x;
    if (list.get(i, k, x) && k == prefix) ++eq;
  }
  const int eq_before = block_scan(eq, sc.warp, sc.total);
  int keep = 0, e = eq_before;
  for (long long i = lo; i < hi; ++i) {
    uint32_t k, x;
    if (!list.get(i, k, x)) continue;
    if (k > prefix) {
      ++keep;
    } else if (k == prefix) {
      keep += e < left;
      ++e;
    }
  }
  int pos = block_scan(keep, sc.warp, sc.total);
  e = eq_before;
  for (long long i = lo; i < hi; ++i) {
    uint32_t k, x;
    if (!list.get(i, k, x)) continue;
    if (k > prefix || (k == prefix && e++ < left)) {
      if (pos < need) out[pos] = static_cast<int>(x);
      ++pos;
    }
  }
  for (int i = need + tid; i < budget; i += kSelectThreads) out[i] = -1;
}

__global__ void __launch_bounds__(kSelectThreads) fasa_select_kernel(FasaParams p) {
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const long long row = static_cast<long long>(b) * p.hq + h;
  const long long L = p.kv_len[b];
  const int need = L < p.budget ? static_cast<int>(L) : p.budget;
  int* out = p.sel + row * p.budget;
  if (need == L) {  // every key is selected, already in order
    for (int i = tid; i < p.budget; i += kSelectThreads) out[i] = i < L ? i : -1;
    return;
  }
  extern __shared__ uint32_t s_list[];  // order keys [kSelectCap], then key indices [kSelectCap]
  __shared__ unsigned int s_hist[kBins];
  __shared__ int s_warp[32];
  __shared__ int s_total, s_digit, s_gt;
  __shared__ float s_q[128];
  const SelectScratch scr{s_hist, s_warp, &s_total, &s_digit, &s_gt};
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
    int carry = 0;
    for (long long w0 = 0; w0 < nseg; w0 += kSelectThreads) {
      const long long w = w0 + tid;
      const int cw = w < nseg ? static_cast<int>(cnt[w]) : 0;
      const int off = carry + block_scan(cw, s_warp, &s_total);
      for (int j = 0; j < cw; ++j) {
        const uint32_t k = order_key(cscore[w * kSegKeys + j]);
        s_key[off + j] = k;
        s_idx[off + j] = cand[w * kSegKeys + j];
        reached += k >= T;
      }
      carry += s_total;
    }
    block_scan(reached, s_warp, &s_total);
    if (s_total >= need) {
      select_emit(SmemList{s_key, s_idx, m}, need, p.budget, out, scr);
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
      select_emit(list, need, p.budget, out, scr);
      return;
    }
  }
  // fewer than `need` keys reached T: every key's score, in the same arithmetic,
  // into the (now unused) candidate arrays, slot n = key n, then select over all
  const int D = p.d, NC = D / 16;
  for (int i = tid; i < D; i += kSelectThreads) s_q[i] = __bfloat162float(p.q[row * D + i]);
  __syncthreads();
  const uint4* kbase = reinterpret_cast<const uint4*>(p.kc) +
                       (static_cast<long long>(b) * p.hkv + h / (p.hq / p.hkv)) * NC * p.n_cache * 2;
  for (long long n = tid; n < L; n += kSelectThreads) {
    float s = 0.f;
    for (int c = 0; c < NC; ++c) {
      const uint32_t bits = static_cast<uint32_t>((p.mask >> (8 * c)) & 0xFFu);
      if (!bits) continue;
      const uint4* r = kbase + (static_cast<long long>(c) * p.n_cache + n) * 2;
      const uint4 lo = __ldg(r), hi = __ldg(r + 1);
      const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (!((bits >> j) & 1u)) continue;
        s = __fmaf_rn(s_q[16 * c + 2 * j], bf16lo_to_f32(w[j]), s);
        s = __fmaf_rn(s_q[16 * c + 2 * j + 1], bf16hi_to_f32(w[j]), s);
      }
    }
    cscore[n] = __fadd_rn(s, 0.f);
    cand[n] = static_cast<uint32_t>(n);
  }
  __syncthreads();
  select_emit(SegmentList{cand, cscore, cnt, L, true}, need, p.budget, out, scr);
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
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
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
  const __nv_bfloat16* kb = p.kc + (static_cast<long long>(b) * p.hkv + kvh) * NC * p.n_cache * 16;
  const __nv_bfloat16* vb = p.v + static_cast<long long>(b) * p.n_cache * p.hkv * D + kvh * D;
  // piece i of the warp's copy: key i / (2 kGran), then its K pieces, then its V pieces
  for (int i = lane; i < 32 * 2 * kGran; i += 32) {
    const int key = i / (2 * kGran), gi = i % (2 * kGran);
    const int n = __shfl_sync(0xffffffffu, n_mine, key);  // warp-uniform loop: every lane shuffles
    const bool kok = __shfl_sync(0xffffffffu, static_cast<int>(ok), key) != 0;
    if (!kok) continue;
    if (gi < kGran) {  // K: chunk gi / 2, half gi % 2
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
  for (int e = 0; e < DPL; ++e) q[e] = __bfloat162float(p.q[row * D + DPL * lane + e]) * scale;
  // partial dot products of all 32 keys over this lane's dims
  float dp[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    float acc = 0.f;
    if (k < nk) {
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
  const float sdot = live ? dp[0] : -INFINITY;
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
  size_t cand, cand_score, seg_cnt, hist, thr, sel, partials, total;
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
  L.partials = off;
  off += align256(rows * n_split * (d + 2) * sizeof(float));
  L.total = off;
  return L;
}

template <int D, int G>
void launch_select_path(const FasaParams& p, long long max_len, cudaStream_t s) {
  const size_t hist_smem = static_cast<size_t>(G) * (kHistBins / 2) * sizeof(unsigned int);
  fasa_sample_kernel<D, G><<<dim3(static_cast<unsigned>((max_len + kSampleCtaKeys - 1) / kSampleCtaKeys), p.hkv,
                                  p.batch),
                             kSampleThreads, hist_smem, s>>>(p);
  fasa_threshold_kernel<<<dim3(p.hq, p.batch), kThresholdThreads, 0, s>>>(p);
  fasa_score_kernel<D, G><<<dim3(static_cast<unsigned>((max_len + kScoreCtaKeys - 1) / kScoreCtaKeys), p.hkv,
                                 p.batch),
                            kScoreThreads, 0, s>>>(p);
}

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
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fasa_select_kernel),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSelectSmem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fasa_attend_kernel<D>),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kAttendSmem));
    if (e != cudaSuccess) return e;
    if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_acq_rel);
  }
  switch (G) {
    case 1: launch_select_path<D, 1>(p, max_len, s); break;
    case 2: launch_select_path<D, 2>(p, max_len, s); break;
    case 3: launch_select_path<D, 3>(p, max_len, s); break;
    case 4: launch_select_path<D, 4>(p, max_len, s); break;
    case 5: launch_select_path<D, 5>(p, max_len, s); break;
    case 6: launch_select_path<D, 6>(p, max_len, s); break;
    case 7: launch_select_path<D, 7>(p, max_len, s); break;
    default: launch_select_path<D, 8>(p, max_len, s); break;
  }
  fasa_select_kernel<<<dim3(p.hq, p.batch), kSelectThreads, kSelectSmem, s>>>(p);
  fasa_attend_kernel<D><<<dim3(p.n_split, p.hq, p.batch), kAttendWarps * 32, kAttendSmem, s>>>(p);
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
  p.cand = reinterpret_cast<uint32_t*>(ws + Lw.cand);
  p.cand_score = reinterpret_cast<float*>(ws + Lw.cand_score);
  p.seg_cnt = reinterpret_cast<unsigned int*>(ws + Lw.seg_cnt);
  p.hist = reinterpret_cast<unsigned int*>(ws + Lw.hist);
  p.thr = reinterpret_cast<uint32_t*>(ws + Lw.thr);
  p.sel = selected ? selected : reinterpret_cast<int*>(ws + Lw.sel);
  p.partials = reinterpret_cast<float*>(ws + Lw.partials);
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
