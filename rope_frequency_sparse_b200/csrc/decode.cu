// decode.cu -- one new query per sequence against a long, already rotated key
// cache, reading only the key pairs that are still inside their window.
//
// "ATFlash: RoPE-Frequenzen kuerzen Attention-Arbeit um bis zu 57 Prozent"
// (sudo-ai.de), section "Was ATFlash anders macht": beyond a pair's window the
// pair's query-key product is left out, while the slow pairs keep far keys
// reachable; section "Die Zahlen - und ihre Grenze": the decode side of the
// method lives in the decode attention kernel, with the online softmax left as
// it is.
//
// Because the windows grow with the pair index, a key at distance Delta needs
// only the pairs i >= i*(Delta).  The key cache is stored pair-chunk-major
// ([b][kv head][chunk of 8 pairs][token][16 elements]), so for a far key only
// the few high chunks are read from HBM: the saving is in bytes, not only in
// multiply-adds.  All value rows are read (a key whose pairs are all outside
// their windows still has logit 0 and weight in the softmax).
//
// Work split: each (sequence, kv head) key range is cut into n_split pieces of
// equal HBM traffic (value bytes plus active key-chunk bytes), one CTA each, in
// a single wave over the SMs; a CTA serves all query heads of its kv head (GQA).
// Inside a CTA one warp streams tiles of 128 keys into a shared-memory ring with
// TMA: the value tile and only the key chunks that some key of the tile still
// needs.  Four warps take 32 keys of each tile apiece and run the contractions on
// the tensor cores with warp-level bf16 MMAs, the G query heads as the M rows:
//   S = Q~ K~^T  over the tile's active chunks.  Each key is a column of the B
//                operand, so a lane zeroes its B registers for the pairs whose
//                window misses its key: the per-pair windows are exact.
//   O += P V     with P taken straight from the S accumulators.
// Each warp keeps the split-softmax state of its keys (running max in log2 units,
// sum, unnormalised output); the CTA merges its warps into one partial, and a
// second kernel merges the partials.
#include <cuda_bf16.h>

#include <atomic>

#include "atf_internal.cuh"
#include "ptx.cuh"

namespace atf {

namespace {

constexpr int kDecConsumers = 4;                       // warps, 32 keys of each tile apiece
constexpr int kDecThreads = (kDecConsumers + 1) * 32;  // plus the TMA producer warp
constexpr int BKD = 128;                               // keys per tile
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct DecCfg {
  static constexpr int NC = D / 16;                       // chunks of 8 pairs
  static constexpr int NP = D / 2;                        // pairs
  static constexpr int NSTG = D == 128 ? 3 : 5;           // ring stages
  static constexpr int BOXES = D / 64;                    // 64-dim boxes of a value tile
  static constexpr int V_BYTES = BKD * D * 2;             // value tile (128B-swizzled boxes)
  static constexpr int KC_BYTES = BKD * 32;               // key chunk tile (32-byte rows, 32B swizzle)
  static constexpr int STAGE_BYTES = V_BYTES + NC * KC_BYTES;
  static constexpr int Q_BYTES = 16 * D * 2;              // rotated queries, 16 rows (heads, zero padded)
};

struct DecShared {
  uint64_t full[5], empty[5];
  int abort;
  int w[kMaxPairs];
  float mw[kDecConsumers][8];  // per warp and query head: running max (log2 units)
  float lw[kDecConsumers][8];  // and row sum
};

template <int D>
constexpr int dec_smem_bytes() {
  return DecCfg<D>::Q_BYTES + DecCfg<D>::NSTG * DecCfg<D>::STAGE_BYTES + static_cast<int>(sizeof(DecShared)) + 1024;
}

// Traffic of keys with distance in [0, x), in units of 32 bytes: each key reads
// its value row (nc units) plus one unit per chunk whose highest pair window
// still reaches it (chunk c is active while Delta <= W_{8c+7}).
__device__ long long traffic_below(long long x, const int* sW, int nc) {
  long long t = static_cast<long long>(nc) * x;
  for (int c = 0; c < nc; ++c) {
    const long long wc = static_cast<long long>(sW[8 * c + 7]) + 1;
    t += x < wc ? x : wc;
  }
  return t;
}

// First key index of split s (of ns) over keys [0, L) whose key 0 lies at
// distance q1 - 1 from the query (q1 = L for a whole sequence, the query at L-1).
// Keys [0, n) have distances [q1 - n, q1), hence traffic T(q1) - T(q1 - n).
__device__ long long split_begin(int s, int ns, long long L, long long q1, const int* sW, int nc) {
  if (s <= 0) return 0;
  if (s >= ns) return L;
  const long long top = traffic_below(q1, sW, nc);
  const long long total = top - traffic_below(q1 - L, sW, nc);
  // the smallest n with traffic of keys [0, n) >= s*total/ns
  const long long target = (total / ns) * s + ((total % ns) * s) / ns;
  long long lo = 0, hi = L;
  while (lo < hi) {
    const long long mid = (lo + hi) / 2;
    if (top - traffic_below(q1 - mid, sW, nc) >= target)
      hi = mid;
    else
      lo = mid + 1;
  }
  return lo & ~static_cast<long long>(BKD - 1);  // whole tiles
}

// Chunks entirely outside every window for the keys of a tile whose smallest
// distance is dmin: chunk c is dead when even its highest pair W_{8c+7} < dmin.
__device__ __forceinline__ int dead_chunks(const int* sW, int nc, long long dmin) {
  int c = 0;
  while (c < nc && static_cast<long long>(sW[8 * c + 7]) < dmin) ++c;
  return c;
}

// Byte offset of element `dim` of row `row` in a 16-row tile stored as 64-dim
// boxes with the 128-byte swizzle.
template <int ROWS>
__device__ __forceinline__ uint32_t sw128_offset(int row, int dim) {
  return (dim >> 6) * (ROWS * 128) + row * 128 + ((((dim & 63) >> 3) ^ (row & 7)) << 4) + (dim & 7) * 2;
}

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_k,
                     const DecodeParams p) {
  using C = DecCfg<D>;
  constexpr int NC = C::NC, NP = C::NP, NSTG = C::NSTG;
  static_assert(G >= 1 && G <= 8, "query heads per kv head");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sStage = smem + C::Q_BYTES;  // [NSTG][STAGE_BYTES]
  DecShared* sh = reinterpret_cast<DecShared*>(sStage + NSTG * C::STAGE_BYTES);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const long long L = p.kv_len[b];
  const long long qpos = p.q_pos[b];              // RoPE angle of the query
  const long long qloc = qpos - p.key_pos0[b];    // the query's distance from slot 0

  if (tid == 0) {
    for (int s = 0; s < NSTG; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], kDecConsumers);
    }
    sh->abort = 0;
    fence_mbar_init();
  }
  if (tid == kDecConsumers * 32) prefetch_tmap(&tm_v), prefetch_tmap(&tm_k);
  for (int i = tid; i < kMaxPairs; i += kDecThreads) sh->w[i] = p.win.w[i];
  // Rotate the G raw queries of this kv head at position qpos (fp64 angle) into
  // bf16 rows of the MMA A operand; rows G..15 stay zero.
  {
    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(p.q);
    for (int idx = tid; idx < 16 * NP; idx += kDecThreads) {
      const int g = idx / NP, i = idx % NP;
      float r0 = 0.f, r1 = 0.f;
      if (g < G) {
        // dims of pair i: (2i, 2i+1), or (i, i + d/2) for rotate-half queries; the
        // rotated pair goes to slots (2i, 2i+1), the cache's order
        const long long row = (static_cast<long long>(b) * p.hq + hk * G + g) * D;
        const long long ea = row + (p.pairing ? i : 2 * i), eb = ea + (p.pairing ? D / 2 : 1);
        const double x0 = __bfloat162float(Q[ea]), x1 = __bfloat162float(Q[eb]);
        double sn, cs;
        sincos(static_cast<double>(qpos) * p.omega[i], &sn, &cs);
        r0 = static_cast<float>(x0 * cs - x1 * sn);
        r1 = static_cast<float>(x0 * sn + x1 * cs);
      }
      *reinterpret_cast<uint32_t*>(sQ + sw128_offset<16>(g, 2 * i)) = pack_bf16x2(r0, r1);
    }
  }
  __syncthreads();

  const long long nb = split_begin(split, p.n_split, L, qloc + 1, sh->w, NC);
  const long long ne = split_begin(split + 1, p.n_split, L, qloc + 1, sh->w, NC);
  const int ntiles = ne > nb ? static_cast<int>((ne - nb + BKD - 1) / BKD) : 0;
  volatile int* abort = &sh->abort;
  auto tile_dead_chunks = [&](int t) {
    const long long last = min(nb + static_cast<long long>(t) * BKD + BKD - 1, ne - 1);
    return dead_chunks(sh->w, NC, qloc - last);
  };

  // per-warp softmax state (consumers): row hrow = lane / 4 of the accumulators
  const int hrow = lane >> 2;
  float mrun = -INFINITY, lsum = 0.f;
  float o[D / 8][4];
#pragma unroll
  for (int u = 0; u < D / 8; ++u) o[u][0] = o[u][1] = o[u][2] = o[u][3] = 0.f;
  unsigned long long cnt = 0;

  if (warp == kDecConsumers) {
    // ================================================================ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int t = 0; t < ntiles; ++t) {
        const int st = t % NSTG;
        if (t >= NSTG && !mbar_wait(&sh->empty[st], ((t / NSTG) - 1) & 1, abort, p.err, 0x401)) break;
        const int n0 = static_cast<int>(nb + static_cast<long long>(t) * BKD);
        const int clo = tile_dead_chunks(t);
        uint8_t* stg = sStage + st * C::STAGE_BYTES;
        mbar_arrive_expect_tx(&sh->full[st], C::V_BYTES + (NC - clo) * C::KC_BYTES);
#pragma unroll
        for (int bx = 0; bx < C::BOXES; ++bx)
          tma_load_4d(stg + bx * (BKD * 128), &tm_v, &sh->full[st], bx * 64, hk, n0, b);
        for (int c = clo; c < NC; ++c)
          tma_load_5d(stg + C::V_BYTES + c * C::KC_BYTES, &tm_k, &sh->full[st], 0, n0, c, hk, b);
        issued = t + 1;
      }
      if (*abort) {
        for (int t = 0; t < issued; ++t) {
          const long long t0 = clock64();
          while (!mbar_try_wait(&sh->full[t % NSTG], (t / NSTG) & 1) && clock64() - t0 < kWaitLimitCycles) {
          }
        }
      }
    }
  } else {
    // ================================================================ consumers
    const int w = warp;
    // windows of the two pairs this lane's B registers hold in each chunk
    int wlo[NC], whi[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      wlo[c] = sh->w[8 * c + (lane & 3)];
      whi[c] = sh->w[8 * c + 4 + (lane & 3)];
    }
    // Q~ A fragments of every chunk (16 rows x 16 dims)
    uint32_t qa[NC][4];
    {
      const int mi = lane >> 3;
      const int row = (lane & 7) + 8 * (mi & 1);
#pragma unroll
      for (int c = 0; c < NC; ++c) ldsm_x4(smem_u32(sQ + sw128_offset<16>(row, 16 * c + 8 * (mi >> 1))), qa[c]);
    }
    const float scale = kLog2e * rsqrtf(static_cast<float>(D));
    for (int t = 0; t < ntiles; ++t) {
      const int st = t % NSTG;
      if (!warp_wait(&sh->full[st], (t / NSTG) & 1, abort, p.err, 0x402)) break;
      const long long n0 = nb + static_cast<long long>(t) * BKD;
      const int clo = tile_dead_chunks(t);
      const uint32_t stg = smem_u32(sStage + st * C::STAGE_BYTES);
      // distance of this lane's B column key in each of the warp's four 8-key n-tiles
      long long dl[4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) dl[nt] = qloc - (n0 + 32 * w + 8 * nt + (lane >> 2));

      // ---- S = Q~ K~^T over the live chunks, B registers zeroed for pairs outside their window
      float sfr[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) sfr[nt][0] = sfr[nt][1] = sfr[nt][2] = sfr[nt][3] = 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        if (c < clo) continue;  // dead for every key of the tile
        const uint32_t kc = stg + C::V_BYTES + c * C::KC_BYTES;
#pragma unroll
        for (int np2 = 0; np2 < 2; ++np2) {
          // matrix lane/8: n-tile 2*np2 + lane/16, 16-byte half (lane/8) & 1 of the key rows
          const int key = 32 * w + 8 * (2 * np2 + (lane >> 4)) + (lane & 7);
          const int half = (lane >> 3) & 1;
          uint32_t bfr[4];
          ldsm_x4(kc + key * 32 + ((half ^ ((key >> 2) & 1)) << 4), bfr);
          const long long d0 = dl[2 * np2], d1 = dl[2 * np2 + 1];
          if (d0 > wlo[c]) bfr[0] = 0u;
          if (d0 > whi[c]) bfr[1] = 0u;
          if (d1 > wlo[c]) bfr[2] = 0u;
          if (d1 > whi[c]) bfr[3] = 0u;
          mma_bf16_16816(sfr[2 * np2], qa[c], bfr[0], bfr[1]);
          mma_bf16_16816(sfr[2 * np2 + 1], qa[c], bfr[2], bfr[3]);
        }
      }
      // ---- online softmax for query head hrow over this warp's 32 keys
      float x[8];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const long long key = n0 + 32 * w + 8 * nt + 2 * (lane & 3) + e;
          x[2 * nt + e] = key < ne ? sfr[nt][e] * scale : -INFINITY;
        }
      float mx = fmaxf(fmax3(x[0], x[1], x[2]), fmaxf(fmax3(x[3], x[4], x[5]), fmax3(x[6], x[7], x[7])));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      if (mx > mrun) {
        const float corr = ex2_approx(mrun - mx);  // 0 while mrun is -inf
        lsum *= corr;
#pragma unroll
        for (int u = 0; u < D / 8; ++u) {
          o[u][0] *= corr;
          o[u][1] *= corr;
        }
        mrun = mx;
      }
      float pr[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        pr[k] = ex2_approx(x[k] - mrun);
        lsum += pr[k];
      }
      // P as A fragments of two 16-key steps (rows 8..15 are padding and stay zero)
      uint32_t pa[2][4];
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) {
        pa[kt][0] = pack_bf16x2(pr[4 * kt], pr[4 * kt + 1]);
        pa[kt][1] = 0u;
        pa[kt][2] = pack_bf16x2(pr[4 * kt + 2], pr[4 * kt + 3]);
        pa[kt][3] = 0u;
      }
      // ---- O += P V
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) {
        const int mi = lane >> 3;
        const int key = 32 * w + 16 * kt + (lane & 7) + 8 * (mi & 1);
#pragma unroll
        for (int u = 0; u < D / 16; ++u) {
          const int dim = 16 * u + 8 * (mi >> 1);
          uint32_t vb[4];
          ldsm_x4_t(stg + (dim >> 6) * (BKD * 128) + key * 128 + ((((dim & 63) >> 3) ^ (key & 7)) << 4), vb);
          mma_bf16_16816(o[2 * u], pa[kt], vb[0], vb[1]);
          mma_bf16_16816(o[2 * u + 1], pa[kt], vb[2], vb[3]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->empty[st]);
      if (p.skipped) {  // pairs outside their window, over this warp's valid keys, times the G heads
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
          int dead = 0;
#pragma unroll
          for (int c = 0; c < NC; ++c) dead += (dl[nt] > wlo[c]) + (dl[nt] > whi[c]);
          dead += __shfl_xor_sync(0xffffffffu, dead, 1);
          dead += __shfl_xor_sync(0xffffffffu, dead, 2);
          if ((lane & 3) == 0 && qloc - dl[nt] < ne) cnt += static_cast<unsigned long long>(dead) * G;
        }
      }
    }
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
  }

  // ---- merge the consumer warps into this split's partial
  __syncthreads();  // every tile consumed: the ring is free for the merge
  float* sO = reinterpret_cast<float*>(sStage);  // [warp][head][D]
  if (warp < kDecConsumers) {
    if ((lane & 3) == 0) {
      sh->mw[warp][hrow] = mrun;
      sh->lw[warp][hrow] = lsum;
    }
#pragma unroll
    for (int u = 0; u < D / 8; ++u) {
      const int dim = 8 * u + 2 * (lane & 3);
      sO[(warp * 8 + hrow) * D + dim] = o[u][0];
      sO[(warp * 8 + hrow) * D + dim + 1] = o[u][1];
    }
  }
  __syncthreads();
  if (!*abort) {
    float* part = p.partials + ((static_cast<long long>(b) * p.hq + hk * G) * p.n_split + split) * (D + 2);
    for (int idx = tid; idx < G * D; idx += kDecThreads) {
      const int g = idx / D, e = idx % D;
      float M = -INFINITY;
      for (int w = 0; w < kDecConsumers; ++w) M = fmaxf(M, sh->mw[w][g]);
      float a = 0.f, l = 0.f;
      if (M != -INFINITY) {
        for (int w = 0; w < kDecConsumers; ++w) {
          if (sh->mw[w][g] == -INFINITY) continue;
          const float f = ex2_approx(sh->mw[w][g] - M);
          a += sO[(w * 8 + g) * D + e] * f;
          l += sh->lw[w][g] * f;
        }
      }
      float* pg = part + static_cast<long long>(g) * p.n_split * (D + 2);
      pg[e] = a;
      if (e == 0) {
        pg[D] = M;
        pg[D + 1] = l;
      }
    }
  }
  if (p.skipped && warp < kDecConsumers) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if (lane == 0 && cnt) atomicAdd(p.skipped, cnt);
  }
}

// Merge the n_split partials of every (sequence, query head) into the output.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(DecodeParams p) {
  const int h = blockIdx.x, b = blockIdx.y, e = threadIdx.x;
  const float* part = p.partials + ((static_cast<long long>(b) * p.hq + h) * p.n_split) * (D + 2);
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
  if (p.partial_out) {  // this key range's merged partial, for a merge with other ranges
    float* pp = p.partial_out + (static_cast<long long>(b) * p.hq + h) * (D + 2);
    pp[e] = a;
    if (e == 0) {
      pp[D] = M;
      pp[D + 1] = l;
    }
    return;
  }
  __nv_bfloat16* O = static_cast<__nv_bfloat16*>(p.out) + (static_cast<long long>(b) * p.hq + h) * D;
  O[e] = __float2bfloat16(l > 0.f ? a / l : 0.f);
}

// Merge n_parts partials [n_parts][rows][D + 2] (sum relative to the max, max in
// log2 units, row sum) into the bf16 output [rows][D].
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const float* parts, int n_parts, long long rows,
                                                         __nv_bfloat16* out) {
  const long long row = blockIdx.x;
  const int e = threadIdx.x;
  float M = -INFINITY;
  for (int r = 0; r < n_parts; ++r) M = fmaxf(M, parts[(r * rows + row) * (D + 2) + D]);
  float a = 0.f, l = 0.f;
  for (int r = 0; r < n_parts; ++r) {
    const float* pr = parts + (r * rows + row) * (D + 2);
    if (pr[D] == -INFINITY) continue;
    const float f = ex2_approx(pr[D] - M);
    a += pr[e] * f;
    l += pr[D + 1] * f;
  }
  out[row * D + e] = __float2bfloat16(l > 0.f ? a / l : 0.f);
}

int decode_num_splits(long long max_kv_len, int batch, int hkv) {
  const int units = batch * hkv;
  if (units <= 0 || max_kv_len <= 0) return 1;
  // one wave of one CTA per SM over the 148 SMs, at least 2048 keys per split
  long long ns = 148LL / units;
  const long long cap = (max_kv_len + 2047) / 2048;
  if (ns > cap) ns = cap;
  if (ns < 1) ns = 1;
  return static_cast<int>(ns);
}

template <int D, int G>
static cudaError_t launch_dec(const DecodeParams& p, const CUtensorMap& tv, const CUtensorMap& tk,
                              cudaStream_t s) {
  auto kern = decode_tc_kernel<D, G>;
  constexpr int bytes = dec_smem_bytes<D>();
  static_assert(bytes <= 227 * 1024, "shared memory budget");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // one bit per device; setting the attribute twice (two threads racing on the
  // first call) is harmless, the atomic keeps the bit updates themselves defined
  static std::atomic<unsigned long long> configured{0};
  if (dev >= 64 || !(configured.load(std::memory_order_acquire) & (1ull << dev))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_acq_rel);
  }
  kern<<<dim3(p.n_split, p.hkv, p.batch), kDecThreads, bytes, s>>>(tv, tk, p);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_decode_d(const DecodeParams& p, const CUtensorMap& tv, const CUtensorMap& tk,
                                   cudaStream_t s) {
  cudaError_t e;
  switch (p.hq / p.hkv) {
    case 1: e = launch_dec<D, 1>(p, tv, tk, s); break;
    case 2: e = launch_dec<D, 2>(p, tv, tk, s); break;
    case 3: e = launch_dec<D, 3>(p, tv, tk, s); break;
    case 4: e = launch_dec<D, 4>(p, tv, tk, s); break;
    case 5: e = launch_dec<D, 5>(p, tv, tk, s); break;
    case 6: e = launch_dec<D, 6>(p, tv, tk, s); break;
    case 7: e = launch_dec<D, 7>(p, tv, tk, s); break;
    case 8: e = launch_dec<D, 8>(p, tv, tk, s); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  decode_combine_kernel<D><<<dim3(p.hq, p.batch), D, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode_merge(const float* parts, int n_parts, long long rows, int d, void* out, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  auto* o = static_cast<__nv_bfloat16*>(out);
  if (d == 64)
    decode_merge_kernel<64><<<static_cast<unsigned>(rows), 64, 0, s>>>(parts, n_parts, rows, o);
  else
    decode_merge_kernel<128><<<static_cast<unsigned>(rows), 128, 0, s>>>(parts, n_parts, rows, o);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tv, const CUtensorMap& tk, cudaStream_t s) {
  if (p.batch == 0) return cudaSuccess;
  return p.d == 64 ? launch_decode_d<64>(p, tv, tk, s) : launch_decode_d<128>(p, tv, tk, s);
}

}  // namespace atf
