// prefill_tc.cu -- causal GQA prefill with one distance window per RoPE
// frequency pair, on the sm_100a tensor cores (tcgen05 MMA, TMEM, TMA).
//
// Method: "ATFlash: RoPE-Frequenzen kuerzen Attention-Arbeit um bis zu 57
// Prozent" (sudo-ai.de).  Section "Was ATFlash anders macht": each frequency
// pair i has a window W_i proportional to its wavelength; for Delta = m - n
// beyond W_i the pair's query-key product is skipped, while slower pairs keep
// the key reachable.  Section "Die Zahlen - und ihre Grenze": the online-softmax
// recurrence is kept as it is.  Logit: s = (1/sqrt d) sum_{i: Delta <= W_i}
// (q~_{2i} k~_{2i} + q~_{2i+1} k~_{2i+1}); no active pair gives s = 0.
//
// Design.  One CTA = two Q tiles of 128 query rows (one query head), sharing
// every K and V tile; 12 warps in three warpgroups:
//   warp 0      TMA producer: both Q~ tiles once, then K and V tiles of 128 keys
//               (128B-swizzled boxes of 64 dims) into separate rings.
//   warp 1      TMEM owner and MMA issuer: the warp runs its loop convergently
//               and one elected lane issues the MMAs and commits; per KV tile j
//               and Q tile g:
//                 S_g(j)  = Q~_g . K~(j)^T      A = Q~_g (smem), B = K tile (smem)
//                 O_g    += P_g(j) . V(j)       A = P_g in TMEM, B = V tile (MN-major)
//   warps 2-3   idle (they complete warpgroup 0 for the register reallocation)
//   warps 4-7   softmax of Q tile 0, warps 8-11 softmax of Q tile 1: one full
//               query row per thread (TMEM lane = row), running max, row sum.
// Warpgroup 0 gives registers to the two softmax warpgroups (setmaxnreg), so a
// thread holds its whole 128-column row of S at once.
// TMEM columns: S_g at [128 g, 128 g + 128) (P_g written back over it as packed
// bf16, in two pieces of 64 keys), O_g at [256 + g d, 256 + (g + 1) d).
// Issue order: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1), ... so one Q tile's
// exponentials overlap the other tile's MMAs.
//
// Window structure.  W is non-decreasing in i (wavelengths grow), so the active
// pairs of any element form a suffix {i >= i*(Delta)}.  KV tiles are visited
// from the diagonal towards key 0, so a Q tile's centre distance c = m0 - n0
// grows monotonically.  Each warp (32 rows) zeroes, in its rows of the Q tile's
// shared-memory copy, the pairs whose windows end before about the median
// distance its rows see on the tile, once and for all, and whole 8-pair chunks
// zeroed in every row are not issued to the MMA (the contraction depth shrinks
// tile by tile).  Elements of a tile that straddles a window boundary are fixed on
// the CUDA cores before the softmax reads S: a zeroed pair whose window still
// covers the element is added back, an issued pair whose window does not is
// subtracted; only straddling pairs, and only 32-column chunks a warp's rows
// reach, are touched.  The window counts come from the W table held across each
// warp's lanes (ballots), with no per-tile table.
// The softmax loop has two bodies.  The correcting body runs only on the tiles
// where a window boundary crosses the warp's elements or where pairs die at the
// next tile; between those, runs of clean tiles (every pair dead or live for
// all of the warp's elements) go through a body that is the dense kernel's loop
// plus one counter update, with none of the correction code in it.
//
// Exponentials.  The SFU evaluates 16 ex2 per clock per SM, as many as the
// tensor core needs cycles for a 128x128 tile's two MMAs.  A share of the column
// pairs can evaluate 2^x on the FMA pipe instead (x = j + f with j = round(x) and
// f in [-1/2, 1/2], 2^f by a cubic, j added to the exponent field); the share is a
// compile-time mask, off by default (see ATF_EXP_FMA_MASK).
#include <cuda_bf16.h>

#include <atomic>
#include <type_traits>

#include "atf_internal.cuh"
#include "ptx.cuh"

namespace atf {

namespace {

constexpr int BM = 128;        // query rows per Q tile (MMA M, TMEM lanes)
constexpr int NQ = 2;          // Q tiles per CTA
constexpr int BN = 128;        // keys per KV tile (four 32-column chunks)
static_assert(BN == 128, "the correction code selects among four 32-column chunks");
constexpr int kThreads = 384;  // 12 warps = 3 warpgroups
constexpr int kRegsLaunch = 168;   // registers per thread at launch (checked by the launcher)
constexpr int kRegsCtl = 64;       // warpgroup 0 after reallocation
constexpr int kRegsSoftmax = 216;  // softmax warpgroups after reallocation
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split exceeds the launch");
constexpr uint32_t kTmemCols = 512;
constexpr int kStash = 12;        // zeroed query pairs kept per row (more are re-read from global memory)

// 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on [-1/2, 1/2]: coefficients chosen for the
// smallest maximum relative error (7.5e-5, Lawson's iteratively reweighted least
// squares in float64, then rounded to float; exp2_poly_fit.py beside the package).
constexpr float kExpC0 = 0.9999280571937561f;
constexpr float kExpC1 = 0.6932609677314758f;
constexpr float kExpC2 = 0.24261093139648438f;
constexpr float kExpC3 = 0.05517149344086647f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23: x + magic rounds x to an integer

template <int D>
struct Cfg {
  static constexpr int NSK = D == 128 ? 2 : 4;   // K ring stages
  static constexpr int NSV = D == 128 ? 2 : 4;   // V ring stages
  static constexpr int BOXES = D / 64;           // 64-dim swizzle boxes per tile
  static constexpr int TILE_BYTES = BN * D * 2;  // one Q, K or V tile
  static constexpr int NCH = D / 16;             // 8-pair chunks = MMA K-steps
  static constexpr int NP = D / 2;
  static constexpr uint32_t COL_S = 0, COL_O = 256;
  static constexpr int SMEM_TILES = (NQ + NSK + NSV) * TILE_BYTES;
};

struct Shared {
  uint64_t q_full[NQ], q_ready[NQ], s_full[NQ], p_bar[NQ][2], o_done[NQ];
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int w[kMaxPairs];
  // Per Q tile, the query pairs most recently zeroed in its shared-memory copy
  // ([slot][row], slot = pair - first zeroed pair), read back by add-back corrections.
  uint32_t stash[NQ][kStash][BM];
};

template <int D>
constexpr int smem_bytes() {
  return Cfg<D>::SMEM_TILES + static_cast<int>(sizeof(Shared)) + 1024;
}

// The rows of one warp (a 32-row quarter q of the Q tile) see, on a KV tile with
// centre distance `center` (= m0 - n0), the distances Delta = center + 32q + [-127, 31].
// Their pair ranges:
//   a: pairs below a lie outside every element's window (W_i < center + 32q - 127)
//   z: pairs zeroed in these rows of Q~ (W_i < center + 32q + kZeroOffset)
//   u: pairs from u on lie inside every element's window (W_i >= center + 32q + 31)
// Pairs in [a, z) are added back where Delta <= W_i, pairs in [z, u) subtracted
// where Delta > W_i.  kZeroOffset sits near the median distance of a full tile, which
// keeps both kinds of correction small, and must be <= 1 so that the pairs added
// back on a tile were zeroed at the step just before it (a(j+1) >= z(j)).
constexpr int kZeroOffset = -48;
// A warp's clean tile (every pair dead for all of its elements or live for all of
// them, nothing zeroed after it) holds no window W_i >= lo within [lo, lo + kCleanSpan),
// lo = center + 32q - 127 its smallest distance: the span covers the tile's own
// distances (lo .. lo + BN + 30) and reaches the next tile's zero point
// (lo + 2 BN - 1 + kZeroOffset), so no pair dies during a run of clean tiles and
// the zeroed pairs after the run are still those before it.
constexpr int kCleanSpan = 2 * BN - 1 + kZeroOffset;
static_assert(kZeroOffset <= 1 && kCleanSpan >= BN + 31,
              "zero point between the tile's element distances and the next tile's add-back range");

// The window table held across a warp: lane l keeps W_l and W_{l+32} (a pair
// index past the head's pairs holds a sentinel that is never below a threshold).
struct WarpWindows {
  long long w0, w1;
  __device__ __forceinline__ WarpWindows(const int* w, int np, int lane) {
    w0 = lane < np ? w[lane] : 0x7fffffffffffffffLL;
    w1 = lane + 32 < np ? w[lane + 32] : 0x7fffffffffffffffLL;
  }
  // number of pairs with W_i < x (W is non-decreasing); warp-collective
  __device__ __forceinline__ int below(long long x) const {
    return __popc(__ballot_sync(0xffffffffu, w0 < x)) + __popc(__ballot_sync(0xffffffffu, w1 < x));
  }
  // W_i (i warp-uniform, i < 64); warp-collective
  __device__ __forceinline__ long long at(int i) const {
    return __shfl_sync(0xffffffffu, i < 32 ? w0 : w1, i & 31);
  }
  __device__ __forceinline__ uint32_t quarter_ranges(long long center, int q) const {
    const long long lo = center + 32 * q;
    const uint32_t z = below(lo + kZeroOffset);
    const uint32_t a = below(lo - (BN - 1));
    const uint32_t u = below(lo + 31);
    return z | (a << 8) | (u << 16);
  }
};

// The 32 key words of one pair (columns c_lo .. c_lo+31) in a 128-byte-swizzled
// K tile: column cc at kb[cc % 8] + 128 cc.
template <int CC>
__device__ __forceinline__ void load_key_words(uint32_t (&kw)[32], const uint32_t (&kb)[8]) {
  if constexpr (CC < 32) {
    kw[CC] = lds32_at<CC * 128>(kb[CC & 7]);
    load_key_words<CC + 1>(kw, kb);
  }
}

// Adds (q_2i k_2i + q_2i+1 k_2i+1)(cc), q signed, to the columns cc of the chunk
// whose bit of `mask` is set.
template <int CC>
__device__ __forceinline__ void correct_columns(float (&x)[32], const uint32_t (&kw)[32], uint32_t mask,
                                                uint32_t qs) {
  if constexpr (CC < 32) {
    x[CC] = fma_bf16x2_f32_if<CC>(mask, qs, kw[CC], x[CC]);
    correct_columns<CC + 1>(x, kw, mask, qs);
  }
}

// Byte offset of pair i (4 bytes) of row r inside a 128-row tile stored as
// 64-dim boxes with the 128-byte swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t pair_offset(int r, int i) {
  return (i >> 5) * (BN * 128) + r * 128 + ((((i & 31) >> 2) ^ (r & 7)) << 4) + (i & 3) * 4;
}

// Zero the query pairs [lo, hi) of row r in a Q~ tile (swizzled layout above),
// keeping the old values of pairs lo .. lo+kStash-1 in stash[pair - lo][r].
// Works on whole 16-byte chunks (4 pairs) of the row.
__device__ __forceinline__ void zero_pairs(uint8_t* tile, uint32_t (*stash)[BM], int r, int lo, int hi) {
#pragma unroll 1
  for (int c4 = lo >> 2; c4 < (hi + 3) >> 2; ++c4) {
    uint4* p4 = reinterpret_cast<uint4*>(tile + pair_offset(r, 4 * c4));
    uint4 q = *p4;
    uint32_t* e = reinterpret_cast<uint32_t*>(&q);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = 4 * c4 + k;
      if (i >= lo && i < hi) {
        if (i - lo < kStash) stash[i - lo][r] = e[k];
        e[k] = 0u;
      }
    }
    *p4 = q;
  }
}

// Bounded wait that ignores the abort flag (used only while draining).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t0 < kWaitLimitCycles) {
  }
}

// 2^x for a pair of floats on the FMA pipe.  x <= 9 here; x is clamped at -126
// so that the scaled result keeps a valid exponent (2^-126 stands in for 0).
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  float x0, x1;
  unpack2(x2, x0, x1);
  const uint64_t xc = pack2(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t t = fadd2(xc, pack2(kRoundMagic, kRoundMagic));  // low mantissa bits = round(x)
  const uint64_t f = ffma2(fadd2(t, pack2(-kRoundMagic, -kRoundMagic)), pack2(-1.f, -1.f), xc);
  uint64_t q = ffma2(pack2(kExpC3, kExpC3), f, pack2(kExpC2, kExpC2));
  q = ffma2(q, f, pack2(kExpC1, kExpC1));
  q = ffma2(q, f, pack2(kExpC0, kExpC0));
  float q0, q1, t0, t1;
  unpack2(q, q0, q1);
  unpack2(t, t0, t1);
  // (bits(t) << 23) == round(x) << 23 modulo 2^32: the magic's own bits shift out
  return pack2(__uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23)),
               __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23)));
}

// column pairs k (columns 2k, 2k+1) whose exponentials use the FMA pipe: bit k % 8.
// Off by default: measured on B200, this kernel is bound by its softmax -> MMA
// dependency chain with the SFU about half busy, and every share moved to the FMA
// pipe made both the dense and the windowed kernel slower (3/8: +7 %, 1/2: +13 %).
#ifndef ATF_EXP_FMA_MASK
#define ATF_EXP_FMA_MASK 0x00
#endif
__host__ __device__ constexpr bool exp_on_fma(int k) { return (ATF_EXP_FMA_MASK >> (k & 7)) & 1; }

// P goes to the MMA warp in two pieces of 64 keys (the P.V of the first runs while
// the softmax computes the second).
constexpr int kPPieces = 2;

}  // namespace

template <int D, bool SPARSE>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using C = Cfg<D>;
  constexpr int NSK = C::NSK, NSV = C::NSV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                      // [NQ][TILE_BYTES]
  uint8_t* sK = sQ + NQ * C::TILE_BYTES;   // [NSK][TILE_BYTES]
  uint8_t* sV = sK + NSK * C::TILE_BYTES;  // [NSV][TILE_BYTES]
  Shared* sh = reinterpret_cast<Shared*>(smem + C::SMEM_TILES);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- coordinates: Q tiles 2 pr and 2 pr + 1 of one (batch, head); heaviest CTAs first
  const int nqt = (p.q_len + BM - 1) / BM;
  const int npr = (nqt + NQ - 1) / NQ;
  int idx = blockIdx.x;
  const int h = idx % p.hq;
  idx /= p.hq;
  const int b = idx % p.batch;
  const int pr = npr - 1 - idx / p.batch;
  const int hk = h / (p.hq / p.hkv);
  const int t0 = pr * NQ * BM;             // first query row of the CTA
  const long long m0 = p.q_offset + t0;    // its position
  const int rows1 = max(0, min(BM, p.q_len - t0 - BM));
  const int nq = rows1 > 0 ? 2 : 1;        // Q tiles with rows
  const long long kv_last = static_cast<long long>(p.kv_len) - 1;
  const long long maxkey0 = min(m0 + min(BM, p.q_len - t0) - 1, kv_last);
  const long long maxkey = nq == 2 ? min(m0 + BM + rows1 - 1, kv_last) : maxkey0;
  const int T = static_cast<int>(maxkey / BN) + 1;              // KV tiles, visited j = 0..T-1
  const int jstart0 = T - 1 - static_cast<int>(maxkey0 / BN);  // Q tile 0 starts one tile later or not
  auto jstart = [&](int g) { return g == 0 ? jstart0 : 0; };
  auto tile_n0 = [&](int j) { return static_cast<long long>(T - 1 - j) * BN; };
  // Q tile g on KV tile j has centre m0 + 128 g - n0(j) = m0 - n0(j + g): entry j + g.
  auto centre = [&](int e) { return m0 - static_cast<long long>(T - 1 - e) * BN; };


  // ---- setup
  if (tid == 0) {
    for (int g = 0; g < NQ; ++g) {
      mbar_init(&sh->q_full[g], 1);
      mbar_init(&sh->q_ready[g], 128);
      mbar_init(&sh->s_full[g], 1);
      for (int pc = 0; pc < 2; ++pc) mbar_init(&sh->p_bar[g][pc], 128);
      mbar_init(&sh->o_done[g], 1);
    }
    for (int s = 0; s < NSK; ++s) {
      mbar_init(&sh->k_full[s], 1);
      mbar_init(&sh->k_empty[s], 8);  // every softmax warp, once per KV tile
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(&sh->v_full[s], 1);
      mbar_init(&sh->v_empty[s], 1);
    }
    mbar_init(&sh->drain, 1);
    sh->abort = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < kMaxPairs; i += kThreads) sh->w[i] = p.win.w[i];
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  __syncthreads();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  volatile int* abort = &sh->abort;

  if (warp < 4) {
    setmaxnreg_dec<kRegsCtl>();
    if (warp == 0 && lane == 0) {
      // ============================================================== TMA producer
      for (int g = 0; g < nq; ++g) {
        mbar_arrive_expect_tx(&sh->q_full[g], C::TILE_BYTES);
#pragma unroll
        for (int bx = 0; bx < C::BOXES; ++bx)
          tma_load_4d(sQ + g * C::TILE_BYTES + bx * (BN * 128), &tm_q, &sh->q_full[g], bx * 64, h, t0 + g * BM, b);
      }
      int k_issued = 0, v_issued = 0;
      // Only the active chunk columns of K are loaded: the first 64-dim box (pairs
      // 0-31) is skipped for a tile where pair 31's window, the widest of them, is
      // below every query-key distance of every Q tile that reads the tile (Q tile g
      // at KV tile j spans centre(j + g) +- (BN - 1)).  Then no MMA issues those
      // chunks (its depth starts past every pair with W_i < centre - 48) and no
      // boundary correction reads them (none of them straddles).
      const long long w_box0 = SPARSE && C::BOXES > 1 ? static_cast<long long>(sh->w[31]) : 0x7fffffffffffffffLL;
      for (int j = 0; j < T; ++j) {
        const int n0 = static_cast<int>(tile_n0(j));
        {
          const int s = j % NSK, use = j / NSK;
          if (j >= NSK && !mbar_wait(&sh->k_empty[s], (use - 1) & 1, abort, p.err, 0x101)) break;
          long long dmin = 0x7fffffffffffffffLL;
          for (int g = 0; g < nq; ++g)
            if (j >= jstart(g)) dmin = min(dmin, centre(j + g) - (BN - 1));
          const int bx0 = w_box0 < dmin ? 1 : 0;
          mbar_arrive_expect_tx(&sh->k_full[s], C::TILE_BYTES / C::BOXES * (C::BOXES - bx0));
#pragma unroll
          for (int bx = 0; bx < C::BOXES; ++bx)
            if (bx >= bx0)
              tma_load_4d(sK + s * C::TILE_BYTES + bx * (BN * 128), &tm_k, &sh->k_full[s], bx * 64, hk, n0, b);
          k_issued = j + 1;
        }
        {
          const int s = j % NSV, use = j / NSV;
          if (j >= NSV && !mbar_wait(&sh->v_empty[s], (use - 1) & 1, abort, p.err, 0x102)) break;
          mbar_arrive_expect_tx(&sh->v_full[s], C::TILE_BYTES);
#pragma unroll
          for (int bx = 0; bx < C::BOXES; ++bx)
            tma_load_4d(sV + s * C::TILE_BYTES + bx * (BN * 128), &tm_v, &sh->v_full[s], bx * 64, hk, n0, b);
          v_issued = j + 1;
        }
      }
      if (*abort) {
        // let every load already issued land before the CTA leaves
        for (int g = 0; g < nq; ++g) drain_wait(&sh->q_full[g], 0);
        for (int j = 0; j < k_issued; ++j) drain_wait(&sh->k_full[j % NSK], (j / NSK) & 1);
        for (int j = 0; j < v_issued; ++j) drain_wait(&sh->v_full[j % NSV], (j / NSV) & 1);
      }
    } else if (warp == 1) {
      // ============================================================== MMA issuer
      // The whole warp runs the loop (warp-uniform descriptors and waits); one
      // elected lane, always the same one, issues the MMAs and their commits.
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, false, true);
      constexpr uint64_t kTileStep = C::TILE_BYTES >> 4;  // descriptor address units
      const uint64_t dq0 = smem_desc(smem_u32(sQ), smem_desc_bits(16, 1024, kLayoutSW128));
      const uint64_t dk0 = smem_desc(smem_u32(sK), smem_desc_bits(16, 1024, kLayoutSW128));
      const uint64_t dv0 = smem_desc(smem_u32(sV), smem_desc_bits(BN * 128, 1024, kLayoutSW128));
      const WarpWindows ww(sh->w, C::NP, lane);
      bool ok = true;
      for (int g = 0; ok && g < nq; ++g) ok = warp_wait(&sh->q_ready[g], 0, abort, p.err, 0x201);
      tc_fence_after();
      int k_seen = 0;  // K tiles whose arrival this warp has observed
      // S_g(j) = Q~_g . K(j)^T over the active 8-pair chunks
      auto issue_s = [&](int g, int j) -> bool {
        const int s = j % NSK;
        if (j >= k_seen) {
          if (!warp_wait(&sh->k_full[s], (j / NSK) & 1, abort, p.err, 0x202)) return false;
          k_seen = j + 1;
          tc_fence_after();
        }
        // pairs zeroed in every row of Q~_g (those of its first quarter): chunks below are skipped
        const int c0 = SPARSE ? ww.below(centre(j + g) + kZeroOffset) >> 3 : 0;
        const uint32_t d_tmem = tmem + C::COL_S + g * BN;
        const uint64_t aq = dq0 + g * kTileStep, bk = dk0 + s * kTileStep;
        if (elect_one()) {
#pragma unroll
          for (int c = 0; c < C::NCH; ++c) {
            const uint64_t off = static_cast<uint64_t>((c >> 2) * (BN * 128) + (c & 3) * 32) >> 4;
            if (SPARSE)
              mma_ss_if(d_tmem, aq + off, bk + off, idesc_qk, c > c0 ? 1u : 0u, c >= c0 ? 1u : 0u);
            else
              mma_ss(d_tmem, aq + off, bk + off, idesc_qk, c > 0 ? 1u : 0u);
          }
          mma_commit(&sh->s_full[g]);
        }
        __syncwarp();
        return true;
      };
      for (int g = 0; ok && g < nq; ++g)
        if (jstart(g) == 0) ok = issue_s(g, 0);
      for (int j = 0; ok && j < T; ++j) {
        const int sv = j % NSV;
        bool v_seen = false;
        for (int g = 0; g < nq; ++g) {
          if (j >= jstart(g)) {
            if (!v_seen) {
              if (!(ok = warp_wait(&sh->v_full[sv], (j / NSV) & 1, abort, p.err, 0x205))) break;
              v_seen = true;
            }
            const uint32_t p_tmem = tmem + C::COL_S + g * BN;  // P_g(j), packed bf16 over S_g(j)
            const uint32_t o_tmem = tmem + C::COL_O + g * D;
            const uint64_t bv = dv0 + sv * kTileStep;
            const bool first = j == jstart(g);
            // P arrives in kPPieces pieces of BN / kPPieces keys: the P.V of a piece
            // runs while the softmax still computes the later ones
            constexpr int KK = BN / 16 / kPPieces;  // K-steps (16 keys) per piece
#pragma unroll
            for (int pc = 0; pc < kPPieces; ++pc) {
              if (!(ok = warp_wait(&sh->p_bar[g][pc], (j - jstart(g)) & 1, abort, p.err, 0x210 + pc))) break;
              tc_fence_after();
              if (elect_one()) {
#pragma unroll
                for (int kk = KK * pc; kk < KK * pc + KK; ++kk)
                  mma_ts(o_tmem, p_tmem + 8 * kk, bv + ((kk * 2048) >> 4), idesc_pv, (!first || kk > 0) ? 1u : 0u);
                if (pc == kPPieces - 1 && j == T - 1) mma_commit(&sh->o_done[g]);
              }
              __syncwarp();
            }
            if (!ok) break;
          }
          // S_g(j+1) overwrites P_g(j); PV_g(j) was issued first and tcgen05.mma
          // operations of one thread execute in issue order.
          if (j + 1 < T && j + 1 >= jstart(g) && !(ok = issue_s(g, j + 1))) break;
        }
        if (!ok) break;
        if (elect_one()) mma_commit(&sh->v_empty[sv]);
        __syncwarp();
      }
      if (!ok) {
        if (elect_one()) mma_commit(&sh->drain);
        __syncwarp();
        drain_wait(&sh->drain, 0);
      }
    }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ================================================================ softmax (warps 4..11)
    const int g = (warp - 4) >> 2;      // Q tile
    const int quarter = warp & 3;       // TMEM lanes 32*quarter.. of this warp
    const int r = quarter * 32 + lane;  // query row in the tile == TMEM lane
    const WarpWindows ww(sh->w, C::NP, lane);
    if (g >= nq) {
      // no rows in this Q tile: only keep the K ring's release count
      for (int j = 0; j < T; ++j) {
        if (!warp_wait(&sh->k_full[j % NSK], (j / NSK) & 1, abort, p.err, 0x300)) break;
        if (lane == 0) mbar_arrive(&sh->k_empty[j % NSK]);
      }
    } else {
      uint8_t* sQg = sQ + g * C::TILE_BYTES;
      const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t s_tmem = tmem + lane_off + C::COL_S + g * BN;
      const int t = t0 + g * BM + r;
      const bool row_ok = t < p.q_len;
      const long long m = m0 + g * BM + r;
      const long long q_elem = ((static_cast<long long>(b) * p.q_len + (row_ok ? t : 0)) * p.hq + h) * D;
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(p.q) + q_elem);
      constexpr float kLog2e = 1.4426950408889634f;
      const float scale = kLog2e * rsqrtf(static_cast<float>(D));
      const int j0 = jstart(g);

      bool ok = warp_wait(&sh->q_full[g], 0, abort, p.err, 0x301);
      if (ok) {
        if (SPARSE) {  // pairs dead in this Q tile's first KV tile
          const int z0 = static_cast<int>(ww.quarter_ranges(centre(j0 + g), quarter) & 0xFF);
          zero_pairs(sQg, sh->stash[g], r, 0, z0);
          fence_proxy_async_smem();
        }
        mbar_arrive(&sh->q_ready[g]);
      }
      for (int j = 0; ok && j < j0; ++j) {  // KV tiles entirely after this Q tile's rows
        if ((ok = warp_wait(&sh->k_full[j % NSK], (j / NSK) & 1, abort, p.err, 0x302)) && lane == 0)
          mbar_arrive(&sh->k_empty[j % NSK]);
      }

      float mrun = -INFINITY;
      uint64_t lsum2 = 0ull;  // packed partial row sums
      unsigned long long cnt = 0;
      int zst = 0;  // first pair held in this warp's rows of the stash

      // The softmax of one KV tile j.  CORR = true: the correcting body, for tiles
      // on which a window boundary crosses this warp's rows (straddling pairs are
      // added back or subtracted on S) or after which pairs die (zeroed in Q~);
      // CORR = false: the clean body, on which every pair is dead for all of this
      // warp's elements (the first a_run pairs) or live for all of them -- the
      // dense kernel's loop plus one counter update.
      auto tile = [&](const int j, auto corr_tag, const int a_run) -> bool {
        constexpr bool CORR = decltype(corr_tag)::value;
        const int s = j % NSK;
        const long long n0 = tile_n0(j);
        const long long center = m0 + g * BM - n0;
        // valid columns of this row form the prefix [0, cmax]
        int cmax = -1;
        if (row_ok) cmax = static_cast<int>(min(static_cast<long long>(BN - 1), min(m, kv_last) - n0));
        const bool partial = __any_sync(0xffffffffu, cmax < BN - 1);
        const int nv = cmax + 1;  // valid columns of this row
        if constexpr (SPARSE && !CORR) cnt += static_cast<unsigned long long>(a_run) * nv;
        // (everything up to the wait is independent of S, off the softmax -> MMA chain)
        uint32_t qr = 0u, qr_next = 0u;
        int z = 0, a = 0, u = 0, cmax_w = 0, cw = 0, wl0 = 0;
        bool has_mma = true;
        uint32_t tb0[BN / 32] = {}, fb0[BN / 32] = {};
        // Classification of pairs hb .. hb+31 (lane l: pair hb + l) for this warp's
        // rows: per 32-column chunk, the pairs some row must correct (tb) and those
        // every row corrects entirely (fb).  Chunks past every row's last valid column
        // (beyond the causal diagonal or the last key, cmax_w) are masked out whole:
        // nothing there needs correcting.  For pairs in [a, u) the windows lie within
        // 127 of the centre, so the thresholds fit in 32 bits.
        auto classify = [&](int hb, int& wl, uint32_t (&tb)[BN / 32], uint32_t (&fb)[BN / 32]) {
          const int il = hb + lane;
          const bool valid = il < u;
          wl = valid ? sh->w[il] : 0;
          const int twl = cw - wl;  // smallest threshold among the warp's rows
          const bool addl = il < z;
#pragma unroll
          for (int qc = 0; qc < BN / 32; ++qc) {
            const int c_lo = 32 * qc;
            tb[qc] = __ballot_sync(0xffffffffu,
                                   valid && c_lo <= cmax_w && (addl ? (c_lo + 31 >= twl) : (c_lo < twl + 31)));
            fb[qc] = __ballot_sync(0xffffffffu, valid && (addl ? (c_lo >= twl + 31) : (c_lo + 31 < twl)));
          }
        };
        if constexpr (CORR) {
          qr = ww.quarter_ranges(center, quarter);
          z = static_cast<int>(qr & 0xFF);
          a = static_cast<int>((qr >> 8) & 0xFF);
          u = static_cast<int>((qr >> 16) & 0xFF);
          // the next tile's zero point, computed while S is still on its way
          qr_next = j + 1 < T ? ww.quarter_ranges(center + BN, quarter) : 0u;
          // no S MMA when every pair is zeroed in every row
          has_mma = (ww.below(center + kZeroOffset) >> 3) < C::NCH;
          cnt += static_cast<unsigned long long>(a) * nv;
          cmax_w = a < u ? __reduce_max_sync(0xffffffffu, cmax) : 0;
          cw = quarter * 32 + static_cast<int>(center);  // threshold offset of row 0 of the warp
          // the first batch is classified before S arrives, off the softmax -> MMA chain
          if (a < u) classify(a, wl0, tb0, fb0);
        }
        if (!warp_wait(&sh->s_full[g], (j - j0) & 1, abort, p.err, 0x303)) return false;
        tc_fence_after();
        if constexpr (CORR) {
          uint32_t s_chunks = has_mma ? 0xFu : 0u;  // 32-column chunks of S held in TMEM
          if (a < u) {
            // ---- boundary corrections, in place on S in TMEM, 32 columns at a time.
            const int cen = static_cast<int>(center);
            const uint32_t kbase = smem_u32(sK + s * C::TILE_BYTES);
            const uint32_t q_base = smem_u32(sQg);
            const uint32_t stash_base = smem_u32(&sh->stash[g][0][r]);
#pragma unroll 1
            for (int hb = a; hb < u; hb += 32) {
              int wl = wl0;
              uint32_t tb[BN / 32], fb[BN / 32];
#pragma unroll
              for (int qc = 0; qc < BN / 32; ++qc) {
                tb[qc] = tb0[qc];
                fb[qc] = fb0[qc];
              }
              if (hb != a) classify(hb, wl, tb, fb);
#pragma unroll 1
              for (int qc = 0; qc < BN / 32; ++qc) {
                const int c_lo = 32 * qc;
                uint32_t tbits = qc == 0 ? tb[0] : qc == 1 ? tb[1] : qc == 2 ? tb[2] : tb[3];
                const uint32_t fbits = qc == 0 ? fb[0] : qc == 1 ? fb[1] : qc == 2 ? fb[2] : fb[3];
                if (!tbits) continue;
                float x[32];
                if ((s_chunks >> qc) & 1u) {
                  tmem_ld32(s_tmem + c_lo, reinterpret_cast<uint32_t*>(x));
                  tmem_ld_wait();
                } else {
#pragma unroll
                  for (int cc = 0; cc < 32; ++cc) x[cc] = 0.f;
                }
                // The key words (k_2i(c), k_2i+1(c)) of the chunk's 32 columns are read
                // straight from the K tile: the address depends only on the column, so
                // every lane issues the same broadcast loads, with no staging and no
                // warp synchronisation.
                // this row's (q_2i, q_2i+1) as a bf16x2 word: from Q~ while the pair is
                // issued, else from the stash of recently zeroed pairs, else from memory
                auto load_qpair = [&](int i) -> uint32_t {
                  uint32_t qv = 0u;
                  if (row_ok) {
                    if (i >= z)
                      qv = lds32(q_base + pair_offset(r, i));
                    else if (static_cast<unsigned>(i - zst) < static_cast<unsigned>(kStash))
                      qv = lds32(stash_base + static_cast<uint32_t>((i - zst) * BM) * 4u);
                    else
                      qv = __ldg(qrow + i);
                  }
                  return qv;
                };
                int k = __ffs(tbits) - 1;
                tbits &= tbits - 1;
                uint32_t qp = load_qpair(hb + k);
#pragma unroll 1
                while (true) {
                  const int i = hb + k;
                  // column cc's key word sits at kb[cc % 8] + 128 cc (the swizzle
                  // permutes the 16-byte chunks of a row by row % 8)
                  const uint32_t kp = kbase + (i >> 5) * (BN * 128) + c_lo * 128 + (i & 3) * 4;
                  const uint32_t ci = static_cast<uint32_t>((i & 31) >> 2);
                  uint32_t kb[8];
#pragma unroll
                  for (int sw = 0; sw < 8; ++sw) kb[sw] = kp + ((ci ^ sw) << 4);
                  uint32_t kw[32];
                  load_key_words<0>(kw, kb);
                  const int wi = __shfl_sync(0xffffffffu, wl, k);
                  const bool more = tbits != 0u;
                  int kn = 0;
                  uint32_t qpn = 0u;
                  if (more) {  // the next item's query pair, in flight during this one
                    kn = __ffs(tbits) - 1;
                    tbits &= tbits - 1;
                    qpn = load_qpair(hb + kn);
                  }
                  const bool add = i < z;  // zeroed pair: add back where cc >= tc; else subtract where cc < tc
                  const uint32_t qs = add ? qp : (qp ^ 0x80008000u);  // both bf16 halves negated to subtract
                  const int tc = r + cen - wi - c_lo;  // chunk columns cc < tc lie outside the window
                  const uint32_t ge = tc <= 0 ? ~0u : (tc >= 32 ? 0u : (~0u << tc));
                  const uint32_t mk = ((fbits >> k) & 1u) ? ~0u : (add ? ge : ~ge);
                  correct_columns<0>(x, kw, mk, qs);
                  if (!more) break;
                  k = kn;
                  qp = qpn;
                }
                tmem_st32(s_tmem + c_lo, reinterpret_cast<uint32_t*>(x));
                s_chunks |= 1u << qc;
              }
              if (p.skipped) {  // skipped pair-MACs of this row among the batch's pairs
                const int nb = min(32, u - hb);
#pragma unroll 1
                for (int k = 0; k < nb; ++k) {
                  const int tl = r + cen - __shfl_sync(0xffffffffu, wl, k);
                  cnt += static_cast<unsigned long long>(tl <= 0 ? 0 : (tl < nv ? tl : nv));
                }
              }
            }
            tmem_st_wait();
          }
          if (s_chunks != 0xFu) {
            // no S MMA on this tile: the chunks no correction wrote hold zero logits
            uint32_t zw[32];
#pragma unroll
            for (int cc = 0; cc < 32; ++cc) zw[cc] = 0u;
#pragma unroll 1
            for (int qc = 0; qc < BN / 32; ++qc)
              if (!((s_chunks >> qc) & 1u)) tmem_st32(s_tmem + 32 * qc, zw);
            tmem_st_wait();
          }
        }
        // ---- the whole row of S in registers
        float v[BN];
#pragma unroll
        for (int c = 0; c < BN; c += 32) tmem_ld32(s_tmem + c, reinterpret_cast<uint32_t*>(v + c));
        tmem_ld_wait();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->k_empty[s]);  // this warp is done with K(j)
        if constexpr (CORR) {
          if (j + 1 < T) {
            // S_g(j) is done reading Q~_g and this tile's corrections are done with
            // the stash: zero (and stash) the pairs that die at the next tile.
            // S_g(j+1) is issued only after this warpgroup's last P arrival below.
            const int zn = static_cast<int>(qr_next & 0xFF);
            if (zn > z) {
              zero_pairs(sQg, sh->stash[g], r, z, zn);
              fence_proxy_async_smem();
            }
            zst = z;
          }
        }

        // ---- mask, max, exponentials
        if (partial) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c > cmax) v[c] = -INFINITY;
        }
        // Row max in eight accumulators: columns 0..7, then 60 steps of two columns.
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = v[e];
        auto max_step = [&](int st) { acc[st & 7] = fmax3(acc[st & 7], v[8 + 2 * st], v[9 + 2 * st]); };
        auto row_max = [&]() {
          return fmaxf(fmax3(acc[0], acc[1], acc[2]), fmax3(acc[3], acc[4], fmax3(acc[5], acc[6], acc[7]))) * scale;
        };
        uint64_t ls[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pw[BN / 2];
        const uint64_t sc2 = pack2(scale, scale);
        uint64_t nm2 = 0ull;  // (-reference, -reference), set once the tile's max is known
        // P of columns 2k, 2k+1 against the current reference
        auto exp_pair = [&](int k) {
          const uint64_t x2 = ffma2(pack2(v[2 * k], v[2 * k + 1]), sc2, nm2);
          float p0, p1;
          if (exp_on_fma(k)) {
            unpack2(exp2_poly2(x2), p0, p1);
          } else {
            float x0, x1;
            unpack2(x2, x0, x1);
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          ls[k & 3] = fadd2(ls[k & 3], pack2(p0, p1));
          pw[k] = pack_bf16x2(p0, p1);
        };
        // Conditional rescale: the reference (mrun) moves only when the row max has
        // grown by more than 2^8; the final 1/l uses the same reference, so this is
        // exact.
        constexpr int KP = BN / 2 / kPPieces;  // column pairs per piece of P
        // a row's reference moves to mnew: O and l are rescaled by 2^(old - new)
        // (0 from a row that had no valid column yet, where O and l are 0)
        auto rescale = [&](float mnew, bool need) {
          const float corr = need ? ex2_approx(mrun - mnew) : 1.f;
          // O_g holds PV_g up to tile j-1, issued before S_g(j); S_g(j)'s commit
          // covers every earlier MMA, so O_g is complete here.
#pragma unroll 1
          for (int k = 0; k < D / 32; ++k) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + C::COL_O + g * D + 32 * k, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
            tmem_st32(tmem + lane_off + C::COL_O + g * D + 32 * k, o);
          }
          if (need) {
            lsum2 = fmul2(lsum2, pack2(corr, corr));
            mrun = mnew;
          }
        };
#pragma unroll
        for (int st = 0; st < 60; ++st) max_step(st);
        const float mnew = fmaxf(mrun, row_max());
        if (j == j0) {
          mrun = mnew;  // no reference yet: it is this tile's max
        } else {
          // a row that had no valid column yet (mrun = -inf) takes its first reference
          const bool need = mrun == -INFINITY ? mnew != -INFINITY : mnew > mrun + 8.f;
          if (__any_sync(0xffffffffu, need)) rescale(mnew, need);
        }
        const float mref = mrun == -INFINITY ? 0.f : mrun;
        nm2 = pack2(-mref, -mref);
#pragma unroll
        for (int k = 0; k < KP; ++k) exp_pair(k);
        // the first piece of P (keys 0..63) goes over while the second is computed
        tmem_st32(s_tmem, pw);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sh->p_bar[g][0]);
#pragma unroll
        for (int k = KP; k < BN / 2; ++k) exp_pair(k);
        tmem_st32(s_tmem + KP, pw + KP);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sh->p_bar[g][1]);
        lsum2 = fadd2(lsum2, fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3])));
        return true;
      };

      // Tiles are visited from the diagonal towards key 0.  A run of clean tiles
      // for this warp ends at the first tile whose range [lo, lo + kCleanSpan)
      // -- lo = centre + 32 quarter - 127, the smallest distance of the warp's
      // elements -- holds some window W_i: there a boundary crosses the warp's
      // elements or pairs die next tile.  The first window not below lo is the
      // next one to enter that range (W is non-decreasing), so the run length
      // follows from it directly.
      int j = j0;
      while (ok && j < T) {
        int jn = T, a_run = 0;
        if constexpr (SPARSE) {
          const long long lo = centre(j + g) + 32 * quarter - (BN - 1);
          a_run = ww.below(lo);  // pairs dead for every element of the run
          if (a_run >= C::NP) {
            jn = j;  // every pair dead: the correcting body handles tiles without S
          } else {
            const long long excess = ww.at(a_run) - lo - (kCleanSpan - 1);  // tile j + t holds W when BN t >= excess
            jn = excess <= 0 ? j : j + static_cast<int>(min((excess + BN - 1) / BN, static_cast<long long>(T - j)));
          }
        }
        for (; ok && j < jn; ++j) ok = tile(j, std::false_type{}, a_run);
        if (ok && j < T) {
          ok = tile(j, std::true_type{}, 0);
          ++j;
        }
      }
      // ---- epilogue: O_g / l -> bf16
      if (ok && warp_wait(&sh->o_done[g], 0, abort, p.err, 0x304)) {
        tc_fence_after();
        float l0, l1;
        unpack2(lsum2, l0, l1);
        const float l = l0 + l1;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + q_elem;
#pragma unroll
        for (int k = 0; k < D / 32; ++k) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + C::COL_O + g * D + 32 * k, o);
          tmem_ld_wait();
          uint32_t ow[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            ow[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * k);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(ow[4 * v4], ow[4 * v4 + 1], ow[4 * v4 + 2], ow[4 * v4 + 3]);
          }
        }
      }
      if (SPARSE && p.skipped) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
        if (lane == 0 && cnt) atomicAdd(p.skipped, cnt);
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool SPARSE>
static cudaError_t launch_tc(const PrefillParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                             const CUtensorMap& tv, cudaStream_t s) {
  auto kern = prefill_tc_kernel<D, SPARSE>;
  constexpr int bytes = smem_bytes<D>();
  static_assert(bytes <= 227 * 1024, "shared memory budget");
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // one bit per device; two threads racing on the first call both check and set
  // the attribute, which is harmless, and the atomic keeps the bit updates defined
  static std::atomic<unsigned long long> configured{0};
  if (dev >= 64 || !(configured.load(std::memory_order_acquire) & (1ull << dev))) {
    // The register reallocation inside the kernel needs exactly the launch
    // allocation it was written for; anything else could leave setmaxnreg.inc
    // waiting, so refuse to launch.
    cudaFuncAttributes attr{};
    e = cudaFuncGetAttributes(&attr, kern);
    if (e != cudaSuccess) return e;
    if (attr.numRegs != kRegsLaunch) return cudaErrorInvalidKernelImage;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    if (dev < 64) configured.fetch_or(1ull << dev, std::memory_order_acq_rel);
  }
  const long long nqt = (p.q_len + BM - 1) / BM;
  const long long ctas = (nqt + NQ - 1) / NQ * p.hq * p.batch;
  if (ctas == 0) return cudaSuccess;
  kern<<<static_cast<unsigned>(ctas), kThreads, bytes, s>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_prefill_tc(const PrefillParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                              const CUtensorMap& tv, bool dense, cudaStream_t s) {
  if (p.d == 64) return dense ? launch_tc<64, false>(p, tq, tk, tv, s) : launch_tc<64, true>(p, tq, tk, tv, s);
  return dense ? launch_tc<128, false>(p, tq, tk, tv, s) : launch_tc<128, true>(p, tq, tk, tv, s);
}

}  // namespace atf
