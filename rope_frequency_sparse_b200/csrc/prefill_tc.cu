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
// Design (one CTA = 128 query rows of one query head; 10 warps):
//   warp 0     TMA producer: the Q~ tile once, then K and V tiles of 128 keys
//              (128B-swizzled boxes of 64 dims) into separate rings.
//   warp 1     TMEM owner and MMA issuer (one thread):
//                S(j)  = Q~ . K~(j)^T            A = Q~ tile, B = K tile (both K-major, smem)
//                O_g  += P(j) . V(j), g = j & 1  A = P in TMEM, B = V tile (MN-major)
//   warps 2-9  softmax, two groups of four warps; group g takes the KV tiles
//              j = g, g+2, g+4, ... with one full query row per thread (TMEM
//              lane = row) and its own running max, row sum and accumulator O_g.
//              The groups run out of phase, so one group's exponentials overlap
//              the other group's loads, reductions and corrections; the two
//              partial results are merged once at the end.
// TMEM columns: S(j) in buffer j&1 at [128(j&1), 128(j&1)+128) (P(j) is written
// back over it as packed bf16), O_0 at [256, 256+d), O_1 at [256+d, 256+2d).
//
// Window structure.  W is non-decreasing in i (wavelengths grow), so the active
// pairs of any element form a suffix {i >= i*(Delta)}.  KV tiles are visited
// from the diagonal towards key 0, so the tile's centre distance
// c_j = m0 - n0_j grows monotonically.  Pairs with W_i < c_j are zeroed in the
// shared-memory copy of Q~ once and for all, and whole 8-pair chunks below the
// first non-zeroed pair are not issued to the MMA at all (the contraction depth
// shrinks tile by tile).  Elements of a tile that straddles a window boundary
// are fixed on the CUDA cores: a zeroed pair whose window still covers the
// element is added back, an issued pair whose window does not is subtracted.
// Each such region is at most half a tile (the side of the boundary away from
// the tile centre), and only straddling pairs have one.  The per-tile pair
// ranges are tabulated in shared memory when the CTA starts.
#include <cuda_bf16.h>

#include "atf_internal.cuh"
#include "ptx.cuh"

namespace atf {

namespace {

constexpr int BM = 128;        // query rows per CTA
constexpr int BN = 128;        // keys per KV tile
constexpr int kThreads = 320;  // 10 warps
constexpr uint32_t kTmemCols = 512;
constexpr int kTileTable = 1024;  // tabulated KV tiles per CTA (131072 keys)

template <int D>
struct Cfg {
  static constexpr int NSK = D == 128 ? 3 : 4;   // K ring stages
  static constexpr int NSV = D == 128 ? 2 : 4;   // V ring stages
  static constexpr int BOXES = D / 64;           // 64-dim swizzle boxes per tile
  static constexpr int TILE_BYTES = BN * D * 2;  // one K (or V, or Q) tile
  static constexpr int NCH = D / 16;             // 8-pair chunks = MMA K-steps
  static constexpr int NP = D / 2;
  static constexpr uint32_t COL_S = 0, COL_O = 256;
  static constexpr int SMEM_TILES = (1 + NSK + NSV) * TILE_BYTES;
};

struct Shared {
  uint64_t q_full, k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], p_full[2], o_done, q_ready, xfin, drain;
  uint32_t tmem_base;
  int abort;
  int w[kMaxPairs];
  float fin_m[2][BM];  // per group: running max (log2 units) and row sum, for the final merge
  float fin_l[2][BM];
  uint32_t tinfo[kTileTable];  // per KV tile: zeroed | add-back start << 8 | subtract end << 16
};

template <int D>
constexpr int smem_bytes() {
  return Cfg<D>::SMEM_TILES + static_cast<int>(sizeof(Shared)) + 1024;
}

// number of pairs with W_i < x  (W non-decreasing, W_i >= 1)
__device__ __forceinline__ int lower_bound_w(const int* w, int np, long long x) {
  int lo = 0, hi = np;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (static_cast<long long>(w[mid]) < x)
      lo = mid + 1;
    else
      hi = mid;
  }
  return lo;
}

// Pair ranges of a KV tile with centre distance `center` (= m0 - n0):
//   z: pairs zeroed in Q~ (W_i < center)
//   a: first pair whose window reaches any element (W_i >= center - 127)
//   u: end of the pairs whose window misses some element (W_i < center + 127)
__device__ __forceinline__ uint32_t tile_ranges(const int* w, int np, long long center) {
  const uint32_t z = lower_bound_w(w, np, center);
  const uint32_t a = lower_bound_w(w, np, center - (BN - 1));
  uint32_t u = lower_bound_w(w, np, center + (BM - 1));
  if (u < z) u = z;
  return z | (a << 8) | (u << 16);
}

// Byte offset of pair i (4 bytes) of row r inside a 128-row tile stored as
// 64-dim boxes with the 128-byte swizzle (16-byte chunk index XOR row % 8).
__device__ __forceinline__ uint32_t pair_offset(int r, int i) {
  return (i >> 5) * (BN * 128) + r * 128 + ((((i & 31) >> 2) ^ (r & 7)) << 4) + (i & 3) * 4;
}

// Warp-collective bounded wait: every lane observes the barrier itself (acquire),
// and the warp leaves together, so .sync.aligned tcgen05 ops never see a split warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, unsigned int* err,
                                          unsigned int code) {
  const bool ok = mbar_wait(bar, parity, abort, err, code);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait that ignores the abort flag (used only while draining).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity) && clock64() - t0 < kWaitLimitCycles) {
  }
}

}  // namespace

template <int D, bool SPARSE>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const PrefillParams p) {
  using C = Cfg<D>;
  constexpr int NSK = C::NSK, NSV = C::NSV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                      // Q~ tile
  uint8_t* sK = smem + C::TILE_BYTES;      // [NSK][TILE_BYTES]
  uint8_t* sV = sK + NSK * C::TILE_BYTES;  // [NSV][TILE_BYTES]
  Shared* sh = reinterpret_cast<Shared*>(smem + C::SMEM_TILES);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- tile coordinates: heaviest query tiles first
  const int nqt = (p.q_len + BM - 1) / BM;
  int idx = blockIdx.x;
  const int h = idx % p.hq;
  idx /= p.hq;
  const int b = idx % p.batch;
  const int qt = nqt - 1 - idx / p.batch;
  const int hk = h / (p.hq / p.hkv);
  const long long m0 = p.q_offset + static_cast<long long>(qt) * BM;
  const int rows_here = min(BM, p.q_len - qt * BM);
  const long long max_key = min(m0 + rows_here - 1, static_cast<long long>(p.kv_len) - 1);
  const int T = static_cast<int>(max_key / BN) + 1;  // KV tiles, visited j = 0..T-1
  auto tile_n0 = [&](int j) { return static_cast<long long>(T - 1 - j) * BN; };
  auto ranges = [&](int j) -> uint32_t {
    if (!SPARSE) return 0u;
    if (j < kTileTable) return sh->tinfo[j];
    return tile_ranges(sh->w, C::NP, m0 - tile_n0(j));
  };

  // ---- setup
  if (tid == 0) {
    mbar_init(&sh->q_full, 1);
    for (int s = 0; s < NSK; ++s) {
      mbar_init(&sh->k_full[s], 1);
      mbar_init(&sh->k_empty[s], 4);
    }
    for (int s = 0; s < NSV; ++s) {
      mbar_init(&sh->v_full[s], 1);
      mbar_init(&sh->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh->s_full[s], 1);
      mbar_init(&sh->p_full[s], 128);
    }
    mbar_init(&sh->o_done, 1);
    mbar_init(&sh->q_ready, 128);
    mbar_init(&sh->xfin, 256);
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
  if (SPARSE) {
    const int nt = T < kTileTable ? T : kTileTable;
    for (int j = tid; j < nt; j += kThreads) sh->tinfo[j] = tile_ranges(sh->w, C::NP, m0 - tile_n0(j));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  volatile int* abort = &sh->abort;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&sh->q_full, C::TILE_BYTES);
#pragma unroll
      for (int bx = 0; bx < C::BOXES; ++bx)
        tma_load_4d(sQ + bx * (BN * 128), &tm_q, &sh->q_full, bx * 64, h, qt * BM, b);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < T; ++j) {
        const int n0 = static_cast<int>(tile_n0(j));
        {
          const int s = j % NSK, use = j / NSK;
          if (j >= NSK && !mbar_wait(&sh->k_empty[s], (use - 1) & 1, abort, p.err, 0x101)) break;
          mbar_arrive_expect_tx(&sh->k_full[s], C::TILE_BYTES);
#pragma unroll
          for (int bx = 0; bx < C::BOXES; ++bx)
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
        drain_wait(&sh->q_full, 0);
        for (int j = 0; j < k_issued; ++j) drain_wait(&sh->k_full[j % NSK], (j / NSK) & 1);
        for (int j = 0; j < v_issued; ++j) drain_wait(&sh->v_full[j % NSV], (j / NSV) & 1);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, false, true);
      constexpr uint64_t kdesc_bits = smem_desc_bits(16, 1024, kLayoutSW128);
      constexpr uint64_t vdesc_bits = smem_desc_bits(BN * 128, 1024, kLayoutSW128);
      const uint32_t sQ_addr = smem_u32(sQ), sK_addr = smem_u32(sK), sV_addr = smem_u32(sV);
      int ev = 0;
      bool ok = mbar_wait(&sh->q_ready, ev & 1, abort, p.err, 0x201);
      ++ev;
      tc_fence_after();
      auto issue_s = [&](int j) -> bool {
        const int s = j % NSK;
        if (!mbar_wait(&sh->k_full[s], (j / NSK) & 1, abort, p.err, 0x202)) return false;
        tc_fence_after();
        const int c0 = static_cast<int>(ranges(j) & 0xFF) >> 3;
        const uint32_t d_tmem = tmem + C::COL_S + (j & 1) * BN;
        for (int c = c0; c < C::NCH; ++c) {
          const uint32_t koff = (c >> 2) * (BN * 128) + (c & 3) * 32;
          mma_ss(d_tmem, smem_desc(sQ_addr + koff, kdesc_bits),
                 smem_desc(sK_addr + s * C::TILE_BYTES + koff, kdesc_bits), idesc_qk, c > c0 ? 1u : 0u);
        }
        mma_commit(&sh->s_full[j & 1]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T) {
          if (SPARSE && (ranges(j + 1) & 0xFF) > (ranges(j) & 0xFF)) {
            ok = mbar_wait(&sh->q_ready, ev & 1, abort, p.err, 0x203);
            ++ev;
            if (!ok) break;
            tc_fence_after();
          }
          // S(j+1) overwrites the TMEM buffer that holds P(j-1); PV(j-1) was issued
          // before it by this thread, and tcgen05.mma operations execute in issue order.
          if (!(ok = issue_s(j + 1))) break;
        }
        const int s = j % NSV;
        // V(j) normally landed long ago: check it before blocking on P(j)
        if (!(ok = mbar_wait(&sh->v_full[s], (j / NSV) & 1, abort, p.err, 0x205))) break;
        if (!(ok = mbar_wait(&sh->p_full[j & 1], (j >> 1) & 1, abort, p.err, 0x204))) break;
        tc_fence_after();
        const uint32_t p_tmem = tmem + C::COL_S + (j & 1) * BN;  // P(j) packed bf16 over S(j)
        const uint32_t o_tmem = tmem + C::COL_O + (j & 1) * D;   // this group's accumulator
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t a = sV_addr + s * C::TILE_BYTES + kk * 2048;
          mma_ts(o_tmem, p_tmem + 8 * kk, smem_desc(a, vdesc_bits), idesc_pv, (j >= 2 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sh->v_empty[s]);
        if (j == T - 1) mma_commit(&sh->o_done);
      }
      if (!ok) {
        mma_commit(&sh->drain);
        drain_wait(&sh->drain, 0);
      }
    }
  } else {
    // ================================================================ softmax (warps 2..9)
    const int quarter = warp & 3;
    const int g = (warp - 2) >> 2;      // group: KV tiles j with j % 2 == g
    const int r = quarter * 32 + lane;  // query row in tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int t = qt * BM + r;
    const bool row_ok = t < p.q_len;
    const long long m = m0 + r;
    const long long q_elem = ((static_cast<long long>(b) * p.q_len + (row_ok ? t : 0)) * p.hq + h) * D;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(p.q) + q_elem);
    constexpr float kLog2e = 1.4426950408889634f;
    const float scale = kLog2e * rsqrtf(static_cast<float>(D));

    bool ok = true;
    // Pairs dead in the first tile are zeroed in the Q~ tile before S(0).
    if (g == 0) {
      ok = warp_wait(&sh->q_full, 0, abort, p.err, 0x300);
      if (ok) {
        if (SPARSE) {
          const int z0 = static_cast<int>(ranges(0) & 0xFF);
          for (int i = 0; i < z0; ++i) *reinterpret_cast<uint32_t*>(sQ + pair_offset(r, i)) = 0u;
          fence_proxy_async_smem();
        }
        mbar_arrive(&sh->q_ready);
      }
    }

    float mrun = -INFINITY;
    uint64_t lsum2 = 0ull;  // packed partial row sums
    unsigned long long cnt = 0;
    for (int j = g; ok && j < T; j += 2) {
      const int s = j % NSK;
      const long long n0 = tile_n0(j);
      const long long center = m0 - n0;
      const uint32_t rg = ranges(j);
      const int z = static_cast<int>(rg & 0xFF);
      const int a = static_cast<int>((rg >> 8) & 0xFF);
      const int u = static_cast<int>((rg >> 16) & 0xFF);
      // prefetch the query pairs of this tile's first boundary corrections
      uint32_t qpf[4] = {0u, 0u, 0u, 0u};
      if (SPARSE && row_ok) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (a + k < u) qpf[k] = __ldg(qrow + a + k);
      }
      if (!(ok = warp_wait(&sh->s_full[j & 1], (j >> 1) & 1, abort, p.err, 0x301))) break;
      tc_fence_after();
      if (SPARSE && j + 1 < T) {
        const int zn = static_cast<int>(ranges(j + 1) & 0xFF);
        if (zn > z) {  // S(j) is done reading Q~: zero the newly dead pairs for S(j+1)
          for (int i = z; i < zn; ++i) *reinterpret_cast<uint32_t*>(sQ + pair_offset(r, i)) = 0u;
          fence_proxy_async_smem();
          mbar_arrive(&sh->q_ready);
        }
      }
      const uint32_t s_tmem = tmem + lane_off + C::COL_S + (j & 1) * BN;
      const bool has_mma = (z >> 3) < C::NCH;  // a tile whose pairs are all zeroed has no S MMA
      // valid columns of this row form the prefix [0, cmax]
      int cmax = -1;
      if (row_ok) {
        long long cmx = min(static_cast<long long>(BN - 1), m - n0);
        cmx = min(cmx, static_cast<long long>(p.kv_len) - 1 - n0);
        cmax = static_cast<int>(cmx);
      }
      const bool partial = __any_sync(0xffffffffu, cmax < BN - 1);
      // ---- pass 1 over S in chunks of 64 columns: boundary corrections (written
      // back to TMEM) and the row max (eight independent 3-input max chains)
      float acc[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] = -INFINITY;
      bool stored = false;
      // the K tile is read only by boundary corrections
      if (SPARSE && a < u && !(ok = warp_wait(&sh->k_full[s], (j / NSK) & 1, abort, p.err, 0x302))) break;
      if (SPARSE) {
        const int nv = cmax + 1;  // valid columns of this row
        cnt += static_cast<unsigned long long>(a) * nv;
        for (int i = a; i < u; ++i) {
          const long long tl = r + center - sh->w[i];
          const int tli = static_cast<int>(tl < -1 ? -1 : (tl > BN ? BN : tl));
          cnt += static_cast<unsigned long long>(tli <= 0 ? 0 : (tli < nv ? tli : nv));
        }
      }
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        float v[64];
        if (has_mma) {
          tmem_ld32(s_tmem + 64 * hc, reinterpret_cast<uint32_t*>(v));
          tmem_ld32(s_tmem + 64 * hc + 32, reinterpret_cast<uint32_t*>(v + 32));
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) v[c] = 0.f;
        }
        if (SPARSE) {
          bool touched = !has_mma;  // a tile without S MMA must write its (zero) logits
          const uint32_t kbase = smem_u32(sK + s * C::TILE_BYTES);
          for (int i = a; i < u; ++i) {
            const int wi = sh->w[i];
            const long long tl = r + center - wi;             // columns c < tl are outside pair i's window
            const long long tw = quarter * 32 + center - wi;  // smallest tl of the warp
            const int tli = static_cast<int>(tl < -1 ? -1 : (tl > BN ? BN : tl));
            const bool add = i < z;  // zeroed pair: add back where c >= tl; else subtract where c < tl
            // skip this chunk when no row of the warp has an element of it on the corrected side
            if (add ? (64 * hc + 63 < tw) : (64 * hc >= tw + 31)) continue;
            touched = true;
            const int kq = i - a;
            const uint32_t qp = kq == 0   ? qpf[0]
                                : kq == 1 ? qpf[1]
                                : kq == 2 ? qpf[2]
                                : kq == 3 ? qpf[3]
                                          : (row_ok ? __ldg(qrow + i) : 0u);
            const float qa = bf16lo_to_f32(qp), qb = bf16hi_to_f32(qp);
            const float sg = add ? 1.f : -1.f;
            uint32_t xo[8];
            {
              const uint32_t base = kbase + (i >> 5) * (BN * 128) + (i & 3) * 4;
              const uint32_t ch = (i & 31) >> 2;
#pragma unroll
              for (int x = 0; x < 8; ++x) xo[x] = base + ((ch ^ x) << 4);
            }
#pragma unroll
            for (int cc = 0; cc < 64; ++cc) {
              const int c = 64 * hc + cc;
              const uint32_t kp = lds32(xo[cc & 7] + c * 128);
              const float pd = fmaf(qa, bf16lo_to_f32(kp), qb * bf16hi_to_f32(kp));
              const bool inside = add ? (c >= tli) : (c < tli);
              v[cc] = inside ? fmaf(sg, pd, v[cc]) : v[cc];
            }
          }
          if (touched) {
            tmem_st32(s_tmem + 64 * hc, reinterpret_cast<uint32_t*>(v));
            tmem_st32(s_tmem + 64 * hc + 32, reinterpret_cast<uint32_t*>(v + 32));
            stored = true;
          }
        }
        if (partial) {
#pragma unroll
          for (int cc = 0; cc < 64; ++cc)
            if (64 * hc + cc > cmax) v[cc] = -INFINITY;
        }
#pragma unroll
        for (int cc = 0; cc < 64; cc += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) acc[k] = fmax3(acc[k], v[cc + k], v[cc + 8 + k]);
      }
      if (stored) tmem_st_wait();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->k_empty[s]);
      const float mx =
          fmaxf(fmax3(acc[0], acc[1], acc[2]), fmax3(acc[3], acc[4], fmax3(acc[5], acc[6], acc[7]))) * scale;

      const float mnew = fmaxf(mrun, mx);
      // Conditional rescale: keep the stale max until the row max has grown by
      // more than 2^8; the final 1/l uses the same reference, so this is exact.
      bool need = false;
      float corr = 1.f;
      if (mrun == -INFINITY) {
        mrun = mnew;
      } else if (mnew > mrun + 8.f) {
        need = true;
        corr = ex2_approx(mrun - mnew);
      }
      if (__any_sync(0xffffffffu, need)) {
        // O_g holds PV(g), PV(g+2), ..., PV(j-2).  PV(j-2) was issued before S(j)
        // and S(j)'s commit covers every earlier MMA, so O_g is complete here.
#pragma unroll
        for (int k = 0; k < D / 32; ++k) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + C::COL_O + g * D + 32 * k, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
          tmem_st32(tmem + lane_off + C::COL_O + g * D + 32 * k, o);
        }
        tmem_st_wait();
        if (need) {
          lsum2 = fmul2(lsum2, pack2(corr, corr));
          mrun = mnew;
        }
      }
      // ---- pass 2: p = 2^(s*scale - mref) (one packed FMA per two elements, then
      // ex2), written back as packed bf16 P over the columns already read
      const float mref = (mrun == -INFINITY) ? 0.f : mrun;
      const uint64_t sc2 = pack2(scale, scale), nm2 = pack2(-mref, -mref);
      uint64_t ls[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        float v[64];
        tmem_ld32(s_tmem + 64 * hc, reinterpret_cast<uint32_t*>(v));
        tmem_ld32(s_tmem + 64 * hc + 32, reinterpret_cast<uint32_t*>(v + 32));
        tmem_ld_wait();
        if (partial) {
#pragma unroll
          for (int cc = 0; cc < 64; ++cc)
            if (64 * hc + cc > cmax) v[cc] = -INFINITY;
        }
        uint32_t pw[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          float x0, x1;
          unpack2(ffma2(pack2(v[2 * k], v[2 * k + 1]), sc2, nm2), x0, x1);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          ls[k & 3] = fadd2(ls[k & 3], pack2(p0, p1));
          pw[k] = pack_bf16x2(p0, p1);
        }
        tmem_st32(s_tmem + 32 * hc, pw);
      }
      lsum2 = fadd2(lsum2, fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3])));
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&sh->p_full[j & 1]);
    }

    // ---- epilogue: merge the two groups' partial results, O / l -> bf16.  Group g
    // writes output columns [g*d/2, (g+1)*d/2) of every row.
    if (ok) {
      float l0, l1;
      unpack2(lsum2, l0, l1);
      sh->fin_m[g][r] = mrun;
      sh->fin_l[g][r] = l0 + l1;
      mbar_arrive(&sh->xfin);
      if (warp_wait(&sh->xfin, 0, abort, p.err, 0x306) && warp_wait(&sh->o_done, 0, abort, p.err, 0x304)) {
        tc_fence_after();
        const float ma = sh->fin_m[0][r], mb = sh->fin_m[1][r];
        const float mm = fmaxf(ma, mb);
        const float fa = ma == -INFINITY ? 0.f : ex2_approx(ma - mm);
        const float fb = mb == -INFINITY ? 0.f : ex2_approx(mb - mm);
        const float l = sh->fin_l[0][r] * fa + sh->fin_l[1][r] * fb;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        const float wa = fa * inv, wb = fb * inv;
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + q_elem + g * (D / 2);
#pragma unroll
        for (int k = 0; k < D / 64; ++k) {
          const int col = g * (D / 2) + 32 * k;
          uint32_t oa[32], ob[32];
          tmem_ld32(tmem + lane_off + C::COL_O + col, oa);
          tmem_ld32(tmem + lane_off + C::COL_O + D + col, ob);
          tmem_ld_wait();
          uint32_t ow[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            // an accumulator that received no P.V holds stale TMEM: select, never multiply
            const float a0 = wa > 0.f ? __uint_as_float(oa[2 * e]) * wa : 0.f;
            const float a1 = wa > 0.f ? __uint_as_float(oa[2 * e + 1]) * wa : 0.f;
            const float b0 = wb > 0.f ? __uint_as_float(ob[2 * e]) * wb : 0.f;
            const float b1 = wb > 0.f ? __uint_as_float(ob[2 * e + 1]) * wb : 0.f;
            ow[e] = pack_bf16x2(a0 + b0, a1 + b1);
          }
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * k);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4)
              dst[v4] = make_uint4(ow[4 * v4], ow[4 * v4 + 1], ow[4 * v4 + 2], ow[4 * v4 + 3]);
          }
        }
      }
    }
    if (SPARSE && p.skipped) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
      if (lane == 0 && cnt) atomicAdd(p.skipped, cnt);
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
  static unsigned long long configured = 0;  // one bit per device
  if (dev < 64 && !(configured & (1ull << dev))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    configured |= 1ull << dev;
  }
  const long long ctas = static_cast<long long>((p.q_len + BM - 1) / BM) * p.hq * p.batch;
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
