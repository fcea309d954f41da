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
// Design (one CTA = 128 query rows of one query head; 6 warps):
//   warp 0     TMA producer: K and V tiles of 128 keys (128B-swizzled boxes of
//              64 dims) into a 3-stage ring.
//   warp 1     TMEM owner and MMA issuer (one thread):
//                S(j)  = Q~ . K~(j)^T   A = Q~ in TMEM, B = K tile (K-major)
//                O    += P(j) . V(j)    A = P in TMEM,  B = V tile (MN-major)
//   warps 2-5  softmax: one query row per thread (TMEM lane = row).
// TMEM columns: S double buffer [0,256), O [256, 256+d), Q~ [256+d, 256+3d/2).
//
// Window structure.  W is non-decreasing in i (wavelengths grow), so the active
// pairs of any element form a suffix {i >= i*(Delta)}.  KV tiles are visited
// from the diagonal towards key 0, so the tile's centre distance
// c_j = m0 - n0_j grows monotonically.  Pairs with W_i < c_j are zeroed in the
// TMEM copy of Q~ once and for all, and whole 8-pair chunks below the first
// non-zeroed pair are not issued to the MMA at all (the contraction depth
// shrinks tile by tile).  Elements of a tile that straddles a window boundary
// are fixed on the CUDA cores: a zeroed pair whose window still covers the
// element is added back, an issued pair whose window does not is subtracted.
// Each such region is at most half a tile (the side of the boundary away from
// the tile centre), and only straddling pairs have one.
#include <cuda_bf16.h>

#include "atf_internal.cuh"
#include "ptx.cuh"

namespace atf {

namespace {

constexpr int BM = 128;       // query rows per CTA
constexpr int BN = 128;       // keys per KV tile
constexpr int kThreads = 192; // 6 warps
constexpr uint32_t kTmemCols = 512;

template <int D>
struct Cfg {
  static constexpr int NS = D == 128 ? 3 : 4;            // ring stages
  static constexpr int BOXES = D / 64;                   // 64-dim swizzle boxes per tile
  static constexpr int TILE_BYTES = BN * D * 2;          // one K (or V) tile
  static constexpr int NCH = D / 16;                     // 8-pair chunks = MMA K-steps
  static constexpr int NP = D / 2;
  static constexpr uint32_t COL_S = 0, COL_O = 256, COL_Q = 256 + D;
  static constexpr int SMEM_TILES = 2 * NS * TILE_BYTES;
  static constexpr int SMEM_BYTES = SMEM_TILES + 1024 /*bars etc*/ + 1024 /*align*/;
};

struct Bars {
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], p_full[2], pv_done, o_done, q_ready, drain;
  uint32_t tmem_base;
  int abort;
  int w[kMaxPairs];
};

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
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const PrefillParams p) {
  using C = Cfg<D>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;                           // [NS][TILE_BYTES]
  uint8_t* sV = smem + NS * C::TILE_BYTES;      // [NS][TILE_BYTES]
  Bars* bars = reinterpret_cast<Bars*>(smem + C::SMEM_TILES);

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
  auto zeroed = [&](int j) -> int {  // pairs with W_i < tile centre
    if (!SPARSE) return 0;
    return lower_bound_w(bars->w, C::NP, m0 - tile_n0(j));
  };

  // ---- setup
  if (tid == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 4);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], 128);
    }
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->q_ready, 128);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < C::NP; i += kThreads) bars->w[i] = p.win.w[i];
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 0) {
    // ================================================================ TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int j = 0; j < T; ++j) {
        const int s = j % NS, use = j / NS;
        const int n0 = static_cast<int>(tile_n0(j));
        if (j >= NS && !mbar_wait(&bars->k_empty[s], (use - 1) & 1, abort, p.err, 0x101)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], C::TILE_BYTES);
#pragma unroll
        for (int bx = 0; bx < C::BOXES; ++bx)
          tma_load_4d(sK + s * C::TILE_BYTES + bx * (BN * 128), &tm_k, &bars->k_full[s], bx * 64, hk, n0, b);
        if (j >= NS && !mbar_wait(&bars->v_empty[s], (use - 1) & 1, abort, p.err, 0x102)) {
          issued = 2 * j + 1;
          break;
        }
        mbar_arrive_expect_tx(&bars->v_full[s], C::TILE_BYTES);
#pragma unroll
        for (int bx = 0; bx < C::BOXES; ++bx)
          tma_load_4d(sV + s * C::TILE_BYTES + bx * (BN * 128), &tm_v, &bars->v_full[s], bx * 64, hk, n0, b);
        issued = 2 * j + 2;
      }
      if (*abort) {
        // let every load already issued land before the CTA leaves
        for (int q = 0; q < issued; ++q) {
          const int j = q >> 1, s = j % NS;
          drain_wait((q & 1) ? &bars->v_full[s] : &bars->k_full[s], (j / NS) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(BM, D, false, true);
      constexpr uint64_t kdesc_bits = smem_desc_bits(16, 1024, kLayoutSW128);
      constexpr uint64_t vdesc_bits = smem_desc_bits(BN * 128, 1024, kLayoutSW128);
      const uint32_t sK_addr = smem_u32(sK), sV_addr = smem_u32(sV);
      int ev = 0;
      bool ok = mbar_wait(&bars->q_ready, ev & 1, abort, p.err, 0x201);
      ++ev;
      auto issue_s = [&](int j) -> bool {
        const int s = j % NS;
        if (!mbar_wait(&bars->k_full[s], (j / NS) & 1, abort, p.err, 0x202)) return false;
        tc_fence_after();
        const int c0 = zeroed(j) >> 3;
        const uint32_t d_tmem = tmem + C::COL_S + (j & 1) * BN;
        for (int c = c0; c < C::NCH; ++c) {
          const uint32_t a = sK_addr + s * C::TILE_BYTES + (c >> 2) * (BN * 128) + (c & 3) * 32;
          mma_ts(d_tmem, tmem + C::COL_Q + 8 * c, smem_desc(a, kdesc_bits), idesc_qk, c > c0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[j & 1]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T) {
          if (SPARSE && zeroed(j + 1) > zeroed(j)) {
            ok = mbar_wait(&bars->q_ready, ev & 1, abort, p.err, 0x203);
            ++ev;
            if (!ok) break;
            tc_fence_after();
          }
          // S(j+1) overwrites the TMEM buffer that holds P(j-1): let PV(j-1) finish first
          if (j >= 1) {
            if (!(ok = mbar_wait(&bars->pv_done, (j - 1) & 1, abort, p.err, 0x206))) break;
            tc_fence_after();
          }
          if (!(ok = issue_s(j + 1))) break;
        }
        const int s = j % NS;
        if (!(ok = mbar_wait(&bars->p_full[j & 1], (j >> 1) & 1, abort, p.err, 0x204))) break;
        if (!(ok = mbar_wait(&bars->v_full[s], (j / NS) & 1, abort, p.err, 0x205))) break;
        tc_fence_after();
        const uint32_t p_tmem = tmem + C::COL_S + (j & 1) * BN;  // P(j) packed bf16 over S(j)
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint32_t a = sV_addr + s * C::TILE_BYTES + kk * 2048;
          mma_ts(tmem + C::COL_O, p_tmem + 8 * kk, smem_desc(a, vdesc_bits), idesc_pv,
                 (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars->v_empty[s]);
        mma_commit(&bars->pv_done);
        if (j == T - 1) mma_commit(&bars->o_done);
      }
      if (!ok) {
        mma_commit(&bars->drain);
        drain_wait(&bars->drain, 0);
      }
    }
  } else {
    // ================================================================ softmax (warps 2..5)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row in tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int t = qt * BM + r;
    const bool row_ok = t < p.q_len;
    const long long m = m0 + r;
    const long long q_elem = ((static_cast<long long>(b) * p.q_len + (row_ok ? t : 0)) * p.hq + h) * D;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(p.q) + q_elem);
    constexpr float kLog2e = 1.4426950408889634f;
    const float scale = kLog2e * rsqrtf(static_cast<float>(D));

    // Q~ row -> TMEM (pairs below the first tile's zeroed count are stored as 0)
    int zcur = zeroed(0);
    {
      uint32_t w[32];
#pragma unroll
      for (int half = 0; half < D / 64; ++half) {
#pragma unroll
        for (int v4 = 0; v4 < 8; ++v4) {
          uint4 x = row_ok ? __ldg(reinterpret_cast<const uint4*>(qrow) + half * 8 + v4) : make_uint4(0, 0, 0, 0);
          w[4 * v4 + 0] = x.x;
          w[4 * v4 + 1] = x.y;
          w[4 * v4 + 2] = x.z;
          w[4 * v4 + 3] = x.w;
        }
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (half * 32 + k < zcur) w[k] = 0u;
        tmem_st32(tmem + lane_off + C::COL_Q + half * 32, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->q_ready);
    }

    float mrun = -INFINITY, lsum = 0.f;
    unsigned long long cnt = 0;
    int j = 0;
    for (; j < T; ++j) {
      const int s = j % NS;
      const long long n0 = tile_n0(j);
      const long long center = m0 - n0;
      const int z = zcur;
      if (!warp_wait(&bars->s_full[j & 1], (j >> 1) & 1, abort, p.err, 0x301)) break;
      tc_fence_after();
      if (SPARSE && j + 1 < T) {
        const int zn = zeroed(j + 1);
        if (zn > zcur) {  // S(j) is done reading Q~: zero the newly dead pairs for S(j+1)
          for (int i = zcur; i < zn; ++i) tmem_st1(tmem + lane_off + C::COL_Q + i, 0u);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&bars->q_ready);
          zcur = zn;
        }
      }
      const uint32_t s_tmem = tmem + lane_off + C::COL_S + (j & 1) * BN;
      float sv[BN];
      if ((z >> 3) < C::NCH) {
#pragma unroll
        for (int k = 0; k < BN / 32; ++k) tmem_ld32(s_tmem + 32 * k, reinterpret_cast<uint32_t*>(sv + 32 * k));
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int c = 0; c < BN; ++c) sv[c] = 0.f;
      }
      // valid columns of this row form the prefix [0, cmax]
      int cmax = -1;
      if (row_ok) {
        long long cm = min(static_cast<long long>(BN - 1), m - n0);
        cm = min(cm, static_cast<long long>(p.kv_len) - 1 - n0);
        cmax = static_cast<int>(cm);
      }
      if (SPARSE) {
        if (!warp_wait(&bars->k_full[s], (j / NS) & 1, abort, p.err, 0x302)) break;
        const int a = lower_bound_w(bars->w, C::NP, center - (BN - 1));
        const int u = max(z, lower_bound_w(bars->w, C::NP, center + (BM - 1)));
        const uint32_t kbase = smem_u32(sK + s * C::TILE_BYTES);
        const int nvalid = cmax + 1;
        cnt += static_cast<unsigned long long>(a) * (nvalid > 0 ? nvalid : 0);
        for (int i = a; i < u; ++i) {
          const int wi = bars->w[i];
          const long long tl = r + center - wi;  // columns c < tl are outside pair i's window
          const long long tw = quarter * 32 + center - wi;  // this warp's smallest tl
          if (nvalid > 0) cnt += static_cast<unsigned long long>(tl <= 0 ? 0 : (tl >= nvalid ? nvalid : tl));
          const uint32_t qp = row_ok ? __ldg(qrow + i) : 0u;
          const float qa = bf16lo_to_f32(qp), qb = bf16hi_to_f32(qp);
          const int tli = static_cast<int>(tl < -1 ? -1 : (tl > BN ? BN : tl));
          uint32_t xo[8];
          {
            const uint32_t base = kbase + (i >> 5) * (BN * 128) + (i & 3) * 4;
            const uint32_t ch = (i & 31) >> 2;
#pragma unroll
            for (int x = 0; x < 8; ++x) xo[x] = base + ((ch ^ x) << 4);
          }
          if (i < z) {
            // zeroed pair: add it back where Delta <= W_i, i.e. c >= tl
#pragma unroll
            for (int blk = 0; blk < BN / 32; ++blk) {
              if (32 * blk + 31 < tw) continue;  // whole block outside for every row of the warp
#pragma unroll
              for (int cc = 0; cc < 32; ++cc) {
                const int c = 32 * blk + cc;
                const uint32_t kp = lds32(xo[c & 7] + c * 128);
                const float pd = fmaf(qa, bf16lo_to_f32(kp), qb * bf16hi_to_f32(kp));
                sv[c] += (c >= tli) ? pd : 0.f;
              }
            }
          } else {
            // issued pair: subtract it where Delta > W_i, i.e. c < tl
#pragma unroll
            for (int blk = 0; blk < BN / 32; ++blk) {
              if (32 * blk >= tw + 31) continue;  // whole block inside for every row of the warp
#pragma unroll
              for (int cc = 0; cc < 32; ++cc) {
                const int c = 32 * blk + cc;
                const uint32_t kp = lds32(xo[c & 7] + c * 128);
                const float pd = fmaf(qa, bf16lo_to_f32(kp), qb * bf16hi_to_f32(kp));
                sv[c] -= (c < tli) ? pd : 0.f;
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->k_empty[s]);
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->k_empty[s]);
      }

      // masks, running max
      const bool partial = __any_sync(0xffffffffu, cmax < BN - 1);
      float mx = -INFINITY;
      if (partial) {
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          sv[c] = (c <= cmax) ? sv[c] * scale : -INFINITY;
          mx = fmaxf(mx, sv[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < BN; ++c) {
          sv[c] *= scale;
          mx = fmaxf(mx, sv[c]);
        }
      }
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
        // O holds PV(0..j-1); wait for PV(j-1) before touching it.  PV(j-2) is
        // known complete (S(j) was issued after it), so pv_done is within one
        // phase of j-1 and the parity test is exact.
        if (!warp_wait(&bars->pv_done, (j - 1) & 1, abort, p.err, 0x303)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 32; ++k) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + C::COL_O + 32 * k, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * corr);
          tmem_st32(tmem + lane_off + C::COL_O + 32 * k, o);
        }
        tmem_st_wait();
        if (need) {
          lsum *= corr;
          mrun = mnew;
        }
      }
      const float mref = (mrun == -INFINITY) ? 0.f : mrun;
      uint32_t pw[BN / 2];
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        const float p0 = ex2_approx(sv[c] - mref);
        const float p1 = ex2_approx(sv[c + 1] - mref);
        lsum += p0 + p1;
        pw[c / 2] = pack_bf16x2(p0, p1);
      }
      tmem_st32(s_tmem, pw);
      tmem_st32(s_tmem + 32, pw + 32);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->p_full[j & 1]);
    }

    // ---- epilogue: O / l -> bf16.  A one-shot barrier marks the last P.V: a
    // parity wait on pv_done could be fooled here, since PV(T-2) may still be
    // pending (two phases outstanding).
    if (j == T && warp_wait(&bars->o_done, 0, abort, p.err, 0x304)) {
      tc_fence_after();
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(p.out) + q_elem;
#pragma unroll
      for (int k = 0; k < D / 32; ++k) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + C::COL_O + 32 * k, o);
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

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, bool SPARSE>
static cudaError_t launch_tc(const PrefillParams& p, const CUtensorMap& tk, const CUtensorMap& tv, cudaStream_t s) {
  using C = Cfg<D>;
  auto kern = prefill_tc_kernel<D, SPARSE>;
  static bool configured = false;  // per instantiation; attribute is per device function
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const long long ctas = static_cast<long long>((p.q_len + BM - 1) / BM) * p.hq * p.batch;
  if (ctas == 0) return cudaSuccess;
  kern<<<static_cast<unsigned>(ctas), kThreads, C::SMEM_BYTES, s>>>(tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_prefill_tc(const PrefillParams& p, const CUtensorMap& tk, const CUtensorMap& tv, bool dense,
                              cudaStream_t s) {
  if (p.d == 64) return dense ? launch_tc<64, false>(p, tk, tv, s) : launch_tc<64, true>(p, tk, tv, s);
  return dense ? launch_tc<128, false>(p, tk, tv, s) : launch_tc<128, true>(p, tk, tv, s);
}

}  // namespace atf
