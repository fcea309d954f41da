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
// equal HBM traffic (value bytes plus active key-chunk bytes), one CTA each; a
// CTA serves all query heads of its kv head (GQA).  Each CTA writes the usual
// split-softmax partial (running max in log2 units, sum, unnormalised output);
// a second kernel merges them.
#include <cuda_bf16.h>

#include "atf_internal.cuh"
#include "ptx.cuh"

namespace atf {

namespace {

constexpr int kDecWarps = 4;
constexpr float kLog2e = 1.4426950408889634f;

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

// First key index of split s (of ns) over keys [0, L), the query at L-1.
__device__ long long split_begin(int s, int ns, long long L, const int* sW, int nc) {
  if (s <= 0) return 0;
  if (s >= ns) return L;
  const long long total = traffic_below(L, sW, nc);
  // keys [0, n) have traffic total - traffic_below(L - n); find the smallest n
  // with that >= s*total/ns.
  const long long target = (total / ns) * s + ((total % ns) * s) / ns;
  long long lo = 0, hi = L;
  while (lo < hi) {
    const long long mid = (lo + hi) / 2;
    if (total - traffic_below(L - mid, sW, nc) >= target)
      hi = mid;
    else
      lo = mid + 1;
  }
  return lo & ~31LL;  // whole 32-key blocks
}

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(kDecWarps * 32) decode_split_kernel(DecodeParams p) {
  constexpr int NC = D / 16;  // chunks of 8 pairs
  constexpr int NP = D / 2;   // pairs
  constexpr int DPL = D / 32; // value dims per lane
  __shared__ float sQ[G][D];
  __shared__ int sW[NP];
  __shared__ __align__(16) float sP[kDecWarps][32][8];
  __shared__ float sM[kDecWarps][G];
  __shared__ float sL[kDecWarps][G];
  __shared__ float sAcc[kDecWarps][G][D];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const long long L = p.kv_len[b];
  const long long qpos = L - 1;

  for (int i = tid; i < NP; i += blockDim.x) sW[i] = p.win.w[i];
  // Rotate the G raw queries of this kv head at position qpos (fp64 angle).
  {
    const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(p.q);
    for (int idx = tid; idx < G * NP; idx += blockDim.x) {
      const int g = idx / NP, i = idx % NP;
      const long long e = (static_cast<long long>(b) * p.hq + hk * G + g) * D + 2 * i;
      const double x0 = __bfloat162float(Q[e]), x1 = __bfloat162float(Q[e + 1]);
      double sn, cs;
      sincos(static_cast<double>(qpos) * p.omega[i], &sn, &cs);
      sQ[g][2 * i] = static_cast<float>(x0 * cs - x1 * sn);
      sQ[g][2 * i + 1] = static_cast<float>(x0 * sn + x1 * cs);
    }
  }
  __syncthreads();

  const long long nb = split_begin(split, p.n_split, L, sW, NC);
  const long long ne = split_begin(split + 1, p.n_split, L, sW, NC);
  const float scale = kLog2e * rsqrtf(static_cast<float>(D));

  float mrun[G], lsum[G], acc[G][DPL];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    mrun[g] = -INFINITY;
    lsum[g] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[g][e] = 0.f;
  }
  unsigned long long cnt = 0;

  const uint4* KC = static_cast<const uint4*>(p.kc);
  const __nv_bfloat16* V = static_cast<const __nv_bfloat16*>(p.v);
  const long long kc_head = (static_cast<long long>(b) * p.hkv + hk) * NC;

  for (long long n0 = nb + 32LL * warp; n0 < ne; n0 += 32LL * kDecWarps) {
    const long long n = n0 + lane;
    const bool valid = n < ne;
    const long long delta = qpos - n;
    // the block's smallest distance is at its last valid key
    const long long last = (ne - 1 < n0 + 31) ? ne - 1 : n0 + 31;
    const long long dmin = qpos - last;
    int c_lo = 0;
    while (c_lo < NC && static_cast<long long>(sW[8 * c_lo + 7]) < dmin) ++c_lo;

    float s[G];
#pragma unroll
    for (int g = 0; g < G; ++g) s[g] = 0.f;
    int inactive = 8 * c_lo;
    for (int c = c_lo; c < NC; ++c) {
      uint4 k0 = make_uint4(0, 0, 0, 0), k1 = make_uint4(0, 0, 0, 0);
      if (valid) {
        const uint4* src = KC + ((kc_head + c) * p.n_cache + n) * 2;
        k0 = __ldg(src);
        k1 = __ldg(src + 1);
      }
      const uint32_t kw[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
      for (int pr = 0; pr < 8; ++pr) {
        const int i = 8 * c + pr;
        if (delta <= static_cast<long long>(sW[i])) {
          const float ka = bf16lo_to_f32(kw[pr]), kb = bf16hi_to_f32(kw[pr]);
#pragma unroll
          for (int g = 0; g < G; ++g) s[g] = fmaf(sQ[g][2 * i], ka, fmaf(sQ[g][2 * i + 1], kb, s[g]));
        } else {
          ++inactive;
        }
      }
    }
    if (valid) cnt += static_cast<unsigned long long>(inactive) * G;

    // online softmax over this block of 32 keys (log2 domain)
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float x = valid ? s[g] * scale : -INFINITY;
      float bm = x;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
      if (bm > mrun[g]) {  // warp-uniform
        const float corr = ex2_approx(mrun[g] - bm);
        lsum[g] *= corr;
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[g][e] *= corr;
        mrun[g] = bm;
      }
      const float pe = valid ? ex2_approx(x - mrun[g]) : 0.f;
      lsum[g] += pe;
      sP[warp][lane][g] = pe;
    }
    __syncwarp();
    const int nk = static_cast<int>((ne - n0) < 32 ? (ne - n0) : 32);
    const __nv_bfloat16* vrow = V + ((static_cast<long long>(b) * p.n_cache + n0) * p.hkv + hk) * D + DPL * lane;
    const long long vstride = static_cast<long long>(p.hkv) * D;
#pragma unroll 4
    for (int k = 0; k < nk; ++k) {
      float vf[DPL];
      if (DPL == 4) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(vrow + k * vstride));
        vf[0] = bf16lo_to_f32(w.x);
        vf[1] = bf16hi_to_f32(w.x);
        vf[2] = bf16lo_to_f32(w.y);
        vf[3] = bf16hi_to_f32(w.y);
      } else {
        const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(vrow + k * vstride));
        vf[0] = bf16lo_to_f32(w);
        vf[1] = bf16hi_to_f32(w);
      }
      const float4 pa = *reinterpret_cast<const float4*>(&sP[warp][k][0]);
      const float4 pb = *reinterpret_cast<const float4*>(&sP[warp][k][4]);
      const float pk[8] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
      for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[g][e] = fmaf(pk[g], vf[e], acc[g][e]);
    }
    __syncwarp();
  }

  // merge the warps of this CTA
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float l = lsum[g];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
    if (lane == 0) {
      sM[warp][g] = mrun[g];
      sL[warp][g] = l;
    }
#pragma unroll
    for (int e = 0; e < DPL; ++e) sAcc[warp][g][DPL * lane + e] = acc[g][e];
  }
  __syncthreads();
  float* part = p.partials + ((static_cast<long long>(b) * p.hq + hk * G) * p.n_split + split) * (D + 2);
  for (int idx = tid; idx < G * D; idx += blockDim.x) {
    const int g = idx / D, e = idx % D;
    float M = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, sM[w][g]);
    float a = 0.f, l = 0.f;
    if (M != -INFINITY) {
      for (int w = 0; w < kDecWarps; ++w) {
        if (sM[w][g] == -INFINITY) continue;
        const float f = ex2_approx(sM[w][g] - M);
        a += sAcc[w][g][e] * f;
        l += sL[w][g] * f;
      }
    }
    float* pg = part + static_cast<long long>(g) * p.n_split * (D + 2);
    pg[e] = a;
    if (e == 0) {
      pg[D] = M;
      pg[D + 1] = l;
    }
  }
  if (p.skipped) {
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
  __nv_bfloat16* O = static_cast<__nv_bfloat16*>(p.out) + (static_cast<long long>(b) * p.hq + h) * D;
  O[e] = __float2bfloat16(a / l);
}

int decode_num_splits(long long max_kv_len, int batch, int hkv) {
  const int units = batch * hkv;
  if (units <= 0 || max_kv_len <= 0) return 1;
  // about four CTAs per SM over the 148 SMs, at least 2048 keys per split
  long long ns = (148LL * 4 + units - 1) / units;
  const long long cap = (max_kv_len + 2047) / 2048;
  if (ns > cap) ns = cap;
  if (ns < 1) ns = 1;
  return static_cast<int>(ns);
}

template <int D>
static cudaError_t launch_decode_d(const DecodeParams& p, cudaStream_t s) {
  const int G = p.hq / p.hkv;
  dim3 grid(p.n_split, p.hkv, p.batch);
  switch (G) {
#define ATF_DEC_CASE(g) \
  case g: decode_split_kernel<D, g><<<grid, kDecWarps * 32, 0, s>>>(p); break;
    ATF_DEC_CASE(1)
    ATF_DEC_CASE(2)
    ATF_DEC_CASE(3)
    ATF_DEC_CASE(4)
    ATF_DEC_CASE(5)
    ATF_DEC_CASE(6)
    ATF_DEC_CASE(7)
    ATF_DEC_CASE(8)
#undef ATF_DEC_CASE
    default: return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_combine_kernel<D><<<dim3(p.hq, p.batch), D, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t s) {
  if (p.batch == 0) return cudaSuccess;
  return p.d == 64 ? launch_decode_d<64>(p, s) : launch_decode_d<128>(p, s);
}

}  // namespace atf
