// prefill_simt.cu -- fp32 prefill on the CUDA cores, for fp32 inputs.
//
// Per-pair windowed causal attention ("ATFlash: RoPE-Frequenzen kuerzen
// Attention-Arbeit um bis zu 57 Prozent", sudo-ai.de, section "Was ATFlash
// anders macht"): the logit of query m and key n <= m sums, over the frequency
// pairs i whose window W_i >= m - n, the pair's product of rotated q and k,
// scaled by 1/sqrt(d); a key with no active pair gets the logit 0.  Softmax and
// P.V are the ordinary online recurrence (section "Die Zahlen - und ihre
// Grenze": the recurrence is not rebuilt).
//
// Tensor-core MMA is not used here: tf32 rounding of q and k (10-bit mantissa)
// would exceed a 1e-4 output tolerance, so the contraction runs in fp32 FFMA.
// Two threads share a query row, each owning half of the head dimension.
#include "atf_internal.cuh"

namespace atf {

template <int D>
__global__ void __launch_bounds__(128) prefill_simt_kernel(PrefillParams p) {
  constexpr int HALF = D / 2;   // dims per thread
  constexpr int ROWS = 64;      // query rows per block
  constexpr int KT = 32;        // keys per shared-memory tile
  __shared__ float sK[KT][D];
  __shared__ float sV[KT][D];
  __shared__ int sW[D / 2];

  const int tid = threadIdx.x;
  const int r = tid >> 1, hf = tid & 1;
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (p.hq / p.hkv);
  const int t = blockIdx.x * ROWS + r;
  const long long m = p.q_offset + t;
  const bool row_ok = t < p.q_len;
  for (int i = tid; i < D / 2; i += blockDim.x) sW[i] = p.win.w[i];

  const float* Q = static_cast<const float*>(p.q);
  const float* K = static_cast<const float*>(p.k);
  const float* V = static_cast<const float*>(p.v);
  float q[HALF], acc[HALF];
#pragma unroll
  for (int e = 0; e < HALF; ++e) {
    q[e] = row_ok ? Q[(((long long)b * p.q_len + t) * p.hq + h) * D + hf * HALF + e] : 0.f;
    acc[e] = 0.f;
  }
  float mrun = -INFINITY, l = 0.f;
  unsigned long long cnt = 0;
  const float scale = rsqrtf(static_cast<float>(D));

  const int t_last = min(p.q_len, (int)(blockIdx.x + 1) * ROWS) - 1;
  const long long n_last = min(p.q_offset + t_last, (long long)p.kv_len - 1);
  for (long long n0 = 0; n0 <= n_last; n0 += KT) {
    __syncthreads();
    for (int e = tid; e < KT * D; e += blockDim.x) {
      const int kk = e / D, dd = e % D;
      const long long n = n0 + kk;
      const long long gi = (((long long)b * p.kv_len + n) * p.hkv + hk) * D + dd;
      sK[kk][dd] = n < p.kv_len ? K[gi] : 0.f;
      sV[kk][dd] = n < p.kv_len ? V[gi] : 0.f;
    }
    __syncthreads();
    for (int kk = 0; kk < KT; ++kk) {
      const long long n = n0 + kk;
      const bool ok = row_ok && n <= m && n < p.kv_len;
      const long long delta = m - n;
      float part = 0.f;
      int inactive = 0;
#pragma unroll
      for (int j = 0; j < HALF / 2; ++j) {
        const int i = hf * (HALF / 2) + j;  // pair index
        if (delta <= sW[i]) {
          part = fmaf(q[2 * j], sK[kk][2 * i], part);
          part = fmaf(q[2 * j + 1], sK[kk][2 * i + 1], part);
        } else {
          ++inactive;
        }
      }
      const float s = (part + __shfl_xor_sync(0xffffffffu, part, 1)) * scale;
      if (ok) {
        cnt += inactive;
        const float mnew = fmaxf(mrun, s);
        const float corr = expf(mrun - mnew);
        const float pe = expf(s - mnew);
        l = l * corr + pe;
#pragma unroll
        for (int e = 0; e < HALF; ++e) acc[e] = fmaf(pe, sV[kk][hf * HALF + e], acc[e] * corr);
        mrun = mnew;
      }
    }
  }
  if (row_ok) {
    float* O = static_cast<float*>(p.out) + (((long long)b * p.q_len + t) * p.hq + h) * D + hf * HALF;
    const float inv = 1.f / l;
#pragma unroll
    for (int e = 0; e < HALF; ++e) O[e] = acc[e] * inv;
  }
  if (p.skipped) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if ((tid & 31) == 0 && cnt) atomicAdd(p.skipped, cnt);
  }
}

cudaError_t launch_prefill_simt(const PrefillParams& p, cudaStream_t s) {
  if (p.q_len == 0 || p.batch == 0) return cudaSuccess;
  dim3 grid((p.q_len + 63) / 64, p.hq, p.batch);
  if (p.d == 64)
    prefill_simt_kernel<64><<<grid, 128, 0, s>>>(p);
  else
    prefill_simt_kernel<128><<<grid, 128, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace atf
