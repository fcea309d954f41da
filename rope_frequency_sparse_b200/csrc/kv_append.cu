// kv_append.cu -- write new tokens into the decode caches: keys rotated at their
// positions into the pair-chunk-major key cache, values copied into the
// token-major value cache.
//
// "ATFlash: RoPE-Frequenzen kuerzen Attention-Arbeit um bis zu 57 Prozent"
// (sudo-ai.de), section "Was ATFlash anders macht": the decode attention reads
// rotated keys, and for far keys only their low-frequency pairs; the cache keeps
// each 8-pair chunk of consecutive tokens contiguous so that those reads are
// whole 32-byte rows.  This kernel maintains that layout one step at a time.
//
// One thread per (new token, 8-pair chunk c): it evaluates the chunk's eight
// rotation angles once in fp64 and serves every kv head, four heads at a time: it
// loads their chunk's 16 key elements and 16 values with 16-byte loads, then
// rotates the keys in fp64, rounds each once to bf16 (the same values the one-shot
// RoPE kernel produces) and stores the chunk's 32-byte rows of both caches.
#include <cuda_bf16.h>

#include "atf_internal.cuh"

namespace atf {

namespace {

__device__ __forceinline__ double bf16_elem(const uint4& v, int k) {  // element k of 8 packed bf16
  const uint32_t w = (k >> 1) == 0 ? v.x : (k >> 1) == 1 ? v.y : (k >> 1) == 2 ? v.z : v.w;
  return static_cast<double>(__uint_as_float((k & 1) ? (w & 0xFFFF0000u) : (w << 16)));
}

}  // namespace

__global__ void __launch_bounds__(128) kv_append_kernel(AppendParams p) {
  __shared__ double s_omega[kMaxPairs];
  __shared__ long long s_cu[kMaxDecodeBatch + 1];
  const int half = p.d / 2, nchunk = p.d / 16;
  for (int i = threadIdx.x; i < half; i += blockDim.x) s_omega[i] = p.omega[i];
  for (int i = threadIdx.x; i <= p.batch; i += blockDim.x) s_cu[i] = p.cu[i];
  __syncthreads();

  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= s_cu[p.batch] * nchunk) return;
  const int c = static_cast<int>(g % nchunk);  // pairs 8c .. 8c+7
  const long long tok = g / nchunk;            // row in k_new / v_new
  int b = 0;
  while (b + 1 < p.batch && s_cu[b + 1] <= tok) ++b;  // sequence of this row
  const long long slot = p.pos[b] + (tok - s_cu[b]);   // its position and cache slot

  const uint4* K = static_cast<const uint4*>(p.k_new);  // 8 bf16 per uint4
  const uint4* V = static_cast<const uint4*>(p.v_new);
  uint4* KC = static_cast<uint4*>(p.kc);
  uint4* VC = static_cast<uint4*>(p.vc);
  const int row16 = p.d / 8;  // uint4 per head row
  constexpr int kHeads = 4;   // heads whose loads are issued together
  double cs[8], sn[8];
  for (int h0 = 0; h0 < p.hkv; h0 += kHeads) {
    // the chunk's key and value elements of up to kHeads heads, loaded before any
    // store (the caches could alias the inputs as far as the compiler knows)
    uint4 xa[kHeads], xb[kHeads], va[kHeads], vb[kHeads];
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh) {
      if (h0 + hh >= p.hkv) break;
      const long long row = (tok * p.hkv + h0 + hh) * row16;
      // interleaved: elements 16c..16c+15 = (a0 b0 a1 b1 ...); rotate-half: the a and b halves
      xa[hh] = p.pairing ? K[row + c] : K[row + 2 * c];
      xb[hh] = p.pairing ? K[row + p.d / 16 + c] : K[row + 2 * c + 1];
      va[hh] = V[row + 2 * c];
      vb[hh] = V[row + 2 * c + 1];
    }
    if (h0 == 0) {  // the chunk's eight angles, once, while the first loads are in flight
#pragma unroll
      for (int k = 0; k < 8; ++k) sincos(static_cast<double>(slot) * s_omega[8 * c + k], &sn[k], &cs[k]);
    }
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh) {
      const int h = h0 + hh;
      if (h >= p.hkv) break;
      uint32_t o[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        double x0, x1;
        if (p.pairing) {
          x0 = bf16_elem(xa[hh], k);
          x1 = bf16_elem(xb[hh], k);
        } else {
          x0 = bf16_elem(k < 4 ? xa[hh] : xb[hh], (2 * k) & 7);
          x1 = bf16_elem(k < 4 ? xa[hh] : xb[hh], (2 * k + 1) & 7);
        }
        const __nv_bfloat16 y0 = __double2bfloat16(x0 * cs[k] - x1 * sn[k]);
        const __nv_bfloat16 y1 = __double2bfloat16(x0 * sn[k] + x1 * cs[k]);
        o[k] = static_cast<uint32_t>(__bfloat16_as_ushort(y0)) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(y1)) << 16);
      }
      const long long ce = ((((long long)b * p.hkv + h) * nchunk + c) * p.n_cache + slot) * 2;  // uint4 index
      KC[ce] = make_uint4(o[0], o[1], o[2], o[3]);
      KC[ce + 1] = make_uint4(o[4], o[5], o[6], o[7]);
      // values: dims 16c .. 16c+15 of this head, token-major
      const long long vd = (((long long)b * p.n_cache + slot) * p.hkv + h) * row16 + 2 * c;
      VC[vd] = va[hh];
      VC[vd + 1] = vb[hh];
    }
  }
}

cudaError_t launch_kv_append(const AppendParams& p, cudaStream_t s) {
  const long long total = p.cu[p.batch] * (p.d / 16);
  if (total == 0) return cudaSuccess;
  const int threads = 128;
  const long long blocks = (total + threads - 1) / threads;
  kv_append_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace atf
