// rope.cu -- RoPE rotation plus the pair-chunk-major key layout.
//
// "ATFlash: RoPE-Frequenzen kuerzen Attention-Arbeit um bis zu 57 Prozent"
// (sudo-ai.de), section "Was ATFlash anders macht": RoPE encodes position as
// 2-D rotations at several frequencies.  Pair i = (x_{2i}, x_{2i+1}) of a token
// at position p is rotated by the angle p*omega_i, omega_i = theta^(-2i/d):
//   x~_{2i} = x_{2i} cos - x_{2i+1} sin,  x~_{2i+1} = x_{2i} sin + x_{2i+1} cos.
// The angle and the rotation are evaluated in fp64 (positions reach 2^20 and
// beyond, where an fp32 angle would be off by more than the bf16 step), and the
// result is rounded once to the output type.
//
// Rotate-half checkpoints (NeoX style, e.g. the Qwen2.5 family) pair dims
// (i, i + d/2) instead.  The attention kernels only ever take dot products of a
// rotated query with rotated keys, so for them any consistent order of the
// dimensions is the same: in the rotate-half modes this kernel writes pair i to
// slots (2i, 2i+1) of its outputs, the interleaved order the kernels read.
//
// Pair-chunk-major layout: the decode kernel reads, for far keys, only the
// low-frequency pairs.  Keys are therefore also written as
// [batch][head][chunk c = d/16][token][16 elements] so that one chunk of 8
// pairs for consecutive tokens is one contiguous run of 32-byte rows.
#include <cuda_bf16.h>

#include "atf_internal.cuh"

namespace atf {

__global__ void __launch_bounds__(256) rope_kernel(RopeParams p) {
  __shared__ double s_omega[kMaxPairs];
  const int half = p.d / 2;
  for (int i = threadIdx.x; i < half; i += blockDim.x) s_omega[i] = p.omega[i];
  __syncthreads();

  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rows = static_cast<long long>(p.batch) * p.seq;
  if (g >= rows * half) return;
  const int i = static_cast<int>(g % half);
  const long long row = g / half;  // b * seq + t
  const int t = static_cast<int>(row % p.seq);
  const int b = static_cast<int>(row / p.seq);

  // dims of pair i in the input: (2i, 2i+1), or (i, i + d/2) in the rotate-half modes
  const bool half_pairs = p.rotate >= 2;
  double c = 1.0, s = 0.0;
  if (p.rotate == 1 || p.rotate == 2) {
    const double phi = static_cast<double>(p.pos_offset + t) * s_omega[i];
    sincos(phi, &s, &c);
  }
  const int nchunk = p.d / 16;
  for (int h = 0; h < p.heads; ++h) {
    const long long e = (row * p.heads + h) * p.d + 2 * i;  // output slots (2i, 2i+1)
    double x0, x1;
    if (half_pairs) {
      const long long ea = (row * p.heads + h) * p.d + i, eb = ea + p.d / 2;
      if (p.fp32) {
        x0 = static_cast<const float*>(p.x)[ea];
        x1 = static_cast<const float*>(p.x)[eb];
      } else {
        x0 = __bfloat162float(static_cast<const __nv_bfloat16*>(p.x)[ea]);
        x1 = __bfloat162float(static_cast<const __nv_bfloat16*>(p.x)[eb]);
      }
    } else if (p.fp32) {
      const float2 v = *reinterpret_cast<const float2*>(static_cast<const float*>(p.x) + e);
      x0 = v.x;
      x1 = v.y;
    } else {
      const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(static_cast<const __nv_bfloat16*>(p.x) + e);
      x0 = __bfloat162float(v.x);
      x1 = __bfloat162float(v.y);
    }
    const double y0 = x0 * c - x1 * s;
    const double y1 = x0 * s + x1 * c;
    if (p.fp32) {
      if (p.x_rot) *reinterpret_cast<float2*>(static_cast<float*>(p.x_rot) + e) = make_float2((float)y0, (float)y1);
    } else {
      // one rounding: fp64 -> bf16 (round to nearest even)
      __nv_bfloat162 o;
      o.x = __double2bfloat16(y0);
      o.y = __double2bfloat16(y1);
      if (p.x_rot) *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.x_rot) + e) = o;
      if (p.x_chunked) {
        const long long ce = ((((long long)b * p.heads + h) * nchunk + i / 8) * p.seq + t) * 16 + 2 * (i % 8);
        *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.x_chunked) + ce) = o;
      }
    }
  }
}

cudaError_t launch_rope(const RopeParams& p, cudaStream_t s) {
  const long long total = static_cast<long long>(p.batch) * p.seq * (p.d / 2);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  rope_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace atf
