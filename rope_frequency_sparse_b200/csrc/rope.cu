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
// One thread per (token, 8-pair chunk, group of 4 heads): it evaluates the
// chunk's eight angles once in fp64 and moves each head's 16 chunk elements with
// 16-byte loads and stores.  The copy modes move the bits unchanged.
#include <cuda_bf16.h>

#include "atf_internal.cuh"

namespace atf {

namespace {

constexpr int kHeadsPerThread = 4;

// element k (< 16) of a chunk held as 16 values
struct Chunk16 {
  double v[16];
};

// Load the 16 elements of pair chunk c of one head row: interleaved layout
// (elements 16c..16c+15 = a0 b0 a1 b1 ...) or rotate-half (a = dims 8c.., b =
// dims d/2 + 8c..), returned as a[k] = v[2k], b[k] = v[2k+1].
__device__ __forceinline__ void load_chunk(const void* base, long long row_elem, int c, int d, bool half_pairs,
                                           bool fp32, Chunk16& x) {
  if (fp32) {
    const float* f = static_cast<const float*>(base) + row_elem;
    if (half_pairs) {
      const float4* a = reinterpret_cast<const float4*>(f + 8 * c);
      const float4* bb = reinterpret_cast<const float4*>(f + d / 2 + 8 * c);
      const float4 a0 = a[0], a1 = a[1], b0 = bb[0], b1 = bb[1];
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        x.v[2 * k] = av[k];
        x.v[2 * k + 1] = bv[k];
      }
    } else {
      const float4* q = reinterpret_cast<const float4*>(f + 16 * c);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 t = q[j];
        x.v[4 * j] = t.x;
        x.v[4 * j + 1] = t.y;
        x.v[4 * j + 2] = t.z;
        x.v[4 * j + 3] = t.w;
      }
    }
  } else {
    const __nv_bfloat16* h = static_cast<const __nv_bfloat16*>(base) + row_elem;
    uint32_t w[8];
    if (half_pairs) {
      const uint4 a = *reinterpret_cast<const uint4*>(h + 8 * c);
      const uint4 bb = *reinterpret_cast<const uint4*>(h + d / 2 + 8 * c);
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t ea = (k & 1) ? (aw[k >> 1] >> 16) : (aw[k >> 1] & 0xFFFFu);
        const uint32_t eb = (k & 1) ? (bw[k >> 1] >> 16) : (bw[k >> 1] & 0xFFFFu);
        w[k] = ea | (eb << 16);
      }
    } else {
      const uint4 q0 = *reinterpret_cast<const uint4*>(h + 16 * c);
      const uint4 q1 = *reinterpret_cast<const uint4*>(h + 16 * c + 8);
      w[0] = q0.x; w[1] = q0.y; w[2] = q0.z; w[3] = q0.w;
      w[4] = q1.x; w[5] = q1.y; w[6] = q1.z; w[7] = q1.w;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      x.v[2 * k] = __uint_as_float(w[k] << 16);
      x.v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(256) rope_kernel(RopeParams p) {
  __shared__ double s_omega[kMaxPairs];
  const int half = p.d / 2, nchunk = p.d / 16;
  for (int i = threadIdx.x; i < half; i += blockDim.x) s_omega[i] = p.omega[i];
  __syncthreads();

  const int hgroups = (p.heads + kHeadsPerThread - 1) / kHeadsPerThread;
  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long rows = static_cast<long long>(p.batch) * p.seq;
  if (g >= rows * nchunk * hgroups) return;
  const int c = static_cast<int>(g % nchunk);
  const int hg = static_cast<int>((g / nchunk) % hgroups);
  const long long row = g / nchunk / hgroups;  // b * seq + t
  const int t = static_cast<int>(row % p.seq);
  const int b = static_cast<int>(row / p.seq);
  const bool rotate = p.rotate == 1 || p.rotate == 2;
  const bool half_pairs = p.rotate >= 2;  // dims of pair i: (i, i + d/2)

  double cs[8], sn[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    cs[k] = 1.0;
    sn[k] = 0.0;
    if (rotate) sincos(static_cast<double>(p.pos_offset + t) * s_omega[8 * c + k], &sn[k], &cs[k]);
  }
  const int h_end = min(p.heads, (hg + 1) * kHeadsPerThread);
  for (int h = hg * kHeadsPerThread; h < h_end; ++h) {
    const long long re = (row * p.heads + h) * p.d;  // element index of the head row
    Chunk16 x;
    load_chunk(p.x, re, c, p.d, half_pairs, p.fp32, x);
    if (p.fp32) {
      float y[16];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        // fp32 input: one rounding of the fp64 rotation to fp32 (identity when not rotating)
        y[2 * k] = rotate ? static_cast<float>(x.v[2 * k] * cs[k] - x.v[2 * k + 1] * sn[k]) : x.v[2 * k];
        y[2 * k + 1] = rotate ? static_cast<float>(x.v[2 * k] * sn[k] + x.v[2 * k + 1] * cs[k]) : x.v[2 * k + 1];
      }
      if (p.x_rot) {
        float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.x_rot) + re + 16 * c);
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
      }
    } else {
      uint32_t o[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (rotate) {
          // one rounding: fp64 -> bf16 (round to nearest even)
          const __nv_bfloat16 y0 = __double2bfloat16(x.v[2 * k] * cs[k] - x.v[2 * k + 1] * sn[k]);
          const __nv_bfloat16 y1 = __double2bfloat16(x.v[2 * k] * sn[k] + x.v[2 * k + 1] * cs[k]);
          o[k] = static_cast<uint32_t>(__bfloat16_as_ushort(y0)) |
                 (static_cast<uint32_t>(__bfloat16_as_ushort(y1)) << 16);
        } else {  // the bits as they are
          o[k] = (__float_as_uint(static_cast<float>(x.v[2 * k])) >> 16) |
                 (__float_as_uint(static_cast<float>(x.v[2 * k + 1])) & 0xFFFF0000u);
        }
      }
      if (p.x_rot) {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.x_rot) + re + 16 * c);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
      if (p.x_chunked) {
        const long long ce = ((((long long)b * p.heads + h) * nchunk + c) * p.seq + t) * 16;
        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.x_chunked) + ce);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
      }
    }
  }
}

cudaError_t launch_rope(const RopeParams& p, cudaStream_t s) {
  const long long hgroups = (p.heads + kHeadsPerThread - 1) / kHeadsPerThread;
  const long long total = static_cast<long long>(p.batch) * p.seq * (p.d / 16) * hgroups;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  rope_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace atf
