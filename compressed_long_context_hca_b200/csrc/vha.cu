// vha.cu -- the layer's attention output from the heads' attention outputs: the cross-head
// low-rank mixing with an identity skip (Virtual Head Attention, VHA), then the output gate.
//
// [news 二.1] "Virtual Head Attention" and "Low-Rank Gated Attention" paragraphs (and
// [analysis 1], second bullet): after the attention computation the heads' outputs are
// mixed across heads through a light low-rank map with an identity skip, and the attention
// output is multiplied by a learned gate. Reading: per position p and column d,
//   z_r      = sum_g B[g, r] O[p, g, d]                  (rank-r "virtual heads")
//   out[p, h, d] = (O[p, h, d] + sum_r A[h, r] z_r) * G[p, h, d]
// A, B: [hq, rank] float32; the gate is optional (d->gate).
//
// One CTA per position (all heads), one thread per 4 columns: a column's hq head values are
// read once for the virtual heads and once more (L1) for the output. A and B sit in shared
// memory. HBM-bound: O and G are read and out written once.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hca_internal.h"

namespace hca {
namespace {

constexpr int kMaxRank = 16;
constexpr int kMaxHeads = 128;

template <typename T>
__device__ __forceinline__ float ldf(const T* p, int64_t i);
template <>
__device__ __forceinline__ float ldf<float>(const float* p, int64_t i) { return p[i]; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}
template <typename T>
__device__ __forceinline__ T cvt(float v);
template <>
__device__ __forceinline__ float cvt<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 cvt<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

template <typename T>
__global__ void vha_gate_kernel(const T* O, const float* A, const float* B, int rank, int hq,
                                int D, int T_seq, const T* gate, int64_t gs0, int64_t gs1,
                                int64_t gs2, T* out) {
  __shared__ float sA[kMaxHeads * kMaxRank], sB[kMaxHeads * kMaxRank];
  for (int i = threadIdx.x; i < hq * rank; i += blockDim.x) {
    sA[i] = A[i];
    sB[i] = B[i];
  }
  __syncthreads();
  const int64_t pos = blockIdx.x;  // b * T_seq + t
  const int b = (int)(pos / T_seq), t = (int)(pos % T_seq);
  const T* op = O + pos * hq * D;
  T* yp = out + pos * hq * D;
  for (int c = threadIdx.x * 4; c < D; c += blockDim.x * 4) {
    float z[kMaxRank][4];
#pragma unroll
    for (int r = 0; r < kMaxRank; ++r)
#pragma unroll
      for (int e = 0; e < 4; ++e) z[r][e] = 0.f;
    if (rank > 0) {
      for (int g = 0; g < hq; ++g) {
        float o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] = ldf<T>(op, (int64_t)g * D + c + e);
#pragma unroll
        for (int r = 0; r < kMaxRank; ++r) {
          if (r < rank) {
            const float bg = sB[g * rank + r];
#pragma unroll
            for (int e = 0; e < 4; ++e) z[r][e] = fmaf(bg, o[e], z[r][e]);
          }
        }
      }
    }
    for (int h = 0; h < hq; ++h) {
      float y[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) y[e] = ldf<T>(op, (int64_t)h * D + c + e);
#pragma unroll
      for (int r = 0; r < kMaxRank; ++r) {
        if (r < rank) {
          const float ah = sA[h * rank + r];
#pragma unroll
          for (int e = 0; e < 4; ++e) y[e] = fmaf(ah, z[r][e], y[e]);
        }
      }
      if (gate) {
        const int64_t go = (int64_t)b * gs0 + (int64_t)t * gs1 + (int64_t)h * gs2 + c;
#pragma unroll
        for (int e = 0; e < 4; ++e) y[e] *= ldf<T>(gate, go + e);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) yp[(int64_t)h * D + c + e] = cvt<T>(y[e]);
    }
  }
}

}  // namespace

cudaError_t launch_vha_gate(const hca_desc& d, const void* O, const float* A, const float* B,
                            int rank, void* out, cudaStream_t s) {
  const int64_t npos = (int64_t)d.batch * d.seqlen;
  if (npos == 0) return cudaSuccess;
  const int threads = d.head_dim / 4 < 128 ? d.head_dim / 4 : 128;
  if (d.dtype == HCA_F32)
    vha_gate_kernel<float><<<(unsigned)npos, threads, 0, s>>>(
        static_cast<const float*>(O), A, B, rank, d.hq, d.head_dim, d.seqlen,
        static_cast<const float*>(d.gate), d.gate_strides[0], d.gate_strides[1],
        d.gate_strides[2], static_cast<float*>(out));
  else
    vha_gate_kernel<__nv_bfloat16><<<(unsigned)npos, threads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(O), A, B, rank, d.hq, d.head_dim, d.seqlen,
        static_cast<const __nv_bfloat16*>(d.gate), d.gate_strides[0], d.gate_strides[1],
        d.gate_strides[2], static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

}  // namespace hca
