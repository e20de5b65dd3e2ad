// decode_softmax.cuh -- the per-row P pieces of the decode kernels' softmax.
//
// With M = 64 score rows in TMEM lanes 16-31 of each 32-lane subpartition, the softmax warp
// of a subpartition holds row quad * 16 + l in lane l + 16 and the O row of the same head in
// lane l. For the exponentials all 32 lanes work: of each 32-column piece of a score row,
// lane l + 16 takes columns 0..15 and lane l columns 16..31, handed over by a shuffle.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "sm100.cuh"

namespace hca {
namespace dsoft {

// two floats -> f16x2 (round to nearest even), `a` in the low half
__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// the 16 scores this lane turns into P, from a 32-column piece loaded by all 32 lanes
// (v: 32 consecutive columns of TMEM lane `lane`): lane l + 16 keeps columns 0..15 of its
// row, lane l (< 16) receives columns 16..31 of lane l + 16's row
__device__ __forceinline__ void pair_split(const uint32_t (&v)[32], bool s_lane,
                                           float (&x)[16]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const uint32_t o = __shfl_xor_sync(0xffffffffu, v[16 + e], 16);
    x[e] = __uint_as_float(s_lane ? v[e] : o);
  }
}

enum PKind { kPF16 = 0, kPBf16Pair = 1, kPBf16PairScaled = 2 };

// P of the 16 columns col0 .. col0 + 15 of one score row: 2^(x * rs - bb), 0 at columns
// >= vlen when kMask. kPF16: f16 pairs in pk. kPBf16Pair: bf16 hi + lo pairs of P (hi in pk,
// lo = bf16(P - hi) in pl); kPBf16PairScaled: the same of P * vscale. Returns the sum of
// the 16 P values (unscaled).
template <bool kMask, int kKind>
__device__ __forceinline__ float p_piece(const float (&x)[16], float rs, float bb, int col0,
                                         uint32_t vlen, float vscale, uint32_t (&pk)[8],
                                         uint32_t (&pl)[8]) {
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    float p0 = fast_exp2(fmaf(x[2 * e], rs, -bb));
    float p1 = fast_exp2(fmaf(x[2 * e + 1], rs, -bb));
    if (kMask) {
      p0 = (uint32_t)(col0 + 2 * e) < vlen ? p0 : 0.f;
      p1 = (uint32_t)(col0 + 2 * e + 1) < vlen ? p1 : 0.f;
    }
    if (kKind == kPF16)
      pk[e] = pack_f16x2(p0, p1);
    else if (kKind == kPBf16Pair)
      split_bf16x2(p0, p1, pk[e], pl[e]);
    else
      split_bf16x2(p0 * vscale, p1 * vscale, pk[e], pl[e]);
    s0 += p0;
    s1 += p1;
  }
  return s0 + s1;
}

}  // namespace dsoft
}  // namespace hca
