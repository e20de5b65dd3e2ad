// gemm_tc.cu -- C = alpha * A . B^T (+ beta * C) on tcgen05 tensor cores: bf16 operands,
// float32 accumulate, float32 output (or bf16 through a sigmoid: the gate projection from
// the query latent runs on it).
//
// A is M x K and B is N x K in the product's terms; each is stored either K-major (K
// contiguous: a row-major [M, K] / [N, K] array) or MN-major (M or N contiguous: a
// row-major [K, M] / [K, N] array), so that S = Q K^T, dQ = dS K, dK = dS^T Q and the
// like all read their operands where they lie, without a transpose pass.
//
// Design for sm_100a:
//  * One CTA per 128 x 256 output tile (M x N), a K loop in steps of 64 (one 128-byte
//    swizzle row of bf16). Operand tiles arrive through 2-D TMA with 128-byte swizzle into
//    a 4-stage ring (48 KB per stage): a K-major tile as one box (rows x 64 K), an MN-major
//    tile as 64-element chunks of 64 K rows each. Loads past the array edges are zero-filled,
//    so ragged M, N and K need no special case.
//  * Warp 0 issues the TMA loads, warp 1 the UMMAs (M = 128, N = 256, K = 16 each; the
//    accumulator is 256 TMEM columns), warps 2-5 the epilogue: TMEM rows -> registers ->
//    alpha * acc + beta * C -> global, each lane writing 32 consecutive floats of its row.
//  * Batched: grid z is a batch index; every operand's row coordinate (and C's first row)
//    moves by a per-batch stride plus a fixed shift, which is how banded products (a
//    sequence's window keys for a chunk of query rows) run as one launch. Rows of C outside
//    [0, c_rows) are not written. With C's row moving only every c_zdiv batches and atomic
//    accumulation, the batch index also splits a long K over CTAs (split-K).
//  * Every mbarrier wait is bounded; on time-out the CTA sets HCA_ERR_TIMEOUT (bits 8 and up
//    name the role), lets its loads and UMMAs in flight land, and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <string.h>

#include "gemm_tc.h"
#include "hca_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace hca {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr uint32_t kABytes = kBM * kBK * 2;   // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;   // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kMnChunk = 64 * kBK * 2;   // 8 KB: 64 MN elements x 64 K rows
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kOffBar = kStages * kStageBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;

struct Params {
  CUtensorMap tmA, tmB;
  float* C;
  int64_t ldc;
  int32_t M, N, K;
  int32_t a_mn, b_mn;
  // map row of operand element (mn, k): K-major: shift + z * bstride + mn; MN-major:
  // shift + z * bstride + k
  int32_t a_shift, a_bstride, b_shift, b_bstride;
  // C row of tile row m: c_shift + (z / c_zdiv) * c_bstride + m, written if in [0, c_rows)
  int32_t c_shift, c_bstride, c_zdiv, c_rows;
  int32_t atomic;  // C += alpha * acc with float32 atomics (split-K, overlapping bands)
  int32_t sigmoid_bf16;  // C = bf16(sigmoid(alpha * acc)), C a bf16 array
  float alpha, beta;
  int32_t* err_word;
};

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t done, drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ uint32_t idesc_f16(bool a_mn, bool b_mn) {
  // bf16 x bf16 -> f32, M = 128, N = 256; bit 15: A major, bit 16: B major (1 = MN)
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int n0 = blockIdx.x * kBN;
  const int m0 = blockIdx.y * kBM;
  const int z = blockIdx.z;
  const int nk = (p.K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (elect_one()) {
      tma_prefetch_desc(&p.tmA);
      tma_prefetch_desc(&p.tmB);
      bool ok = true;
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kStages;
        const int round = kb / kStages;
        if (round > 0 && !(ok = mbar_wait(&bars->empty[s], (round - 1) & 1, abort))) break;
        mbar_expect_tx(&bars->full[s], kStageBytes);
        uint8_t* sa = smem + s * kStageBytes;
        uint8_t* sb = sa + kABytes;
        const int k0 = kb * kBK;
        if (p.a_mn) {
          const int row = p.a_shift + z * p.a_bstride + k0;
          tma_load_2d_hint(sa, &p.tmA, &bars->full[s], m0, row);
          tma_load_2d_hint(sa + kMnChunk, &p.tmA, &bars->full[s], m0 + 64, row);
        } else {
          tma_load_2d_hint(sa, &p.tmA, &bars->full[s], k0, p.a_shift + z * p.a_bstride + m0);
        }
        if (p.b_mn) {
          const int row = p.b_shift + z * p.b_bstride + k0;
#pragma unroll
          for (int c = 0; c < kBN / 64; ++c)
            tma_load_2d_hint(sb + c * kMnChunk, &p.tmB, &bars->full[s], n0 + 64 * c, row);
        } else {
          tma_load_2d_hint(sb, &p.tmB, &bars->full[s], k0, p.b_shift + z * p.b_bstride + n0);
        }
        ++issued;
      }
      if (!ok) {
        bars->abort = 1;
        if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << 8));
        volatile int no_abort = 0;  // let the loads in flight land
        for (int kb = issued > kStages ? issued - kStages : 0; kb < issued; ++kb)
          mbar_wait(&bars->full[kb % kStages], (kb / kStages) & 1, &no_abort, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ UMMA issuer
    if (elect_one()) {
      const uint32_t idesc = idesc_f16(p.a_mn != 0, p.b_mn != 0);
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kStages;
        if (!(ok = mbar_wait(&bars->full[s], (kb / kStages) & 1, abort))) break;
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * kStageBytes);
        const uint32_t sb = sa + kABytes;
        // K-major: one 128-byte row per operand row, 16 K elements = 32 bytes along it.
        // MN-major: 64-element chunks (LBO = 8 KB apart) of 64 K rows, 16 K rows = 2 KB.
        const uint64_t ad = p.a_mn ? sdesc_sw128(sa, kMnChunk, 1024) : sdesc_sw128(sa, 16, 1024);
        const uint64_t bd = p.b_mn ? sdesc_sw128(sb, kMnChunk, 1024) : sdesc_sw128(sb, 16, 1024);
        const uint32_t astep = p.a_mn ? (2048 >> 4) : (32 >> 4);
        const uint32_t bstep = p.b_mn ? (2048 >> 4) : (32 >> 4);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_ss(tmem, ad + kk * astep, bd + kk * bstep, idesc, (kb | kk) != 0);
        umma_commit(&bars->empty[s]);
      }
      if (ok) {
        umma_commit(&bars->done);
      } else {
        bars->abort = 1;
        if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << 9));
      }
      volatile int no_abort = 0;
      umma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, &no_abort, 100000000ull);
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;
    const bool ok = nk == 0 || mbar_wait(&bars->done, 0, abort);
    if (!ok) {
      if (lane == 0 && p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << 10));
    } else {
      tc_fence_after();
      const int m = m0 + row;
      const int64_t crow = (int64_t)p.c_shift + (int64_t)(z / p.c_zdiv) * p.c_bstride + m;
      const bool valid = m < p.M && crow >= 0 && crow < p.c_rows;
      float* cp = p.C + crow * p.ldc;
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16);
#pragma unroll 1
      for (int q = 0; q < kBN / 32; ++q) {
        uint32_t v[32];
        if (nk > 0) {
          tmem_ld32(taddr + q * 32, v);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = 0u;
        }
        const int c0 = n0 + q * 32;
        if (!valid || c0 >= p.N) continue;
        if (p.sigmoid_bf16) {
          __nv_bfloat16* bp = reinterpret_cast<__nv_bfloat16*>(p.C) + crow * p.ldc;
          float g[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) g[e] = 1.f / (1.f + __expf(-p.alpha * __uint_as_float(v[e])));
          if (c0 + 32 <= p.N && (p.ldc & 7) == 0) {
#pragma unroll
            for (int w = 0; w < 4; ++w)
              *reinterpret_cast<uint4*>(bp + c0 + 8 * w) =
                  make_uint4(pack_bf16x2(g[8 * w], g[8 * w + 1]), pack_bf16x2(g[8 * w + 2], g[8 * w + 3]),
                             pack_bf16x2(g[8 * w + 4], g[8 * w + 5]),
                             pack_bf16x2(g[8 * w + 6], g[8 * w + 7]));
          } else {
            for (int e = 0; e < 32 && c0 + e < p.N; ++e) bp[c0 + e] = __float2bfloat16_rn(g[e]);
          }
        } else if (p.atomic) {
          if (c0 + 32 <= p.N && (p.ldc & 3) == 0) {
#pragma unroll
            for (int w = 0; w < 8; ++w)
              atomicAdd(reinterpret_cast<float4*>(cp + c0) + w,
                        make_float4(p.alpha * __uint_as_float(v[4 * w]),
                                    p.alpha * __uint_as_float(v[4 * w + 1]),
                                    p.alpha * __uint_as_float(v[4 * w + 2]),
                                    p.alpha * __uint_as_float(v[4 * w + 3])));
          } else {
            for (int e = 0; e < 32 && c0 + e < p.N; ++e)
              atomicAdd(cp + c0 + e, p.alpha * __uint_as_float(v[e]));
          }
        } else if (c0 + 32 <= p.N && (p.ldc & 3) == 0) {
          float4* dst = reinterpret_cast<float4*>(cp + c0);
#pragma unroll
          for (int w = 0; w < 8; ++w) {
            float4 x = make_float4(p.alpha * __uint_as_float(v[4 * w]),
                                   p.alpha * __uint_as_float(v[4 * w + 1]),
                                   p.alpha * __uint_as_float(v[4 * w + 2]),
                                   p.alpha * __uint_as_float(v[4 * w + 3]));
            if (p.beta != 0.f) {
              const float4 o = dst[w];
              x.x = fmaf(p.beta, o.x, x.x);
              x.y = fmaf(p.beta, o.y, x.y);
              x.z = fmaf(p.beta, o.z, x.z);
              x.w = fmaf(p.beta, o.w, x.w);
            }
            dst[w] = x;
          }
        } else {
          for (int e = 0; e < 32 && c0 + e < p.N; ++e) {
            float x = p.alpha * __uint_as_float(v[e]);
            if (p.beta != 0.f) x = fmaf(p.beta, cp[c0 + e], x);
            cp[c0 + e] = x;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// 2-D bf16 map over a row-major [rows, cols] array, 128-byte swizzle, box {64, box_rows}
cudaError_t map_2d(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld,
                   uint32_t box_rows) {
  return encode_bf16_2d(m, base, (uint64_t)(rows > 0 ? rows : 1), (uint64_t)cols,
                        (uint64_t)ld, 64, box_rows);
}

}  // namespace

cudaError_t gemm_tc(const GemmOperand& A, const GemmOperand& B, const GemmOutput& C, int M,
                    int N, int K, int batch, float alpha, float beta, int32_t* err_word,
                    cudaStream_t s) {
  if (C.zdiv < 1) return cudaErrorInvalidValue;
  if (M <= 0 || N <= 0 || batch <= 0) return cudaSuccess;
  Params p;
  memset(&p, 0, sizeof(p));
  cudaError_t e;
  // K-major: the map's columns are K, a box is 128 (A) / 256 (B) rows of 64 K elements.
  // MN-major: the map's columns are M / N, a box is 64 K rows of 64 MN elements.
  if ((e = map_2d(&p.tmA, A.ptr, A.rows, A.cols, A.ld, A.mn_major ? kBK : kBM)) != cudaSuccess)
    return e;
  if ((e = map_2d(&p.tmB, B.ptr, B.rows, B.cols, B.ld, B.mn_major ? kBK : kBN)) != cudaSuccess)
    return e;
  p.C = C.ptr;
  p.ldc = C.ld;
  p.M = M;
  p.N = N;
  p.K = K;
  p.a_mn = A.mn_major ? 1 : 0;
  p.b_mn = B.mn_major ? 1 : 0;
  p.a_shift = A.shift;
  p.a_bstride = A.bstride;
  p.b_shift = B.shift;
  p.b_bstride = B.bstride;
  p.c_shift = C.shift;
  p.c_bstride = C.bstride;
  p.c_zdiv = C.zdiv;
  p.c_rows = C.rows;
  p.atomic = C.atomic ? 1 : 0;
  p.sigmoid_bf16 = C.sigmoid_bf16 ? 1 : 0;
  p.alpha = alpha;
  p.beta = beta;
  p.err_word = err_word;
  static PerDevice<int> smem_limit_set;
  if ((e = set_smem_limit_once(smem_limit_set, (const void*)gemm_tc_kernel, (int)kSmemBytes)) !=
      cudaSuccess)
    return e;
  dim3 grid((N + kBN - 1) / kBN, (M + kBM - 1) / kBM, batch);
  gemm_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace hca
