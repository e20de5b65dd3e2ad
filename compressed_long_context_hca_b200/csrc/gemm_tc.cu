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
//  * Persistent CTAs (one per SM), each walking the output tiles (128 x 256, M x N; N tiles
//    fastest so neighbouring CTAs share an A tile in L2) in a static stride. A K loop in
//    steps of 64 (one 128-byte swizzle row of bf16). Operand tiles arrive through 2-D TMA
//    with 128-byte swizzle into a ring: a K-major tile as one box (rows x 64 K), an MN-major
//    tile as 64-element chunks of 64 K rows each. Loads past the array edges are zero-filled,
//    so ragged M, N and K need no special case.
//  * Optional second A operand (the low part of a bf16 pair A = A_hi + A_lo): both A tiles
//    and one B tile per ring stage, two UMMAs into the same accumulator, so a pair product
//    costs one launch, one B stream and one epilogue.
//  * Warp 0 issues the TMA loads, warp 1 the UMMAs (M = 128, N = 256, K = 16 each), warps
//    2-5 the epilogue. The accumulator is double-buffered in TMEM (2 x 256 columns): the
//    epilogue of tile i (TMEM -> registers -> alpha * acc + beta * C -> global, each lane
//    writing 32 consecutive floats of its row) overlaps the K loop of tile i + 1.
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
constexpr uint32_t kABytes = kBM * kBK * 2;   // 16 KB
constexpr uint32_t kBBytes = kBN * kBK * 2;   // 32 KB
// the ring: 4 stages of A, B (48 KB) or, with the second A operand, 3 of A, A_lo, B (64 KB)
constexpr int kStagesMax = 4;
constexpr uint32_t kRingBytes = 4 * (kABytes + kBBytes);
static_assert(3 * (2 * kABytes + kBBytes) == kRingBytes, "both rings fill the same space");
constexpr uint32_t kMnChunk = 64 * kBK * 2;   // 8 KB: 64 MN elements x 64 K rows
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;           // two 256-column accumulators
constexpr uint32_t kOffBar = kRingBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;

struct Params {
  CUtensorMap tmA, tmA2, tmB;
  int32_t has_a2;
  float* C;
  int64_t ldc;
  int32_t M, N, K, batch;
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
  uint64_t full[kStagesMax], empty[kStagesMax];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
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

// One 32-column piece of an epilogue row: alpha * acc (+ beta * C), atomically added, or
// through the sigmoid into bf16.
__device__ __forceinline__ void store_piece(const Params& p, float* cp, int64_t crow, int c0,
                                            const uint32_t (&v)[32]) {
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
    return;
  }
  if (p.atomic) {
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
    return;
  }
  if (c0 + 32 <= p.N && (p.ldc & 3) == 0) {
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

__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int nk = (p.K + kBK - 1) / kBK;
  const int tiles_n = (p.N + kBN - 1) / kBN;
  const int tiles_mn = tiles_n * ((p.M + kBM - 1) / kBM);
  const int ntiles = tiles_mn * p.batch;
  const uint32_t stage_bytes = (p.has_a2 ? 2 * kABytes : kABytes) + kBBytes;
  const int kStages = p.has_a2 ? 3 : 4;
  const uint32_t kStageBytes = stage_bytes;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesMax; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], 4);  // the four epilogue warps
    }
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
      if (p.has_a2) tma_prefetch_desc(&p.tmA2);
      tma_prefetch_desc(&p.tmB);
      bool ok = true;
      uint32_t cnt = 0;  // stages filled, over all tiles
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
        const int z = tile / tiles_mn, rem = tile % tiles_mn;
        const int m0 = (rem / tiles_n) * kBM, n0 = (rem % tiles_n) * kBN;
        for (int kb = 0; kb < nk; ++kb, ++cnt) {
          const int s = cnt % kStages;
          const uint32_t round = cnt / kStages;
          if (round > 0 && !(ok = mbar_wait(&bars->empty[s], (round - 1) & 1, abort))) break;
          mbar_expect_tx(&bars->full[s], stage_bytes);
          uint8_t* sa = smem + s * kStageBytes;
          uint8_t* sa2 = sa + kABytes;
          uint8_t* sb = sa + (p.has_a2 ? 2 : 1) * kABytes;
          const int k0 = kb * kBK;
          if (p.a_mn) {
            const int row = p.a_shift + z * p.a_bstride + k0;
            tma_load_2d_hint(sa, &p.tmA, &bars->full[s], m0, row);
            tma_load_2d_hint(sa + kMnChunk, &p.tmA, &bars->full[s], m0 + 64, row);
            if (p.has_a2) {
              tma_load_2d_hint(sa2, &p.tmA2, &bars->full[s], m0, row);
              tma_load_2d_hint(sa2 + kMnChunk, &p.tmA2, &bars->full[s], m0 + 64, row);
            }
          } else {
            const int row = p.a_shift + z * p.a_bstride + m0;
            tma_load_2d_hint(sa, &p.tmA, &bars->full[s], k0, row);
            if (p.has_a2) tma_load_2d_hint(sa2, &p.tmA2, &bars->full[s], k0, row);
          }
          if (p.b_mn) {
            const int row = p.b_shift + z * p.b_bstride + k0;
#pragma unroll
            for (int c = 0; c < kBN / 64; ++c)
              tma_load_2d_hint(sb + c * kMnChunk, &p.tmB, &bars->full[s], n0 + 64 * c, row);
          } else {
            tma_load_2d_hint(sb, &p.tmB, &bars->full[s], k0, p.b_shift + z * p.b_bstride + n0);
          }
        }
      }
      if (!ok) {
        bars->abort = 1;
        if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << 8));
        volatile int no_abort = 0;  // let the loads in flight land (cnt: the failed stage)
        for (uint32_t q = cnt > kStages ? cnt - kStages : 0; q < cnt; ++q)
          mbar_wait(&bars->full[q % kStages], (q / kStages) & 1, &no_abort, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ UMMA issuer
    if (elect_one()) {
      const uint32_t idesc = idesc_f16(p.a_mn != 0, p.b_mn != 0);
      bool ok = true;
      uint32_t cnt = 0;
      int it = 0;  // tiles of this CTA so far
      for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
        const int buf = it & 1;
        // the epilogue has drained this buffer's previous tile (it - 2)
        if (it >= 2 && !(ok = mbar_wait(&bars->acc_empty[buf], ((it >> 1) - 1) & 1, abort))) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * kBN;
        for (int kb = 0; kb < nk; ++kb, ++cnt) {
          const int s = cnt % kStages;
          if (!(ok = mbar_wait(&bars->full[s], (cnt / kStages) & 1, abort))) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * kStageBytes);
          const uint32_t sa2 = sa + kABytes;
          const uint32_t sb = sa + (p.has_a2 ? 2 : 1) * kABytes;
          // K-major: one 128-byte row per operand row, 16 K elements = 32 bytes along it.
          // MN-major: 64-element chunks (LBO = 8 KB apart) of 64 K rows, 16 K rows = 2 KB.
          const uint64_t ad = p.a_mn ? sdesc_sw128(sa, kMnChunk, 1024) : sdesc_sw128(sa, 16, 1024);
          const uint64_t ad2 = p.a_mn ? sdesc_sw128(sa2, kMnChunk, 1024) : sdesc_sw128(sa2, 16, 1024);
          const uint64_t bd = p.b_mn ? sdesc_sw128(sb, kMnChunk, 1024) : sdesc_sw128(sb, 16, 1024);
          const uint32_t astep = p.a_mn ? (2048 >> 4) : (32 >> 4);
          const uint32_t bstep = p.b_mn ? (2048 >> 4) : (32 >> 4);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            umma_ss(d, ad + kk * astep, bd + kk * bstep, idesc, (kb | kk) != 0);
            if (p.has_a2) umma_ss(d, ad2 + kk * astep, bd + kk * bstep, idesc, 1u);
          }
          umma_commit(&bars->empty[s]);
        }
        if (ok) umma_commit(&bars->acc_full[buf]);
      }
      if (!ok) {
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
    const uint32_t taddr0 = tmem + ((uint32_t)(quad * 32) << 16);
    int it = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
      const int buf = it & 1;
      const bool ok = nk == 0 || mbar_wait(&bars->acc_full[buf], (it >> 1) & 1, abort);
      if (!ok) {
        bars->abort = 1;
        if (lane == 0 && p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << 10));
        break;
      }
      tc_fence_after();
      const int z = tile / tiles_mn, rem = tile % tiles_mn;
      const int m0 = (rem / tiles_n) * kBM, n0 = (rem % tiles_n) * kBN;
      const int m = m0 + row;
      const int64_t crow = (int64_t)p.c_shift + (int64_t)(z / p.c_zdiv) * p.c_bstride + m;
      const bool valid = m < p.M && crow >= 0 && crow < p.c_rows;
      float* cp = p.C + crow * p.ldc;
      const uint32_t taddr = taddr0 + buf * kBN;
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
        if (q == kBN / 32 - 1) {
          // every TMEM read of this warp for the tile is done: hand the buffer back
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
        }
        const int c0 = n0 + q * 32;
        if (!valid || c0 >= p.N) continue;
        store_piece(p, cp, crow, c0, v);
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

cudaError_t gemm_tc(const GemmOperand& A, const GemmOperand* A_lo, const GemmOperand& B,
                    const GemmOutput& C, int M, int N, int K, int batch, float alpha, float beta,
                    int32_t* err_word, cudaStream_t s) {
  if (C.zdiv < 1) return cudaErrorInvalidValue;
  if (M <= 0 || N <= 0 || batch <= 0) return cudaSuccess;
  Params p;
  memset(&p, 0, sizeof(p));
  cudaError_t e;
  // K-major: the map's columns are K, a box is 128 (A) / 256 (B) rows of 64 K elements.
  // MN-major: the map's columns are M / N, a box is 64 K rows of 64 MN elements.
  if ((e = map_2d(&p.tmA, A.ptr, A.rows, A.cols, A.ld, A.mn_major ? kBK : kBM)) != cudaSuccess)
    return e;
  if (A_lo) {
    if ((e = map_2d(&p.tmA2, A_lo->ptr, A_lo->rows, A_lo->cols, A_lo->ld,
                    A_lo->mn_major ? kBK : kBM)) != cudaSuccess)
      return e;
    p.has_a2 = 1;
  }
  if ((e = map_2d(&p.tmB, B.ptr, B.rows, B.cols, B.ld, B.mn_major ? kBK : kBN)) != cudaSuccess)
    return e;
  p.C = C.ptr;
  p.ldc = C.ld;
  p.M = M;
  p.N = N;
  p.K = K;
  p.batch = batch;
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
  const int64_t tiles =
      (int64_t)((N + kBN - 1) / kBN) * ((M + kBM - 1) / kBM) * (int64_t)batch;
  if (tiles >= (int64_t(1) << 31)) return cudaErrorInvalidValue;
  const int sms = device_sm_count();
  const int grid = tiles < sms ? (int)tiles : sms;
  gemm_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace hca
