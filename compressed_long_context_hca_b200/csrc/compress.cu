// compress.cu -- block mean pooling into the paged compressed cache.
//
// [news 二.1] / [analysis 1] (see include/hca.h): every `block` consecutive tokens become
// one cache entry; the pooling rule is the mean over the tokens present (reading).
//
// HBM-bound: each block of K (and V) is read once with 16-byte non-allocating loads and a
// single row of the pool is written. One CTA handles one (block, sequence, tensor): its
// threads split the row into 16-byte vectors and the block's tokens into `groups`
// interleaved row sets; partial float32 sums meet in shared memory. Accumulation is
// float32, the mean is an IEEE division by the token count, rounded once to the storage
// type. An 8-bit cache ([serve fp8] in include/hca.h) stores e4m3(mean / scale): an IEEE
// float32 division by the pool's scale, then round-to-nearest-even with saturation at 448.
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include "hca_internal.h"
#include "sm100.cuh"

namespace hca {
namespace {

constexpr int kThreads = 256;

template <typename T>
struct Vec16;
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void add(const uint4& v, float* acc) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
  __device__ static uint4 pack(const float* x) {
    uint4 v;
    uint32_t* w = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
    return v;
  }
};
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  __device__ static void add(const uint4& v, float* acc) {
    acc[0] += __uint_as_float(v.x);
    acc[1] += __uint_as_float(v.y);
    acc[2] += __uint_as_float(v.z);
    acc[3] += __uint_as_float(v.w);
  }
  __device__ static uint4 pack(const float* x) {
    return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
                      __float_as_uint(x[3]));
  }
};

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

struct CompressArgs {
  const void* src[2];  // K, V: first token of block first_block of sequence 0
  void* pool[2];       // kc_pool, vc_pool
  const int32_t* page_table;
  int32_t* n_entries;
  int32_t* err_word;
  int64_t batch_stride_rows;  // token rows between sequences
  int32_t row_vecs;           // 16-byte vectors per token row (hkv * head_dim)
  int32_t part_vecs;          // of which one CTA handles (row_vecs / column parts)
  int32_t groups;             // row groups per CTA
  int32_t seqlen, block, first_block, n_blocks;
  int32_t page_entries, max_pages, num_pages;
  int32_t e4m3;               // pools hold e4m3 codes (one byte per element)
  float scale[2];             // e4m3: K, V pool scales
};

// N float32 means -> N e4m3 codes of mean / scale (N = 8 or 4), stored at byte offset
// `elem` of the pool (8 or 4 bytes, aligned: rows are a multiple of 8 bytes)
template <int N>
__device__ __forceinline__ void store_e4m3(uint8_t* pool, int64_t elem, const float* x,
                                           float scale) {
  uint32_t w[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < N; i += 2) {
    const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(
        make_float2(__fdiv_rn(x[i], scale), __fdiv_rn(x[i + 1], scale)), __NV_SATFINITE,
        __NV_E4M3);
    w[i >> 2] |= (uint32_t)c << (8 * (i & 3));
  }
  if (N == 8)
    *reinterpret_cast<uint2*>(pool + elem) = make_uint2(w[0], w[1]);
  else
    *reinterpret_cast<uint32_t*>(pool + elem) = w[0];
}

template <typename T>
__global__ void __launch_bounds__(kThreads) compress_kernel(CompressArgs a) {
  using V16 = Vec16<T>;
  constexpr int N = V16::N;
  pdl_wait();  // the kernel before this one on the stream (e.g. the ring update) is done
  pdl_trigger();
  const int jrel = blockIdx.x;
  const int b = blockIdx.y;
  const int which = blockIdx.z & 1;          // 0: K, 1: V
  const int vofs = (blockIdx.z >> 1) * a.part_vecs;  // this CTA's columns of the row
  const int j = a.first_block + jrel;
  const int tok0 = j * a.block;
  const int count = min(a.block, a.seqlen - tok0);

  extern __shared__ float red[];  // [groups][row_vecs*N] partial sums

  const uint4* src = reinterpret_cast<const uint4*>(a.src[which]) +
                     ((int64_t)b * a.batch_stride_rows + (int64_t)jrel * a.block) * a.row_vecs;
  const int lanes = a.part_vecs < kThreads ? a.part_vecs : kThreads;
  const int g = threadIdx.x / lanes;
  const int v0 = threadIdx.x % lanes;
  const bool active = g < a.groups;

  for (int vbase = 0; vbase < a.part_vecs; vbase += lanes) {
    const int v = vbase + v0;
    float acc[N];
#pragma unroll
    for (int i = 0; i < N; ++i) acc[i] = 0.f;
    if (active && v < a.part_vecs) {
      int r = g;
      // 4 independent 16-byte loads in flight per thread
      for (; r + 3 * a.groups < count; r += 4 * a.groups) {
        uint4 x0 = ld_stream(src + (int64_t)r * a.row_vecs + vofs + v);
        uint4 x1 = ld_stream(src + (int64_t)(r + a.groups) * a.row_vecs + vofs + v);
        uint4 x2 = ld_stream(src + (int64_t)(r + 2 * a.groups) * a.row_vecs + vofs + v);
        uint4 x3 = ld_stream(src + (int64_t)(r + 3 * a.groups) * a.row_vecs + vofs + v);
        V16::add(x0, acc);
        V16::add(x1, acc);
        V16::add(x2, acc);
        V16::add(x3, acc);
      }
      for (; r < count; r += a.groups)
        V16::add(ld_stream(src + (int64_t)r * a.row_vecs + vofs + v), acc);
      float* dst = red + ((int64_t)g * lanes + v0) * N;
#pragma unroll
      for (int i = 0; i < N; ++i) dst[i] = acc[i];
    }
    __syncthreads();
    if (g == 0 && v < a.part_vecs) {
      float sum[N];
#pragma unroll
      for (int i = 0; i < N; ++i) sum[i] = 0.f;
      for (int gg = 0; gg < a.groups; ++gg) {
        const float* p = red + ((int64_t)gg * lanes + v0) * N;
#pragma unroll
        for (int i = 0; i < N; ++i) sum[i] += p[i];
      }
      const float cnt = (float)count;
#pragma unroll
      for (int i = 0; i < N; ++i) sum[i] = __fdiv_rn(sum[i], cnt);
      const int page = a.page_table[(int64_t)b * a.max_pages + j / a.page_entries];
      if (page < 0 || page >= a.num_pages) {
        if (a.err_word) atomicOr(a.err_word, kErrPageRange);
      } else {
        const int64_t row = (int64_t)page * a.page_entries + j % a.page_entries;
        if (a.e4m3) {
          store_e4m3<N>(static_cast<uint8_t*>(a.pool[which]),
                        (row * a.row_vecs + vofs + v) * N, sum, a.scale[which]);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(a.pool[which]) + row * a.row_vecs + vofs + v;
          *dst = V16::pack(sum);
        }
      }
    }
    __syncthreads();
  }
  if (which == 0 && vofs == 0 && jrel == a.n_blocks - 1 && threadIdx.x == 0)
    a.n_entries[b] = a.first_block + a.n_blocks;
}

}  // namespace

cudaError_t launch_compress(const hca_desc& d, const void* K, const void* V,
                            int64_t batch_stride_tokens, int32_t first_block,
                            int32_t n_blocks, const hca_cache& c, cudaStream_t s) {
  CompressArgs a;
  a.src[0] = K;
  a.src[1] = V;
  a.pool[0] = c.kc_pool;
  a.pool[1] = c.vc_pool;
  a.page_table = c.page_table;
  a.n_entries = c.n_entries;
  a.err_word = c.err_word;
  const int esize = d.dtype == HCA_BF16 ? 2 : 4;
  a.row_vecs = (int32_t)((int64_t)d.hkv * d.head_dim * esize / 16);
  a.batch_stride_rows = batch_stride_tokens;
  a.seqlen = d.seqlen;
  a.block = d.block;
  a.first_block = first_block;
  a.n_blocks = n_blocks;
  a.page_entries = c.page_entries;
  a.max_pages = c.max_pages;
  a.num_pages = c.num_pages;
  a.e4m3 = c.pool_format == HCA_POOL_E4M3 ? 1 : 0;
  a.scale[0] = c.k_scale;
  a.scale[1] = c.v_scale;
  // Few blocks (a decode step completing one block per sequence): split each row's columns
  // over up to 8 CTAs until there are about two CTAs per SM, so that enough loads are in
  // flight; each CTA then walks the block's rows over fewer columns.
  int csplit = 1;
  const int64_t ctas = (int64_t)n_blocks * d.batch * 2;
  const int64_t want = 2 * (int64_t)device_sm_count();
  while (csplit < 8 && ctas * csplit < want && a.row_vecs % (2 * csplit) == 0) csplit *= 2;
  a.part_vecs = a.row_vecs / csplit;
  const int lanes = a.part_vecs < kThreads ? a.part_vecs : kThreads;
  a.groups = kThreads / lanes;
  if (a.groups > d.block) a.groups = d.block;
  const int vec_elems = 16 / esize;
  const size_t smem = (size_t)a.groups * lanes * vec_elems * sizeof(float);
  // a programmatic dependent of the kernel before it on the stream (it waits for it in the
  // kernel before touching memory), so its launch overlaps that kernel's tail
  cudaLaunchAttribute pdl[1];
  cudaLaunchConfig_t cfg = pdl_config(pdl, s);
  cfg.gridDim = dim3(n_blocks, d.batch, 2 * csplit);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  if (d.dtype == HCA_BF16) {
    if (smem > 48 * 1024)
      cudaFuncSetAttribute(compress_kernel<__nv_bfloat16>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return cudaLaunchKernelEx(&cfg, compress_kernel<__nv_bfloat16>, a);
  }
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(compress_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
  return cudaLaunchKernelEx(&cfg, compress_kernel<float>, a);
}

}  // namespace hca
