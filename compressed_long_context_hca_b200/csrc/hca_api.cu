// hca_api.cu -- the exported C ABI of libhca (see include/hca.h for the contract).
//
// Host code only: argument validation, choice of kernel by dtype, launch on the caller's
// stream. Nothing here allocates device memory or keeps state between calls (apart from
// per-device caches of the SM count and of kernel attributes).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "gemm_tc.h"
#include "hca_internal.h"
#include "tmap.h"

namespace hca {

int device_sm_count() {
  static PerDevice<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  int n = 0;
  if (cache.get(dev, &n)) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  cache.put(dev, n);
  return n;
}

cudaError_t set_smem_limit_once(PerDevice<int>& done, const void* kernel, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int flag = 0;
  if (done.get(dev, &flag)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  done.put(dev, 1);
  return cudaSuccess;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  // looked up once; threads racing on the first lookup store the same pointer
  static std::atomic<EncodeTiledFn> cached{nullptr};
  EncodeTiledFn fn = cached.load(std::memory_order_relaxed);
  if (fn) return fn;
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  fn = reinterpret_cast<EncodeTiledFn>(ptr);
  cached.store(fn, std::memory_order_relaxed);
  return fn;
}

cudaError_t encode_bf16_rows(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                             uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (rows == 0) rows = 1;  // a map needs a non-empty extent; nothing reads past the data
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint64_t ld, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (rows == 0) rows = 1;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_bf16_chunks(CUtensorMap* map, const void* base, uint64_t rows,
                               uint32_t box_rows, uint32_t box_chunks) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (rows == 0) rows = 1;
  cuuint64_t dims[3] = {64, rows, 8};
  cuuint64_t strides[2] = {1024, 128};
  cuuint32_t box[3] = {64, box_rows, box_chunks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_u8_chunks(CUtensorMap* map, const void* base, uint64_t rows,
                             uint32_t box_rows, uint32_t box_chunks) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return cudaErrorNotSupported;
  if (rows == 0) rows = 1;
  cuuint64_t dims[3] = {128, rows, 4};
  cuuint64_t strides[2] = {512, 128};
  cuuint32_t box[3] = {128, box_rows, box_chunks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace hca

using namespace hca;

namespace {

// HCA_ECUDA carries no detail across the ABI; with HCA_DEBUG set in the environment the
// CUDA error string is also written to stderr.
int32_t from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return HCA_OK;
  static const bool debug = getenv("HCA_DEBUG") != nullptr;
  if (debug) fprintf(stderr, "libhca: CUDA error %d: %s\n", (int)e, cudaGetErrorString(e));
  return HCA_ECUDA;
}

int32_t check_desc(const hca_desc* d) {
  if (!d) return HCA_EINVAL;
  if (d->batch < 0 || d->seqlen < 0 || d->hq < 1 || d->hkv < 1 || d->head_dim < 1 ||
      d->block < 1 || d->window < 1 || d->decode_splits < 0)
    return HCA_EINVAL;
  if (d->hq % d->hkv != 0) return HCA_EINVAL;
  if (d->dtype != HCA_BF16 && d->dtype != HCA_F32) return HCA_EUNSUPPORTED;
  if (!(d->scale == d->scale)) return HCA_EINVAL;  // NaN
  return HCA_OK;
}

bool finite_positive(float x) { return x > 0.f && x <= 3.4028234663852886e38f; }

int32_t check_cache(const hca_cache* c) {
  if (!c || !c->kc_pool || !c->vc_pool || !c->page_table || !c->n_entries) return HCA_EINVAL;
  if (c->page_entries < 1 || c->max_pages < 1 || c->num_pages < 1) return HCA_EINVAL;
  if (c->pool_format != HCA_POOL_NATIVE && c->pool_format != HCA_POOL_E4M3) return HCA_EINVAL;
  if (c->pool_format == HCA_POOL_E4M3 && (!finite_positive(c->k_scale) ||
                                          !finite_positive(c->v_scale)))
    return HCA_EINVAL;
  return HCA_OK;
}

bool e4m3_cache(const hca_cache* c) { return c->pool_format == HCA_POOL_E4M3; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

int32_t hca_abi_version(void) { return HCA_ABI_VERSION; }

const char* hca_status_string(int32_t status) {
  switch (status) {
    case HCA_OK: return "HCA_OK";
    case HCA_EINVAL: return "HCA_EINVAL: invalid argument";
    case HCA_EUNSUPPORTED: return "HCA_EUNSUPPORTED: no kernel for this shape/dtype";
    case HCA_ENOSPACE: return "HCA_ENOSPACE: cache or workspace too small";
    case HCA_ECUDA: return "HCA_ECUDA: CUDA call failed";
    default: return "HCA: unknown status";
  }
}

int32_t hca_set_gate(hca_desc* d, const void* gate, const int64_t* strides) {
  if (!d) return HCA_EINVAL;
  if (gate && !strides) return HCA_EINVAL;
  d->gate = gate;
  for (int i = 0; i < 3; ++i) d->gate_strides[i] = gate ? strides[i] : 0;
  return HCA_OK;
}

int32_t hca_compress(const hca_desc* d, const void* K, const void* V,
                     int64_t batch_stride_tokens, int32_t first_block, int32_t n_blocks,
                     const hca_cache* cache, hca_stream_t stream) {
  int32_t st = check_desc(d);
  if (st != HCA_OK) return st;
  if ((st = check_cache(cache)) != HCA_OK) return st;
  if (first_block < 0 || n_blocks < 0 || batch_stride_tokens < 0) return HCA_EINVAL;
  if (n_blocks == 0 || d->batch == 0) return HCA_OK;
  if (!K || !V) return HCA_EINVAL;
  if ((int64_t)(first_block + n_blocks - 1) * d->block >= d->seqlen) return HCA_EINVAL;
  if ((int64_t)first_block + n_blocks > (int64_t)cache->max_pages * cache->page_entries)
    return HCA_ENOSPACE;
  if (d->head_dim % 8 != 0) return HCA_EUNSUPPORTED;
  const int esize = d->dtype == HCA_BF16 ? 2 : 4;
  if (((int64_t)d->hkv * d->head_dim * esize) % 16 != 0) return HCA_EUNSUPPORTED;
  if (!aligned16(K) || !aligned16(V) || !aligned16(cache->kc_pool) ||
      !aligned16(cache->vc_pool))
    return HCA_EINVAL;
  return from_cuda(launch_compress(*d, K, V, batch_stride_tokens, first_block, n_blocks, *cache,
                                   reinterpret_cast<cudaStream_t>(stream)));
}

int32_t hca_ring_append(const hca_desc* d, const void* new_k, const void* new_v,
                        const int32_t* ctx_len, void* ring_k, void* ring_v,
                        hca_stream_t stream) {
  int32_t st = check_desc(d);
  if (st != HCA_OK) return st;
  if (d->batch == 0) return HCA_OK;
  if (!new_k || !new_v || !ctx_len || !ring_k || !ring_v) return HCA_EINVAL;
  if (d->seqlen < 1) return HCA_EINVAL;
  const int esize = d->dtype == HCA_BF16 ? 2 : 4;
  if (((int64_t)d->hkv * d->head_dim * esize) % 16 != 0) return HCA_EUNSUPPORTED;
  if (!aligned16(new_k) || !aligned16(new_v) || !aligned16(ring_k) || !aligned16(ring_v))
    return HCA_EINVAL;
  return from_cuda(launch_ring_append(*d, new_k, new_v, ctx_len, ring_k, ring_v,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

int32_t hca_attn_prefill_range(const hca_desc* d, int32_t q_pos0, int32_t kv_pos0,
                               int32_t kv_len, const void* Q, const void* K, const void* V,
                               const hca_cache* cache, void* O, float* lse, int32_t* dbg_mask,
                               hca_stream_t stream) {
  int32_t st = check_desc(d);
  if (st != HCA_OK) return st;
  if ((st = check_cache(cache)) != HCA_OK) return st;
  if (q_pos0 < 0 || kv_pos0 < 0 || kv_len < 0) return HCA_EINVAL;
  if (e4m3_cache(cache)) return HCA_EUNSUPPORTED;
  if (d->batch == 0 || d->seqlen == 0) return HCA_OK;
  if (!Q || !K || !V || !O) return HCA_EINVAL;
  if ((int64_t)q_pos0 + d->seqlen > INT32_MAX) return HCA_EINVAL;
  // the K/V rows must hold every raw token a query row's window reaches
  const int64_t first_needed = q_pos0 - d->window + 1 > 0 ? q_pos0 - d->window + 1 : 0;
  if (kv_pos0 > first_needed || (int64_t)kv_pos0 + kv_len < (int64_t)q_pos0 + d->seqlen)
    return HCA_EINVAL;
  if (d->gate && (d->gate_strides[0] < 0 || d->gate_strides[1] < 0 || d->gate_strides[2] < 0))
    return HCA_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const PrefillRange r{q_pos0, kv_pos0, kv_len};
  if (d->dtype == HCA_F32) {
    if (d->head_dim % 32 != 0 || d->head_dim > 512) return HCA_EUNSUPPORTED;
    return from_cuda(launch_prefill_simt(*d, Q, K, V, *cache, O, lse, dbg_mask, r, s));
  }
  if (!prefill_tc_supported(*d, *cache)) return HCA_EUNSUPPORTED;
  if ((int64_t)d->batch * kv_len >= (int64_t(1) << 31)) return HCA_EUNSUPPORTED;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) ||
      !aligned16(cache->kc_pool) || !aligned16(cache->vc_pool))
    return HCA_EINVAL;
  if (prefill_pair_supported(*d, *cache))
    return from_cuda(launch_prefill_pair(*d, Q, K, V, *cache, O, lse, dbg_mask, r, s));
  return from_cuda(launch_prefill_tc(*d, Q, K, V, *cache, O, lse, dbg_mask, r, s));
}

int32_t hca_attn_prefill(const hca_desc* d, const void* Q, const void* K, const void* V,
                         const hca_cache* cache, void* O, float* lse, int32_t* dbg_mask,
                         hca_stream_t stream) {
  if (!d) return HCA_EINVAL;
  return hca_attn_prefill_range(d, 0, 0, d->seqlen, Q, K, V, cache, O, lse, dbg_mask, stream);
}

size_t hca_prefill_backward_workspace_bytes(const hca_desc* d) {
  if (check_desc(d) != HCA_OK) return 0;
  return backward_tc_supported(*d) ? backward_tc_workspace_bytes(*d)
                                   : backward_simt_workspace_bytes(*d);
}

int32_t hca_attn_prefill_backward(const hca_desc* d, const void* Q, const void* K,
                                  const void* V, const hca_cache* cache,
                                  const float* lse, const void* dO, void* dQ, void* dK,
                                  void* dV, void* dG, void* workspace, size_t workspace_bytes,
                                  hca_stream_t stream) {
  int32_t st = check_desc(d);
  if (st != HCA_OK) return st;
  if ((st = check_cache(cache)) != HCA_OK) return st;
  if (e4m3_cache(cache)) return HCA_EUNSUPPORTED;
  if (d->batch == 0 || d->seqlen == 0) return HCA_OK;
  if (!Q || !K || !V || !lse || !dO || !dQ || !dK || !dV) return HCA_EINVAL;
  if ((d->gate != nullptr) != (dG != nullptr)) return HCA_EINVAL;
  if (d->gate && (d->gate_strides[0] < 0 || d->gate_strides[1] < 0 || d->gate_strides[2] < 0))
    return HCA_EINVAL;
  if (d->head_dim % 32 != 0 || d->head_dim > 512) return HCA_EUNSUPPORTED;
  if ((int64_t)d->batch * d->seqlen * d->hq >= (int64_t(1) << 31)) return HCA_EUNSUPPORTED;
  const bool tc = backward_tc_supported(*d);
  const size_t need = tc ? backward_tc_workspace_bytes(*d) : backward_simt_workspace_bytes(*d);
  if (!workspace || workspace_bytes < need) return HCA_ENOSPACE;
  if (!aligned16(workspace)) return HCA_EINVAL;
  const BackwardTensors x{Q, K, V, lse, dO, dQ, dK, dV, dG};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (tc) {
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(dO) || !aligned16(dQ) ||
        !aligned16(dK) || !aligned16(dV) || (dG && !aligned16(dG)) ||
        !aligned16(cache->kc_pool) || !aligned16(cache->vc_pool))
      return HCA_EINVAL;
    if (d->gate && (reinterpret_cast<uintptr_t>(d->gate) % 4 || d->gate_strides[2] % 2 ||
                    d->gate_strides[1] % 2 || d->gate_strides[0] % 2))
      return HCA_EINVAL;
    return from_cuda(launch_backward_tc(*d, x, *cache, workspace, s));
  }
  return from_cuda(launch_backward_simt(*d, x, *cache, workspace, s));
}

int32_t hca_gate_from_latent(const hca_desc* d, const void* q_lat, const void* W_g,
                             int32_t latent, void* G, hca_stream_t stream) {
  int32_t st = check_desc(d);
  if (st != HCA_OK) return st;
  if (latent < 1) return HCA_EINVAL;
  const int64_t rows = (int64_t)d->batch * d->seqlen;
  if (rows == 0) return HCA_OK;
  if (!q_lat || !W_g || !G) return HCA_EINVAL;
  const int64_t n = (int64_t)d->hq * d->head_dim;
  if (d->dtype != HCA_BF16) return HCA_EUNSUPPORTED;
  if (latent % 8 != 0 || n % 8 != 0 || rows >= (int64_t(1) << 31) || n >= (int64_t(1) << 31))
    return HCA_EUNSUPPORTED;
  if (!aligned16(q_lat) || !aligned16(W_g) || !aligned16(G)) return HCA_EINVAL;
  // G [rows, n] = sigmoid(q_lat [rows, latent] . W_g [latent, n]): A K-major, B MN-major
  const GemmOperand A{q_lat, rows, latent, latent, false, 0, 0};
  const GemmOperand B{W_g, latent, n, n, true, 0, 0};
  GemmOutput C{static_cast<float*>(G), n, 0, 0, (int32_t)rows, 1, false, true};
  return from_cuda(gemm_tc(A, nullptr, B, C, (int)rows, (int)n, latent, 1, 1.f, 0.f, nullptr,
                           reinterpret_cast<cudaStream_t>(stream)));
}

int32_t hca_vha_gate(const hca_desc* d, const void* O, const float* A, const float* B,
                     int32_t rank, void* out, hca_stream_t stream) {
  int32_t st = check_desc(d);
  if (st != HCA_OK) return st;
  if (rank < 0 || rank > 16 || d->hq > 128) return HCA_EUNSUPPORTED;
  if ((int64_t)d->batch * d->seqlen == 0) return HCA_OK;
  if (!O || !out || (rank > 0 && (!A || !B))) return HCA_EINVAL;
  if (d->head_dim % 4 != 0 || d->head_dim > 512) return HCA_EUNSUPPORTED;
  if (d->gate && (d->gate_strides[0] < 0 || d->gate_strides[1] < 0 || d->gate_strides[2] < 0))
    return HCA_EINVAL;
  return from_cuda(launch_vha_gate(*d, O, A, B, rank, out, reinterpret_cast<cudaStream_t>(stream)));
}

size_t hca_decode_workspace_bytes(const hca_desc* d) {
  if (check_desc(d) != HCA_OK) return 0;
  if (d->dtype != HCA_BF16) return 0;
  return decode_tc_workspace_bytes(*d);
}

int32_t hca_attn_decode(const hca_desc* d, const void* Q, const int32_t* ctx_len,
                        const hca_cache* cache, const void* ring_k, const void* ring_v,
                        void* O, float* lse, void* workspace, size_t workspace_bytes,
                        hca_stream_t stream) {
  int32_t st = check_desc(d);
  if (st != HCA_OK) return st;
  if ((st = check_cache(cache)) != HCA_OK) return st;
  if (d->batch == 0) return HCA_OK;
  if (!Q || !ctx_len || !ring_k || !ring_v || !O) return HCA_EINVAL;
  if (d->seqlen < 1) return HCA_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d->dtype == HCA_F32) {
    if (d->head_dim % 32 != 0 || d->head_dim > 512 || e4m3_cache(cache))
      return HCA_EUNSUPPORTED;
    return from_cuda(launch_decode_simt(*d, Q, ctx_len, *cache, ring_k, ring_v, O, lse, s));
  }
  if (!decode_tc_supported(*d, *cache)) return HCA_EUNSUPPORTED;
  const size_t need = decode_tc_workspace_bytes(*d);
  if (!workspace || workspace_bytes < need) return HCA_ENOSPACE;
  if (!aligned16(Q) || !aligned16(ring_k) || !aligned16(ring_v) || !aligned16(O) ||
      !aligned16(workspace) || !aligned16(cache->kc_pool) || !aligned16(cache->vc_pool))
    return HCA_EINVAL;
  return from_cuda(
      launch_decode_tc(*d, Q, ctx_len, *cache, ring_k, ring_v, O, lse, workspace, s));
}

int32_t hca_attn_decode_append(const hca_desc* d, const void* Q, const int32_t* ctx_len,
                               const hca_cache* cache, const void* new_k, const void* new_v,
                               void* ring_k, void* ring_v, void* O, float* lse,
                               void* workspace, size_t workspace_bytes, hca_stream_t stream) {
  int32_t st = check_desc(d);
  if (st != HCA_OK) return st;
  if ((st = check_cache(cache)) != HCA_OK) return st;
  if (d->batch == 0) return HCA_OK;
  if (!Q || !ctx_len || !ring_k || !ring_v || !O || !new_k || !new_v) return HCA_EINVAL;
  if (d->seqlen < 1) return HCA_EINVAL;
  if (!aligned16(new_k) || !aligned16(new_v)) return HCA_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d->dtype == HCA_F32) {
    if (d->head_dim % 32 != 0 || d->head_dim > 512 || e4m3_cache(cache))
      return HCA_EUNSUPPORTED;
    if ((int64_t)d->hkv * d->head_dim * 4 % 16 != 0) return HCA_EUNSUPPORTED;
    if (!aligned16(ring_k) || !aligned16(ring_v)) return HCA_EINVAL;
    cudaError_t e = launch_ring_append(*d, new_k, new_v, ctx_len, ring_k, ring_v, s);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(launch_decode_simt(*d, Q, ctx_len, *cache, ring_k, ring_v, O, lse, s));
  }
  if (!decode_tc_supported(*d, *cache)) return HCA_EUNSUPPORTED;
  const size_t need = decode_tc_workspace_bytes(*d);
  if (!workspace || workspace_bytes < need) return HCA_ENOSPACE;
  if (!aligned16(Q) || !aligned16(ring_k) || !aligned16(ring_v) || !aligned16(O) ||
      !aligned16(workspace) || !aligned16(cache->kc_pool) || !aligned16(cache->vc_pool))
    return HCA_EINVAL;
  DecodePart whole{0, INT32_MAX, 1, nullptr};
  whole.new_k = new_k;
  whole.new_v = new_v;
  return from_cuda(
      launch_decode_part(*d, Q, ctx_len, *cache, ring_k, ring_v, whole, O, lse, workspace, s));
}

size_t hca_decode_partial_bytes(const hca_desc* d) {
  if (check_desc(d) != HCA_OK || d->dtype != HCA_BF16) return 0;
  return decode_partial_bytes(*d);
}

int32_t hca_attn_decode_partial(const hca_desc* d, const void* Q, const int32_t* ctx_len,
                                const hca_cache* cache, const void* ring_k, const void* ring_v,
                                int32_t entry_begin, int32_t entry_end, int32_t with_window,
                                void* partial, void* workspace, size_t workspace_bytes,
                                hca_stream_t stream) {
  int32_t st = check_desc(d);
  if (st != HCA_OK) return st;
  if ((st = check_cache(cache)) != HCA_OK) return st;
  if (entry_begin < 0 || entry_end < entry_begin || entry_begin % 128 != 0) return HCA_EINVAL;
  if (d->batch == 0) return HCA_OK;
  if (!Q || !ctx_len || !ring_k || !ring_v || !partial) return HCA_EINVAL;
  if (d->seqlen < 1) return HCA_EINVAL;
  if (d->dtype != HCA_BF16 || !decode_tc_supported(*d, *cache)) return HCA_EUNSUPPORTED;
  const DecodePart part{entry_begin, entry_end, with_window ? 1 : 0, partial};
  const size_t need = decode_part_workspace_bytes(*d, part);
  if (need > 0 && (!workspace || workspace_bytes < need)) return HCA_ENOSPACE;
  if (!aligned16(Q) || !aligned16(ring_k) || !aligned16(ring_v) || !aligned16(partial) ||
      (need > 0 && !aligned16(workspace)) || !aligned16(cache->kc_pool) ||
      !aligned16(cache->vc_pool))
    return HCA_EINVAL;
  return from_cuda(launch_decode_part(*d, Q, ctx_len, *cache, ring_k, ring_v, part, nullptr,
                                      nullptr, workspace, reinterpret_cast<cudaStream_t>(stream)));
}

int32_t hca_decode_merge(const hca_desc* d, const void* parts, int32_t n_parts,
                         int64_t part_stride, void* O, float* lse, hca_stream_t stream) {
  int32_t st = check_desc(d);
  if (st != HCA_OK) return st;
  if (n_parts < 1) return HCA_EINVAL;
  if (d->batch == 0) return HCA_OK;
  if (!parts || !O) return HCA_EINVAL;
  if (d->dtype != HCA_BF16 || d->head_dim != 512 || d->hq < 1 || d->hq > 64)
    return HCA_EUNSUPPORTED;
  if (n_parts > 1 && (part_stride < (int64_t)decode_partial_bytes(*d) || part_stride % 16 != 0))
    return HCA_EINVAL;
  if (!aligned16(parts) || !aligned16(O)) return HCA_EINVAL;
  if (d->gate) {
    const uintptr_t ga = reinterpret_cast<uintptr_t>(d->gate);
    if (ga % 4 || d->gate_strides[0] % 2 || d->gate_strides[2] % 2 || d->gate_strides[0] < 0 ||
        d->gate_strides[2] < 0)
      return HCA_EINVAL;
  }
  return from_cuda(launch_decode_merge(*d, parts, n_parts, part_stride, O, lse,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

int32_t hca_attn_decode_noalloc(const hca_desc* d, const void* Q, const int32_t* ctx_len,
                                const hca_cache* cache, const void* ring_k, const void* ring_v,
                                void* O, float* lse, hca_stream_t stream) {
  int32_t st = check_desc(d);
  if (st != HCA_OK) return st;
  if ((st = check_cache(cache)) != HCA_OK) return st;
  if (d->batch == 0) return HCA_OK;
  if (!Q || !ctx_len || !ring_k || !ring_v || !O) return HCA_EINVAL;
  if (d->seqlen < 1) return HCA_EINVAL;
  if (d->dtype != HCA_BF16 || !decode_tc_supported(*d, *cache)) return HCA_EUNSUPPORTED;
  if (decode_tc_workspace_bytes(*d) > (size_t)HCA_DECODE_NOALLOC_SCRATCH_BYTES)
    return HCA_ENOSPACE;
  if (!aligned16(Q) || !aligned16(ring_k) || !aligned16(ring_v) || !aligned16(O) ||
      !aligned16(cache->kc_pool) || !aligned16(cache->vc_pool))
    return HCA_EINVAL;
  return from_cuda(launch_decode_tc_noalloc(*d, Q, ctx_len, *cache, ring_k, ring_v, O, lse,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
