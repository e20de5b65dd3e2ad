// hca_internal.h -- launch functions behind the C ABI (host side, not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/hca.h"

namespace hca {

// Number of SMs of the current device (cached per device).
int device_sm_count();

cudaError_t launch_compress(const hca_desc& d, const void* K, const void* V,
                            int64_t batch_stride_tokens, int32_t first_block,
                            int32_t n_blocks, const hca_cache& c, cudaStream_t s);

// float32, CUDA cores, any shape with head_dim % 32 == 0 && head_dim <= 512
cudaError_t launch_prefill_simt(const hca_desc& d, const void* Q, const void* K,
                                const void* V, const hca_cache& c, void* O, float* lse,
                                int32_t* dbg_mask, cudaStream_t s);
cudaError_t launch_decode_simt(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                               const hca_cache& c, const void* ring_k, const void* ring_v,
                               void* O, float* lse, cudaStream_t s);

// bf16, tcgen05 tensor cores
bool prefill_tc_supported(const hca_desc& d, const hca_cache& c);
cudaError_t launch_prefill_tc(const hca_desc& d, const void* Q, const void* K, const void* V,
                              const hca_cache& c, void* O, float* lse, int32_t* dbg_mask,
                              cudaStream_t s);
// bf16, 2-CTA clusters on the 2-SM UMMA (hq in 16..128); preferred over the one-CTA kernel
bool prefill_pair_supported(const hca_desc& d, const hca_cache& c);
cudaError_t launch_prefill_pair(const hca_desc& d, const void* Q, const void* K, const void* V,
                                const hca_cache& c, void* O, float* lse, int32_t* dbg_mask,
                                cudaStream_t s);

bool decode_tc_supported(const hca_desc& d, const hca_cache& c);
int decode_num_splits(const hca_desc& d);
size_t decode_tc_workspace_bytes(const hca_desc& d);
cudaError_t launch_decode_tc(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                             const hca_cache& c, const void* ring_k, const void* ring_v,
                             void* O, float* lse, void* ws, cudaStream_t s);
cudaError_t launch_decode_tc_noalloc(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                                     const hca_cache& c, const void* ring_k,
                                     const void* ring_v, void* O, float* lse, cudaStream_t s);

}  // namespace hca
