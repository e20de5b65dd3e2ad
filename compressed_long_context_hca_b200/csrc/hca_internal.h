// hca_internal.h -- launch functions behind the C ABI (host side, not exported).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "../../include/hca.h"

namespace hca {

// Per-device memo of a value that a device's first call computes (a kernel attribute set,
// a symbol address, a count); T() means "not computed yet". The slots are relaxed atomics:
// host threads whose first calls on one device race each compute the same value and store
// it, which is harmless. Devices numbered kMaxDevices and up are not memoised: every call
// computes the value again.
constexpr int kMaxDevices = 64;
template <typename T>
struct PerDevice {
  std::atomic<T> slot[kMaxDevices];
  bool get(int dev, T* out) const {
    if (dev < 0 || dev >= kMaxDevices) return false;
    const T v = slot[dev].load(std::memory_order_relaxed);
    if (v == T()) return false;
    *out = v;
    return true;
  }
  void put(int dev, T v) {
    if (dev >= 0 && dev < kMaxDevices) slot[dev].store(v, std::memory_order_relaxed);
  }
};

// Raises the dynamic shared-memory limit of `kernel` on the current device, once per device.
cudaError_t set_smem_limit_once(PerDevice<int>& done, const void* kernel, int bytes);

// Number of SMs of the current device (cached per device).
int device_sm_count();

cudaError_t launch_compress(const hca_desc& d, const void* K, const void* V,
                            int64_t batch_stride_tokens, int32_t first_block,
                            int32_t n_blocks, const hca_cache& c, cudaStream_t s);
cudaError_t launch_ring_append(const hca_desc& d, const void* new_k, const void* new_v,
                               const int32_t* ctx_len, void* ring_k, void* ring_v,
                               cudaStream_t s);

// Query rows of a prefill call: row t of a sequence is position q_pos0 + t; K/V row u is
// position kv_pos0 + u, kv_len rows per sequence (a whole sequence: 0, 0, seqlen).
struct PrefillRange {
  int32_t q_pos0, kv_pos0, kv_len;
};

// float32, CUDA cores, any shape with head_dim % 32 == 0 && head_dim <= 512
cudaError_t launch_prefill_simt(const hca_desc& d, const void* Q, const void* K,
                                const void* V, const hca_cache& c, void* O, float* lse,
                                int32_t* dbg_mask, const PrefillRange& r, cudaStream_t s);
cudaError_t launch_decode_simt(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                               const hca_cache& c, const void* ring_k, const void* ring_v,
                               void* O, float* lse, cudaStream_t s);

// bf16, tcgen05 tensor cores
bool prefill_tc_supported(const hca_desc& d, const hca_cache& c);
cudaError_t launch_prefill_tc(const hca_desc& d, const void* Q, const void* K, const void* V,
                              const hca_cache& c, void* O, float* lse, int32_t* dbg_mask,
                              const PrefillRange& r, cudaStream_t s);
// bf16, 2-CTA clusters on the 2-SM UMMA (hq in 16..128); preferred over the one-CTA kernel
bool prefill_pair_supported(const hca_desc& d, const hca_cache& c);
cudaError_t launch_prefill_pair(const hca_desc& d, const void* Q, const void* K, const void* V,
                                const hca_cache& c, void* O, float* lse, int32_t* dbg_mask,
                                const PrefillRange& r, cudaStream_t s);

// Tensors of a prefill backward call (device pointers; dtype of the descriptor, lse f32).
struct BackwardTensors {
  const void* Q;
  const void* K;
  const void* V;
  const float* lse;
  const void* dO;
  void* dQ;
  void* dK;
  void* dV;
  void* dG;
};

// CUDA cores, float32 arithmetic, float32 or bf16 tensors (head_dim % 32 == 0, <= 512)
size_t backward_simt_workspace_bytes(const hca_desc& d);
cudaError_t launch_backward_simt(const hca_desc& d, const BackwardTensors& x, const hca_cache& c,
                                 void* ws, cudaStream_t s);

// bf16 on tcgen05 GEMMs (head_dim 512, hkv 1, window <= 128)
bool backward_tc_supported(const hca_desc& d);
size_t backward_tc_workspace_bytes(const hca_desc& d);
cudaError_t launch_backward_tc(const hca_desc& d, const BackwardTensors& x, const hca_cache& c,
                               void* ws, cudaStream_t s);

// VHA mixing + gate over [batch * seqlen positions, hq, head_dim] (vha.cu)
cudaError_t launch_vha_gate(const hca_desc& d, const void* O, const float* A, const float* B,
                            int rank, void* out, cudaStream_t s);

// The key part of a decode call: visible compressed entries [e0, e1) (e0 a multiple of 128)
// and the raw window if with_ring. out_partial == nullptr: the call writes the final output;
// else it writes an unnormalised float32 partial result there (decode_partial_bytes).
// new_k / new_v (with_ring only; nullptr = none): the new token's rows [batch, 512], written
// into ring slot t % window by the CTA that reads the window, before it reads it.
struct DecodePart {
  int32_t e0, e1, with_ring;
  void* out_partial;
  const void* new_k = nullptr;
  const void* new_v = nullptr;
};

bool decode_tc_supported(const hca_desc& d, const hca_cache& c);
size_t decode_partial_bytes(const hca_desc& d);
size_t decode_part_workspace_bytes(const hca_desc& d, const DecodePart& part);
cudaError_t launch_decode_part(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                               const hca_cache& c, const void* ring_k, const void* ring_v,
                               const DecodePart& part, void* O, float* lse, void* ws,
                               cudaStream_t s);
cudaError_t launch_decode_merge(const hca_desc& d, const void* parts, int n_parts,
                                int64_t part_stride_bytes, void* O, float* lse, cudaStream_t s);
int decode_num_splits(const hca_desc& d);
size_t decode_tc_workspace_bytes(const hca_desc& d);
cudaError_t launch_decode_tc(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                             const hca_cache& c, const void* ring_k, const void* ring_v,
                             void* O, float* lse, void* ws, cudaStream_t s);
// Shared by the 16-bit and 8-bit decode launches (decode_tc.cu): the split count of a part,
// the float count of the (m, l) block of a workspace of nsplit splits, the PDL launch
// attribute, and the merge of nsplit split partials (ws_ml, ws_o) into the final output or,
// when pml != nullptr, into one partial (pml, po).
int part_num_splits(const hca_desc& d, const DecodePart& part);
size_t ml_floats(const hca_desc& d, int nsplit);
cudaLaunchConfig_t pdl_config(cudaLaunchAttribute* pdl, cudaStream_t s);
cudaError_t launch_split_merge(const hca_desc& d, const float* ws_ml, const float* ws_o,
                               int nsplit, float* pml, float* po, void* O, float* lse,
                               cudaStream_t s);
// 8-bit compressed pools (hca_cache.pool_format == HCA_POOL_E4M3; decode_fp8.cu): same
// arguments, workspace layout and split rule as launch_decode_part.
cudaError_t launch_decode_fp8(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                              const hca_cache& c, const void* ring_k, const void* ring_v,
                              const DecodePart& part, void* O, float* lse, void* ws,
                              cudaStream_t s);
cudaError_t launch_decode_tc_noalloc(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                                     const hca_cache& c, const void* ring_k,
                                     const void* ring_v, void* O, float* lse, cudaStream_t s);

}  // namespace hca
