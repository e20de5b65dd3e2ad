// ring.cu -- the raw-window ring update of a decode step, one launch for every sequence.
//
// Operation ([news 二.1] in include/hca.h: the newest `window` raw tokens are attended as
// they are; the decode path keeps them in a ring of `window` slots, token u in slot
// u % window): the new token of sequence b, at position t = ctx_len[b] - 1, has its key and
// value rows written to slot t % window of the K and V rings. ctx_len is clamped into
// [1, seqlen] exactly as the decode kernels clamp it, so both agree on the slot.
//
// Pure data movement (2 x hkv x head_dim elements per sequence): one CTA per sequence
// copies both rows in 16-byte units. Launched as a programmatic dependent of the kernel
// before it (the previous step's merge or decode) and letting the next one (the step's
// decode) be scheduled early; each waits for its predecessor before touching memory.
#include <cuda_runtime.h>
#include <stdint.h>

#include "hca_internal.h"
#include "sm100.cuh"

namespace hca {
namespace {

struct RingArgs {
  const uint4* k;      // [batch, row_units]
  const uint4* v;
  const int32_t* ctx_len;
  uint4* rk;           // [batch, window, row_units]
  uint4* rv;
  int32_t row_units;   // 16-byte units of one token row (hkv * head_dim elements)
  int32_t window, seqlen;
};

__global__ void __launch_bounds__(128) ring_append_kernel(const RingArgs a) {
  pdl_wait();  // the previous step's reads of the ring are complete
  pdl_trigger();
  const int b = blockIdx.x;
  int ctx = a.ctx_len[b];
  ctx = ctx < 1 ? 1 : (ctx > a.seqlen ? a.seqlen : ctx);
  const int64_t slot = (int64_t)(ctx - 1) % a.window;
  const int64_t src = (int64_t)b * a.row_units;
  const int64_t dst = ((int64_t)b * a.window + slot) * a.row_units;
  for (int i = threadIdx.x; i < a.row_units; i += blockDim.x) {
    a.rk[dst + i] = a.k[src + i];
    a.rv[dst + i] = a.v[src + i];
  }
}

}  // namespace

cudaError_t launch_ring_append(const hca_desc& d, const void* new_k, const void* new_v,
                               const int32_t* ctx_len, void* ring_k, void* ring_v,
                               cudaStream_t s) {
  const int esize = d.dtype == HCA_BF16 ? 2 : 4;
  RingArgs a;
  a.k = reinterpret_cast<const uint4*>(new_k);
  a.v = reinterpret_cast<const uint4*>(new_v);
  a.ctx_len = ctx_len;
  a.rk = reinterpret_cast<uint4*>(ring_k);
  a.rv = reinterpret_cast<uint4*>(ring_v);
  a.row_units = (int32_t)((int64_t)d.hkv * d.head_dim * esize / 16);
  a.window = d.window;
  a.seqlen = d.seqlen;
  cudaLaunchAttribute pdl[1];
  cudaLaunchConfig_t cfg = pdl_config(pdl, s);
  cfg.gridDim = dim3(d.batch);
  cfg.blockDim = dim3(128);
  return cudaLaunchKernelEx(&cfg, ring_append_kernel, a);
}

}  // namespace hca
