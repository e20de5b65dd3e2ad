// backward_simt.cu -- gradients of the HCA prefill on CUDA cores (float32 arithmetic,
// float32 or bf16 tensors).
//
// The operation is the exact derivative of the prefill output ([news 二.1] / [analysis 1] /
// [gate] in include/hca.h; the pages quote the backward kernel's speed-up, [analysis infra
// 3], and print no formulas). Per query row (sequence b, position t, head h) with visible
// keys k_i, values v_i (compressed entries j < n_c(t), then the raw window):
//   s_i = scale q.k_i,  p_i = exp(s_i - lse),  O_pre = sum_i p_i v_i,  O = O_pre * G
//   dG = dO * O_pre,  dO' = dO * G,  Delta = dO' . O_pre
//   dp_i = dO' . v_i,  ds_i = p_i (dp_i - Delta)
//   dq = scale sum_i ds_i k_i,   dk_i += scale ds_i q,   dv_i += p_i dO'
// and an entry's gradient reaches every token of its block divided by the block's token
// count (the entry is their mean). O_pre is recomputed from the forward's lse.
//
// Kernels, in launch order:
//   prep       one warp per row: O_pre recomputed in float32, Delta (and dG)
//   entries    one warp per (entry, KV head, chunk of query positions): dKc, dVc partial
//              sums over the rows that see the entry, float32 atomics into the workspace
//   raw        one warp per (token, KV head): dK, dV over the window rows that see the
//              token, plus the token's share of its block's entry gradient; final output
//   dq         one warp per row: dQ
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hca_internal.h"
#include "sm100.cuh"

namespace hca {
namespace {

constexpr int kMaxVpl = 16;  // head_dim <= 512
constexpr int kWarps = 4;
constexpr int kEntryChunk = 256;  // query positions per warp in the entries kernel

struct BwdArgs {
  const void* Q;
  const void* K;
  const void* V;
  const void* kc;
  const void* vc;
  const float* lse;
  const void* dO;
  const void* gate;
  int64_t gs0, gs1, gs2;
  void* dQ;
  void* dK;
  void* dV;
  void* dG;
  const int32_t* page_table;
  const int32_t* n_entries;
  int32_t* err_word;
  float* delta;   // [b, T, hq]
  float* dkc;     // [b, n_ent, hkv, D]
  float* dvc;
  int32_t n_ent;  // entries per sequence in dkc / dvc: ceil(T / block)
  int32_t batch, T, hq, hkv, D, block, window, page_entries, max_pages, num_pages;
  float scale;
};

template <typename T>
__device__ __forceinline__ float ld(const void* p, int64_t i);
template <>
__device__ __forceinline__ float ld<float>(const void* p, int64_t i) {
  return static_cast<const float*>(p)[i];
}
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const void* p, int64_t i) {
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}
template <typename T>
__device__ __forceinline__ void st(void* p, int64_t i, float v);
template <>
__device__ __forceinline__ void st<float>(void* p, int64_t i, float v) {
  static_cast<float*>(p)[i] = v;
}
template <>
__device__ __forceinline__ void st<__nv_bfloat16>(void* p, int64_t i, float v) {
  static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

__device__ __forceinline__ int visible(int t, int block, int window) {
  const int x = t + 1 - window;
  return x < 0 ? 0 : x / block;
}

// lane's elements lane + 32 i of a row of D values
template <typename T>
__device__ __forceinline__ void load_row(float (&r)[kMaxVpl], const void* base, int64_t off,
                                         int lane, int vpl) {
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i) r[i] = i < vpl ? ld<T>(base, off + lane + 32 * i) : 0.f;
}

// dO' = dO * G of row (b, t, h) (dO itself without a gate)
template <typename T>
__device__ __forceinline__ void load_dop(float (&r)[kMaxVpl], const BwdArgs& a, int b, int t,
                                         int h, int lane, int vpl) {
  const int64_t row = (((int64_t)b * a.T + t) * a.hq + h) * a.D;
  load_row<T>(r, a.dO, row, lane, vpl);
  if (a.gate) {
    const int64_t goff = (int64_t)b * a.gs0 + (int64_t)t * a.gs1 + (int64_t)h * a.gs2;
#pragma unroll
    for (int i = 0; i < kMaxVpl; ++i)
      if (i < vpl) r[i] *= ld<T>(a.gate, goff + lane + 32 * i);
  }
}

__device__ __forceinline__ float dot(const float (&x)[kMaxVpl], const float (&y)[kMaxVpl],
                                     int vpl) {
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i)
    if (i < vpl) s = fmaf(x[i], y[i], s);
  return warp_sum(s);
}

// pool row of entry j of sequence b, KV head g (-1 when the page id is out of range)
__device__ __forceinline__ int64_t entry_row(const BwdArgs& a, int b, int j, int g) {
  const int page = a.page_table[(int64_t)b * a.max_pages + j / a.page_entries];
  if (page < 0 || page >= a.num_pages) {
    if (a.err_word && (threadIdx.x & 31) == 0) atomicOr(a.err_word, kErrPageRange);
    return -1;
  }
  return ((int64_t)page * a.page_entries + j % a.page_entries) * a.hkv + g;
}

// visible entries of position t, clamped to what the cache holds
__device__ __forceinline__ int entries_of(const BwdArgs& a, int b, int t) {
  const int nc = visible(t, a.block, a.window);
  const int have = min(a.n_entries[b], a.max_pages * a.page_entries);
  if (nc > have) {
    if (a.err_word && (threadIdx.x & 31) == 0) atomicOr(a.err_word, kErrCacheShort);
    return have;
  }
  return nc;
}

// ------------------------------------------------------------------------------ prep
// The ungated output O_pre = sum_i p_i v_i is recomputed in float32 from the lse (a stored
// bf16 output carries 2^-9 of |O| of rounding, which Delta = dO' . O_pre would multiply by
// |dO'| summed over head_dim), then Delta and dG = dO * O_pre.
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) bwd_prep_kernel(const BwdArgs a) {
  const int64_t row = (int64_t)blockIdx.x * kWarps + threadIdx.x / 32;
  if (row >= (int64_t)a.batch * a.T * a.hq) return;
  const int lane = threadIdx.x & 31;
  const int vpl = a.D / 32;
  const int h = (int)(row % a.hq);
  const int t = (int)((row / a.hq) % a.T);
  const int b = (int)(row / ((int64_t)a.hq * a.T));
  const int g = h * a.hkv / a.hq;
  float q[kMaxVpl], o[kMaxVpl], d[kMaxVpl];
  load_row<T>(q, a.Q, row * a.D, lane, vpl);
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i) o[i] = 0.f;
  const float lse = a.lse[row];
  auto key = [&](const void* kb, const void* vb, int64_t off) {
    float k[kMaxVpl];
    load_row<T>(k, kb, off, lane, vpl);
    const float p = expf(dot(q, k, vpl) * a.scale - lse);
#pragma unroll
    for (int i = 0; i < kMaxVpl; ++i)
      if (i < vpl) o[i] = fmaf(p, ld<T>(vb, off + lane + 32 * i), o[i]);
  };
  const int nc = entries_of(a, b, t);
  for (int j = 0; j < nc; ++j) {
    const int64_t erow = entry_row(a, b, j, g);
    if (erow >= 0) key(a.kc, a.vc, erow * a.D);
  }
  for (int u = max(0, t - a.window + 1); u <= t; ++u)
    key(a.K, a.V, (((int64_t)b * a.T + u) * a.hkv + g) * a.D);
  load_row<T>(d, a.dO, row * a.D, lane, vpl);
  if (a.gate) {
    const int64_t goff = (int64_t)b * a.gs0 + (int64_t)t * a.gs1 + (int64_t)h * a.gs2;
#pragma unroll
    for (int i = 0; i < kMaxVpl; ++i) {
      if (i < vpl) {
        const float gv = ld<T>(a.gate, goff + lane + 32 * i);
        st<T>(a.dG, row * a.D + lane + 32 * i, d[i] * o[i]);
        d[i] *= gv;  // dO'
      }
    }
  }
  const float delta = dot(o, d, vpl);
  if (lane == 0) a.delta[row] = delta;
}

// ------------------------------------------------------------------------------ entries
// warp = (sequence b, entry j, KV head g, chunk c of query positions)
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) bwd_entries_kernel(const BwdArgs a, int nchunk) {
  const int64_t w = (int64_t)blockIdx.x * kWarps + threadIdx.x / 32;
  if (w >= (int64_t)a.batch * a.n_ent * a.hkv * nchunk) return;
  const int lane = threadIdx.x & 31;
  const int vpl = a.D / 32;
  const int c = (int)(w % nchunk);
  const int g = (int)((w / nchunk) % a.hkv);
  const int j = (int)((w / ((int64_t)nchunk * a.hkv)) % a.n_ent);
  const int b = (int)(w / ((int64_t)nchunk * a.hkv * a.n_ent));
  // entry j is visible to t iff (j + 1) * block <= t + 1 - window
  const int t_first = (j + 1) * a.block + a.window - 1;
  const int t0 = max(t_first, c * kEntryChunk);
  const int t1 = min(a.T, (c + 1) * kEntryChunk);
  if (t0 >= t1) return;
  const int64_t erow = entry_row(a, b, j, g);
  if (erow < 0) return;
  float kc[kMaxVpl], vc[kMaxVpl], dk[kMaxVpl], dv[kMaxVpl];
  load_row<T>(kc, a.kc, erow * a.D, lane, vpl);
  load_row<T>(vc, a.vc, erow * a.D, lane, vpl);
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i) dk[i] = dv[i] = 0.f;
  const int hpg = a.hq / a.hkv;
  for (int t = t0; t < t1; ++t) {
    if (j >= entries_of(a, b, t)) continue;  // a cache shorter than the visible count
    for (int h = g * hpg; h < (g + 1) * hpg; ++h) {
      const int64_t row = ((int64_t)b * a.T + t) * a.hq + h;
      float q[kMaxVpl], dop[kMaxVpl];
      load_row<T>(q, a.Q, row * a.D, lane, vpl);
      load_dop<T>(dop, a, b, t, h, lane, vpl);
      const float p = expf(dot(q, kc, vpl) * a.scale - a.lse[row]);
      const float ds = p * (dot(dop, vc, vpl) - a.delta[row]) * a.scale;
#pragma unroll
      for (int i = 0; i < kMaxVpl; ++i) {
        dk[i] = fmaf(ds, q[i], dk[i]);
        dv[i] = fmaf(p, dop[i], dv[i]);
      }
    }
  }
  const int64_t o = (((int64_t)b * a.n_ent + j) * a.hkv + g) * a.D;
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i) {
    if (i < vpl) {
      atomicAdd(a.dkc + o + lane + 32 * i, dk[i]);
      atomicAdd(a.dvc + o + lane + 32 * i, dv[i]);
    }
  }
}

// ------------------------------------------------------------------------------ raw
// warp = (sequence b, token u, KV head g): the window rows that see u, then the token's
// share of its block's entry gradient; writes dK, dV
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) bwd_raw_kernel(const BwdArgs a) {
  const int64_t w = (int64_t)blockIdx.x * kWarps + threadIdx.x / 32;
  if (w >= (int64_t)a.batch * a.T * a.hkv) return;
  const int lane = threadIdx.x & 31;
  const int vpl = a.D / 32;
  const int g = (int)(w % a.hkv);
  const int u = (int)((w / a.hkv) % a.T);
  const int b = (int)(w / ((int64_t)a.hkv * a.T));
  const int64_t krow = (((int64_t)b * a.T + u) * a.hkv + g) * a.D;
  float k[kMaxVpl], v[kMaxVpl], dk[kMaxVpl], dv[kMaxVpl];
  load_row<T>(k, a.K, krow, lane, vpl);
  load_row<T>(v, a.V, krow, lane, vpl);
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i) dk[i] = dv[i] = 0.f;
  const int hpg = a.hq / a.hkv;
  const int t1 = min(a.T, u + a.window);  // token u is in the window of t in [u, u + W - 1]
  for (int t = u; t < t1; ++t) {
    for (int h = g * hpg; h < (g + 1) * hpg; ++h) {
      const int64_t row = ((int64_t)b * a.T + t) * a.hq + h;
      float q[kMaxVpl], dop[kMaxVpl];
      load_row<T>(q, a.Q, row * a.D, lane, vpl);
      load_dop<T>(dop, a, b, t, h, lane, vpl);
      const float p = expf(dot(q, k, vpl) * a.scale - a.lse[row]);
      const float ds = p * (dot(dop, v, vpl) - a.delta[row]) * a.scale;
#pragma unroll
      for (int i = 0; i < kMaxVpl; ++i) {
        dk[i] = fmaf(ds, q[i], dk[i]);
        dv[i] = fmaf(p, dop[i], dv[i]);
      }
    }
  }
  // the entry of u's block is the mean of the block's tokens
  const int j = u / a.block;
  if (j < a.n_ent) {
    const float inv = 1.f / (float)(min(a.T, (j + 1) * a.block) - j * a.block);
    const int64_t o = (((int64_t)b * a.n_ent + j) * a.hkv + g) * a.D;
#pragma unroll
    for (int i = 0; i < kMaxVpl; ++i) {
      if (i < vpl) {
        dk[i] = fmaf(a.dkc[o + lane + 32 * i], inv, dk[i]);
        dv[i] = fmaf(a.dvc[o + lane + 32 * i], inv, dv[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i) {
    if (i < vpl) {
      st<T>(a.dK, krow + lane + 32 * i, dk[i]);
      st<T>(a.dV, krow + lane + 32 * i, dv[i]);
    }
  }
}

// ------------------------------------------------------------------------------ dq
template <typename T>
__global__ void __launch_bounds__(kWarps * 32) bwd_dq_kernel(const BwdArgs a) {
  const int64_t row = (int64_t)blockIdx.x * kWarps + threadIdx.x / 32;
  if (row >= (int64_t)a.batch * a.T * a.hq) return;
  const int lane = threadIdx.x & 31;
  const int vpl = a.D / 32;
  const int h = (int)(row % a.hq);
  const int t = (int)((row / a.hq) % a.T);
  const int b = (int)(row / ((int64_t)a.hq * a.T));
  const int g = h * a.hkv / a.hq;
  float q[kMaxVpl], dop[kMaxVpl], dq[kMaxVpl];
  load_row<T>(q, a.Q, row * a.D, lane, vpl);
  load_dop<T>(dop, a, b, t, h, lane, vpl);
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i) dq[i] = 0.f;
  const float lse = a.lse[row], delta = a.delta[row];
  auto key = [&](const void* kb, const void* vb, int64_t off) {
    float k[kMaxVpl], v[kMaxVpl];
    load_row<T>(k, kb, off, lane, vpl);
    load_row<T>(v, vb, off, lane, vpl);
    const float p = expf(dot(q, k, vpl) * a.scale - lse);
    const float ds = p * (dot(dop, v, vpl) - delta) * a.scale;
#pragma unroll
    for (int i = 0; i < kMaxVpl; ++i) dq[i] = fmaf(ds, k[i], dq[i]);
  };
  const int nc = entries_of(a, b, t);
  for (int j = 0; j < nc; ++j) {
    const int64_t erow = entry_row(a, b, j, g);
    if (erow >= 0) key(a.kc, a.vc, erow * a.D);
  }
  for (int u = max(0, t - a.window + 1); u <= t; ++u)
    key(a.K, a.V, (((int64_t)b * a.T + u) * a.hkv + g) * a.D);
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i)
    if (i < vpl) st<T>(a.dQ, row * a.D + lane + 32 * i, dq[i]);
}

template <typename T>
cudaError_t launch_all(const BwdArgs& a, cudaStream_t s) {
  const int64_t rows = (int64_t)a.batch * a.T * a.hq;
  const unsigned thr = kWarps * 32;
  auto blocks = [](int64_t n) { return (unsigned)((n + kWarps - 1) / kWarps); };
  cudaError_t e;
  bwd_prep_kernel<T><<<blocks(rows), thr, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int nchunk = (a.T + kEntryChunk - 1) / kEntryChunk;
  const int64_t ew = (int64_t)a.batch * a.n_ent * a.hkv * nchunk;
  if (ew > 0) {
    bwd_entries_kernel<T><<<blocks(ew), thr, 0, s>>>(a, nchunk);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  bwd_raw_kernel<T><<<blocks((int64_t)a.batch * a.T * a.hkv), thr, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_dq_kernel<T><<<blocks(rows), thr, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t backward_simt_workspace_bytes(const hca_desc& d) {
  const size_t n_ent = (size_t)((d.seqlen + d.block - 1) / d.block);
  const size_t delta = (size_t)d.batch * d.seqlen * d.hq;
  const size_t ent = (size_t)d.batch * n_ent * d.hkv * d.head_dim;
  return (((delta + 3) & ~size_t(3)) + 2 * ent) * sizeof(float);
}

cudaError_t launch_backward_simt(const hca_desc& d, const BackwardTensors& x, const hca_cache& c,
                                 void* ws, cudaStream_t s) {
  BwdArgs a{};
  a.Q = x.Q;
  a.K = x.K;
  a.V = x.V;
  a.kc = c.kc_pool;
  a.vc = c.vc_pool;
  a.lse = x.lse;
  a.dO = x.dO;
  a.gate = d.gate;
  a.gs0 = d.gate_strides[0];
  a.gs1 = d.gate_strides[1];
  a.gs2 = d.gate_strides[2];
  a.dQ = x.dQ;
  a.dK = x.dK;
  a.dV = x.dV;
  a.dG = x.dG;
  a.page_table = c.page_table;
  a.n_entries = c.n_entries;
  a.err_word = c.err_word;
  a.batch = d.batch;
  a.T = d.seqlen;
  a.hq = d.hq;
  a.hkv = d.hkv;
  a.D = d.head_dim;
  a.block = d.block;
  a.window = d.window;
  a.page_entries = c.page_entries;
  a.max_pages = c.max_pages;
  a.num_pages = c.num_pages;
  a.scale = d.scale;
  a.n_ent = (d.seqlen + d.block - 1) / d.block;
  const size_t delta = (size_t)d.batch * d.seqlen * d.hq;
  const size_t ent = (size_t)d.batch * a.n_ent * d.hkv * d.head_dim;
  a.delta = static_cast<float*>(ws);
  a.dkc = a.delta + ((delta + 3) & ~size_t(3));
  a.dvc = a.dkc + ent;
  cudaError_t e = cudaMemsetAsync(a.dkc, 0, 2 * ent * sizeof(float), s);
  if (e != cudaSuccess) return e;
  return d.dtype == HCA_F32 ? launch_all<float>(a, s) : launch_all<__nv_bfloat16>(a, s);
}

}  // namespace hca
