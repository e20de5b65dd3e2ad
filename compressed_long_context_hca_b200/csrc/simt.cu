// simt.cu -- float32 HCA attention on CUDA cores (no tensor cores, no TF32).
//
// This is the path for float32 inputs, where the tolerance (1e-5 absolute) rules out
// reduced-precision tensor-core arithmetic. One warp owns one (sequence, position, head)
// row: each lane holds head_dim/32 query elements, a key's score is a warp all-reduce of
// the lane partial dot products, and a single-pass online softmax keeps (max, sum, out).
//
// Key set of position t ([news 二.1] / [analysis 1] in include/hca.h): compressed entries
// j < n_c(t) = max(0, floor((t+1-window)/block)) read through the page table, then raw
// tokens max(0, t-window+1) .. t. Decode reads the raw tokens from a ring of `window`
// slots (token u in slot u % window).
#include <cuda_runtime.h>

#include "hca_internal.h"
#include "sm100.cuh"

namespace hca {
namespace {

constexpr int kMaxVpl = 16;  // head_dim <= 512
constexpr int kWarps = 4;

struct SimtArgs {
  const float* Q;
  const float* K;       // prefill raw keys [b, T, hkv, D]   | decode ring [n, W, hkv, D]
  const float* V;
  const float* kc;      // pools
  const float* vc;
  const int32_t* page_table;
  const int32_t* n_entries;
  int32_t* err_word;
  const int32_t* ctx_len;  // decode only
  const float* gate;
  int64_t gs0, gs1, gs2;
  float* O;
  float* lse;
  int32_t* dbg;
  int32_t batch, T, hq, hkv, D, block, window, page_entries, max_pages, num_pages;
  // prefill: query row t is position q0 + t; K/V row u is position kv0 + u, of Tk rows
  int32_t q0, kv0, Tk;
  float scale;
};

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

struct RowState {
  float m, l;
  float acc[kMaxVpl];
};

__device__ __forceinline__ void consume_key(RowState& st, const float (&q)[kMaxVpl],
                                            const float* k, const float* v, int lane, int vpl,
                                            float scale) {
  float part = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i)
    if (i < vpl) part = fmaf(q[i], k[lane + 32 * i], part);
  const float s = warp_sum(part) * scale;
  const float mn = fmaxf(st.m, s);
  const float alpha = expf(st.m - mn);  // st.m = -inf on the first key -> 0
  const float p = expf(s - mn);
  st.l = st.l * alpha + p;
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i)
    if (i < vpl) st.acc[i] = fmaf(st.acc[i], alpha, p * v[lane + 32 * i]);
  st.m = mn;
}

// Shared body: one warp, one row: position t of sequence b, head h, written at out_row.
template <bool kDecode>
__device__ void attend_row(const SimtArgs& a, int b, int t, int h, int64_t out_row,
                           int64_t gate_off, int64_t dbg_row) {
  const int lane = threadIdx.x & 31;
  const int vpl = a.D / 32;
  const int g = h * a.hkv / a.hq;
  float q[kMaxVpl];
  const float* qp = a.Q + out_row * a.D;
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i) q[i] = i < vpl ? qp[lane + 32 * i] : 0.f;

  RowState st;
  st.m = -INFINITY;
  st.l = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i) st.acc[i] = 0.f;

  int nc = (t + 1 - a.window) / a.block;
  if (t + 1 - a.window < 0) nc = 0;
  const int have = min(a.n_entries[b], a.max_pages * a.page_entries);
  if (nc > have) {
    if (lane == 0 && a.err_word) atomicOr(a.err_word, kErrCacheShort);
    nc = have;
  }
  for (int j = 0; j < nc; ++j) {
    const int page = a.page_table[(int64_t)b * a.max_pages + j / a.page_entries];
    if (page < 0 || page >= a.num_pages) {
      if (lane == 0 && a.err_word) atomicOr(a.err_word, kErrPageRange);
      continue;
    }
    const int64_t row = ((int64_t)page * a.page_entries + j % a.page_entries) * a.hkv + g;
    consume_key(st, q, a.kc + row * a.D, a.vc + row * a.D, lane, vpl, a.scale);
  }
  const int lo = max(0, t - a.window + 1);
  for (int u = lo; u <= t; ++u) {
    int64_t row;
    if (kDecode)
      row = ((int64_t)b * a.window + (u % a.window)) * a.hkv + g;
    else
      row = ((int64_t)b * a.Tk + (u - a.kv0)) * a.hkv + g;
    consume_key(st, q, a.K + row * a.D, a.V + row * a.D, lane, vpl, a.scale);
  }
  const float inv = 1.f / st.l;
  float* op = a.O + out_row * a.D;
  const float* gp = a.gate ? a.gate + gate_off : nullptr;
#pragma unroll
  for (int i = 0; i < kMaxVpl; ++i) {
    if (i < vpl) {
      float o = st.acc[i] * inv;
      if (gp) o *= gp[lane + 32 * i];
      op[lane + 32 * i] = o;
    }
  }
  if (lane == 0) {
    if (a.lse) a.lse[out_row] = st.m + logf(st.l);
    if (!kDecode && a.dbg && h == 0) {
      int32_t* dp = a.dbg + dbg_row * 3;
      dp[0] = nc;
      dp[1] = lo;
      dp[2] = t;
    }
  }
}

__global__ void __launch_bounds__(kWarps * 32) prefill_simt_kernel(SimtArgs a) {
  const int64_t row = (int64_t)blockIdx.x * kWarps + threadIdx.x / 32;
  const int64_t rows = (int64_t)a.batch * a.T * a.hq;
  if (row >= rows) return;
  const int h = (int)(row % a.hq);
  const int64_t bt = row / a.hq;
  const int tq = (int)(bt % a.T);  // query row; position q0 + tq
  const int b = (int)(bt / a.T);
  const int64_t goff = (int64_t)b * a.gs0 + (int64_t)tq * a.gs1 + (int64_t)h * a.gs2;
  attend_row<false>(a, b, tq + a.q0, h, row, goff, bt);
}

__global__ void __launch_bounds__(kWarps * 32) decode_simt_kernel(SimtArgs a) {
  const int64_t row = (int64_t)blockIdx.x * kWarps + threadIdx.x / 32;
  const int64_t rows = (int64_t)a.batch * a.hq;
  if (row >= rows) return;
  const int h = (int)(row % a.hq);
  const int b = (int)(row / a.hq);
  // ctx_len is clamped into [1, seqlen] (flagged), the same rule as the tensor-core decode
  const int ctx = a.ctx_len[b];
  if ((ctx < 1 || ctx > a.T) && h == 0 && (threadIdx.x & 31) == 0 && a.err_word)
    atomicOr(a.err_word, kErrCtxRange);
  const int t = min(max(ctx, 1), a.T) - 1;
  const int64_t goff = (int64_t)b * a.gs0 + (int64_t)h * a.gs2;
  attend_row<true>(a, b, t, h, row, goff, 0);
}

SimtArgs make_args(const hca_desc& d, const hca_cache& c) {
  SimtArgs a{};
  a.kc = static_cast<const float*>(c.kc_pool);
  a.vc = static_cast<const float*>(c.vc_pool);
  a.page_table = c.page_table;
  a.n_entries = c.n_entries;
  a.err_word = c.err_word;
  a.gate = static_cast<const float*>(d.gate);
  a.gs0 = d.gate_strides[0];
  a.gs1 = d.gate_strides[1];
  a.gs2 = d.gate_strides[2];
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
  return a;
}

}  // namespace

cudaError_t launch_prefill_simt(const hca_desc& d, const void* Q, const void* K,
                                const void* V, const hca_cache& c, void* O, float* lse,
                                int32_t* dbg_mask, const PrefillRange& r, cudaStream_t s) {
  SimtArgs a = make_args(d, c);
  a.q0 = r.q_pos0;
  a.kv0 = r.kv_pos0;
  a.Tk = r.kv_len;
  a.Q = static_cast<const float*>(Q);
  a.K = static_cast<const float*>(K);
  a.V = static_cast<const float*>(V);
  a.O = static_cast<float*>(O);
  a.lse = lse;
  a.dbg = dbg_mask;
  const int64_t rows = (int64_t)d.batch * d.seqlen * d.hq;
  const int64_t blocks = (rows + kWarps - 1) / kWarps;
  if (blocks == 0) return cudaSuccess;
  prefill_simt_kernel<<<(unsigned)blocks, kWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_decode_simt(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                               const hca_cache& c, const void* ring_k, const void* ring_v,
                               void* O, float* lse, cudaStream_t s) {
  SimtArgs a = make_args(d, c);
  a.Q = static_cast<const float*>(Q);
  a.K = static_cast<const float*>(ring_k);
  a.V = static_cast<const float*>(ring_v);
  a.ctx_len = ctx_len;
  a.O = static_cast<float*>(O);
  a.lse = lse;
  const int64_t rows = (int64_t)d.batch * d.hq;
  const int64_t blocks = (rows + kWarps - 1) / kWarps;
  if (blocks == 0) return cudaSuccess;
  decode_simt_kernel<<<(unsigned)blocks, kWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace hca
