// backward_tc.cu -- gradients of the HCA prefill for bf16 on tcgen05 tensor cores: the
// contractions run on gemm_tc (bf16 operands, float32 accumulation), the softmax part on
// CUDA cores.
//
// The operation is the one of backward_simt.cu (the exact derivative of the prefill output;
// [analysis infra 3] in include/hca.h). At head_dim 512 a 128-row tile's float32 dQ fills
// all of TMEM, so instead of one fused kernel the backward materialises the score-shaped
// quantities of a group of query positions in the workspace and runs every product as a
// dense GEMM:
//   per sequence b: gather the entries Kc, Vc into contiguous rows; zero the float32
//   accumulators dKc, dVc [entries, 512] and dK, dV [T, 512] (window part);
//   per group of G positions (R = G * hq query rows):
//     Sc = Q Kc^T, dPc = dO' Vc^T           [R, E]    (E = entries visible to the group)
//     Sw = Q K_band^T, dPw = dO' V_band^T   [R, 256]  (per 128 positions, the 256 raw keys
//                                                      that hold their windows)
//     softmax kernel: P = exp(scale S - lse), Delta = sum P dP over the row's visible keys,
//       dS = scale P (dP - Delta); P and dS written as bf16 pairs hi + lo
//     dQ = dSc Kc + dSw K_band;  dKc += dSc^T Q;  dVc += Pc^T dO';  dK_band += dSw^T Q;
//     dV_band += Pw^T dO'  (the K-long products split over CTAs with float32 atomics)
//     with a gate: dO' = dO * G (bf16 pair), O_pre = Pc Vc + Pw V_band, dG = dO * O_pre
//   then dK[u] = dK_band[u] + dKc[u / block] / count, the same for dV, cast to bf16.
// Every bf16 operand that is not an input (P, dS, dO') enters as hi + lo, two products:
// the gradients are long sums whose terms can be far larger than the result, and one bf16
// rounding (2^-9) of each term would swamp it.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <string.h>

#include <utility>

#include "gemm_tc.h"
#include "hca_internal.h"
#include "sm100.cuh"

namespace hca {
namespace {

constexpr int kD = 512;
constexpr int kBand = 256;   // raw keys per 128 query positions: 128 before them + theirs
constexpr int kSub = 128;    // query positions per band
constexpr int kGroup = 1024; // query positions per group

__host__ __device__ __forceinline__ int visible_count(int t, int block, int window) {
  const int x = t + 1 - window;
  return x < 0 ? 0 : x / block;
}

// entries j < n_ent of sequence b into contiguous rows; missing ones are zero and flagged
__global__ void gather_entries_kernel(const __nv_bfloat16* kc_pool, const __nv_bfloat16* vc_pool,
                                      const int32_t* page_table, const int32_t* n_entries,
                                      int b, int n_ent, int PE, int max_pages, int num_pages,
                                      __nv_bfloat16* kc, __nv_bfloat16* vc, int32_t* err) {
  const int j = blockIdx.x;
  const int have = min(n_entries[b], max_pages * PE);
  int64_t row = -1;
  if (j < have) {
    const int page = page_table[(int64_t)b * max_pages + j / PE];
    if (page >= 0 && page < num_pages)
      row = (int64_t)page * PE + j % PE;
    else if (threadIdx.x == 0 && err)
      atomicOr(err, kErrPageRange);
  }
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (int i = threadIdx.x; i < kD / 8; i += blockDim.x) {
    uint4 a = z, v = z;
    if (row >= 0) {
      a = reinterpret_cast<const uint4*>(kc_pool + row * kD)[i];
      v = reinterpret_cast<const uint4*>(vc_pool + row * kD)[i];
    }
    reinterpret_cast<uint4*>(kc + (int64_t)j * kD)[i] = a;
    reinterpret_cast<uint4*>(vc + (int64_t)j * kD)[i] = v;
  }
}

// dO' = dO * G of the group's rows as a bf16 pair
__global__ void gate_dop_kernel(const __nv_bfloat16* dO, const __nv_bfloat16* G, int64_t gs0,
                                int64_t gs1, int64_t gs2, int b, int p0, int hq, int R,
                                __nv_bfloat16* hi, __nv_bfloat16* lo, int64_t r0) {
  const int r = blockIdx.x;
  if (r >= R) return;
  const int t = p0 + r / hq, h = r % hq;
  const __nv_bfloat16* d = dO + (r0 + r) * kD;
  const __nv_bfloat16* g = G + (int64_t)b * gs0 + (int64_t)t * gs1 + (int64_t)h * gs2;
  for (int c = threadIdx.x * 2; c < kD; c += blockDim.x * 2) {
    const float x0 = __bfloat162float(d[c]) * __bfloat162float(g[c]);
    const float x1 = __bfloat162float(d[c + 1]) * __bfloat162float(g[c + 1]);
    uint32_t h2, l2;
    split_bf16x2(x0, x1, h2, l2);
    *reinterpret_cast<uint32_t*>(hi + (int64_t)r * kD + c) = h2;
    *reinterpret_cast<uint32_t*>(lo + (int64_t)r * kD + c) = l2;
  }
}

struct SoftmaxArgs {
  const float* sc;
  const float* dpc;
  const float* sw;
  const float* dpw;
  const float* lse;  // [b T hq] natural log
  __nv_bfloat16 *pc_hi, *pc_lo, *dsc_hi, *dsc_lo, *pw_hi, *pw_lo, *dsw_hi, *dsw_lo;
  int64_t r0;        // global row of the group's row 0
  int R, E, Ep, hq, p0, block, window;
  float scale;
};

// one warp per row: Delta over the row's visible keys, then P and dS as bf16 pairs
__global__ void __launch_bounds__(128) softmax_bwd_kernel(const SoftmaxArgs a) {
  const int r = blockIdx.x * 4 + threadIdx.x / 32;
  if (r >= a.R) return;
  const int lane = threadIdx.x & 31;
  const int t = a.p0 + r / a.hq;
  const float l2e = 1.4426950408889634f;
  const float sl2 = a.scale * l2e;
  const float lse2 = a.lse[a.r0 + r] * l2e;
  const int nc = min(visible_count(t, a.block, a.window), a.E);
  const int lo = max(0, t - a.window + 1);
  const int kb = a.p0 + ((t - a.p0) / kSub) * kSub - kSub;  // position of band column 0
  const float* sc = a.sc + (int64_t)r * a.Ep;
  const float* dpc = a.dpc + (int64_t)r * a.Ep;
  const float* sw = a.sw + (int64_t)r * kBand;
  const float* dpw = a.dpw + (int64_t)r * kBand;
  float delta = 0.f;
  for (int j = lane; j < nc; j += 32) delta = fmaf(exp2f(fmaf(sc[j], sl2, -lse2)), dpc[j], delta);
  for (int j = lane; j < kBand; j += 32) {
    const int u = kb + j;
    if (u >= lo && u <= t) delta = fmaf(exp2f(fmaf(sw[j], sl2, -lse2)), dpw[j], delta);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) delta += __shfl_xor_sync(0xffffffffu, delta, o);
  const int64_t oc = (int64_t)r * a.Ep;
  for (int j = 2 * lane; j < a.Ep; j += 64) {
    float p[2], ds[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const bool in = j + e < nc;
      p[e] = in ? exp2f(fmaf(sc[j + e], sl2, -lse2)) : 0.f;
      ds[e] = in ? a.scale * p[e] * (dpc[j + e] - delta) : 0.f;
    }
    uint32_t ph, pl, dh, dl;
    split_bf16x2(p[0], p[1], ph, pl);
    split_bf16x2(ds[0], ds[1], dh, dl);
    *reinterpret_cast<uint32_t*>(a.pc_hi + oc + j) = ph;
    *reinterpret_cast<uint32_t*>(a.pc_lo + oc + j) = pl;
    *reinterpret_cast<uint32_t*>(a.dsc_hi + oc + j) = dh;
    *reinterpret_cast<uint32_t*>(a.dsc_lo + oc + j) = dl;
  }
  const int64_t ow = (int64_t)r * kBand;
  for (int j = 2 * lane; j < kBand; j += 64) {
    float p[2], ds[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int u = kb + j + e;
      const bool in = u >= lo && u <= t;
      p[e] = in ? exp2f(fmaf(sw[j + e], sl2, -lse2)) : 0.f;
      ds[e] = in ? a.scale * p[e] * (dpw[j + e] - delta) : 0.f;
    }
    uint32_t ph, pl, dh, dl;
    split_bf16x2(p[0], p[1], ph, pl);
    split_bf16x2(ds[0], ds[1], dh, dl);
    *reinterpret_cast<uint32_t*>(a.pw_hi + ow + j) = ph;
    *reinterpret_cast<uint32_t*>(a.pw_lo + ow + j) = pl;
    *reinterpret_cast<uint32_t*>(a.dsw_hi + ow + j) = dh;
    *reinterpret_cast<uint32_t*>(a.dsw_lo + ow + j) = dl;
  }
}

// float32 rows -> bf16 rows (dQ of a group; dG = dO * O_pre with mul != nullptr)
__global__ void rows_to_bf16_kernel(const float* src, const __nv_bfloat16* mul, int64_t n,
                                    __nv_bfloat16* dst) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    float v = src[i];
    if (mul) v *= __bfloat162float(mul[i]);
    dst[i] = __float2bfloat16_rn(v);
  }
}

// dK[u] = dKw[u] + dKc[u / block] / count(block), the same for dV; bf16 out
__global__ void finalize_kv_kernel(const float* dkw, const float* dvw, const float* dkc,
                                   const float* dvc, int T, int block, int n_ent,
                                   __nv_bfloat16* dK, __nv_bfloat16* dV) {
  const int u = blockIdx.x;
  const int j = u / block;
  const float inv = 1.f / (float)(min(T, (j + 1) * block) - j * block);
  for (int c = threadIdx.x; c < kD; c += blockDim.x) {
    float k = dkw[(int64_t)u * kD + c], v = dvw[(int64_t)u * kD + c];
    if (j < n_ent) {
      k = fmaf(dkc[(int64_t)j * kD + c], inv, k);
      v = fmaf(dvc[(int64_t)j * kD + c], inv, v);
    }
    dK[(int64_t)u * kD + c] = __float2bfloat16_rn(k);
    dV[(int64_t)u * kD + c] = __float2bfloat16_rn(v);
  }
}

// ------------------------------------------------------------------------------ plan
struct Plan {
  int G, R, Ep, NE;
  size_t kc, vc, dkc, dvc, dkw, dvw;                        // per sequence
  size_t sc, dpc, pch, pcl, dsch, dscl;                     // [R, Ep]
  size_t sw, dpw, pwh, pwl, dswh, dswl;                     // [R, 256]
  size_t dq, doph, dopl, opre;                              // [R, 512]
  size_t total;
};

Plan make_plan(const hca_desc& d) {
  Plan p;
  memset(&p, 0, sizeof(p));
  p.G = d.seqlen < kGroup ? ((d.seqlen + kSub - 1) / kSub) * kSub : kGroup;
  p.R = p.G * d.hq;
  p.NE = (d.seqlen + d.block - 1) / d.block;
  const int nvis = visible_count(d.seqlen - 1, d.block, d.window);
  p.Ep = ((nvis > 0 ? nvis : 1) + 7) & ~7;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += (bytes + 255) & ~size_t(255);
    return o;
  };
  const size_t T = (size_t)d.seqlen, NE = (size_t)p.NE, R = (size_t)p.R, Ep = (size_t)p.Ep;
  p.kc = take(NE * kD * 2);
  p.vc = take(NE * kD * 2);
  p.dkc = take(NE * kD * 4);
  p.dvc = take(NE * kD * 4);
  p.dkw = take(T * kD * 4);
  p.dvw = take(T * kD * 4);
  p.sc = take(R * Ep * 4);
  p.dpc = take(R * Ep * 4);
  p.pch = take(R * Ep * 2);
  p.pcl = take(R * Ep * 2);
  p.dsch = take(R * Ep * 2);
  p.dscl = take(R * Ep * 2);
  p.sw = take(R * kBand * 4);
  p.dpw = take(R * kBand * 4);
  p.pwh = take(R * kBand * 2);
  p.pwl = take(R * kBand * 2);
  p.dswh = take(R * kBand * 2);
  p.dswl = take(R * kBand * 2);
  p.dq = take(R * kD * 4);
  if (d.gate) {
    p.doph = take(R * kD * 2);
    p.dopl = take(R * kD * 2);
    p.opre = take(R * kD * 4);
  }
  p.total = off;
  return p;
}

GemmOperand kmajor(const void* ptr, int64_t rows, int64_t cols, int64_t ld, int32_t shift = 0,
                   int32_t bstride = 0) {
  return GemmOperand{ptr, rows, cols, ld, false, shift, bstride};
}
GemmOperand mnmajor(const void* ptr, int64_t rows, int64_t cols, int64_t ld, int32_t shift = 0,
                    int32_t bstride = 0) {
  return GemmOperand{ptr, rows, cols, ld, true, shift, bstride};
}
GemmOutput out_rows(float* ptr, int64_t ld, int32_t rows, int32_t shift = 0, int32_t bstride = 0,
                    int32_t zdiv = 1, bool atomic = false) {
  return GemmOutput{ptr, ld, shift, bstride, rows, zdiv, atomic, false};
}

}  // namespace

bool backward_tc_supported(const hca_desc& d) {
  return d.dtype == HCA_BF16 && d.head_dim == kD && d.hkv == 1 && d.window >= 1 &&
         d.window <= kSub && d.hq >= 1 && d.hq <= 128 &&
         (int64_t)d.batch * d.seqlen * d.hq < (int64_t(1) << 31);
}

size_t backward_tc_workspace_bytes(const hca_desc& d) { return make_plan(d).total; }

cudaError_t launch_backward_tc(const hca_desc& d, const BackwardTensors& x, const hca_cache& c,
                               void* ws, cudaStream_t s) {
  const Plan pl = make_plan(d);
  uint8_t* w = static_cast<uint8_t*>(ws);
  auto F = [&](size_t o) { return reinterpret_cast<float*>(w + o); };
  auto H = [&](size_t o) { return reinterpret_cast<__nv_bfloat16*>(w + o); };
  const int T = d.seqlen, hq = d.hq;
  const int64_t rowsQ = (int64_t)d.batch * T * hq, rowsK = (int64_t)d.batch * T;
  const bool gated = d.gate != nullptr;
  const auto* Gp = static_cast<const __nv_bfloat16*>(d.gate);
  int32_t* err = c.err_word;
  cudaError_t e;
#define HCA_TRY(x)                       \
  do {                                   \
    if ((e = (x)) != cudaSuccess) return e; \
  } while (0)
  for (int b = 0; b < d.batch; ++b) {
    if (pl.NE > 0)
      gather_entries_kernel<<<pl.NE, 64, 0, s>>>(
          static_cast<const __nv_bfloat16*>(c.kc_pool), static_cast<const __nv_bfloat16*>(c.vc_pool),
          c.page_table, c.n_entries, b, pl.NE, c.page_entries, c.max_pages, c.num_pages,
          H(pl.kc), H(pl.vc), err);
    HCA_TRY(cudaGetLastError());
    HCA_TRY(cudaMemsetAsync(F(pl.dkc), 0, (size_t)pl.NE * kD * 4, s));
    HCA_TRY(cudaMemsetAsync(F(pl.dvc), 0, (size_t)pl.NE * kD * 4, s));
    HCA_TRY(cudaMemsetAsync(F(pl.dkw), 0, (size_t)T * kD * 4, s));
    HCA_TRY(cudaMemsetAsync(F(pl.dvw), 0, (size_t)T * kD * 4, s));
    for (int p0 = 0; p0 < T; p0 += pl.G) {
      const int p1 = p0 + pl.G < T ? p0 + pl.G : T;
      const int R = (p1 - p0) * hq;
      const int64_t r0 = ((int64_t)b * T + p0) * hq;
      const int E = visible_count(p1 - 1, d.block, d.window);
      const int nsub = (p1 - p0 + kSub - 1) / kSub;
      const int Mw = kSub * hq;  // rows of one band
      const int32_t kv_row0 = (int32_t)((int64_t)b * T + p0 - kSub);
      // dO' (pair) of the group: dO itself without a gate
      GemmOperand dop_hi = kmajor(x.dO, rowsQ, kD, kD, (int32_t)r0);
      GemmOperand dop_lo = dop_hi;
      GemmOperand dop_hi_mn = mnmajor(x.dO, rowsQ, kD, kD, (int32_t)r0);
      GemmOperand dop_lo_mn = dop_hi_mn;
      if (gated) {
        gate_dop_kernel<<<R, 128, 0, s>>>(static_cast<const __nv_bfloat16*>(x.dO), Gp,
                                          d.gate_strides[0], d.gate_strides[1],
                                          d.gate_strides[2], b, p0, hq, R, H(pl.doph), H(pl.dopl),
                                          r0);
        HCA_TRY(cudaGetLastError());
        dop_hi = kmajor(H(pl.doph), R, kD, kD);
        dop_lo = kmajor(H(pl.dopl), R, kD, kD);
        dop_hi_mn = mnmajor(H(pl.doph), R, kD, kD);
        dop_lo_mn = mnmajor(H(pl.dopl), R, kD, kD);
      }
      const GemmOperand Qg = kmajor(x.Q, rowsQ, kD, kD, (int32_t)r0);
      const GemmOperand Qg_mn = mnmajor(x.Q, rowsQ, kD, kD, (int32_t)r0);
      // ---- scores and dP: compressed part [R, E], window bands [R, 256]
      const GemmOperand* dop_lo_p = gated ? &dop_lo : nullptr;
      if (E > 0) {
        HCA_TRY(gemm_tc(Qg, nullptr, kmajor(H(pl.kc), pl.NE, kD, kD), out_rows(F(pl.sc), pl.Ep, R),
                        R, E, kD, 1, 1.f, 0.f, err, s));
        HCA_TRY(gemm_tc(dop_hi, dop_lo_p, kmajor(H(pl.vc), pl.NE, kD, kD),
                        out_rows(F(pl.dpc), pl.Ep, R), R, E, kD, 1, 1.f, 0.f, err, s));
      }
      const GemmOperand Qb = kmajor(x.Q, rowsQ, kD, kD, (int32_t)r0, Mw);
      const GemmOperand Kband = kmajor(x.K, rowsK, kD, kD, kv_row0, kSub);
      const GemmOperand Vband = kmajor(x.V, rowsK, kD, kD, kv_row0, kSub);
      HCA_TRY(gemm_tc(Qb, nullptr, Kband, out_rows(F(pl.sw), kBand, R, 0, Mw), Mw, kBand, kD,
                      nsub, 1.f, 0.f, err, s));
      {
        GemmOperand a = dop_hi, al = dop_lo;
        a.bstride = al.bstride = Mw;
        HCA_TRY(gemm_tc(a, gated ? &al : nullptr, Vband, out_rows(F(pl.dpw), kBand, R, 0, Mw), Mw,
                        kBand, kD, nsub, 1.f, 0.f, err, s));
      }
      // ---- P, Delta, dS
      SoftmaxArgs sa;
      sa.sc = F(pl.sc);
      sa.dpc = F(pl.dpc);
      sa.sw = F(pl.sw);
      sa.dpw = F(pl.dpw);
      sa.lse = x.lse;
      sa.pc_hi = H(pl.pch);
      sa.pc_lo = H(pl.pcl);
      sa.dsc_hi = H(pl.dsch);
      sa.dsc_lo = H(pl.dscl);
      sa.pw_hi = H(pl.pwh);
      sa.pw_lo = H(pl.pwl);
      sa.dsw_hi = H(pl.dswh);
      sa.dsw_lo = H(pl.dswl);
      sa.r0 = r0;
      sa.R = R;
      sa.E = E;
      sa.Ep = pl.Ep;
      sa.hq = hq;
      sa.p0 = p0;
      sa.block = d.block;
      sa.window = d.window;
      sa.scale = d.scale;
      softmax_bwd_kernel<<<(R + 3) / 4, 128, 0, s>>>(sa);
      HCA_TRY(cudaGetLastError());
      // ---- products with a bf16 pair operand X = hi + lo (one pass of gemm_tc each)
      auto pair = [&](size_t hi, size_t lo, int64_t rows, int64_t cols, bool mn, int32_t bst) {
        return std::make_pair(GemmOperand{H(hi), rows, cols, cols, mn, 0, bst},
                              GemmOperand{H(lo), rows, cols, cols, mn, 0, bst});
      };
      // dQ = dSc Kc + dSw K_band  (float32 rows, then bf16)
      {
        bool first = true;
        if (E > 0) {
          auto ds = pair(pl.dsch, pl.dscl, R, pl.Ep, false, 0);
          const GemmOperand kc_mn = mnmajor(H(pl.kc), pl.NE, kD, kD);
          HCA_TRY(gemm_tc(ds.first, &ds.second, kc_mn, out_rows(F(pl.dq), kD, R), R, kD, E, 1,
                          1.f, 0.f, err, s));
          first = false;
        }
        auto dsw = pair(pl.dswh, pl.dswl, R, kBand, false, Mw);
        const GemmOperand kb_mn = mnmajor(x.K, rowsK, kD, kD, kv_row0, kSub);
        HCA_TRY(gemm_tc(dsw.first, &dsw.second, kb_mn, out_rows(F(pl.dq), kD, R, 0, Mw), Mw, kD,
                        kBand, nsub, 1.f, first ? 0.f : 1.f, err, s));
        const int64_t n = (int64_t)R * kD;
        rows_to_bf16_kernel<<<1184, 256, 0, s>>>(F(pl.dq), nullptr, n,
                                                 static_cast<__nv_bfloat16*>(x.dQ) + r0 * kD);
        HCA_TRY(cudaGetLastError());
      }
      // dG = dO * O_pre, O_pre = Pc Vc + Pw V_band
      if (gated) {
        bool first = true;
        if (E > 0) {
          auto pc = pair(pl.pch, pl.pcl, R, pl.Ep, false, 0);
          const GemmOperand vc_mn = mnmajor(H(pl.vc), pl.NE, kD, kD);
          HCA_TRY(gemm_tc(pc.first, &pc.second, vc_mn, out_rows(F(pl.opre), kD, R), R, kD, E, 1,
                          1.f, 0.f, err, s));
          first = false;
        }
        auto pw = pair(pl.pwh, pl.pwl, R, kBand, false, Mw);
        const GemmOperand vb_mn = mnmajor(x.V, rowsK, kD, kD, kv_row0, kSub);
        HCA_TRY(gemm_tc(pw.first, &pw.second, vb_mn, out_rows(F(pl.opre), kD, R, 0, Mw), Mw, kD,
                        kBand, nsub, 1.f, first ? 0.f : 1.f, err, s));
        // dG rows of the group: dO * O_pre (dG is dense [b, T, hq, D])
        rows_to_bf16_kernel<<<1184, 256, 0, s>>>(F(pl.opre),
                                                 static_cast<const __nv_bfloat16*>(x.dO) + r0 * kD,
                                                 (int64_t)R * kD,
                                                 static_cast<__nv_bfloat16*>(x.dG) + r0 * kD);
        HCA_TRY(cudaGetLastError());
      }
      // dKc += dSc^T Q, dVc += Pc^T dO'  (K = R rows, split over CTAs)
      if (E > 0) {
        const int ksplit = 1024;
        const int nspl = (R + ksplit - 1) / ksplit;
        auto dsT = pair(pl.dsch, pl.dscl, R, pl.Ep, true, ksplit);
        auto pT = pair(pl.pch, pl.pcl, R, pl.Ep, true, ksplit);
        GemmOperand q = Qg_mn;
        q.bstride = ksplit;
        GemmOperand dh = dop_hi_mn, dl = dop_lo_mn;
        dh.bstride = dl.bstride = ksplit;
        const GemmOutput okc = out_rows(F(pl.dkc), kD, pl.NE, 0, 0, 1, true);
        const GemmOutput ovc = out_rows(F(pl.dvc), kD, pl.NE, 0, 0, 1, true);
        HCA_TRY(gemm_tc(dsT.first, &dsT.second, q, okc, E, kD, ksplit, nspl, 1.f, 0.f, err, s));
        HCA_TRY(gemm_tc(pT.first, &pT.second, dh, ovc, E, kD, ksplit, nspl, 1.f, 0.f, err, s));
        if (gated) HCA_TRY(gemm_tc(pT.first, nullptr, dl, ovc, E, kD, ksplit, nspl, 1.f, 0.f, err, s));
      }
      // dK_band += dSw^T Q_band, dV_band += Pw^T dO'_band  (K = 128 hq rows per band,
      // split in 4; bands of neighbouring sub-chunks overlap: atomics)
      {
        const int sp = 4;
        const int kb = Mw / sp;
        auto dsT = pair(pl.dswh, pl.dswl, R, kBand, true, kb);
        auto pT = pair(pl.pwh, pl.pwl, R, kBand, true, kb);
        GemmOperand q = Qg_mn;
        q.bstride = kb;
        GemmOperand dh = dop_hi_mn, dl = dop_lo_mn;
        dh.bstride = dl.bstride = kb;
        const GemmOutput ok = out_rows(F(pl.dkw), kD, T, p0 - kSub, kSub, sp, true);
        const GemmOutput ov = out_rows(F(pl.dvw), kD, T, p0 - kSub, kSub, sp, true);
        const int nb = nsub * sp;
        HCA_TRY(gemm_tc(dsT.first, &dsT.second, q, ok, kBand, kD, kb, nb, 1.f, 0.f, err, s));
        HCA_TRY(gemm_tc(pT.first, &pT.second, dh, ov, kBand, kD, kb, nb, 1.f, 0.f, err, s));
        if (gated) HCA_TRY(gemm_tc(pT.first, nullptr, dl, ov, kBand, kD, kb, nb, 1.f, 0.f, err, s));
      }
    }
    finalize_kv_kernel<<<T, 128, 0, s>>>(F(pl.dkw), F(pl.dvw), F(pl.dkc), F(pl.dvc), T, d.block,
                                         pl.NE, static_cast<__nv_bfloat16*>(x.dK) + (int64_t)b * T * kD,
                                         static_cast<__nv_bfloat16*>(x.dV) + (int64_t)b * T * kD);
    HCA_TRY(cudaGetLastError());
  }
#undef HCA_TRY
  return cudaSuccess;
}

}  // namespace hca
