// decode_fp8.cu -- one HCA decode step over an 8-bit (e4m3) compressed cache, on tcgen05
// tensor cores, followed (with several splits) by the merge of the 16-bit decode.
//
// Operation ([news 二.1] / [analysis 1] / [gate] / [serve fp8] in include/hca.h): the newest
// token t = ctx_len - 1 attends with one softmax to the compressed entries j < n_c(t),
// stored as e4m3 codes with one float32 scale per pool (value = value(code) * scale), and
// to the last `window` raw tokens, which stay bf16 in a ring of `window` slots.
//
// Design for sm_100a (HBM-bound; a compressed tile of 128 entries is 64 KB of keys and
// 64 KB of values, half of the 16-bit cache):
//  * Scores of a compressed tile run on kind::f8f6f4 UMMAs straight from the stored codes
//    (K-major, as TMA lands them). The query is carried as two e4m3 parts: with
//    r_h a power of two per head that puts the head's largest |q| in [128, 256),
//    q / r_h = Q1 + Q2, Q1 = e4m3(q / r_h), Q2 = e4m3(q / r_h - Q1). A bf16 q has 8
//    significant bits; Q1 takes the top 4 and the remainder has at most 4, so the two parts
//    are exact for every element within 2^9 of the head's largest (|q / r_h| >= 1/4, where
//    the remainder's last bit is still an e4m3 step); below, the part error is at most 2^-10,
//    i.e. 2^-17 of the largest |q / r_h|. Both parts accumulate into one TMEM accumulator,
//    S = Q1 K + Q2 K (two UMMAs per 32-code step), and the softmax forms
//    s = S * r_h * k_scale * scale.
//  * P.V runs on kind::f16 with f16 operands. The e4m3 values arrive by TMA in a ring of
//    their own (one 16 KB box = 32 keys x 512 codes); converter warps widen each 16-key
//    group to f16 values times 2^-8 (exact, by moving the code's bits) into two MN-major
//    128-byte-swizzled buffers (each warp hands its part of a group over on its own; the
//    P.V warp releases a box once both of its groups are in).
//    P enters as one f16 value (11 significant bits: its rounding moves the output by at
//    most 2^-12 of the value spread, a quarter of the bf16 output's own rounding),
//    pre-scaled by 2^7 so that small P stay clear of the f16 subnormal range while the
//    largest (2^15 between lazy rescales) stays finite. O accumulates in units of the
//    widened values; v_scale * 2^8 multiplies it once at the end.
//  * The ring tile (the raw window, bf16) is the last tile of the last split and runs the
//    16-bit way inside the same CTA: once the last e4m3 score MMA has completed, the bf16
//    query replaces Q1/Q2 in shared memory, its scores accumulate in the score buffer
//    (kind::f16 bf16), its P goes to bf16 hi + lo parts divided by v_scale * 2^8 (O keeps
//    its units), and its values land in the same V buffers by TMA.
//  * Roles: warp 0 loads the K boxes into a 3-slot K ring (128 keys x one 128-byte column
//    chunk; the window tile's bf16 K in 64-column chunks) and the bf16 query (staged for
//    the converters at the start, and again for the window tile); warp 11 loads the e4m3 V
//    boxes into a 3-slot V ring; warp 1 issues the score UMMAs, warp 10 the P.V UMMAs;
//    warps 2-5 run the softmax (lazy rescale, as the 16-bit kernel) and the epilogue;
//    warps 6-9 widen V; warps 2-9 together prepare Q1/Q2 at the start. With a ring update
//    requested, warp 0 writes the new K row and the thread of warp 6 that loads the
//    window's values the new V row, each before its own loads of the window.
//  * TMEM: O (64 x 512 f32, M = 64 layout) in lanes 0-15 of each 32-lane subpartition;
//    two score buffers (128 columns each) in lanes 16-31.
//  * All mbarrier waits are bounded (HCA_ERR_TIMEOUT on give-up); on give-up every issuing
//    thread waits (bounded) for its own copies still in flight before the CTA leaves.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <string.h>

#include "decode_keys.cuh"
#include "decode_softmax.cuh"
#include "hca_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace hca {
namespace {

using namespace dkeys;
using namespace dsoft;

constexpr int kM = 64;    // head rows
constexpr int kD = 512;
// K load warp, score-MMA warp, 4 softmax warps, 4 converter warps, P.V-MMA warp,
// V load warp
constexpr int kThreads = 384;
constexpr int kPvWarp = 10;
constexpr int kVLoadWarp = 11;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kLaneS = 16u << 16;   // lane offset of the score accumulators

constexpr uint32_t kQChunkBytes = kM * 128;     // 8 KB: 64 rows x 128 bytes (either type)
constexpr uint32_t kQPartBytes = 4 * kQChunkBytes;  // 32 KB: one e4m3 part of the query
constexpr uint32_t kQ16Bytes = 8 * kQChunkBytes;    // 64 KB: the bf16 query
constexpr uint32_t kPChunkBytes = kM * 128;     // 8 KB: 64 rows x 64 keys (16-bit)
constexpr uint32_t kPBytes = 2 * kPChunkBytes;  // 16 KB: one part of P (128 keys)
constexpr int kKStages = 3;                     // K ring: 16 KB boxes
constexpr int kV8Stages = 3;                    // V ring: 16 KB boxes of e4m3 values
constexpr uint32_t kSlot = 16384;               // 16 KB ring slot
constexpr int kVRows = 32;                      // keys of one e4m3 V box (4 chunks x 4 KB)
constexpr uint32_t kV8Chunk = kVRows * 128;     // 4 KB: 32 keys x 128 codes
constexpr int kVStages = 2;
constexpr uint32_t kVChunkBytes = 16 * 128;     // 2 KB: 16 keys x 64 values (16-bit)
constexpr uint32_t kVSlot = 8 * kVChunkBytes;   // 16 KB: 16 keys x 512 values

constexpr uint32_t kOffQ = 0;                           // Q1 | Q2, later the bf16 query
constexpr uint32_t kOffP = kQ16Bytes;                   // P hi | P lo
constexpr uint32_t kOffRing = kOffP + 2 * kPBytes;      // K ring
constexpr uint32_t kOffVRing = kOffRing + kKStages * kSlot;
constexpr uint32_t kOffV = kOffVRing + kV8Stages * kSlot;
constexpr uint32_t kOffBar = kOffV + kVStages * kVSlot;
constexpr uint32_t kOffRowScale = kOffBar + 512;        // 64 floats
constexpr uint32_t kSmemBytes = kOffRowScale + 256 + 1024;
static_assert(2 * kQPartBytes == kQ16Bytes, "Q1 | Q2 and the bf16 query share one region");

constexpr float kRescaleThreshold = 8.0f;  // log2 units, as the 16-bit kernel
constexpr float kPShift = 7.0f;            // P = 2^(s - max + 7) <= 2^15 between rescales
// End of a CTA: O is staged row-major in the P + K + V region (free once the last PV is
// done) with a padded row stride, then written out coalesced.
constexpr int kORow = kD + 4;
constexpr uint32_t kOffStage = kOffP;
static_assert(kM * kORow * 4 + 3 * kM * 4 <= kOffBar - kOffStage, "staging space");

struct Params8 {
  CUtensorMap tmK8;  // e4m3 Kc pool {128 bytes, rows, 4 chunks}, box {128, 128, 1}
  CUtensorMap tmV8;  // e4m3 Vc pool {128 bytes, rows, 4 chunks}, box {128, 32, 4}
  CUtensorMap tmQb;  // bf16 Q {64, batch*hq, 8}, box {64, 64, 4}
  CUtensorMap tmRk;  // bf16 ring K {64, batch*W, 8}, box {64, 128, 1}
  CUtensorMap tmRv;  // bf16 ring V {64, batch*W, 8}, box {64, 16, 8}
  const int32_t* ctx_len;
  const int32_t* page_table;
  const int32_t* n_entries;
  int32_t* err_word;
  float* ws_ml;  // [nseq, nsplit, hq, 2]
  float* ws_o;   // [nseq, nsplit, hq, 512]
  __nv_bfloat16* O;  // nsplit == 1 && !partial: the final output
  float* lse;
  const __nv_bfloat16* gate;
  int64_t gs0, gs2;
  // the new token's rows and the raw rings, for the in-kernel ring update (nullptr = none)
  const uint4* new_k;
  const uint4* new_v;
  uint4* ring_k;
  uint4* ring_v;
  int32_t nseq, seqlen, hq, W, block, PE, max_pages, num_pages, nsplit;
  int32_t e0, e1, with_ring, partial;
  float scale_log2, k_scale, v_scale;
};

struct Bars8 {
  uint64_t qs_full;   // the bf16 query staged for the converters landed (TMA)
  uint64_t q_ready;   // Q1, Q2 and the row scales written (converters)
  uint64_t qb_full;   // bf16 query of the ring tile landed (TMA)
  uint64_t q8_free;   // the last e4m3 score MMA completed: the query region may be reused
  // K boxes and e4m3 V boxes stream through rings of their own, each filled by its own
  // load warp, so that V boxes waiting to be widened never hold back the K stream
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v8_full[kV8Stages], v8_empty[kV8Stages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t drain, drain_pv;  // each UMMA issuer's MMAs complete (end of the CTA)
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars8) <= 512, "barrier block too large");

// Two e4m3 codes of a word (bytes 0-1 for sel 0, 2-3 for sel 1; the lower byte to the lower
// half) -> f16x2 of their values times 2^-8, exactly, by moving bits: the code's exponent and
// fraction fields (bits 0-6) become the f16 exponent and fraction fields shifted left by 7
// (same exponent field, biases 7 and 15: the value is 2^-8 times the code's; the subnormal
// codes land on f16 subnormals), the sign bit goes to bit 15.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2_s8(uint32_t w, int sel) {
  const uint32_t y = __byte_perm(w, 0u, sel ? 0x3424u : 0x1404u);  // codes in bytes 1 and 3
  return (y & 0x80008000u) | ((y >> 1) & 0x3f803f80u);
}
constexpr float kV16Scale = 256.f;  // the widened values are the codes' values times 2^-8

// 2^k as a float for k in [-126, 127] (exact; the exponent field built directly)
__device__ __forceinline__ float exp2i(int k) {
  k = k < -126 ? -126 : (k > 127 ? 127 : k);
  return __int_as_float((k + 127) << 23);
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) decode_fp8_kernel(const __grid_constant__ Params8 p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sP = smem + kOffP;
  uint8_t* sRing = smem + kOffRing;
  uint8_t* sVRing = smem + kOffVRing;
  uint8_t* sV = smem + kOffV;
  Bars8* bars = reinterpret_cast<Bars8*>(smem + kOffBar);
  float* sRS = reinterpret_cast<float*>(smem + kOffRowScale);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&bars->qs_full, 1);
    mbar_init(&bars->q_ready, 1);
    mbar_init(&bars->qb_full, 1);
    mbar_init(&bars->q8_free, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kV8Stages; ++s) {
      mbar_init(&bars->v8_full[s], 1);
      mbar_init(&bars->v8_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars->v_full[s], 4);  // one arrival per converter warp
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_full[x], 4);
      mbar_init(&bars->o_done[x], 1);
    }
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->drain_pv, 1);
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
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int split = blockIdx.x;
  // where a partial result goes: [b, split] of the workspace (with one split and a partial
  // call, the workspace is the call's partial output)
  float* dst_ml = p.ws_ml + ((int64_t)b * p.nsplit + split) * p.hq * 2;
  float* dst_o = p.ws_o + ((int64_t)b * p.nsplit + split) * p.hq * kD;
  const Seq sq = make_seq(p, b, split);
  const int ntiles = sq.j1 - sq.j0;
  const bool has_ring = ntiles > 0 && tile_of(p, sq, sq.j1 - 1).kind == kRing;
  const int nct = ntiles - (has_ring ? 1 : 0);  // compressed (e4m3) tiles of this split

  // Q1, Q2 and the per-head scale r_h of the two-part query, computed by the softmax and
  // converter warps together (qt = 0..255 over warps 2-9, four threads per head row, 128
  // elements each) from the bf16 query staged in shared memory (chunk c of row h at
  // stage(c) + (c % 4) * 8 KB + h * 128, stage(c) the P buffer for c < 4 and the V buffers
  // after; 16-byte units swizzled by h % 8). Ends with a barrier of the 256 threads; one of
  // them then announces q_ready to the score-MMA warp. Returns false on a time-out.
  auto prep_query = [&](int qt) -> bool {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars->qs_full, 0, abort));
    const int h = qt >> 2, quarter = qt & 3;
    const bool live = h < p.hq && ok;
    const uint8_t* stage = quarter < 2 ? sP : sV;
    auto unit = [&](int i) {  // 16-byte unit i (8 elements) of this thread's 128
      const int gc = 2 * quarter + (i >> 3);  // chunk of the row
      const uint8_t* rowp = stage + (gc & 3) * kQChunkBytes + h * 128;
      return *reinterpret_cast<const uint4*>(rowp + (((i & 7) ^ (h & 7)) << 4));
    };
    // the four threads of a row walk their units in staggered orders: unit i of every
    // chunk sits in the same banks, so equal i in the four quarters would conflict
    float amax = 0.f;
    if (live)
      for (int i0 = 0; i0 < 16; ++i0) {
        const uint4 x = unit((i0 + 2 * quarter) & 15);
        const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(x2[k]);
          amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    // r_h = 2^e puts the head's largest |q| / r_h in [128, 256)
    // (the exponent field of amax; e is kept in [-126, 126] so that r_h and 1 / r_h are
    // both normal floats: a row whose largest |q| is below 2^-119 keeps a smaller range)
    const int ebits = (__float_as_int(amax) >> 23) & 0xff;
    int e = amax > 0.f ? (ebits > 0 ? ebits - 127 : -126) - 7 : 0;
    e = e < -126 ? -126 : (e > 126 ? 126 : e);
    const float rinv = exp2i(-e);  // 1 / r_h, exact
    for (int u0 = 0; u0 < 8; ++u0) {  // 16-element units of the e4m3 parts
      const int u = (u0 + 2 * quarter) & 7;
      uint32_t w1[4] = {0u, 0u, 0u, 0u}, w2[4] = {0u, 0u, 0u, 0u};
      if (live) {
#pragma unroll
        for (int hv = 0; hv < 2; ++hv) {
          const uint4 x = unit(2 * u + hv);
          const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(x2[k]);
            const float a0 = f.x * rinv, a1 = f.y * rinv;
            const __nv_fp8x2_storage_t q1 =
                __nv_cvt_float2_to_fp8x2(make_float2(a0, a1), __NV_SATFINITE, __NV_E4M3);
            const __half2_raw h1 = __nv_cvt_fp8x2_to_halfraw2(q1, __NV_E4M3);
            const float2 v1 = __half22float2(__half2(h1));
            const __nv_fp8x2_storage_t q2 = __nv_cvt_float2_to_fp8x2(
                make_float2(a0 - v1.x, a1 - v1.y), __NV_SATFINITE, __NV_E4M3);
            const int pos = hv * 8 + 2 * k;  // code index within the 16-byte unit
            w1[pos >> 2] |= (uint32_t)q1 << (8 * (pos & 3));
            w2[pos >> 2] |= (uint32_t)q2 << (8 * (pos & 3));
          }
        }
      }
      const int elem = quarter * 128 + 16 * u;
      const uint32_t off = (elem >> 7) * kQChunkBytes + h * 128 +
                           ((((elem & 127) >> 4) ^ (h & 7)) << 4);
      *reinterpret_cast<uint4*>(sQ + off) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
      *reinterpret_cast<uint4*>(sQ + kQPartBytes + off) = make_uint4(w2[0], w2[1], w2[2], w2[3]);
    }
    if (quarter == 0) sRS[h] = p.scale_log2 * p.k_scale * exp2i(e);
    fence_proxy_async_smem();
    named_sync(2, 256);
    if (qt == 0) mbar_arrive(&bars->q_ready);
    return ok;
  };

  if (ntiles <= 0) {
    // empty split: an all-zero partial that the merge skips
    for (int h = threadIdx.x; h < p.hq; h += blockDim.x) {
      dst_ml[2 * h] = -INFINITY;
      dst_ml[2 * h + 1] = 0.f;
    }
  } else if (warp == 0 || warp == kVLoadWarp) {
    // ------------------------------------------------------------------ loads
    // Warp 0 streams the K boxes of the split's tiles into the K ring (and the queries),
    // warp kVLoadWarp the e4m3 V boxes into the V ring; the window tile's values go to the
    // f16 V buffers directly (converter warps). Box n of a ring sits in slot n % stages and
    // completes phase n / stages of that slot's full barrier.
    if (elect_one()) {
      const uint64_t pol = policy_evict_first();  // every cache row is read once
      const bool kw = warp == 0;
      const int stages = kw ? kKStages : kV8Stages;
      uint64_t* full = kw ? bars->k_full : bars->v8_full;
      uint64_t* empty = kw ? bars->k_empty : bars->v8_empty;
      uint8_t* ring = kw ? sRing : sVRing;
      if (kw) {
        if (split == 0 && p.err_word) {
          const int ctx = p.ctx_len[b];
          if (ctx < 1 || ctx > p.seqlen) atomicOr(p.err_word, kErrCtxRange);
          const int x = sq.t + 1 - p.W;
          if ((x < 0 ? 0 : x / p.block) > p.n_entries[b]) atomicOr(p.err_word, kErrCacheShort);
        }
        // the bf16 query, staged for the converter warps in the P buffer (box of chunks
        // 0-3) and the V buffers (chunks 4-7): both are free until Q1/Q2 are ready
        mbar_expect_tx(&bars->qs_full, kQ16Bytes);
        tma_load_3d(sP, &p.tmQb, &bars->qs_full, 0, b * p.hq, 0, pol);
        tma_load_3d(sV, &p.tmQb, &bars->qs_full, 0, b * p.hq, 4, pol);
      }
      uint32_t cnt = 0;  // boxes issued into this ring
      bool ok = true, q_issued = false;
      auto load = [&](const CUtensorMap* map, int row, int chunk) -> bool {
        const uint32_t s = cnt % stages;
        if (cnt >= (uint32_t)stages &&
            !mbar_wait(&empty[s], ((cnt / stages) - 1) & 1, abort))
          return false;
        mbar_expect_tx(&full[s], kSlot);
        tma_load_3d(ring + s * kSlot, map, &full[s], 0, row, chunk, pol);
        ++cnt;
        return true;
      };
      for (int c = 0; c < ntiles && ok; ++c) {
        const Tile t = tile_of(p, sq, sq.j0 + c);
        if (t.kind == kCompressed) {
          int page = p.page_table[(int64_t)b * p.max_pages + t.key0 / p.PE];
          if (page < 0 || page >= p.num_pages) {
            if (p.err_word && kw) atomicOr(p.err_word, kErrPageRange);
            page = 0;
          }
          const int row = page * p.PE + t.key0 % p.PE;
          if (kw) {
            for (int q = 0; q < 4 && ok; ++q) ok = load(&p.tmK8, row, q);
          } else {
            for (int q = 0; q < (t.n + kVRows - 1) / kVRows && ok; ++q)
              ok = load(&p.tmV8, row + q * kVRows, 0);
          }
        } else if (kw) {
          // the bf16 query replaces Q1/Q2 once the last e4m3 score MMA has completed
          if (!(ok = mbar_wait(&bars->q8_free, 0, abort))) break;
          mbar_expect_tx(&bars->qb_full, kQ16Bytes);
          for (int h = 0; h < 2; ++h)
            tma_load_3d(sQ + h * (kQ16Bytes / 2), &p.tmQb, &bars->qb_full, 0, b * p.hq, 4 * h,
                        pol);
          q_issued = true;
          if (p.new_k) append_ring_row(p, p.new_k, p.ring_k, b, sq.t);  // the new token
          for (int q = 0; q < 8 && ok; ++q) ok = load(&p.tmRk, b * p.W, q);
        }
      }
      if (!ok) {
        bars->abort = 1;
        if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << (kw ? 9 : 15)));
        // box n could only be issued once box n - stages had been released: at most the
        // last `stages` boxes are in flight, plus the queries
        volatile int no_abort = 0;
        const uint32_t first = cnt > (uint32_t)stages ? cnt - stages : 0u;
        for (uint32_t n = first; n < cnt; ++n)
          mbar_wait(&full[n % stages], (n / stages) & 1, &no_abort, 100000000ull);
        if (q_issued) mbar_wait(&bars->qb_full, 0, &no_abort, 100000000ull);
        if (kw) mbar_wait(&bars->qs_full, 0, &no_abort, 100000000ull);
      }
    }
  } else if (warp == 1 || warp == kPvWarp) {
    // ------------------------------------------------------------------ UMMA issuers
    // Warp 1 issues the score MMAs S(c) in tile order, warp kPvWarp the P.V MMAs PV(c):
    // S(c + 1) goes out as soon as its K boxes have landed and the softmax has released
    // score buffer (c + 1) & 1, not behind PV(c - 1), which is paced by the widening of V.
    // The two streams touch different TMEM columns and shared memory; each warp's commits
    // track its own MMAs.
    if (elect_one()) {
      bool ok = true;
      const uint32_t qbase = smem_u32(sQ);
      const uint32_t pbase = smem_u32(sP);
      const uint32_t rbase = smem_u32(sRing);
      const uint32_t vbase = smem_u32(sV);
      if (warp == 1) {
        ok = mbar_wait(&bars->q_ready, 0, abort);
        tc_fence_after();
        uint32_t n = 0;  // K boxes consumed
        bool q8_released = false;
        for (int c = 0; c < ntiles && ok; ++c) {
          // S(c) overwrites score buffer c & 1: the softmax of tile c - 2 is done with it
          if (c >= 2 && !(ok = mbar_wait(&bars->p_full[c & 1], ((c - 2) >> 1) & 1, abort)))
            break;
          const Tile t = tile_of(p, sq, sq.j0 + c);
          const uint32_t sb = tmem + kLaneS + (c & 1) * 128;  // score buffer c & 1
          if (t.kind == kCompressed) {
            const uint32_t idesc = idesc_e4m3_f32(kM, t.n);
            for (int q = 0; q < 4 && ok; ++q) {
              const uint32_t s = n % kKStages;
              if (!(ok = mbar_wait(&bars->k_full[s], (n / kKStages) & 1, abort))) break;
              tc_fence_after();
              const uint32_t kaddr = rbase + s * kSlot;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {  // K = 32 codes per UMMA
                const uint64_t kd = sdesc_sw128(kaddr + kk * 32, 16, 1024);
                const uint32_t acc = (q | kk) != 0;
                const uint32_t qa = qbase + q * kQChunkBytes + kk * 32;
                umma_ss_f8(sb, sdesc_sw128(qa, 16, 1024), kd, idesc, acc);
                umma_ss_f8(sb, sdesc_sw128(qa + kQPartBytes, 16, 1024), kd, idesc, 1u);
              }
              umma_commit(&bars->k_empty[s]);
              ++n;
            }
          } else {
            if (!q8_released) {  // a split whose only tile is the ring tile
              umma_commit(&bars->q8_free);
              q8_released = true;
            }
            if (!(ok = mbar_wait(&bars->qb_full, 0, abort))) break;
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(kM, t.n, false);
            for (int q = 0; q < 8 && ok; ++q) {
              const uint32_t s = n % kKStages;
              if (!(ok = mbar_wait(&bars->k_full[s], (n / kKStages) & 1, abort))) break;
              tc_fence_after();
              const uint32_t kaddr = rbase + s * kSlot;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)  // K = 16 bf16 per UMMA
                umma_ss(sb, sdesc_sw128(qbase + q * kQChunkBytes + kk * 32, 16, 1024),
                        sdesc_sw128(kaddr + kk * 32, 16, 1024), idesc, (q | kk) != 0);
              umma_commit(&bars->k_empty[s]);
              ++n;
            }
          }
          if (ok) umma_commit(&bars->s_full[c & 1]);
          // after the last e4m3 score MMAs of a split that ends with the ring tile, the
          // bf16 query may replace Q1/Q2 as soon as they complete
          if (ok && has_ring && c + 1 == nct && !q8_released) {
            umma_commit(&bars->q8_free);
            q8_released = true;
          }
        }
      } else {
        uint32_t nv = 0, cv = 0;  // V boxes before the tile, V groups consumed
        for (int pc = 0; pc < ntiles && ok; ++pc) {
          const Tile t = tile_of(p, sq, sq.j0 + pc);
          const uint32_t vstart = nv;  // V ring index of the tile's first box
          if (t.kind == kCompressed) nv += (t.n + kVRows - 1) / kVRows;
          if (!(ok = mbar_wait(&bars->p_full[pc & 1], (pc >> 1) & 1, abort))) break;
          tc_fence_after();
          const uint32_t idesc = t.kind == kCompressed ? idesc_f16_f32(kM, 256, true)
                                                       : idesc_bf16_f32(kM, 256, true);
          // O[:, 256 h .. 256 h + 255] += P(group) V(group, columns of half h): one N = 256
          // UMMA per half and part of P
          const bool f8 = t.kind == kCompressed;
          const int ng = t.n / 16;
          for (int g = 0; g < ng && ok; ++g) {
            const uint32_t s = cv % kVStages;
            if (!(ok = mbar_wait(&bars->v_full[s], (cv / kVStages) & 1, abort))) break;
            // every converter warp has widened this group: an e4m3 box is free once both of
            // its groups (or the tile's last) are in
            if (f8 && ((g & 1) == 1 || g == ng - 1))
              mbar_arrive(&bars->v8_empty[(vstart + (g >> 1)) % kV8Stages]);
            tc_fence_after();
            const uint32_t vaddr = vbase + s * kVSlot;
            const uint32_t paddr =
                pbase + (f8 ? (pc & 1) * kPBytes : 0u) + (g >> 2) * kPChunkBytes + (g & 3) * 32;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t vd = sdesc_sw128(vaddr + h * 4 * kVChunkBytes, kVChunkBytes, 1024);
              umma_ss(tmem + h * 256, sdesc_sw128(paddr, 16, 1024), vd, idesc,
                      (pc > 0 || g > 0));
              if (!f8)
                umma_ss(tmem + h * 256, sdesc_sw128(paddr + kPBytes, 16, 1024), vd, idesc, 1u);
            }
            umma_commit(&bars->v_empty[s]);
            ++cv;
          }
          if (ok) umma_commit(&bars->o_done[pc & 1]);
        }
      }
      if (!ok) {
        bars->abort = 1;
        if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << (warp == 1 ? 11 : 14)));
      }
      // each issuer waits for its own MMAs before the CTA may release TMEM
      volatile int no_abort = 0;
      uint64_t* drain = warp == 1 ? &bars->drain : &bars->drain_pv;
      umma_commit(drain);
      mbar_wait(drain, 0, &no_abort, 100000000ull);
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------------ softmax + partials
    // Lane l + 16 of a warp holds score row quad * 16 + l; lane l (< 16) holds the O row of
    // the same head. Per tile c: wait S(c); row max; wait for the P buffer (PV(c - 2), or
    // PV(c - 1) for the window tile or a rescale); lazy rescale of O; P(c); arrive p_full,
    // which also releases score buffer c & 1 to S(c + 2).
    const int quad = warp & 3;
    const bool s_lane = lane >= 16;
    const int hrow = quad * 16 + (lane & 15);
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    // Q1, Q2 and r_h with the converter warps (the barrier at its end orders sRS)
    bool ok = prep_query(threadIdx.x - 64);
    const float rs8 = sRS[hrow];            // r_h * k_scale * scale * log2(e)
    // ring values enter O in the units of the widened e4m3 values (value / (v_scale * 2^8))
    const float inv_vs = 1.f / (p.v_scale * kV16Scale);
    float base = -INFINITY, l = 0.f;
    for (int c = 0; c < ntiles && ok; ++c) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[c & 1], (c >> 1) & 1, abort));
      if (!ok) break;
      tc_fence_after();
      const Tile tl = tile_of(p, sq, sq.j0 + c);
      const bool f8 = tl.kind == kCompressed;
      const uint32_t sbuf = tmem + lane_addr + (c & 1) * 128;
      // visible columns: a prefix of a compressed tile, or ring slots 0..min(W,t+1)-1
      const int vhi = f8 ? min(tl.n, sq.e1 - tl.key0) : min(p.W, sq.t + 1);
      const uint32_t vlen = vhi > 0 ? (uint32_t)vhi : 0u;
      const float rs = f8 ? rs8 : p.scale_log2;
      // 32 raw scores of columns q*32 .. q*32+31
      auto load_scores = [&](int q, uint32_t (&v)[32]) {
        tmem_ld32(sbuf + q * 32, v);
        tmem_wait_ld();
      };
      // pass 1: row max over the visible keys
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
      for (int q = 0; q < kTN / 32; ++q) {
        if (q * 32 >= tl.n) break;
        uint32_t v[32];
        load_scores(q, v);
        if ((uint32_t)(q * 32 + 32) <= vlen) {  // a fully visible piece: no masks
#pragma unroll
          for (int e = 0; e < 32; ++e) mx[e & 7] = fmaxf(mx[e & 7], __uint_as_float(v[e]));
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const bool in = (uint32_t)(q * 32 + e) < vlen;
            mx[e & 7] = fmaxf(mx[e & 7], in ? __uint_as_float(v[e]) : -INFINITY);
          }
        }
      }
      const float cmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                         rs;
      const bool grow = s_lane && (c == 0 || cmax > base + kRescaleThreshold);
      float factor = 1.f;
      if (grow) {
        factor = c == 0 ? 1.f : fast_exp2(base - cmax);
        l *= factor;
        base = cmax;
      }
      // The P of an e4m3 tile goes to buffer c & 1, free once PV(c - 2) is done, so that
      // this pass overlaps PV(c - 1); the window tile's hi and lo parts take both buffers,
      // and rescaling O needs every earlier PV done: both wait for PV(c - 1).
      const bool rescale = c > 0 && __any_sync(0xffffffffu, grow);
      const int pv_wait = (rescale || !f8) ? c - 1 : c - 2;
      if (pv_wait >= 0) {
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bars->o_done[pv_wait & 1], (pv_wait >> 1) & 1, abort));
        if (!ok) break;
      }
      if (rescale) {
        // the 32-lane read-modify-write also rewrites the score lanes (unchanged): no UMMA
        // may be in flight, so S(c + 1) (if issued) must have completed. PV(c) waits for
        // our p_full.
        if (c + 1 < ntiles)
          ok = mbar_wait(&bars->s_full[(c + 1) & 1], ((c + 1) >> 1) & 1, abort);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const float f_o = __shfl_sync(0xffffffffu, factor, (lane & 15) + 16);
        const float f = s_lane ? 1.f : f_o;
#pragma unroll 1
        for (int q = 0; q < kD / 32; ++q) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_addr + q * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
          tmem_st32(tmem + lane_addr + q * 32, v);
        }
        tmem_wait_st();
      }
      // pass 2: P = 2^(s - base + 7) into the K-major 128B-swizzled P buffer: one f16 value
      // for an e4m3 tile; hi + lo bf16 parts (two buffers) times 1/v_scale for the ring tile.
      // All 32 lanes work: of each 32-column piece of row hrow, lane l + 16 takes columns
      // 0..15 and lane l columns 16..31, handed over by a shuffle.
      const float b_own = base == -INFINITY ? 0.f : base - kPShift;
      const float b_pair = __shfl_xor_sync(0xffffffffu, b_own, 16);
      const float bb = s_lane ? b_own : b_pair;
      const int half = s_lane ? 0 : 16;
      uint8_t* pbuf = sP + (f8 ? (c & 1) * kPBytes : 0u);
      float ps = 0.f;
      for (int q = 0; q < kTN / 32; ++q) {
        if (q * 32 >= tl.n) break;
        uint32_t v[32];
        load_scores(q, v);
        float x[16];
        pair_split(v, s_lane, x);
        const int col0 = q * 32 + half;
        uint32_t pk[8], pl[8];
        const bool visible = (uint32_t)(q * 32 + 32) <= vlen;  // the whole piece: no masks
        if (f8)
          ps += visible ? p_piece<false, kPF16>(x, rs, bb, col0, vlen, inv_vs, pk, pl)
                        : p_piece<true, kPF16>(x, rs, bb, col0, vlen, inv_vs, pk, pl);
        else
          ps += visible ? p_piece<false, kPBf16PairScaled>(x, rs, bb, col0, vlen, inv_vs, pk, pl)
                        : p_piece<true, kPBf16PairScaled>(x, rs, bb, col0, vlen, inv_vs, pk, pl);
        // keys col0 .. col0 + 15 -> 64-key P chunk q/2, 16-byte units (q&1)*4 + half/8 + w
        uint8_t* rowp = pbuf + (q >> 1) * kPChunkBytes + hrow * 128;
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          const int u = (q & 1) * 4 + (half >> 3) + w;
          const int us = u ^ (hrow & 7);
          *reinterpret_cast<uint4*>(rowp + us * 16) =
              make_uint4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
          if (!f8)
            *reinterpret_cast<uint4*>(rowp + kPBytes + us * 16) =
                make_uint4(pl[4 * w], pl[4 * w + 1], pl[4 * w + 2], pl[4 * w + 3]);
        }
      }
      l += ps + __shfl_xor_sync(0xffffffffu, ps, 16);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[c & 1]);
    }
    // the last PV's commit covers every earlier P.V MMA; every score MMA completed before
    // its s_full was seen
    if (ok) ok = mbar_wait(&bars->o_done[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1, abort);
    ok = __all_sync(0xffffffffu, ok);
    float* sO = reinterpret_cast<float*>(smem + kOffStage);  // [64][kORow]
    float* sM = sO + kM * kORow;                               // reference max (log2 units)
    float* sL = sM + kM;                                       // row sum
    float* sInv = sL + kM;                                     // v_scale / row sum
    if (ok) {
      tc_fence_after();
      if (s_lane) {
        sM[hrow] = base - kPShift;  // l and O carry the 2^7 of P
        sL[hrow] = l;
        sInv[hrow] = 1.f / l;
      }
      const float vs = p.v_scale * kV16Scale;
      float* orow = sO + hrow * kORow;
#pragma unroll 1
      for (int q = 0; q < kD / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_addr + q * 32, v);
        tmem_wait_ld();
        if (!s_lane) {
          float4* o4 = reinterpret_cast<float4*>(orow + q * 32);
#pragma unroll
          for (int w = 0; w < 8; ++w)
            o4[w] = make_float4(__uint_as_float(v[4 * w]) * vs, __uint_as_float(v[4 * w + 1]) * vs,
                                __uint_as_float(v[4 * w + 2]) * vs,
                                __uint_as_float(v[4 * w + 3]) * vs);
        }
      }
    } else {
      bars->abort = 1;
      if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << 12));
    }
    named_sync(1, 128);
    const int tid = threadIdx.x - 64;  // 0..127 over the four softmax warps
    if (p.nsplit == 1 && !p.partial) {
      // final output: O / l, gate, bf16 in 16-byte units; lse in natural log
      __nv_bfloat16* ob = p.O + (int64_t)b * p.hq * kD;
#pragma unroll 4
      for (int i = tid; i < p.hq * (kD / 8); i += 128) {
        const int h = i / (kD / 8);
        const int c = 8 * (i % (kD / 8));
        const float4 x0 = *reinterpret_cast<const float4*>(sO + h * kORow + c);
        const float4 x1 = *reinterpret_cast<const float4*>(sO + h * kORow + c + 4);
        const float inv = sInv[h];
        float o[8] = {x0.x * inv, x0.y * inv, x0.z * inv, x0.w * inv,
                      x1.x * inv, x1.y * inv, x1.z * inv, x1.w * inv};
        if (p.gate) {
          const __nv_bfloat162* gp = reinterpret_cast<const __nv_bfloat162*>(
              p.gate + (int64_t)b * p.gs0 + (int64_t)h * p.gs2 + c);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 g = __bfloat1622float2(gp[k]);
            o[2 * k] *= g.x;
            o[2 * k + 1] *= g.y;
          }
        }
        *reinterpret_cast<uint4*>(ob + (int64_t)h * kD + c) =
            make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]),
                       pack_bf16x2(o[4], o[5]), pack_bf16x2(o[6], o[7]));
      }
      if (p.lse)
        for (int h = tid; h < p.hq; h += 128)
          p.lse[(int64_t)b * p.hq + h] = (sM[h] + __log2f(sL[h])) * 0.69314718055994531f;
    } else {
      // split partial: unnormalised O (value units), (reference max, sum) per head
      for (int i = tid; i < p.hq * (kD / 4); i += 128) {
        const int h = i / (kD / 4);
        const int c = 4 * (i % (kD / 4));
        *reinterpret_cast<float4*>(dst_o + (int64_t)h * kD + c) =
            *reinterpret_cast<const float4*>(sO + h * kORow + c);
      }
      for (int h = tid; h < p.hq; h += 128) {
        dst_ml[h * 2] = sM[h];
        dst_ml[h * 2 + 1] = sL[h];
      }
    }
  } else {
    // ------------------------------------------------------------------ converters
    const int ct = threadIdx.x - 192;  // 0..127
    const int cw = ct >> 5;
    // (1) Q1, Q2 and the per-head scale, with the softmax warps
    const bool q_ok = prep_query(threadIdx.x - 64);

    // (2) V groups of 16 keys in key order into the f16 V buffers: e4m3 boxes of the V
    // ring widened, the window tile's bf16 values by TMA. Thread (cw, lane) widens keys kr
    // and kr + 8 of a group at values 32*c32 .. 32*c32 + 31.
    const int kr = lane & 7;
    const int c32 = cw * 4 + (lane >> 3);
    bool ok = q_ok;
    uint32_t n = 0, cv = 0;  // V ring boxes before the tile, V groups produced
    for (int c = 1; c <= ntiles && ok; ++c) {
      const Tile t = tile_of(p, sq, sq.j0 + c - 1);
      const int ng = t.n / 16;
      if (t.kind == kCompressed) {
        // keys at or past the visible end of the tile are written as 0 (their P is 0, and
        // the pool rows behind them may hold anything)
        const int vlen = min(t.n, sq.e1 - t.key0);
        for (int g = 0; g < ng && ok; ++g, ++cv) {
          const uint32_t sidx = n + (g >> 1);
          const uint32_t rs = sidx % kV8Stages;
          bool w_ok = true;
          if ((g & 1) == 0)
            w_ok = __all_sync(0xffffffffu,
                              mbar_wait(&bars->v8_full[rs], (sidx / kV8Stages) & 1, abort));
          const uint32_t vs = cv % kVStages;
          if (w_ok && cv >= (uint32_t)kVStages)
            w_ok = __all_sync(0xffffffffu,
                              mbar_wait(&bars->v_empty[vs], ((cv / kVStages) - 1) & 1, abort));
          if (w_ok) {
            const uint8_t* box = sVRing + rs * kSlot + (c32 >> 2) * kV8Chunk;
            uint8_t* dst = sV + vs * kVSlot + (c32 >> 1) * kVChunkBytes;
#pragma unroll
            for (int it = 0; it < 2; ++it) {
              const int k = kr + 8 * it;              // key within the group
              const int r = 16 * (g & 1) + k;         // row within the box
              uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
              if (16 * g + k < vlen) {
                const uint8_t* rowp = box + r * 128;
                const int u0 = 2 * (c32 & 3);
                lo = *reinterpret_cast<const uint4*>(rowp + ((u0 ^ (r & 7)) << 4));
                hi = *reinterpret_cast<const uint4*>(rowp + (((u0 + 1) ^ (r & 7)) << 4));
              }
              const uint32_t cw8[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
              uint8_t* rowd = dst + it * 1024 + kr * 128;
#pragma unroll
              for (int w = 0; w < 4; ++w) {
                const uint32_t a = cw8[2 * w], bq = cw8[2 * w + 1];
                const int unit = ((c32 & 1) << 2) + w;
                *reinterpret_cast<uint4*>(rowd + ((unit ^ (k & 7)) << 4)) =
                    make_uint4(e4m3x2_to_f16x2_s8(a, 0), e4m3x2_to_f16x2_s8(a, 1),
                               e4m3x2_to_f16x2_s8(bq, 0), e4m3x2_to_f16x2_s8(bq, 1));
              }
            }
            fence_proxy_async_smem();
          }
          // each warp hands its quarter of the group over on its own (v_full counts four
          // arrivals); a warp that gave up stops, and the others' bounded waits end on the
          // abort flag
          ok = w_ok;
          __syncwarp();
          if (ok && lane == 0) mbar_arrive(&bars->v_full[vs]);
        }
        n += (t.n + kVRows - 1) / kVRows;
      } else if (ct == 0) {
        // the window's values, bf16, one TMA box of 16 rows x 512 values per group (the new
        // token's row written into its slot first)
        if (p.new_v) append_ring_row(p, p.new_v, p.ring_v, b, sq.t);
        const uint64_t pol = policy_evict_first();
        uint32_t issued = 0;
        const uint32_t cv0 = cv;
        for (int g = 0; g < ng && ok; ++g) {
          const uint32_t vs = (cv0 + g) % kVStages;
          if (cv0 + g >= (uint32_t)kVStages &&
              !(ok = mbar_wait(&bars->v_empty[vs], (((cv0 + g) / kVStages) - 1) & 1, abort)))
            break;
          // the four arrivals of a converted group: this one with the bytes, three plain
          mbar_expect_tx(&bars->v_full[vs], kVSlot);
          mbar_arrive(&bars->v_full[vs]);
          mbar_arrive(&bars->v_full[vs]);
          mbar_arrive(&bars->v_full[vs]);
          tma_load_3d(sV + vs * kVSlot, &p.tmRv, &bars->v_full[vs], 0, b * p.W + 16 * g, 0,
                      pol);
          ++issued;
        }
        if (!ok) {
          volatile int no_abort = 0;
          const uint32_t end = cv0 + issued;
          const uint32_t first = issued > (uint32_t)kVStages ? end - kVStages : cv0;
          for (uint32_t m = first; m < end; ++m)
            mbar_wait(&bars->v_full[m % kVStages], (m / kVStages) & 1, &no_abort,
                      100000000ull);
        }
        cv += ng;
      }
    }
    if (!ok && lane == 0) {
      bars->abort = 1;
      if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << 13));
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

}  // namespace

cudaError_t launch_decode_fp8(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                              const hca_cache& c, const void* ring_k, const void* ring_v,
                              const DecodePart& part, void* O, float* lse, void* ws,
                              cudaStream_t s) {
  Params8 p;
  memset(&p, 0, sizeof(p));
  const int nsplit = part_num_splits(d, part);
  cudaError_t e;
  const uint64_t rowsC = (uint64_t)c.num_pages * c.page_entries;
  const uint64_t rowsR = (uint64_t)d.batch * d.window;
  if ((e = encode_u8_chunks(&p.tmK8, c.kc_pool, rowsC, kTN, 1)) != cudaSuccess) return e;
  if ((e = encode_u8_chunks(&p.tmV8, c.vc_pool, rowsC, kVRows, 4)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmQb, Q, (uint64_t)d.batch * d.hq, kM, 4)) != cudaSuccess)
    return e;
  if ((e = encode_bf16_chunks(&p.tmRk, ring_k, rowsR, kTN, 1)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmRv, ring_v, rowsR, 16, 8)) != cudaSuccess) return e;
  float* pml = static_cast<float*>(part.out_partial);
  float* po = pml ? pml + ml_floats(d, 1) : nullptr;
  p.ctx_len = ctx_len;
  p.page_table = c.page_table;
  p.n_entries = c.n_entries;
  p.err_word = c.err_word;
  if (pml && nsplit == 1) {  // the decode CTAs write the partial result themselves
    p.ws_ml = pml;
    p.ws_o = po;
  } else {
    p.ws_ml = static_cast<float*>(ws);
    p.ws_o = p.ws_ml + ml_floats(d, nsplit);
  }
  p.nseq = d.batch;
  p.seqlen = d.seqlen;
  p.hq = d.hq;
  p.W = d.window;
  p.block = d.block;
  p.PE = c.page_entries;
  p.max_pages = c.max_pages;
  p.num_pages = c.num_pages;
  p.nsplit = nsplit;
  p.e0 = part.e0;
  p.e1 = part.e1;
  p.with_ring = part.with_ring ? 1 : 0;
  p.partial = pml ? 1 : 0;
  p.new_k = static_cast<const uint4*>(part.new_k);
  p.new_v = static_cast<const uint4*>(part.new_v);
  p.ring_k = static_cast<uint4*>(const_cast<void*>(ring_k));
  p.ring_v = static_cast<uint4*>(const_cast<void*>(ring_v));
  p.scale_log2 = d.scale * 1.4426950408889634f;
  p.k_scale = c.k_scale;
  p.v_scale = c.v_scale;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.gate = static_cast<const __nv_bfloat16*>(d.gate);
  p.gs0 = d.gate_strides[0];
  p.gs2 = d.gate_strides[2];
  static PerDevice<int> smem_limit_set;
  if ((e = set_smem_limit_once(smem_limit_set, (const void*)decode_fp8_kernel,
                               (int)kSmemBytes)) != cudaSuccess)
    return e;
  cudaLaunchAttribute pdl[1];
  cudaLaunchConfig_t cfg = pdl_config(pdl, s);
  cfg.gridDim = dim3(nsplit, d.batch);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  if ((e = cudaLaunchKernelEx(&cfg, decode_fp8_kernel, p)) != cudaSuccess) return e;
  if (nsplit == 1) return cudaSuccess;
  return launch_split_merge(d, p.ws_ml, p.ws_o, nsplit, pml, po, O, lse, s);
}

}  // namespace hca
