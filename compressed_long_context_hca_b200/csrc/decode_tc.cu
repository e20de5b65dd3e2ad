// decode_tc.cu -- one HCA decode step on tcgen05 tensor cores, split over the key list,
// followed by a merge of the split partials.
//
// Operation ([news 二.1] / [analysis 1] / [gate] in include/hca.h): the newest token of a
// sequence (position t = ctx_len - 1) attends with one softmax to the compressed entries
// j < n_c(t) and to the last `window` raw tokens, held in a ring of `window` slots.
//
// Design for sm_100a (HBM-bound: every key row is read once, ~63 flop per byte):
//  * The hq <= 64 query heads of a sequence share its KV head, so they form the M = 64 rows
//    of every UMMA. An M = 64 accumulator occupies TMEM lanes 0-15 of each 32-lane
//    subpartition; a second one sits at lane offset 16. O (64 x 512 f32) takes lanes
//    0-15 x 512 columns; two score buffers of 128 keys take lanes 16-31.
//  * The key list (compressed tiles of 128 entries, then the ring tile) is cut into
//    `nsplit` contiguous splits; grid = (nsplit, sequences). A split is walked in chunks
//    of one tile (128 keys) with a running softmax (lazy rescale).
//  * One load stream per CTA, in the order K(0), K(1), V(0), K(2), V(1), ...: the scores of
//    chunk c + 1 are computed while the softmax of chunk c runs, and V(c) arrives after it,
//    so the stream of 3-D TMA boxes (128 rows x two 128-byte chunks, two issuing warps)
//    does not wait on the softmax. P goes to shared memory as two bf16 parts, P_hi = bf16(P)
//    and P_lo = bf16(P - P_hi) (UMMA K-major swizzled layout), and O += P_hi V + P_lo V runs
//    as two UMMAs with V N-major: the rounding of P costs ~2^-17 of the value spread instead
//    of 2^-9. One buffer pair is enough: P(c) is written once PV(c - 1) is done, and V(c)
//    only arrives after K(c + 1).
//  * The softmax computes P on all 32 lanes of its warps: the score row of lane l + 16 is
//    shared with lane l by shuffles (decode_softmax.cuh).
//  * With a ring update requested (hca_attn_decode_append), the two producer threads of
//    the CTA holding the window tile write the new token's K and V rows into slot t % W
//    before their first load of that tile, then fence the async proxy.
//  * Each CTA writes float32 partials (unnormalised O, base max m in log2 units, sum l) to
//    the workspace; merge_kernel combines them per head, applies the gate and casts.
//  * All mbarrier waits are bounded (HCA_ERR_TIMEOUT on give-up).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <string.h>

#include "hca_internal.h"
#include "sm100.cuh"
#include "decode_keys.cuh"
#include "decode_softmax.cuh"
#include "tmap.h"

namespace hca {
namespace {

using namespace dkeys;
using namespace dsoft;

constexpr int kM = 64;                    // head rows
constexpr int kD = 512;
constexpr int kKC = 64;                   // elements per 128-byte swizzle row ("chunk")
constexpr int kNCh = kD / kKC;            // 8
constexpr uint32_t kChunk128 = 128 * kKC * 2;           // 16 KB: 128 rows x one chunk
constexpr uint32_t kSlotBytes = 2 * kChunk128;          // 32 KB: one 3-D box, 2 chunks
constexpr int kSlotsPerTile = kNCh / 2;                 // 4 for K, 4 for V
constexpr uint32_t kQChunkBytes = kM * kKC * 2;         // 8 KB
constexpr uint32_t kQBytes = kNCh * kQChunkBytes;       // 64 KB (two 32 KB boxes)
constexpr uint32_t kPChunkBytes = kM * kKC * 2;         // 8 KB (64 rows x 64 keys)
constexpr int kCT = 1;                    // tiles per softmax chunk (128 keys)
constexpr uint32_t kPBytes = kCT * (kTN / kKC) * kPChunkBytes;  // 16 KB: one part of P
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P stays below 2^8 between rescales
constexpr int kStages = 4;  // = kSlotsPerTile: the slots of a tile are ring slots 0..3
static_assert(kStages == kSlotsPerTile, "P.V pairs ring slots (0,1) and (2,3) of a V tile");
constexpr int kThreads = 224;             // 2 TMA warps, UMMA warp, 4 softmax warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kLaneS = 16u << 16;   // lane offset of the score accumulator

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffP = kQBytes;
constexpr uint32_t kOffRing = kOffP + 2 * kPBytes;  // P_hi, then P_lo
constexpr uint32_t kOffBar = kOffRing + kStages * kSlotBytes;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
// End of a CTA: O (64 x 512 f32) is staged row-major in the P + ring region (free once the
// last PV is done) with a padded row stride, then written out coalesced.
constexpr int kORow = kD + 4;  // floats per staged row: rows r and r + 8 share banks only
constexpr uint32_t kOffStage = kOffP;
static_assert(kOffRing == kOffP + 2 * kPBytes, "P and ring must be adjacent");
static_assert(kM * kORow * 4 + 3 * kM * 4 <= 2 * kPBytes + kStages * kSlotBytes, "staging space");

struct Params {
  // 3-D maps {64 elements, rows, 8 chunks}
  CUtensorMap tmQ, tmKc, tmVc, tmRk, tmRv;
  const int32_t* ctx_len;
  const int32_t* page_table;
  const int32_t* n_entries;
  int32_t* err_word;
  float* ws_ml;   // [nseq, nsplit, hq, 2]
  float* ws_o;    // [nseq, nsplit, hq, 512]
  // nsplit == 1: the CTA writes the final output itself (no merge launch)
  __nv_bfloat16* O;
  float* lse;
  const __nv_bfloat16* gate;
  int64_t gs0, gs2;
  // the new token's rows and the raw rings, for the in-kernel ring update (nullptr = none)
  const uint4* new_k;
  const uint4* new_v;
  uint4* ring_k;
  uint4* ring_v;
  int32_t nseq, seqlen, hq, W, block, PE, max_pages, num_pages, nsplit;
  // key part of the call: visible compressed entries [e0, e1) (e0 % 128 == 0), and the raw
  // window if with_ring; partial != 0: the result is an unnormalised float32 partial
  // (written to ws_ml / ws_o at split 0 when nsplit == 1, else merged into one by the merge)
  int32_t e0, e1, with_ring, partial;
  float scale_log2;
};

struct Bars {
  uint64_t q_full;
  uint64_t ring_full[kStages], ring_empty[kStages];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block too large");

__global__ void __launch_bounds__(kThreads, 1) decode_tc_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sP = smem + kOffP;
  uint8_t* sRing = smem + kOffRing;
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int b = blockIdx.y;
  const int split = blockIdx.x;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->ring_full[s], 1);
      mbar_init(&bars->ring_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->s_full[x], 1);
      mbar_init(&bars->p_full[x], 4);
      mbar_init(&bars->o_done[x], 1);
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
  // launched as a programmatic dependent: the previous grid on the stream (a merge reading
  // this workspace, or whatever wrote the inputs) must be complete before the first global
  // access; then the merge grid may be scheduled as SMs free up
  pdl_wait();
  pdl_trigger();
  const Seq sq = make_seq(p, b, split);
  const int ntiles = sq.j1 - sq.j0;
  const int nchunks = (ntiles + kCT - 1) / kCT;
  // tiles [chunk_t0(c), chunk_t1(c)) of the split form chunk c
  auto chunk_t0 = [&](int c) { return sq.j0 + c * kCT; };
  auto chunk_t1 = [&](int c) { return min(sq.j0 + (c + 1) * kCT, sq.j1); };

  if (ntiles <= 0) {
    // empty split: an all-zero partial that the merge skips
    for (int h = threadIdx.x; h < p.hq; h += blockDim.x) {
      float* ml = p.ws_ml + (((int64_t)b * p.nsplit + split) * p.hq + h) * 2;
      ml[0] = -INFINITY;
      ml[1] = 0.f;
    }
  } else if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------------ TMA producers
    // Two producer warps take turns over one load sequence (even / odd loads): one issuing
    // thread's bulk-tensor copies are served one after another.
    if (elect_one()) {
      const uint32_t mine = warp == 0 ? 0u : 1u;
      const uint64_t pol = policy_evict_first();  // every cache row is read once
      bool ok = true;
      if (mine == 0) {
        if (split == 0 && p.err_word) {
          const int ctx = p.ctx_len[b];
          if (ctx < 1 || ctx > p.seqlen) atomicOr(p.err_word, kErrCtxRange);
          const int x = sq.t + 1 - p.W;
          if ((x < 0 ? 0 : x / p.block) > p.n_entries[b]) atomicOr(p.err_word, kErrCacheShort);
        }
        mbar_expect_tx(&bars->q_full, kQBytes);
        for (int h = 0; h < 2; ++h)
          tma_load_3d(sQ + h * (kQBytes / 2), &p.tmQ, &bars->q_full, 0, b * p.hq, 4 * h, pol);
      }
      uint32_t cnt = 0;
      auto load_tile = [&](int j, bool is_v) -> bool {
        const Tile t = tile_of(p, sq, j);
        int row;
        if (t.kind == kCompressed) {
          int page = p.page_table[(int64_t)b * p.max_pages + t.key0 / p.PE];
          if (page < 0 || page >= p.num_pages) {
            if (p.err_word) atomicOr(p.err_word, kErrPageRange);
            page = 0;
          }
          row = page * p.PE + t.key0 % p.PE;
        } else {
          row = b * p.W;
          // the new token into the ring (both producers write the same rows, each before
          // its own first load of the window tile)
          if (!is_v && p.new_k) {
            append_ring_row(p, p.new_k, p.ring_k, b, sq.t);
            append_ring_row(p, p.new_v, p.ring_v, b, sq.t);
          }
        }
        const CUtensorMap* map = t.kind == kCompressed ? (is_v ? &p.tmVc : &p.tmKc)
                                                       : (is_v ? &p.tmRv : &p.tmRk);
        for (int q = 0; q < kSlotsPerTile; ++q) {
          const uint32_t n = cnt++;
          if ((n & 1u) != mine) continue;
          const uint32_t s = n % kStages;
          const uint32_t round = n / kStages;
          if (round > 0 && !mbar_wait(&bars->ring_empty[s], (round - 1) & 1, abort)) return false;
          mbar_expect_tx(&bars->ring_full[s], kSlotBytes);
          tma_load_3d(sRing + s * kSlotBytes, map, &bars->ring_full[s], 0, row, 2 * q, pol);
        }
        return true;
      };
      // K(0), then per step c >= 1: K(c) (if any), V(c - 1)
      for (int c = 0; c <= nchunks && ok; ++c) {
        if (c < nchunks)
          for (int j = chunk_t0(c); j < chunk_t1(c) && ok; ++j) ok = load_tile(j, false);
        if (c >= 1)
          for (int j = chunk_t0(c - 1); j < chunk_t1(c - 1) && ok; ++j) ok = load_tile(j, true);
      }
      if (!ok) {
        bars->abort = 1;
        if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << 9));
        volatile int no_abort = 0;
        const uint32_t first = cnt > kStages ? cnt - kStages : 0;
        for (uint32_t q = first; q < cnt; ++q)
          if ((q & 1u) == mine)
            mbar_wait(&bars->ring_full[q % kStages], (q / kStages) & 1, &no_abort, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ UMMA issuer
    // Same order as the loads: S(0), then per step c >= 1: S(c) (if any), PV(c - 1).
    // S(c) writes score buffer c & 1, which the softmax of chunk c - 2 has released:
    // PV(c - 2), issued earlier, waited for that softmax's p_full.
    if (elect_one()) {
      bool ok = mbar_wait(&bars->q_full, 0, abort);
      tc_fence_after();
      uint32_t cnt = 0;
      const uint32_t qbase = smem_u32(sQ);
      const uint32_t pbase = smem_u32(sP);
      const uint32_t rbase = smem_u32(sRing);
      const uint32_t idesc_pv = idesc_bf16_f32(kM, 256, true);
      for (int c = 0; c <= nchunks && ok; ++c) {
        if (c < nchunks) {
          const uint32_t sbuf = tmem + kLaneS + (c & 1) * (kCT * kTN);
          for (int j = chunk_t0(c); j < chunk_t1(c) && ok; ++j) {
            const Tile t = tile_of(p, sq, j);
            const uint32_t d_tmem = sbuf + (j - chunk_t0(c)) * kTN;
            const uint32_t idesc = idesc_bf16_f32(kM, t.n, false);
            for (int q = 0; q < kSlotsPerTile && ok; ++q) {
              const uint32_t s = cnt % kStages;
              if (!(ok = mbar_wait(&bars->ring_full[s], (cnt / kStages) & 1, abort))) break;
              tc_fence_after();
              const uint32_t sbase = rbase + s * kSlotBytes;
              for (int cc = 0; cc < 2; ++cc) {
                const int d = 2 * q + cc;
                const uint32_t kaddr = sbase + cc * kChunk128;
                const uint32_t qaddr = qbase + d * kQChunkBytes;
#pragma unroll
                for (int kk = 0; kk < kKC / 16; ++kk)
                  umma_ss(d_tmem, sdesc_sw128(qaddr + kk * 32, 16, 1024),
                          sdesc_sw128(kaddr + kk * 32, 16, 1024), idesc, (d | kk) != 0);
              }
              umma_commit(&bars->ring_empty[s]);
              ++cnt;
            }
          }
          if (ok) umma_commit(&bars->s_full[c & 1]);
        }
        if (c >= 1 && ok) {
          const int pc = c - 1;
          if (!(ok = mbar_wait(&bars->p_full[pc & 1], (pc >> 1) & 1, abort))) break;
          tc_fence_after();
          const uint32_t pbuf = pbase;
          // O[:, 256 h .. 256 h + 255] += P(tile) V(tile, slots 2h and 2h + 1): a V tile fills
          // ring slots 0..3 in order (every tile is 4 loads), so slots 2h and 2h + 1 are
          // adjacent and their four 128-column chunks have one stride (16 KB): one N = 256
          // MMA per 16-key group and part of P
          for (int j = chunk_t0(pc); j < chunk_t1(pc) && ok; ++j) {
            const Tile t = tile_of(p, sq, j);
            const int jt = j - chunk_t0(pc);
            for (int h = 0; h < kSlotsPerTile / 2 && ok; ++h) {
              const uint32_t s = cnt % kStages;  // == 2 h
              if (!(ok = mbar_wait(&bars->ring_full[s], (cnt / kStages) & 1, abort))) break;
              if (!(ok = mbar_wait(&bars->ring_full[s + 1], ((cnt + 1) / kStages) & 1, abort)))
                break;
              tc_fence_after();
              const uint32_t vaddr = rbase + s * kSlotBytes;
              for (int kk = 0; kk < t.n / 16; ++kk) {
                const int key16 = jt * (kTN / 16) + kk;  // 16-key group within the chunk
                const uint32_t paddr = pbuf + (key16 >> 2) * kPChunkBytes + (key16 & 3) * 32;
                const uint64_t vd = sdesc_sw128(vaddr + kk * 2048, kChunk128, 1024);
                umma_ss(tmem + h * 256, sdesc_sw128(paddr, 16, 1024), vd, idesc_pv,
                        (pc > 0 || jt > 0 || kk > 0));
                umma_ss(tmem + h * 256, sdesc_sw128(paddr + kPBytes, 16, 1024), vd, idesc_pv, 1u);
              }
              umma_commit(&bars->ring_empty[s]);
              umma_commit(&bars->ring_empty[s + 1]);
              cnt += 2;
            }
          }
          if (ok) umma_commit(&bars->o_done[pc & 1]);
        }
      }
      if (!ok) {
        bars->abort = 1;
        if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << 11));
      }
      volatile int no_abort = 0;
      umma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, &no_abort, 100000000ull);
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------------ softmax + partials
    // Lane l + 16 of a warp holds score row quad * 16 + l; lane l (< 16) holds the O row of
    // the same head. Per chunk c: wait S(c); row max; wait PV(c - 1) (frees P, and lets O
    // be rescaled); lazy rescale; P(c); arrive p_full. PV(c - 1) is awaited at every chunk,
    // so each o_done[x] phase is awaited in order and a parity wait never sees a barrier
    // that is two phases away.
    const int quad = warp & 3;
    const bool s_lane = lane >= 16;
    const int hrow = quad * 16 + (lane & 15);
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const int t = sq.t;
    const int W = p.W;
    bool ok = true;
    float base = -INFINITY, l = 0.f;
    for (int c = 0; c < nchunks && ok; ++c) {
      ok = __all_sync(0xffffffffu, mbar_wait(&bars->s_full[c & 1], (c >> 1) & 1, abort));
      if (!ok) break;
      tc_fence_after();
      const uint32_t sbuf = tmem + lane_addr + (c & 1) * (kCT * kTN);
      // pass 1: row max over the visible keys of the chunk (branch-free selects)
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
      for (int j = chunk_t0(c); j < chunk_t1(c); ++j) {
        const Tile tl = tile_of(p, sq, j);
        // visible columns: a prefix of a compressed tile, or ring slots 0..min(W,t+1)-1
        const int vhi = tl.kind == kCompressed ? min(tl.n, sq.e1 - tl.key0) : min(W, t + 1);
        const uint32_t vlen = vhi > 0 ? (uint32_t)vhi : 0u;
        const uint32_t col0 = (j - chunk_t0(c)) * kTN;
        for (int q = 0; q < kTN / 32; ++q) {
          if (q * 32 >= tl.n) break;
          uint32_t v[32];
          tmem_ld32(sbuf + col0 + q * 32, v);
          tmem_wait_ld();
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
      }
      const float cmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                         p.scale_log2;
      // lazy rescale: move the base only when the max grew by more than the threshold
      const bool grow = s_lane && (c == 0 || cmax > base + kRescaleThreshold);
      float factor = 1.f;
      if (grow) {
        factor = c == 0 ? 1.f : fast_exp2(base - cmax);
        l *= factor;
        base = cmax;
      }
      if (c > 0) {
        // PV(c - 1) done: the P buffer is free and O holds every earlier chunk
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&bars->o_done[(c - 1) & 1], ((c - 1) >> 1) & 1, abort));
        if (!ok) break;
      }
      if (c > 0 && __any_sync(0xffffffffu, grow)) {
        // O rows live in lanes 0-15 next to score lanes 16-31 of the same columns: the
        // 32-lane read-modify-write below is safe only with no UMMA in flight, i.e. also
        // after S(c + 1) (if issued) has completed. PV(c) waits for our p_full.
        if (c + 1 < nchunks)
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
      // pass 2: P = exp2(s * scale - base) -> bf16 parts P_hi = bf16(P), P_lo = bf16(P - P_hi)
      // in two K-major 128B-swizzled buffers; O += P_hi V + P_lo V keeps ~16 bits of P.
      // All 32 lanes work: of each 32-column piece of row hrow, lane l + 16 takes columns
      // 0..15 and lane l columns 16..31.
      uint8_t* pbuf = sP;
      const float b_own = base == -INFINITY ? 0.f : base;
      const float b_pair = __shfl_xor_sync(0xffffffffu, b_own, 16);
      const float bb = s_lane ? b_own : b_pair;
      const int half = s_lane ? 0 : 16;
      float ps = 0.f;
      for (int j = chunk_t0(c); j < chunk_t1(c); ++j) {
        const Tile tl = tile_of(p, sq, j);
        const int vhi = tl.kind == kCompressed ? min(tl.n, sq.e1 - tl.key0) : min(W, t + 1);
        const uint32_t vlen = vhi > 0 ? (uint32_t)vhi : 0u;
        const int jt = j - chunk_t0(c);
        for (int q = 0; q < kTN / 32; ++q) {
          if (q * 32 >= tl.n) break;
          uint32_t v[32];
          tmem_ld32(sbuf + jt * kTN + q * 32, v);
          tmem_wait_ld();
          float x[16];
          pair_split(v, s_lane, x);
          const int col0 = q * 32 + half;
          uint32_t pk[8], pl[8];
          const bool visible = (uint32_t)(q * 32 + 32) <= vlen;  // the whole piece: no masks
          ps += visible ? p_piece<false, kPBf16Pair>(x, p.scale_log2, bb, col0, vlen, 1.f, pk, pl)
                        : p_piece<true, kPBf16Pair>(x, p.scale_log2, bb, col0, vlen, 1.f, pk, pl);
          // chunk keys jt*128 + col0 .. -> 64-key P chunk (jt*2 + q/2), 16-byte units
          // (q&1)*4 + half/8 + w
          uint8_t* rowp = pbuf + (jt * 2 + (q >> 1)) * kPChunkBytes + hrow * 128;
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            const int u = (q & 1) * 4 + (half >> 3) + w;
            const int us = u ^ (hrow & 7);
            *reinterpret_cast<uint4*>(rowp + us * 16) =
                make_uint4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]);
            *reinterpret_cast<uint4*>(rowp + kPBytes + us * 16) =
                make_uint4(pl[4 * w], pl[4 * w + 1], pl[4 * w + 2], pl[4 * w + 3]);
          }
        }
      }
      l += ps + __shfl_xor_sync(0xffffffffu, ps, 16);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[c & 1]);
    }
    // the last PV's commit covers every earlier UMMA of this CTA
    if (ok) ok = mbar_wait(&bars->o_done[(nchunks - 1) & 1], ((nchunks - 1) >> 1) & 1, abort);
    ok = __all_sync(0xffffffffu, ok);
    float* sO = reinterpret_cast<float*>(smem + kOffStage);  // [64][kORow]
    float* sM = sO + kM * kORow;                               // row max (log2 units)
    float* sL = sM + kM;                                       // row sum
    float* sInv = sL + kM;                                     // 1 / row sum
    if (ok) {
      tc_fence_after();
      if (s_lane) {
        sM[hrow] = base;
        sL[hrow] = l;
        sInv[hrow] = 1.f / l;
      }
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
            o4[w] = make_float4(__uint_as_float(v[4 * w]), __uint_as_float(v[4 * w + 1]),
                                __uint_as_float(v[4 * w + 2]), __uint_as_float(v[4 * w + 3]));
        }
      }
    } else {
      bars->abort = 1;
      if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << 12));
    }
    // every softmax warp arrives here exactly once (also after a time-out: the output is
    // then invalid and flagged)
    asm volatile("bar.sync 1, 128;" ::: "memory");
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
          // the gate is only guaranteed 4-byte aligned: four bf16x2 loads
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
      // split partial: unnormalised O, (max, sum) per head
      const int64_t slot0 = ((int64_t)b * p.nsplit + split) * p.hq;
      float* ob = p.ws_o + slot0 * kD;
      for (int i = tid; i < p.hq * (kD / 4); i += 128) {
        const int h = i / (kD / 4);
        const int c = 4 * (i % (kD / 4));
        *reinterpret_cast<float4*>(ob + (int64_t)h * kD + c) =
            *reinterpret_cast<const float4*>(sO + h * kORow + c);
      }
      for (int h = tid; h < p.hq; h += 128) {
        p.ws_ml[(slot0 + h) * 2] = sM[h];
        p.ws_ml[(slot0 + h) * 2 + 1] = sL[h];
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

// Combine the partials of one sequence: per head, M = max_s m_s over the parts holding keys,
// L = sum_s 2^(m_s - M) l_s, acc = sum_s 2^(m_s - M) O_s. Final output: acc / L, then the
// gate and the cast to bf16, lse = (M + log2 L) ln 2. Partial output (one part that stands
// for all of them): (M, L) and acc, float32. One block per (head, sequence), 4 output
// columns per thread. The non-empty parts are listed in order (ballot compaction, so the
// sums are deterministic) with their weights in shared memory; every thread then walks the
// list with independent loads.
constexpr int kMergeThreads = kD / 4;  // 128

struct MergeArgs {
  const float* ml;             // (m, l) of part s, sequence b, head h at
  const float* o;              //   ml + s * ml_ss + b * ml_bs + 2 h;  o: + s * o_ss + b * o_bs
  int64_t ml_ss, ml_bs, o_ss, o_bs;  // + h * 512
  int nsplit, hq;
  const __nv_bfloat16* gate;
  int64_t gs0, gs2;
  __nv_bfloat16* O;            // final output (when pml == nullptr)
  float* lse;
  float* pml;                  // partial output [b, h, 2] and [b, h, 512] (or nullptr)
  float* po;
};

__global__ void __launch_bounds__(kMergeThreads) merge_kernel(const MergeArgs a) {
  __shared__ float s_w[kMergeThreads], s_l[kMergeThreads];
  __shared__ int s_idx[kMergeThreads];
  __shared__ float s_red[kMergeThreads / 32];
  __shared__ int s_cnt[kMergeThreads / 32];
  pdl_wait();  // the decode grid's partials are complete and visible
  pdl_trigger();
  const int b = blockIdx.y;
  const int h = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int wid = tid >> 5;
  const int nsplit = a.nsplit;
  const float* ml = a.ml + (int64_t)b * a.ml_bs + (int64_t)h * 2;
  const float* ob = a.o + (int64_t)b * a.o_bs + (int64_t)h * kD + tid * 4;

  float m = -INFINITY;
  for (int s = tid; s < nsplit; s += kMergeThreads) {
    const float2 v = *reinterpret_cast<const float2*>(ml + s * a.ml_ss);
    if (v.y > 0.f) m = fmaxf(m, v.x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) s_red[wid] = m;
  __syncthreads();
  float M = s_red[0];
#pragma unroll
  for (int w = 1; w < kMergeThreads / 32; ++w) M = fmaxf(M, s_red[w]);

  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < nsplit; s0 += kMergeThreads) {
    const int s = s0 + tid;
    float2 v = make_float2(-INFINITY, 0.f);
    if (s < nsplit) v = *reinterpret_cast<const float2*>(ml + s * a.ml_ss);
    const bool live = v.y > 0.f;
    const unsigned bal = __ballot_sync(0xffffffffu, live);
    __syncthreads();  // the previous chunk's list has been consumed
    if (lane == 0) s_cnt[wid] = __popc(bal);
    __syncthreads();
    int off = 0, n = 0;
#pragma unroll
    for (int w = 0; w < kMergeThreads / 32; ++w) {
      off += w < wid ? s_cnt[w] : 0;
      n += s_cnt[w];
    }
    if (live) {
      const int k = off + __popc(bal & ((1u << lane) - 1u));
      s_w[k] = exp2f(v.x - M);
      s_l[k] = v.y;
      s_idx[k] = s;
    }
    __syncthreads();
    int k = 0;
    for (; k + 4 <= n; k += 4) {
      float4 x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        x[u] = *reinterpret_cast<const float4*>(ob + s_idx[k + u] * a.o_ss);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float w = s_w[k + u];
        acc.x = fmaf(w, x[u].x, acc.x);
        acc.y = fmaf(w, x[u].y, acc.y);
        acc.z = fmaf(w, x[u].z, acc.z);
        acc.w = fmaf(w, x[u].w, acc.w);
        L = fmaf(w, s_l[k + u], L);
      }
    }
    for (; k < n; ++k) {
      const float4 x = *reinterpret_cast<const float4*>(ob + s_idx[k] * a.o_ss);
      const float w = s_w[k];
      acc.x = fmaf(w, x.x, acc.x);
      acc.y = fmaf(w, x.y, acc.y);
      acc.z = fmaf(w, x.z, acc.z);
      acc.w = fmaf(w, x.w, acc.w);
      L = fmaf(w, s_l[k], L);
    }
  }
  const int d = tid * 4;
  const int64_t bh = (int64_t)b * a.hq + h;
  if (a.pml) {
    *reinterpret_cast<float4*>(a.po + bh * kD + d) = acc;
    if (tid == 0) *reinterpret_cast<float2*>(a.pml + bh * 2) = make_float2(M, L);
    return;
  }
  const float inv = 1.f / L;
  float o[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
  if (a.gate) {
    const __nv_bfloat16* gp = a.gate + (int64_t)b * a.gs0 + (int64_t)h * a.gs2 + d;
    const float2 g0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(gp));
    const float2 g1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(gp + 2));
    o[0] *= g0.x;
    o[1] *= g0.y;
    o[2] *= g1.x;
    o[3] *= g1.y;
  }
  *reinterpret_cast<uint2*>(a.O + bh * kD + d) =
      make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
  if (a.lse && tid == 0) a.lse[bh] = (M + __log2f(L)) * 0.69314718055994531f;
}

}  // namespace

bool decode_tc_supported(const hca_desc& d, const hca_cache& c) {
  if (d.dtype != HCA_BF16 || d.head_dim != kD || d.hkv != 1) return false;
  if (d.hq < 1 || d.hq > kM) return false;
  if (d.window < 1 || d.window > kTN || d.block < 1) return false;
  if (c.page_entries % 128 != 0) return false;
  // TMA row coordinates and row indices are 32-bit
  if ((int64_t)c.num_pages * c.page_entries >= (int64_t(1) << 31)) return false;
  if ((int64_t)d.batch * (d.hq > d.window ? d.hq : d.window) >= (int64_t(1) << 31)) return false;
  if (d.gate) {
    const uintptr_t ga = reinterpret_cast<uintptr_t>(d.gate);
    if (ga % 4 || d.gate_strides[0] % 2 || d.gate_strides[2] % 2) return false;
  }
  return true;
}

// Splits per sequence for a key list of `tiles` 128-key tiles (d.decode_splits if > 0,
// capped at the tiles). Automatic rule: the time of a step is about the largest number of
// tiles one CTA streams, plus, once a sequence is split, its float32 partials and the merge
// (about two tiles' worth, measured). Among the split counts that keep every CTA in one
// wave (splits x batch <= SMs), take the one with the fewest tiles per CTA + 2 if split;
// ties go to fewer splits. 16 sequences at 1M context (65 tiles) -> 9 splits; 128
// sequences of up to 9 tiles -> 1.
static int splits_for_tiles(const hca_desc& d, int tiles) {
  if (tiles < 1) tiles = 1;
  if (d.decode_splits > 0) return d.decode_splits < tiles ? d.decode_splits : tiles;
  const int64_t sms = device_sm_count();
  const int64_t batch = d.batch > 0 ? d.batch : 1;
  int64_t smax = sms / batch;
  if (smax < 1) smax = 1;
  if (smax > tiles) smax = tiles;
  int best = 1;
  int64_t best_cost = tiles;
  for (int64_t sp = 2; sp <= smax; ++sp) {
    const int64_t cost = (tiles + sp - 1) / sp + 2;
    if (cost < best_cost) {
      best_cost = cost;
      best = (int)sp;
    }
  }
  return best;
}

// visible compressed entries of the longest context d.seqlen
static int64_t max_visible_entries(const hca_desc& d) {
  const int64_t x = (int64_t)d.seqlen - d.window;
  return x < 0 ? 0 : x / d.block;
}

int decode_num_splits(const hca_desc& d) {
  return splits_for_tiles(d, (int)((max_visible_entries(d) + kTN - 1) / kTN) + 1);
}

// Split count of a call over the key part: at most that of the whole key list, so the
// workspace of hca_decode_workspace_bytes(d) always suffices.
int part_num_splits(const hca_desc& d, const DecodePart& part) {
  const int64_t nc = max_visible_entries(d);
  const int64_t e1 = part.e1 < nc ? part.e1 : nc;
  const int64_t n = e1 > part.e0 ? e1 - part.e0 : 0;
  const int tiles = (int)((n + kTN - 1) / kTN) + (part.with_ring ? 1 : 0);
  const int ns = splits_for_tiles(d, tiles);
  const int full = decode_num_splits(d);
  return ns < full ? ns : full;
}

// Workspace layout: ws_ml [batch, nsplit, hq, 2] float, padded to a multiple of 4 floats so
// that ws_o [batch, nsplit, hq, 512] float (read and written as float4) starts 16-byte
// aligned whatever batch * nsplit * hq is. A partial result is this layout with nsplit 1.
size_t ml_floats(const hca_desc& d, int nsplit) {
  const size_t n = (size_t)d.batch * nsplit * d.hq * 2;
  return (n + 3) & ~size_t(3);
}

size_t decode_tc_workspace_bytes(const hca_desc& d) {
  const int ns = decode_num_splits(d);
  return (ml_floats(d, ns) + (size_t)d.batch * ns * d.hq * kD) * sizeof(float);
}

size_t decode_partial_bytes(const hca_desc& d) {
  return (ml_floats(d, 1) + (size_t)d.batch * d.hq * kD) * sizeof(float);
}

size_t decode_part_workspace_bytes(const hca_desc& d, const DecodePart& part) {
  const int ns = part_num_splits(d, part);
  if (ns == 1 && part.out_partial) return 0;
  return (ml_floats(d, ns) + (size_t)d.batch * ns * d.hq * kD) * sizeof(float);
}

cudaLaunchConfig_t pdl_config(cudaLaunchAttribute* pdl, cudaStream_t s) {
  // programmatic dependent of the grid before it on the stream (each kernel waits for it
  // with griddepcontrol.wait before touching memory)
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = s;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  return cfg;
}

cudaError_t launch_decode_part(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                               const hca_cache& c, const void* ring_k, const void* ring_v,
                               const DecodePart& part, void* O, float* lse, void* ws,
                               cudaStream_t s) {
  if (c.pool_format == HCA_POOL_E4M3)
    return launch_decode_fp8(d, Q, ctx_len, c, ring_k, ring_v, part, O, lse, ws, s);
  Params p;
  memset(&p, 0, sizeof(p));
  const int nsplit = part_num_splits(d, part);
  cudaError_t e;
  const uint64_t rowsC = (uint64_t)c.num_pages * c.page_entries;
  if ((e = encode_bf16_chunks(&p.tmQ, Q, (uint64_t)d.batch * d.hq, kM, 4)) != cudaSuccess)
    return e;
  if ((e = encode_bf16_chunks(&p.tmKc, c.kc_pool, rowsC, kTN, 2)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmVc, c.vc_pool, rowsC, kTN, 2)) != cudaSuccess) return e;
  const uint64_t rowsR = (uint64_t)d.batch * d.window;
  if ((e = encode_bf16_chunks(&p.tmRk, ring_k, rowsR, kTN, 2)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmRv, ring_v, rowsR, kTN, 2)) != cudaSuccess) return e;
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
  p.O = static_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.gate = static_cast<const __nv_bfloat16*>(d.gate);
  p.gs0 = d.gate_strides[0];
  p.gs2 = d.gate_strides[2];
  static PerDevice<int> smem_limit_set;
  if ((e = set_smem_limit_once(smem_limit_set, (const void*)decode_tc_kernel, (int)kSmemBytes)) !=
      cudaSuccess)
    return e;
  // both grids are programmatic dependents of the grid before them on the stream: the merge
  // is scheduled while decode CTAs drain, and a following decode step's prologue overlaps
  // the merge
  cudaLaunchAttribute pdl[1];
  cudaLaunchConfig_t cfg = pdl_config(pdl, s);
  cfg.gridDim = dim3(nsplit, d.batch);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  if ((e = cudaLaunchKernelEx(&cfg, decode_tc_kernel, p)) != cudaSuccess) return e;
  if (nsplit == 1) return cudaSuccess;  // the decode CTAs wrote their result themselves
  return launch_split_merge(d, p.ws_ml, p.ws_o, nsplit, pml, po, O, lse, s);
}

cudaError_t launch_split_merge(const hca_desc& d, const float* ws_ml, const float* ws_o,
                               int nsplit, float* pml, float* po, void* O, float* lse,
                               cudaStream_t s) {
  MergeArgs m;
  memset(&m, 0, sizeof(m));
  m.ml = ws_ml;
  m.o = ws_o;
  m.ml_ss = (int64_t)d.hq * 2;
  m.ml_bs = (int64_t)nsplit * d.hq * 2;
  m.o_ss = (int64_t)d.hq * kD;
  m.o_bs = (int64_t)nsplit * d.hq * kD;
  m.nsplit = nsplit;
  m.hq = d.hq;
  m.gate = static_cast<const __nv_bfloat16*>(d.gate);
  m.gs0 = d.gate_strides[0];
  m.gs2 = d.gate_strides[2];
  m.O = static_cast<__nv_bfloat16*>(O);
  m.lse = lse;
  m.pml = pml;
  m.po = po;
  cudaLaunchAttribute pdl[1];
  cudaLaunchConfig_t mcfg = pdl_config(pdl, s);
  mcfg.gridDim = dim3(d.hq, d.batch);
  mcfg.blockDim = dim3(kMergeThreads);
  return cudaLaunchKernelEx(&mcfg, merge_kernel, m);
}

cudaError_t launch_decode_tc(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                             const hca_cache& c, const void* ring_k, const void* ring_v,
                             void* O, float* lse, void* ws, cudaStream_t s) {
  const DecodePart whole{0, INT32_MAX, 1, nullptr};
  return launch_decode_part(d, Q, ctx_len, c, ring_k, ring_v, whole, O, lse, ws, s);
}

cudaError_t launch_decode_merge(const hca_desc& d, const void* parts, int n_parts,
                                int64_t part_stride_bytes, void* O, float* lse,
                                cudaStream_t s) {
  MergeArgs m;
  memset(&m, 0, sizeof(m));
  const int64_t stride = part_stride_bytes / (int64_t)sizeof(float);
  m.ml = static_cast<const float*>(parts);
  m.o = m.ml + ml_floats(d, 1);
  m.ml_ss = stride;
  m.ml_bs = (int64_t)d.hq * 2;
  m.o_ss = stride;
  m.o_bs = (int64_t)d.hq * kD;
  m.nsplit = n_parts;
  m.hq = d.hq;
  m.gate = static_cast<const __nv_bfloat16*>(d.gate);
  m.gs0 = d.gate_strides[0];
  m.gs2 = d.gate_strides[2];
  m.O = static_cast<__nv_bfloat16*>(O);
  m.lse = lse;
  cudaLaunchAttribute pdl[1];
  cudaLaunchConfig_t mcfg = pdl_config(pdl, s);
  mcfg.gridDim = dim3(d.hq, d.batch);
  mcfg.blockDim = dim3(kMergeThreads);
  return cudaLaunchKernelEx(&mcfg, merge_kernel, m);
}

// ---------------------------------------------------------------------------------------
// Decode without a caller-provided workspace.
//
// Some callers cannot hand this library a workspace: their device memory belongs to
// another allocator (a framework's caching pool, or a serving engine that reserves all of
// HBM up front and has no free block to lend), or their decode loop must not call the CUDA
// allocator at all, because cudaMalloc/cudaFree can synchronise the device and stall every
// other stream. For them the split partials live in one fixed array inside the library,
// sized for HCA_DECODE_NOALLOC_SCRATCH_BYTES (include/hca.h). The array is created when the
// library's device code is loaded on a GPU and stays allocated on that GPU until the
// process exits. Every call reuses it, so two calls whose kernels overlap on the GPU (two
// streams, or two host threads) overwrite each other's partials; callers must serialise
// them. Nothing in it has to start at zero: each split writes its partial before the merge
// reads it.
static __device__ __align__(256) unsigned char g_decode_scratch[HCA_DECODE_NOALLOC_SCRATCH_BYTES];

// The array's name is only a host-side stand-in; its device address is looked up once per
// device (on that device's first call, with that device current) and memoised.
static cudaError_t decode_scratch_address(void** out) {
  static PerDevice<void*> cached;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (cached.get(dev, out)) return cudaSuccess;
  void* ptr = nullptr;
  e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
  if (e != cudaSuccess) return e;
  cached.put(dev, ptr);
  *out = ptr;
  return cudaSuccess;
}

cudaError_t launch_decode_tc_noalloc(const hca_desc& d, const void* Q, const int32_t* ctx_len,
                                     const hca_cache& c, const void* ring_k,
                                     const void* ring_v, void* O, float* lse, cudaStream_t s) {
  void* ws = nullptr;
  cudaError_t e = decode_scratch_address(&ws);
  if (e != cudaSuccess) return e;
  return launch_decode_tc(d, Q, ctx_len, c, ring_k, ring_v, O, lse, ws, s);
}

}  // namespace hca
