// prefill_tc.cu -- HCA prefill attention on tcgen05 tensor cores (bf16 in, f32 accumulate).
//
// Operation ([news 二.1] / [analysis 1] / [gate] in include/hca.h): every query position t
// attends with one softmax to the compressed entries j < n_c(t) (blocks that end before its
// window) and to the raw tokens max(0, t-W+1) .. t, head_dim 512; the output is optionally
// multiplied by a supplied gate.
//
// Design for sm_100a:
//  * A tile is 128 rows = (128 / hq) consecutive positions x hq query heads. All rows share
//    the single KV head, so one K/V tile in shared memory serves 128 rows.
//  * head_dim 512 in float32 would fill all 512 TMEM columns for 128 rows, leaving no room
//    for scores. Each CTA therefore owns one 256-wide half of the output: TMEM holds the
//    output half (256 columns) and two 128-column score buffers. Both halves compute the
//    full scores (the price of the split: 1.5x tensor work; a later design removes it).
//  * Q (128 x 512 bf16, 128 KB) stays in shared memory for the tile; K and V stream through
//    a ring of three 32 KB slots (3-D TMA boxes of 128 rows x two 128-byte chunks, 128-byte
//    swizzle).
//  * Warp roles: warps 0 and 10 stream K/V and warp 11 streams Q through TMA, warp 1 issues
//    UMMA (single thread), warps 2-5 run the online softmax (one row per thread, TMEM
//    lane = row), warps 6-9 the epilogue (O / l, gate, bf16) of the previous item.
//  * S = Q K^T runs as kind::f16 with both operands in shared memory; P is split into two
//    bf16 parts (P_hi = bf16(P), P_lo = bf16(P - P_hi)) written back into the score columns
//    of TMEM, and O += P_hi V + P_lo V runs as two UMMAs with A from TMEM and V (N-major)
//    from shared memory, so the rounding of P costs ~2^-17 of the value spread, not 2^-9.
//  * The key list of a tile is: compressed tiles of up to 128 entries (the last one cut to
//    a multiple of 16), an optional 16-row raw tile for the keys that only the first
//    position of the tile still sees, then one 128-row raw tile ending at the last position.
//  * Online softmax in base 2 with lazy rescaling: the running reference only moves when
//    the row max grows by more than 8 (a factor of 256), so O is rarely touched.
//  * Persistent grid, one CTA per SM, row tiles in decreasing-work order handed out in a
//    snake so that every CTA gets a similar share; a CTA runs both output halves of a row
//    tile back to back, the second on the Q tile already in shared memory.
//  * Every mbarrier wait is bounded; on time-out the CTA raises HCA_ERR_TIMEOUT (4) in the
//    error word and unwinds, releasing its TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <string.h>

#include "hca_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace hca {
namespace {

constexpr int kBM = 128;               // rows per tile
constexpr int kD = 512;                // head_dim
constexpr int kDH = 256;               // output half per CTA
constexpr int kKC = 64;                // elements per 128-byte swizzle row (one "chunk")
constexpr int kNCh = kD / kKC;         // 8 chunks of Q / K
constexpr int kBN = 128;               // max keys per tile
constexpr uint32_t kChunk128 = kBN * kKC * 2;  // 16 KB: 128 rows x one chunk
constexpr uint32_t kChunk16 = 16 * kKC * 2;    // 2 KB: 16 rows x one chunk
constexpr uint32_t kSlotBytes = 2 * kChunk128;  // 32 KB: 128 rows x two chunks
constexpr int kStages = 3;
constexpr int kQPairs = 4;                     // Q loaded as 4 boxes of two chunks
constexpr uint32_t kQBytes = kNCh * kChunk128;  // 128 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmS0 = 0, kTmO = 256;
constexpr int kThreads = 384;  // 3 TMA warps, UMMA, 4 softmax warps, 4 epilogue warps
constexpr float kRescaleThreshold = 8.0f;  // log2 units

enum TileKind { kCompressed = 0, kRaw16 = 1, kRaw128 = 2 };

struct Params {
  // 3-D maps {64 elements, rows, 8 chunks}: one box = rows x (chunks x 128 B)
  CUtensorMap tmQ, tmK, tmV, tmK16, tmV16, tmKc, tmVc;
  __nv_bfloat16* O;
  float* lse;
  int32_t* dbg;
  const __nv_bfloat16* gate;
  int64_t gs0, gs1, gs2;
  const int32_t* page_table;
  const int32_t* n_entries;
  int32_t* err_word;
  int32_t batch, T, hq, P, W, block, PE, max_pages, num_pages;
  // query row t of a sequence is position q0 + t; K/V row u is position kv0 + u, of Tk rows
  int32_t q0, kv0, Tk;
  int32_t n_rt;     // row tiles per sequence
  int32_t n_items;  // 2 * batch * n_rt
  float scale_log2;
};

struct Item {
  int b, i, half;
  int t0, tl;       // first / last valid query row of the tile
  int nc_last;      // compressed entries visible to the last position (clamped)
  int nct;          // compressed tiles
  int lo, hi;       // raw key range of the tile (positions)
  int rawA_n;       // keys used from the 128-row raw tile
  int strag;        // 1 if the 16-row raw tile exists
  int ntiles;
};

struct Tile {
  int kind;
  int n;       // keys (MMA N), multiple of 16
  int rowoff;  // first used row inside the loaded box
  int key0;    // compressed: first entry; raw: token of the first used row
};

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

__device__ __forceinline__ int visible_count(int t, int block, int W) {
  const int x = t + 1 - W;
  return x < 0 ? 0 : x / block;
}

__device__ __forceinline__ int item_index(int r, int G, int c) {
  return r * G + ((r & 1) ? (G - 1 - c) : c);  // snake over the CTAs
}

// The r-th item of CTA c: row tiles are dealt out in the snake above, and a CTA takes both
// output halves of a row tile one after the other (items 2 rt and 2 rt + 1), so the second
// half reuses the Q tile already in shared memory.
__device__ __forceinline__ int cta_item(int r, int G, int c) {
  return 2 * item_index(r >> 1, G, c) + (r & 1);
}

__device__ __forceinline__ Item make_item(const Params& p, int k) {
  Item it;
  it.half = k & 1;
  const int rt = k >> 1;
  it.b = rt % p.batch;
  it.i = p.n_rt - 1 - rt / p.batch;  // heaviest tiles first
  it.t0 = it.i * p.P;
  it.tl = min(it.t0 + p.P - 1, p.T - 1);
  // never trust the device count beyond what the page table can address
  const int have = min(p.n_entries[it.b], p.max_pages * p.PE);
  it.nc_last = min(visible_count(it.tl + p.q0, p.block, p.W), have);
  it.nct = (it.nc_last + kBN - 1) / kBN;
  it.lo = max(0, it.t0 + p.q0 - p.W + 1);
  it.hi = it.tl + p.q0;
  const int R = it.hi - it.lo + 1;
  it.rawA_n = min(kBN, round16(min(R, kBN)));
  it.strag = R > kBN ? 1 : 0;
  it.ntiles = it.nct + it.strag + 1;
  return it;
}

__device__ __forceinline__ Tile tile_of(const Item& it, int j) {
  Tile t;
  if (j < it.nct) {
    t.kind = kCompressed;
    t.key0 = j * kBN;
    t.n = min(kBN, round16(it.nc_last - j * kBN));
    t.rowoff = 0;
  } else if (it.strag && j == it.nct) {
    t.kind = kRaw16;
    t.key0 = it.hi - 143;
    t.n = 16;
    t.rowoff = 0;
  } else {
    t.kind = kRaw128;
    t.n = it.rawA_n;
    t.rowoff = kBN - it.rawA_n;
    t.key0 = it.hi - kBN + 1 + t.rowoff;
  }
  return t;
}

// K slots of a tile: 4 boxes of two chunks (128-row kinds) or 1 box of all 8 chunks
// (16-row kind); V slots: 2 boxes of two chunks of this CTA's half, or 1 box of its 4.
__device__ __forceinline__ int k_slots(const Tile& t) { return t.kind == kRaw16 ? 1 : 4; }
__device__ __forceinline__ int v_slots(const Tile& t) { return t.kind == kRaw16 ? 1 : 2; }

// Shared-memory carve-up (offsets from a 1024-byte aligned base).
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffRing = kQBytes;
constexpr uint32_t kOffBar = kOffRing + kStages * kSlotBytes;
constexpr uint32_t kOffL = kOffBar + 256;               // row sums l, 2 items x 128 rows
constexpr uint32_t kSmemBytes = kOffL + 2 * kBM * 4 + 1024;  // + alignment slack

struct Bars {
  uint64_t q_full[kQPairs], q_empty[kQPairs];
  uint64_t ring_full[kStages], ring_empty[kStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done, o_free, o_final, drain;
  uint64_t l_full[2];  // per item parity: a single barrier could run two phases ahead
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 256, "barrier block too large");

// role: 1 K/V producer, 2 Q producer, 3 UMMA issuer, 4 softmax, 5 epilogue; recorded in
// bit (8 + role) next to HCA_ERR_TIMEOUT so a report names the role that gave up first.
__device__ __forceinline__ void raise_timeout(const Params& p, Bars* bars, int role) {
  bars->abort = 1;
  if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << (8 + role)));
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t row, int32_t chunk, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(0), "r"(row), "r"(chunk),
      "l"(policy)
      : "memory");
}

// L2 policies: streams read or written once (Q, gate, O) leave L2 first; K/V tiles, read
// by every row tile of a sequence, stay.
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint4 ld_stream_hint(const void* ptr, uint64_t pol) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr), "l"(pol));
  return v;
}
__device__ __forceinline__ void st_stream_hint(void* ptr, const uint4& v, uint64_t pol) {
  asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.u32 [%0], {%1,%2,%3,%4}, %5;" ::"l"(ptr),
               "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "l"(pol)
               : "memory");
}

__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sRing = smem + kOffRing;
  Bars* bars = reinterpret_cast<Bars*>(smem + kOffBar);
  float* sL = reinterpret_cast<float*>(smem + kOffL);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int q = 0; q < kQPairs; ++q) {
      mbar_init(&bars->q_full[q], 1);
      mbar_init(&bars->q_empty[q], 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->ring_full[s], 1);
      mbar_init(&bars->ring_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->p_full[s], 4);
    }
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->o_free, 4);
    mbar_init(&bars->o_final, 1);
    mbar_init(&bars->l_full[0], 4);
    mbar_init(&bars->l_full[1], 4);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmQ);
    tma_prefetch_desc(&p.tmK);
    tma_prefetch_desc(&p.tmV);
    tma_prefetch_desc(&p.tmK16);
    tma_prefetch_desc(&p.tmV16);
    tma_prefetch_desc(&p.tmKc);
    tma_prefetch_desc(&p.tmVc);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int G = gridDim.x;
  const int c = blockIdx.x;

  if (warp == 0 || warp == 10) {
    // ------------------------------------------------------------------ K/V TMA producers
    // Two producer warps walk the same load sequence and take turns (even / odd loads):
    // one issuing thread's bulk-tensor copies are served one after another, so two
    // issuers double the fill rate. The sequence is the order the UMMA warp consumes,
    // one stream over all items of the CTA: K of tile g, then V of tile g-1.
    if (elect_one()) {
      const uint32_t mine = warp == 0 ? 0u : 1u;
      const uint64_t pol_kv = policy_evict_last();
      uint32_t cnt = 0;  // ring loads in the sequence so far (both producers)
      bool ok = true;
      // returns the slot to fill, -2 when the other producer owns this load, -1 on time-out
      auto next_slot = [&](uint32_t bytes) -> int {
        const uint32_t n = cnt++;
        if ((n & 1u) != mine) return -2;
        const uint32_t s = n % kStages;
        const uint32_t round = n / kStages;
        if (round > 0 && !mbar_wait(&bars->ring_empty[s], (round - 1) & 1, abort)) return -1;
        mbar_expect_tx(&bars->ring_full[s], bytes);
        return (int)s;
      };
      auto load_tile = [&](const Item& it, int j, bool is_v) -> bool {
        const Tile t = tile_of(it, j);
        const int nsl = is_v ? v_slots(t) : k_slots(t);
        for (int q = 0; q < nsl; ++q) {
          if (t.kind == kRaw16) {
            const int s = next_slot(is_v ? 4 * kChunk16 : kNCh * kChunk16);
            if (s == -1) return false;
            if (s >= 0)
              tma_load_3d(sRing + s * kSlotBytes, is_v ? &p.tmV16 : &p.tmK16,
                          &bars->ring_full[s], it.b * p.Tk + t.key0 - p.kv0,
                          is_v ? it.half * 4 : 0,
                          pol_kv);
            continue;
          }
          const int s = next_slot(kSlotBytes);
          if (s == -1) return false;
          if (s < 0) continue;
          const int chunk = is_v ? it.half * 4 + 2 * q : 2 * q;
          int row;
          const CUtensorMap* map;
          if (t.kind == kCompressed) {
            int page = p.page_table[(int64_t)it.b * p.max_pages + t.key0 / p.PE];
            if (page < 0 || page >= p.num_pages) {
              if (p.err_word) atomicOr(p.err_word, kErrPageRange);
              page = 0;
            }
            row = page * p.PE + (t.key0 % p.PE);
            map = is_v ? &p.tmVc : &p.tmKc;
          } else {
            row = it.b * p.Tk + it.hi - kBN + 1 - p.kv0;
            map = is_v ? &p.tmV : &p.tmK;
          }
          tma_load_3d(sRing + s * kSlotBytes, map, &bars->ring_full[s], row, chunk, pol_kv);
        }
        return true;
      };
      // The UMMA warp consumes one stream across items: K of tile g, then V of tile g-1
      // (which may belong to the previous item), so the next item's first K tile does not
      // wait for the current item's last softmax.
      Item pit;
      int pj = -1;
      for (int r = 0; ok; ++r) {
        const int k = cta_item(r, G, c);
        if (k >= p.n_items) break;
        const Item it = make_item(p, k);
        if (mine == 0 && p.err_word &&
            visible_count(it.tl + p.q0, p.block, p.W) > p.n_entries[it.b])
          atomicOr(p.err_word, kErrCacheShort);
        for (int j = 0; j < it.ntiles && ok; ++j) {
          ok = load_tile(it, j, false);
          if (ok && pj >= 0) ok = load_tile(pit, pj, true);
          pit = it;
          pj = j;
        }
      }
      if (ok && pj >= 0) ok = load_tile(pit, pj, true);
      if (!ok) {
        raise_timeout(p, bars, 1);
        // let this producer's loads already in flight land before shared memory goes away
        volatile int no_abort = 0;
        const uint32_t first = cnt > kStages ? cnt - kStages : 0;
        for (uint32_t q = first; q < cnt; ++q)
          if ((q & 1u) == mine)
            mbar_wait(&bars->ring_full[q % kStages], (q / kStages) & 1, &no_abort, 100000000ull);
      }
    }
  } else if (warp == 11) {
    // ------------------------------------------------------------------ Q TMA producer
    // Q of an item: 4 boxes of two chunks, each reloaded as soon as the previous item's
    // last score UMMA on that pair has finished. The second half of a row tile has the
    // same Q: its pairs are only handed over again (an arrival without a copy).
    if (elect_one()) {
      const uint64_t pol_q = policy_evict_first();
      int nitem = 0;
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int k = cta_item(r, G, c);
        if (k >= p.n_items) break;
        const Item it = make_item(p, k);
        const int qrow = (it.b * p.T + it.t0) * p.hq;
        const bool reuse = (r & 1) != 0;  // same row tile as the previous item
        for (int q = 0; q < kQPairs && ok; ++q) {
          if (nitem > 0 && !(ok = mbar_wait(&bars->q_empty[q], (nitem - 1) & 1, abort))) break;
          if (reuse) {
            mbar_arrive(&bars->q_full[q]);
          } else {
            mbar_expect_tx(&bars->q_full[q], kSlotBytes);
            tma_load_3d(sQ + q * kSlotBytes, &p.tmQ, &bars->q_full[q], qrow, 2 * q, pol_q);
          }
        }
        ++nitem;
      }
      if (!ok) {
        raise_timeout(p, bars, 2);
        volatile int no_abort = 0;
        for (int q = 0; q < kQPairs; ++q)
          mbar_wait(&bars->q_full[q], (nitem - 1) & 1, &no_abort, 100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ UMMA issuer
    if (elect_one()) {
      uint32_t cnt = 0;   // ring slots consumed
      uint32_t g = 0;     // tiles processed (score buffer / phase counter)
      int nitem = 0;
      bool ok = true;
      const uint32_t qbase = smem_u32(sQ);
      const uint32_t rbase = smem_u32(sRing);
      auto issue_s = [&](const Item& it, int j, uint32_t gg, int ni) -> bool {
        const Tile t = tile_of(it, j);
        const int last = it.ntiles - 1;
        const uint32_t sb = gg & 1;
        const uint32_t d_tmem = tmem + kTmS0 + sb * 128;
        const uint32_t idesc = idesc_bf16_f32(kBM, t.n, false);
        if (j == 0) {
          for (int q = 0; q < kQPairs; ++q)
            if (!mbar_wait(&bars->q_full[q], ni & 1, abort)) return false;
        }
        const int nsl = k_slots(t);
        for (int q = 0; q < nsl; ++q) {
          const uint32_t s = cnt % kStages;
          if (!mbar_wait(&bars->ring_full[s], (cnt / kStages) & 1, abort)) return false;
          tc_fence_after();
          const uint32_t sbase = rbase + s * kSlotBytes;
          // chunks of this slot: 2 (128-row kinds, chunk pair q) or all 8 (16-row kind)
          const int nchunks = t.kind == kRaw16 ? kNCh : 2;
          const uint32_t cstride = t.kind == kRaw16 ? kChunk16 : kChunk128;
          for (int cc = 0; cc < nchunks; ++cc) {
            const int d = t.kind == kRaw16 ? cc : 2 * q + cc;
            const uint32_t qaddr = qbase + d * kChunk128;
            const uint32_t kaddr = sbase + cc * cstride + t.rowoff * 128;
#pragma unroll
            for (int kk = 0; kk < kKC / 16; ++kk) {
              const uint64_t ad = sdesc_sw128(qaddr + kk * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(kaddr + kk * 32, 16, 1024);
              umma_ss(d_tmem, ad, bd, idesc, (d | kk) != 0);
            }
          }
          umma_commit(&bars->ring_empty[s]);
          if (j == last) umma_commit(&bars->q_empty[q]);  // the last tile is 128-row
          ++cnt;
        }
        umma_commit(&bars->s_full[sb]);
        return true;
      };
      auto issue_pv = [&](const Item& it, int j, uint32_t gg, int ni) -> bool {
        const Tile t = tile_of(it, j);
        const uint32_t sb = gg & 1;
        if (!mbar_wait(&bars->p_full[sb], (gg >> 1) & 1, abort)) return false;
        // the first P.V of an item overwrites O: the epilogue must have read the last one
        if (j == 0 && ni > 0 && !mbar_wait(&bars->o_free, (ni - 1) & 1, abort)) return false;
        tc_fence_after();
        const uint32_t a_tmem = tmem + kTmS0 + sb * 128;
        const int nsl = v_slots(t);
        for (int q = 0; q < nsl; ++q) {
          const uint32_t s = cnt % kStages;
          if (!mbar_wait(&bars->ring_full[s], (cnt / kStages) & 1, abort)) return false;
          tc_fence_after();
          const uint32_t vaddr = rbase + s * kSlotBytes + t.rowoff * 128;
          // 16-row kind: one N=256 MMA over the 4 chunks (stride 2 KB); 128-row kinds:
          // N=128 over the slot's 2 chunks (stride 16 KB) into columns 128q..128q+127
          const uint32_t ncols = t.kind == kRaw16 ? 256 : 128;
          const uint32_t lbo = t.kind == kRaw16 ? kChunk16 : kChunk128;
          const uint32_t idesc = idesc_bf16_f32(kBM, ncols, true);
          const uint32_t d_tmem = tmem + kTmO + q * 128;
          for (int kk = 0; kk < t.n / 16; ++kk) {
            // 16 keys = two 8-row swizzle atoms = 2 KB; P_hi then P_lo of the group
            const uint64_t bd = sdesc_sw128(vaddr + kk * 2048, lbo, 1024);
            umma_ts(d_tmem, a_tmem + kk * 16, bd, idesc, (j > 0 || kk > 0));
            umma_ts(d_tmem, a_tmem + kk * 16 + 8, bd, idesc, 1u);
          }
          umma_commit(&bars->ring_empty[s]);
          ++cnt;
        }
        umma_commit(&bars->o_done);
        if (j == it.ntiles - 1) umma_commit(&bars->o_final);
        return true;
      };
      // One stream across items: S of tile g, then P.V of tile g-1 (possibly of the
      // previous item), so the tensor pipe keeps working over item boundaries.
      Item pit;
      int pj = -1, pni = 0;
      uint32_t pgg = 0;
      for (int r = 0; ok; ++r) {
        const int k = cta_item(r, G, c);
        if (k >= p.n_items) break;
        const Item it = make_item(p, k);
        for (int j = 0; j < it.ntiles && ok; ++j) {
          ok = issue_s(it, j, g + j, nitem);
          if (ok && pj >= 0) ok = issue_pv(pit, pj, pgg, pni);
          pit = it;
          pj = j;
          pgg = g + j;
          pni = nitem;
        }
        g += it.ntiles;
        ++nitem;
      }
      if (ok && pj >= 0) ok = issue_pv(pit, pj, pgg, pni);
      if (!ok) raise_timeout(p, bars, 3);
      // drain: every UMMA issued above has finished before TMEM is released
      volatile int no_abort = 0;
      umma_commit(&bars->drain);
      mbar_wait(&bars->drain, 0, &no_abort, 100000000ull);
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------------ softmax
    const int quad = warp & 3;               // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;        // tile row == TMEM lane
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    uint32_t g = 0;
    int nitem = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int k = cta_item(r, G, c);
      if (k >= p.n_items) break;
      const Item it = make_item(p, k);
      const int pos = it.t0 + row / p.hq;
      const int h = row % p.hq;
      const bool row_valid = pos < p.T;
      const int tq = min(pos, p.T - 1);  // query row
      const int t = tq + p.q0;           // its position
      const int nc_row =
          min(visible_count(t, p.block, p.W), min(p.n_entries[it.b], p.max_pages * p.PE));
      const int lo_row = max(0, t - p.W + 1);
      float m = -INFINITY;  // reference of the stored P / O (log2 domain)
      float l = 0.f;
      for (int j = 0; j < it.ntiles; ++j) {
        const Tile tl = tile_of(it, j);
        const uint32_t gg = g + j;
        const uint32_t sb = gg & 1;
        if (!(ok = mbar_wait(&bars->s_full[sb], (gg >> 1) & 1, abort))) break;
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_addr + kTmS0 + sb * 128;
        // all scores of the tile in registers (one TMEM pass)
        // visible columns of this row form one range [vlo, vhi) of the tile
        int vlo, vhi;
        if (tl.kind == kCompressed) {
          vlo = 0;
          vhi = min(tl.n, nc_row - tl.key0);
        } else {
          vlo = max(0, lo_row - tl.key0);
          vhi = min(tl.n, t - tl.key0 + 1);
        }
        const uint32_t vlen = vhi > vlo ? (uint32_t)(vhi - vlo) : 0u;
        const int npieces = (tl.n + 31) >> 5;
        // pass 1: row max of the raw scores (scale > 0 applies after); 32-column pieces,
        // the next piece's TMEM load in flight while this one is reduced
        float mx[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
        uint32_t cur[32], nxt[32];
        tmem_ld32(s_addr, cur);
        tmem_wait_ld();
#pragma unroll 1
        for (int q = 0; q < npieces; ++q) {
          if (q + 1 < npieces) tmem_ld32(s_addr + (q + 1) * 32, nxt);
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const bool in = (uint32_t)(q * 32 + e - vlo) < vlen;
            mx[e & 7] = fmaxf(mx[e & 7], in ? __uint_as_float(cur[e]) : -INFINITY);
          }
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) cur[e] = nxt[e];
        }
        const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                         p.scale_log2;
        const float mn = fmaxf(m, mt);
        float ref = m;
        float alpha = 1.f;
        bool rescale = false;
        if (m == -INFINITY) {
          ref = mn;
        } else if (mn > m + kRescaleThreshold) {
          ref = mn;
          alpha = fast_exp2(m - mn);
          rescale = true;
        }
        const float base = ref == -INFINITY ? 0.f : ref;
        // P = exp2(s * scale - ref) as a bf16 pair hi + lo (A of the two P.V products),
        // written over the score columns. The scores are re-read 32 columns at a time, the
        // next piece's load in flight while this one is converted; 16-key group k keeps hi
        // in columns [16k, 16k+8) and lo in [16k+8, 16k+16), so piece q lands on its own
        // columns, already read.
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
        tmem_ld32(s_addr, cur);
        tmem_wait_ld();
#pragma unroll 1
        for (int q = 0; q < npieces; ++q) {
          if (q + 1 < npieces) tmem_ld32(s_addr + (q + 1) * 32, nxt);
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c0 = q * 32 + 2 * e;
            const bool in0 = (uint32_t)(c0 - vlo) < vlen;
            const bool in1 = (uint32_t)(c0 + 1 - vlo) < vlen;
            const float p0 =
                in0 ? fast_exp2(fmaf(__uint_as_float(cur[2 * e]), p.scale_log2, -base)) : 0.f;
            const float p1 =
                in1 ? fast_exp2(fmaf(__uint_as_float(cur[2 * e + 1]), p.scale_log2, -base)) : 0.f;
            split_bf16x2(p0, p1, pk[(e & 8) * 2 + (e & 7)], pk[(e & 8) * 2 + 8 + (e & 7)]);
            ps[e & 3] += p0 + p1;
          }
          tmem_st32(s_addr + q * 32, pk);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) cur[e] = nxt[e];
        }
        l = l * alpha + (ps[0] + ps[1]) + (ps[2] + ps[3]);
        m = ref;
        // Observe the completion of the previous P.V (of this item, or the previous item's
        // last one). Every o_done phase is consumed in order: a parity wait is exact only
        // while the barrier is at most one phase away. A rescale of O must not race it.
        if (gg > 0) {
          if (!(ok = mbar_wait(&bars->o_done, (gg - 1) & 1, abort))) break;
          tc_fence_after();
        }
        // rescale O (all lanes of the warp take part in the TMEM round trip)
        if (__any_sync(0xffffffffu, rescale) && j > 0) {
          const uint32_t o_addr = tmem + lane_addr + kTmO;
#pragma unroll 1
          for (int q = 0; q < kDH / 32; ++q) {
            uint32_t o[32];
            tmem_ld32(o_addr + q * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(o_addr + q * 32, o);
          }
        }
        if (j == it.ntiles - 1) {
          // hand the row sum to the epilogue warps; LSE and the debug mask go out here
          sL[(nitem & 1) * kBM + row] = l;
          if (row_valid && it.half == 0) {
            const int64_t orow = ((int64_t)it.b * p.T + tq) * p.hq + h;
            if (p.lse) p.lse[orow] = (m + __log2f(l)) * 0.69314718055994531f;
            if (p.dbg && h == 0) {
              int32_t* dp = p.dbg + ((int64_t)it.b * p.T + tq) * 3;
              dp[0] = nc_row;
              dp[1] = lo_row;
              dp[2] = t;
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->l_full[nitem & 1]);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[sb]);
      }
      g += it.ntiles;
      ++nitem;
    }
    if (!ok) raise_timeout(p, bars, 4);
  } else if (warp >= 6 && warp < 10) {
    // ------------------------------------------------------------------ epilogue
    // O half / l (* gate) -> bf16, overlapping the next item's softmax
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint64_t pol_stream = policy_evict_first();
    int nitem = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int k = cta_item(r, G, c);
      if (k >= p.n_items) break;
      const Item it = make_item(p, k);
      const int pos = it.t0 + row / p.hq;
      const int h = row % p.hq;
      const bool row_valid = pos < p.T;
      const int t = min(pos, p.T - 1);
      if (!(ok = mbar_wait(&bars->o_final, nitem & 1, abort))) break;
      if (!(ok = mbar_wait(&bars->l_full[nitem & 1], (nitem >> 1) & 1, abort))) break;
      tc_fence_after();
      const float inv = 1.f / sL[(nitem & 1) * kBM + row];
      const int64_t orow = ((int64_t)it.b * p.T + t) * p.hq + h;
      __nv_bfloat16* op = p.O + orow * kD + it.half * kDH;
      const __nv_bfloat16* gp =
          p.gate ? p.gate + (int64_t)it.b * p.gs0 + (int64_t)t * p.gs1 + (int64_t)h * p.gs2 +
                       it.half * kDH
                 : nullptr;
      const uint32_t o_addr = tmem + lane_addr + kTmO;
#pragma unroll 1
      for (int q = 0; q < kDH / 32; ++q) {
        uint4 gv[4];
        if (gp) {
#pragma unroll
          for (int w = 0; w < 4; ++w) gv[w] = ld_stream_hint(gp + q * 32 + w * 8, pol_stream);
        }
        uint32_t v[32];
        tmem_ld32(o_addr + q * 32, v);
        tmem_wait_ld();
        float o[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(v[e]) * inv;
        if (gp) {
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv[w]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(g2[e]);
              o[w * 8 + 2 * e] *= f.x;
              o[w * 8 + 2 * e + 1] *= f.y;
            }
          }
        }
        if (row_valid) {
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint4 pk;
            pk.x = pack_bf16x2(o[w * 8 + 0], o[w * 8 + 1]);
            pk.y = pack_bf16x2(o[w * 8 + 2], o[w * 8 + 3]);
            pk.z = pack_bf16x2(o[w * 8 + 4], o[w * 8 + 5]);
            pk.w = pack_bf16x2(o[w * 8 + 6], o[w * 8 + 7]);
            st_stream_hint(op + q * 32 + w * 8, pk, pol_stream);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->o_free);
      ++nitem;
    }
    if (!ok) raise_timeout(p, bars, 5);
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

bool prefill_tc_supported(const hca_desc& d, const hca_cache& c) {
  if (d.dtype != HCA_BF16 || d.head_dim != kD || d.hkv != 1) return false;
  if (d.hq < 8 || d.hq > 128 || (128 % d.hq) != 0) return false;
  if (d.window < 1 || d.window > 128 || d.block < 1) return false;
  if (c.page_entries % kBN != 0) return false;
  // TMA row coordinates and row indices are 32-bit
  if ((int64_t)d.batch * d.seqlen * d.hq >= (int64_t(1) << 31)) return false;
  if ((int64_t)c.num_pages * c.page_entries >= (int64_t(1) << 31)) return false;
  if (d.gate) {
    const uintptr_t ga = reinterpret_cast<uintptr_t>(d.gate);
    if (ga % 16 || d.gate_strides[0] % 8 || d.gate_strides[1] % 8 || d.gate_strides[2] % 8)
      return false;
  }
  return true;
}

cudaError_t launch_prefill_tc(const hca_desc& d, const void* Q, const void* K, const void* V,
                              const hca_cache& c, void* O, float* lse, int32_t* dbg_mask,
                              const PrefillRange& r, cudaStream_t s) {
  Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t rowsQ = (uint64_t)d.batch * d.seqlen * d.hq;
  const uint64_t rowsK = (uint64_t)d.batch * r.kv_len;
  const uint64_t rowsC = (uint64_t)c.num_pages * c.page_entries;
  cudaError_t e;
  if ((e = encode_bf16_chunks(&p.tmQ, Q, rowsQ, kBM, 2)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmK, K, rowsK, kBN, 2)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmV, V, rowsK, kBN, 2)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmK16, K, rowsK, 16, 8)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmV16, V, rowsK, 16, 4)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmKc, c.kc_pool, rowsC, kBN, 2)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmVc, c.vc_pool, rowsC, kBN, 2)) != cudaSuccess) return e;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.dbg = dbg_mask;
  p.gate = static_cast<const __nv_bfloat16*>(d.gate);
  p.gs0 = d.gate_strides[0];
  p.gs1 = d.gate_strides[1];
  p.gs2 = d.gate_strides[2];
  p.page_table = c.page_table;
  p.n_entries = c.n_entries;
  p.err_word = c.err_word;
  p.batch = d.batch;
  p.T = d.seqlen;
  p.q0 = r.q_pos0;
  p.kv0 = r.kv_pos0;
  p.Tk = r.kv_len;
  p.hq = d.hq;
  p.P = kBM / d.hq;
  p.W = d.window;
  p.block = d.block;
  p.PE = c.page_entries;
  p.max_pages = c.max_pages;
  p.num_pages = c.num_pages;
  p.n_rt = (d.seqlen + p.P - 1) / p.P;
  p.n_items = 2 * d.batch * p.n_rt;
  p.scale_log2 = d.scale * 1.4426950408889634f;
  if (p.n_items == 0) return cudaSuccess;
  static PerDevice<int> smem_limit_set;
  if ((e = set_smem_limit_once(smem_limit_set, (const void*)prefill_tc_kernel, (int)kSmemBytes)) !=
      cudaSuccess)
    return e;
  const int grid = min(p.n_items / 2, device_sm_count());  // row tiles (pairs of items)
  prefill_tc_kernel<<<grid, kThreads, kSmemBytes, s>>>(p);
  return cudaGetLastError();
}

}  // namespace hca
