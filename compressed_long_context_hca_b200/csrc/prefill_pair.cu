// prefill_pair.cu -- HCA prefill attention on pairs of SMs: tcgen05 2-CTA UMMA
// (cta_group::2), bf16 in, f32 accumulate.
//
// Operation ([news 二.1] / [analysis 1] / [gate] in include/hca.h): every query position t
// attends with one softmax to the compressed entries j < n_c(t) (blocks that end before its
// window) and to the raw tokens max(0, t-W+1) .. t, head_dim 512; the output is optionally
// multiplied by a supplied gate.
//
// Design for sm_100a:
//  * A cluster of two CTAs on two SMs drives one 2-SM UMMA stream. A work item is a pair row
//    tile of 256 rows: CTA rank r holds the 128 rows (128 / hq consecutive positions x hq
//    heads) of the r-th half in its shared memory (Q) and TMEM (scores, output). All rows
//    share the single KV head.
//  * The 2-SM UMMA splits its B operand between the two CTAs along N. For S = Q K^T each
//    CTA loads half of the keys of a K tile; for O += P V each CTA loads V for its half of
//    the output columns. Each SM thus streams half of every K and V tile that a one-CTA
//    kernel streams, and that stream (from L2, where the window and the compressed cache
//    stay) is what bounds the one-CTA kernel.
//  * TMEM per CTA: one 256-column output half and two 128-column score buffers, as in the
//    one-CTA kernel; the two output halves of a pair row tile are two items run back to
//    back, the second on the Q tiles already resident.
//  * The key list of an item is the union over its positions: compressed tiles of up to
//    128 entries (the last cut to a multiple of 16), a 16-key raw tile when the earliest
//    positions see keys beyond the last 128, and one raw tile of up to 128 keys ending at
//    the last position. Each row masks its own visible range.
//  * Roles per CTA: warps 0 and 10 K/V TMA (taking turns), warp 11 Q TMA, warp 1 UMMA issue
//    (the leader CTA; the peer's warp 1 only shares the TMEM allocation), warps 2-5 online
//    softmax (TMEM lane = row), warps 6-9 the epilogue (O / l, gate, bf16). The peer's TMA
//    loads complete on the leader's barriers; the leader's UMMA commits arrive on the same
//    barrier of both CTAs; the peer's softmax and epilogue warps arrive on the leader's.
//  * P is carried as two bf16 parts, P = P_hi + P_lo (P_lo the bf16 of the remainder), and
//    O += P.V runs as two TS-UMMAs per 16-key group, one per part: a peaked softmax (a few
//    keys of large, far-apart values) then loses ~2^-17 of the value spread to the rounding
//    of P instead of 2^-9 with one bf16 P.
//  * One UMMA stream across items: S of tile g, then P.V of tile g-1. The softmax hands
//    P(g) over before it observes the completion of P.V(g-1) unless O must be rescaled
//    (lazy rescale: only when the row max grows by more than 2^8), so P.V(g) queues behind
//    P.V(g-1) instead of waiting for a round trip through the softmax warps. The epilogue
//    hands O back as soon as its last TMEM piece is in registers.
//  * Every mbarrier wait is bounded; on time-out a CTA raises HCA_ERR_TIMEOUT (4) and
//    unwinds. Both CTAs leave through one cluster barrier, after the leader's last UMMA has
//    completed, so neither's shared memory or TMEM goes away while the other can reach it.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <string.h>

#include "hca_internal.h"
#include "sm100.cuh"
#include "tmap.h"

namespace hca {
namespace {

constexpr int kBM = 128;         // rows per CTA
constexpr int kD = 512;          // head_dim
constexpr int kDH = 256;         // output half per item
constexpr int kNCh = kD / 64;    // 8 chunks of 64 elements (128 bytes)
constexpr int kBN = 128;         // max keys per tile (both CTAs together)
constexpr uint32_t kSlotBytes = 32768;
// per-CTA boxes (3-D {64 elements, rows, chunks}, 128-byte swizzle, chunk-major in smem)
constexpr uint32_t kKChunk = 64 * 128;      // K of a 128-key tile: 64 keys x 4 chunks per slot
constexpr uint32_t kKBox = 4 * kKChunk;     // 32 KB
constexpr uint32_t kVChunk = 128 * 128;     // V of a 128-key tile: 128 keys x 2 chunks
constexpr uint32_t kVBox = 2 * kVChunk;     // 32 KB
constexpr uint32_t kK8Chunk = 8 * 128;      // K of the 16-key tile: 8 keys x 8 chunks
constexpr uint32_t kK8Box = kNCh * kK8Chunk;  // 8 KB
constexpr uint32_t kV16Chunk = 16 * 128;    // V of the 16-key tile: 16 keys x 2 chunks
constexpr uint32_t kV16Box = 2 * kV16Chunk;   // 4 KB
constexpr int kStages = 3;
constexpr int kQPairs = 4;                  // Q loaded as 4 boxes of two chunks
constexpr uint32_t kQChunk = kBM * 128;     // 16 KB
constexpr uint32_t kQBytes = kNCh * kQChunk;  // 128 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmS0 = 0, kTmO = 256;
constexpr int kThreads = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr uint16_t kPairMask = 0x3;

static_assert(kKBox == kSlotBytes && kVBox == kSlotBytes, "ring slot holds one box");

enum TileKind { kCompressed = 0, kRaw16 = 1, kRaw128 = 2 };

struct Params {
  CUtensorMap tmQ, tmK, tmV, tmK8, tmV16, tmKc, tmVc;
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
  int32_t o32;      // O is 32-byte aligned: the epilogue stores 32 bytes per lane
  int32_t n_pt;     // pair row tiles per sequence (2 P positions each)
  int32_t n_items;  // 2 * batch * n_pt
  float scale_log2;
};

struct Item {
  int b, half;
  int t0, tl;   // first query row, last valid query row of the pair row tile
  int nc_last;  // compressed entries visible to the last position (clamped)
  int nct;      // compressed tiles
  int lo, hi;   // raw key range of the pair row tile (positions)
  int rawA_n;   // keys of the last raw tile
  int strag;    // 1 if the 16-key raw tile exists
  int ntiles;
};

struct Tile {
  int kind;
  int n;     // keys (MMA N, both CTAs), multiple of 16
  int key0;  // first key: compressed entry or raw token
};

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

__device__ __forceinline__ int visible_count(int t, int block, int W) {
  const int x = t + 1 - W;
  return x < 0 ? 0 : x / block;
}

// The r-th item of cluster c: pair row tiles are dealt out in a snake over the clusters,
// and a cluster takes both output halves of one pair row tile back to back.
__device__ __forceinline__ int cluster_item(int r, int G, int c) {
  const int rr = r >> 1;
  const int idx = rr * G + ((rr & 1) ? (G - 1 - c) : c);
  return 2 * idx + (r & 1);
}

__device__ __forceinline__ Item make_item(const Params& p, int k) {
  Item it;
  it.half = k & 1;
  const int pt = k >> 1;
  it.b = pt % p.batch;
  const int i = p.n_pt - 1 - pt / p.batch;  // heaviest tiles first
  it.t0 = i * 2 * p.P;
  it.tl = min(it.t0 + 2 * p.P - 1, p.T - 1);
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
  } else if (it.strag && j == it.nct) {
    t.kind = kRaw16;
    t.key0 = it.hi - kBN - 15;
    t.n = 16;
  } else {
    t.kind = kRaw128;
    t.n = it.rawA_n;
    t.key0 = it.hi - it.rawA_n + 1;
  }
  return t;
}

// K slots of a tile per CTA: 2 boxes of 4 chunks (128-key kinds) or 1 box of all 8 chunks
// (16-key kind); V: one box of this CTA's two chunks.
__device__ __forceinline__ int k_slots(const Tile& t) { return t.kind == kRaw16 ? 1 : 2; }

// Shared-memory carve-up (offsets from a 1024-byte aligned base; identical in both CTAs,
// which the 2-SM UMMA relies on: its descriptors name one offset for both).
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffRing = kQBytes;
constexpr uint32_t kOffBar = kOffRing + kStages * kSlotBytes;
constexpr uint32_t kOffL = kOffBar + 512;
constexpr uint32_t kSmemBytes = kOffL + 2 * kBM * 4 + 1024;

struct Bars {
  uint64_t q_full[kQPairs], q_empty[kQPairs];
  uint64_t ring_full[kStages], ring_empty[kStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_done[2];  // P.V of tiles of even / odd index
  uint64_t o_free, o_final, drain;
  uint64_t l_full[2];
  // leader only: where each load stream stopped issuing (see drain_loads), 4 K/V producers
  // (rank * 2 + parity) and 2 Q producers (rank), and the barrier they arrive on
  uint64_t stops_full;
  int32_t kv_stop[4];
  int32_t q_stop[2];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars) <= 512, "barrier block too large");

// ------------------------------------------------------------------------ cluster PTX
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// shared::cluster address of the same offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_rank(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// arrive on a barrier of either CTA (shared::cluster address). The TMEM data it hands over
// (P, or O read back) is ordered by tcgen05.wait::st / fence::before_thread_sync before it
// and fence::after_thread_sync after the wait, as for a local hand-off.
__device__ __forceinline__ void mbar_arrive_cl(uint32_t bar_cl) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cl) : "memory");
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr_cl, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr_cl), "r"(v) : "memory");
}
// arrive with release at cluster scope: a store to the other CTA's shared memory made
// before it is visible to whoever observes the phase
__device__ __forceinline__ void mbar_arrive_release_cl(uint32_t bar_cl) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cl)
               : "memory");
}
__device__ __forceinline__ void mbar_complete_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// A role gave up waiting: every role of both CTAs stops at its next wait.
__device__ __forceinline__ void raise_timeout(const Params& p, Bars* bars, int role) {
  bars->abort = 1;
  st_cluster_u32(map_rank(&bars->abort, cluster_rank() ^ 1u), 1u);
  if (p.err_word) atomicOr(p.err_word, kErrTimeout | (1 << (8 + role)));
}

// A load stream publishes, in the leader CTA, the first sequence number it did not issue.
__device__ __forceinline__ void publish_stop(Bars* bars, int32_t* slot, int32_t stop) {
  st_cluster_u32(map_rank(slot, 0), (uint32_t)stop);
  mbar_arrive_release_cl(map_rank(&bars->stops_full, 0));
}

// ------------------------------------------------------------------------ 2-SM tcgen05
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D (+)= A[smem] B[smem]^T over the pair: M = 256 (128 rows of A in each CTA), B split by N
__device__ __forceinline__ void umma2_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D (+)= A[tmem] B[smem]^T over the pair (A: 128 TMEM lanes of each CTA, 2 bf16 per column)
__device__ __forceinline__ void umma2_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive once on the barrier at this offset in both CTAs when the UMMAs issued so far are done
__device__ __forceinline__ void umma2_commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(kPairMask)
      : "memory");
}
__device__ __forceinline__ void umma2_commit_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Tiled 3-D TMA load into this CTA's shared memory whose completion is counted on a barrier
// of the leader CTA (bar_cl: shared::cluster address). No multicast.
__device__ __forceinline__ void tma_load_pair(void* dst, const CUtensorMap* map, uint32_t bar_cl,
                                              int32_t row, int32_t chunk, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cl), "r"(0), "r"(row), "r"(chunk),
      "l"(policy)
      : "memory");
}

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
// 32-byte store (ptr 32-byte aligned): each lane of an epilogue warp writes its own row, so
// a warp's store touches 32 rows; wider stores halve the instructions the LSU processes
__device__ __forceinline__ void st_stream_hint32(void* ptr, const uint32_t* v, uint64_t pol) {
  asm volatile(
      "st.global.L1::no_allocate.L2::cache_hint.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8}, %9;" ::"l"(
          ptr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "l"(pol)
      : "memory");
}

// Per-CTA bytes of K/V load n of cluster c: the producers' load sequence walked again (K of
// tile j of an item, then V of the tile before it, possibly of the previous item; the V of
// the very last tile closes the sequence). Returns 0 past the end.
__device__ uint32_t kv_load_bytes(const Params& p, int G, int c, int32_t n) {
  int32_t cnt = 0;
  Item pit;
  int pj = -1;
  auto v_bytes = [&](const Item& it, int j) { return tile_of(it, j).kind == kRaw16 ? kV16Box : kVBox; };
  for (int r = 0;; ++r) {
    const int k = cluster_item(r, G, c);
    if (k >= p.n_items) break;
    const Item it = make_item(p, k);
    for (int j = 0; j < it.ntiles; ++j) {
      const Tile t = tile_of(it, j);
      const int nk = k_slots(t);
      if (n < cnt + nk) return t.kind == kRaw16 ? kK8Box : kKBox;
      cnt += nk;
      if (pj >= 0) {
        if (n == cnt) return v_bytes(pit, pj);
        ++cnt;
      }
      pit = it;
      pj = j;
    }
  }
  if (pj >= 0 && n == cnt) return v_bytes(pit, pj);
  return 0;
}

// After a time-out (leader, one thread): wait, bounded, until every bulk load either CTA
// has issued has landed, so that neither CTA's shared memory goes away under a copy.
// The peer's loads complete on the leader's barriers, which the peer cannot wait on; each
// load stream published the first sequence number it did not issue (kv_stop, q_stop).
// A stream issues load n of a ring slot only after the slot's previous phase completed, so
// on each barrier at most its last issued load can be outstanding: n* = the largest issued
// sequence number on the slot, and no load after it exists, which keeps the parity wait
// exact. The leader armed 2 x the bytes of every load it issued: a half the peer never
// issued is completed by hand; a load only the peer issued is armed now.
__device__ void drain_loads(const Params& p, Bars* bars, int G, int c) {
  volatile int no_abort = 0;
  if (!mbar_wait(&bars->stops_full, 0, &no_abort, 3000000000ull)) return;
  // every stop is now visible (release arrives, acquire here)
  asm volatile("fence.acq_rel.cluster;" ::: "memory");
  const volatile int32_t* kv = bars->kv_stop;
  for (int s = 0; s < kStages; ++s) {
    int32_t nstar = -1;
    for (int cm = 0; cm < 4; ++cm) {  // stream (rank cm / 2, parity cm % 2)
      for (int32_t n = kv[cm] - 1; n >= 0 && n >= kv[cm] - 6; --n)
        if ((n & 1) == (cm & 1) && n % kStages == s) {
          nstar = max(nstar, n);
          break;
        }
    }
    if (nstar < 0) continue;
    const bool L = nstar < kv[0 * 2 + (nstar & 1)];
    const bool P = nstar < kv[1 * 2 + (nstar & 1)];
    const uint32_t b = kv_load_bytes(p, G, c, nstar);
    if (L && !P) mbar_complete_tx(&bars->ring_full[s], b);
    if (!L && P) mbar_expect_tx(&bars->ring_full[s], b);
    mbar_wait(&bars->ring_full[s], (uint32_t)(nstar / kStages) & 1, &no_abort, 100000000ull);
  }
  // Q: box q of walked item r is sequence number 4 r + q; only even items load (odd ones
  // reuse the tile and only the leader arrives, without bytes)
  const volatile int32_t* qs = bars->q_stop;
  for (int q = 0; q < kQPairs; ++q) {
    int r0 = -1, r1 = -1;
    if (qs[0] > q) r0 = (qs[0] - 1 - q) / kQPairs;
    if (qs[1] > q) r1 = (qs[1] - 1 - q) / kQPairs;
    const int rstar = max(r0, r1);
    if (rstar < 0 || (rstar & 1)) continue;
    const bool L = rstar <= r0, P = rstar <= r1;
    if (L && !P) mbar_complete_tx(&bars->q_full[q], kSlotBytes);
    if (!L && P) mbar_expect_tx(&bars->q_full[q], kSlotBytes);
    mbar_wait(&bars->q_full[q], (uint32_t)rstar & 1, &no_abort, 100000000ull);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_pair_kernel(const __grid_constant__ Params p) {
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
  const uint32_t rank = cluster_rank();  // 0: leader (issues the UMMAs), 1: peer
  const bool leader = rank == 0;

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
      mbar_init(&bars->p_full[s], 8);  // 4 softmax warps of each CTA (leader's barrier)
    }
    mbar_init(&bars->o_done[0], 1);
    mbar_init(&bars->o_done[1], 1);
    mbar_init(&bars->o_free, 8);  // 4 epilogue warps of each CTA (leader's barrier)
    mbar_init(&bars->o_final, 1);
    mbar_init(&bars->l_full[0], 4);
    mbar_init(&bars->l_full[1], 4);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->stops_full, 6);  // 4 K/V producers and 2 Q producers of the pair
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmQ);
    tma_prefetch_desc(&p.tmK);
    tma_prefetch_desc(&p.tmV);
    tma_prefetch_desc(&p.tmK8);
    tma_prefetch_desc(&p.tmV16);
    tma_prefetch_desc(&p.tmKc);
    tma_prefetch_desc(&p.tmVc);
  }
  if (warp == 1) {
    // one warp of each CTA, same warp index and destination offset in both
    tmem_alloc_pair(&bars->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int G = (int)cluster_count();
  const int c = (int)cluster_id();

  if (warp == 0 || warp == 10) {
    // ------------------------------------------------------------------ K/V TMA producers
    // Two producer warps per CTA walk the same load sequence and take turns (even / odd
    // loads); both CTAs walk the same sequence, the order the UMMA warp consumes: K of
    // tile g, then V of tile g-1. Each CTA loads its own half of every box; the leader's
    // producer announces the bytes of both halves on its barrier.
    if (elect_one()) {
      const uint32_t mine = warp == 0 ? 0u : 1u;
      const uint64_t pol_kv = policy_evict_last();
      uint32_t full_cl[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) full_cl[s] = map_rank(&bars->ring_full[s], 0);
      uint32_t cnt = 0;  // ring loads in the sequence so far (both producers)
      bool ok = true;
      // returns the slot to fill, -2 when the other producer owns this load, -1 on time-out
      auto next_slot = [&](uint32_t bytes) -> int {
        const uint32_t n = cnt++;
        if ((n & 1u) != mine) return -2;
        const uint32_t s = n % kStages;
        const uint32_t round = n / kStages;
        if (round > 0 && !mbar_wait(&bars->ring_empty[s], (round - 1) & 1, abort)) return -1;
        if (leader) mbar_expect_tx(&bars->ring_full[s], 2 * bytes);
        return (int)s;
      };
      auto load_tile = [&](const Item& it, int j, bool is_v) -> bool {
        const Tile t = tile_of(it, j);
        // first row of the tile in the source array
        int row0;
        const CUtensorMap* mk;
        const CUtensorMap* mv;
        if (t.kind == kCompressed) {
          int page = p.page_table[(int64_t)it.b * p.max_pages + t.key0 / p.PE];
          if (page < 0 || page >= p.num_pages) {
            if (p.err_word) atomicOr(p.err_word, kErrPageRange);
            page = 0;
          }
          row0 = page * p.PE + (t.key0 % p.PE);
          mk = &p.tmKc;
          mv = &p.tmVc;
        } else {
          row0 = it.b * p.Tk + t.key0 - p.kv0;
          mk = &p.tmK;
          mv = &p.tmV;
        }
        if (is_v) {
          // all keys of the tile, this CTA's two of the half's four chunks
          const bool small = t.kind == kRaw16;
          const int s = next_slot(small ? kV16Box : kVBox);
          if (s == -1) return false;
          if (s >= 0)
            tma_load_pair(sRing + s * kSlotBytes, small ? &p.tmV16 : mv, full_cl[s], row0,
                          it.half * 4 + 2 * (int)rank, pol_kv);
          return true;
        }
        if (t.kind == kRaw16) {
          // keys [8 rank, 8 rank + 8) of the 16, all 8 chunks
          const int s = next_slot(kK8Box);
          if (s == -1) return false;
          if (s >= 0)
            tma_load_pair(sRing + s * kSlotBytes, &p.tmK8, full_cl[s], row0 + 8 * (int)rank, 0,
                          pol_kv);
          return true;
        }
        // keys [n/2 rank, n/2 rank + n/2) of the tile (a 64-key box), chunks 4q .. 4q+3
        for (int q = 0; q < 2; ++q) {
          const int s = next_slot(kKBox);
          if (s == -1) return false;
          if (s >= 0)
            tma_load_pair(sRing + s * kSlotBytes, mk, full_cl[s], row0 + (t.n >> 1) * (int)rank,
                          4 * q, pol_kv);
        }
        return true;
      };
      Item pit;
      int pj = -1;
      for (int r = 0; ok; ++r) {
        const int k = cluster_item(r, G, c);
        if (k >= p.n_items) break;
        const Item it = make_item(p, k);
        if (leader && mine == 0 && p.err_word &&
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
      if (!ok) raise_timeout(p, bars, 1);
      // every sequence number of this producer's parity below the stop was issued; the one
      // whose slot wait failed (cnt - 1) was not. The leader waits for what is in flight
      // (drain_loads) before either CTA leaves.
      publish_stop(bars, &bars->kv_stop[rank * 2 + mine], (int32_t)(ok ? cnt : cnt - 1));
    }
  } else if (warp == 11) {
    // ------------------------------------------------------------------ Q TMA producer
    // Q of an item: 4 boxes of two chunks of this CTA's 128 rows, each reloaded once the
    // previous item's last score UMMA on it has finished. The second output half of a pair
    // row tile has the same Q: the leader only hands the boxes over again.
    if (elect_one()) {
      const uint64_t pol_q = policy_evict_first();
      uint32_t qfull_cl[kQPairs];
#pragma unroll
      for (int q = 0; q < kQPairs; ++q) qfull_cl[q] = map_rank(&bars->q_full[q], 0);
      int nitem = 0;
      int32_t qstop = 0;  // boxes walked (item-major, 4 per item), then the first not issued
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int k = cluster_item(r, G, c);
        if (k >= p.n_items) break;
        const Item it = make_item(p, k);
        const int qrow = (it.b * p.T + it.t0 + (int)rank * p.P) * p.hq;
        const bool reuse = (r & 1) != 0;
        for (int q = 0; q < kQPairs && ok; ++q) {
          if (nitem > 0 && !(ok = mbar_wait(&bars->q_empty[q], (nitem - 1) & 1, abort))) break;
          ++qstop;
          if (reuse) {
            if (leader) mbar_arrive(&bars->q_full[q]);
          } else {
            if (leader) mbar_expect_tx(&bars->q_full[q], 2 * kSlotBytes);
            tma_load_pair(sQ + q * kSlotBytes, &p.tmQ, qfull_cl[q], qrow, 2 * q, pol_q);
          }
        }
        ++nitem;
      }
      if (!ok) raise_timeout(p, bars, 2);
      publish_stop(bars, &bars->q_stop[rank], qstop);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ UMMA issuer
    // The leader's thread issues every 2-SM UMMA of the pair; the peer's warp idles.
    if (leader && elect_one()) {
      uint32_t cnt = 0;  // ring slots consumed
      uint32_t g = 0;    // tiles processed (score buffer / phase counter)
      int nitem = 0;
      bool ok = true;
      const uint32_t rbase = smem_u32(sRing);
      const uint64_t qd0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      auto issue_s = [&](const Item& it, int j, uint32_t gg, int ni) -> bool {
        const Tile t = tile_of(it, j);
        const int last = it.ntiles - 1;
        const uint32_t sb = gg & 1;
        const uint32_t d_tmem = tmem + kTmS0 + sb * 128;
        const uint32_t idesc = idesc_bf16_f32(2 * kBM, t.n, false);
        const int nsl = k_slots(t);
        for (int q = 0; q < nsl; ++q) {
          // an item's first tile waits for its Q boxes slot by slot: a 64-key K slot reads Q
          // pairs 2q and 2q+1 only (the 16-key slot reads all four), so the first slot's MMAs
          // start while the later boxes of a new Q tile are still landing
          if (j == 0) {
            const int q0 = t.kind == kRaw16 ? 0 : 2 * q;
            const int q1 = t.kind == kRaw16 ? kQPairs : 2 * q + 2;
            for (int qq = q0; qq < q1; ++qq)
              if (!mbar_wait(&bars->q_full[qq], ni & 1, abort)) return false;
          }
          const uint32_t s = cnt % kStages;
          if (!mbar_wait(&bars->ring_full[s], (cnt / kStages) & 1, abort)) return false;
          tc_fence_after();
          // Descriptors are built once per slot and stepped by constant offsets (the start
          // address field is address >> 4; every shared address here is below 256 KB, so the
          // addition never carries out of the field).
          const uint64_t kd0 = sdesc_sw128(rbase + s * kSlotBytes, 16, 1024);
          if (t.kind == kRaw16) {
            // all 8 chunks of 8 keys in one slot
#pragma unroll
            for (int cc = 0; cc < kNCh; ++cc)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma2_ss(d_tmem, qd0 + ((cc * kQChunk + kk * 32) >> 4),
                         kd0 + ((cc * kK8Chunk + kk * 32) >> 4), idesc, (cc | kk) != 0);
          } else {
            // chunks 4q .. 4q+3 of 64 keys
            const uint64_t qdq = qd0 + ((uint32_t)(4 * q) * (kQChunk >> 4));
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma2_ss(d_tmem, qdq + ((cc * kQChunk + kk * 32) >> 4),
                         kd0 + ((cc * kKChunk + kk * 32) >> 4), idesc, (q | cc | kk) != 0);
          }
          umma2_commit_both(&bars->ring_empty[s]);
          if (j == last) {  // the last tile is a 128-key kind: slot q held Q pairs 2q, 2q+1
            umma2_commit_both(&bars->q_empty[2 * q]);
            umma2_commit_both(&bars->q_empty[2 * q + 1]);
          }
          ++cnt;
        }
        umma2_commit_both(&bars->s_full[sb]);
        return true;
      };
      auto issue_pv = [&](const Item& it, int j, uint32_t gg, int ni) -> bool {
        const Tile t = tile_of(it, j);
        const uint32_t sb = gg & 1;
        if (!mbar_wait(&bars->p_full[sb], (gg >> 1) & 1, abort)) return false;
        // the first P.V of an item overwrites O: both epilogues must have read the last one
        if (j == 0 && ni > 0 && !mbar_wait(&bars->o_free, (ni - 1) & 1, abort)) return false;
        tc_fence_after();
        const uint32_t a_tmem = tmem + kTmS0 + sb * 128;
        const uint32_t s = cnt % kStages;
        if (!mbar_wait(&bars->ring_full[s], (cnt / kStages) & 1, abort)) return false;
        tc_fence_after();
        // N = 256 output columns, 128 in each CTA (two chunks, N-major, chunk stride lbo);
        // 16 keys = two 8-row swizzle atoms = 2 KB of each chunk
        const uint32_t lbo = t.kind == kRaw16 ? kV16Chunk : kVChunk;
        const uint32_t idesc = idesc_bf16_f32(2 * kBM, kDH, true);
        const uint64_t vd0 = sdesc_sw128(rbase + s * kSlotBytes, lbo, 1024);
        const uint32_t acc0 = j > 0 ? 1u : 0u;
        // per 16-key group: O += P_hi V, then O += P_lo V (A columns 16 kk and 16 kk + 8)
        if (t.n == kBN) {
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            umma2_ts(tmem + kTmO, a_tmem + kk * 16, vd0 + kk * (2048 >> 4), idesc, acc0 | kk);
            umma2_ts(tmem + kTmO, a_tmem + kk * 16 + 8, vd0 + kk * (2048 >> 4), idesc, 1u);
          }
        } else {
          for (int kk = 0; kk < t.n / 16; ++kk) {
            umma2_ts(tmem + kTmO, a_tmem + kk * 16, vd0 + kk * (2048 >> 4), idesc, acc0 | kk);
            umma2_ts(tmem + kTmO, a_tmem + kk * 16 + 8, vd0 + kk * (2048 >> 4), idesc, 1u);
          }
        }
        umma2_commit_both(&bars->ring_empty[s]);
        ++cnt;
        umma2_commit_both(&bars->o_done[gg & 1]);
        if (j == it.ntiles - 1) umma2_commit_both(&bars->o_final);
        return true;
      };
      // One stream across items: S of tile g, then P.V of tile g-1 (possibly of the
      // previous item), so the tensor pipe keeps working over item boundaries.
      Item pit;
      int pj = -1, pni = 0;
      uint32_t pgg = 0;
      for (int r = 0; ok; ++r) {
        const int k = cluster_item(r, G, c);
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
      // drain: every UMMA issued above has finished before either CTA releases anything
      volatile int no_abort = 0;
      umma2_commit_local(&bars->drain);
      mbar_wait(&bars->drain, 0, &no_abort, 100000000ull);
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------------ softmax
    const int quad = warp & 3;         // TMEM lane quadrant of this warp
    const int row = quad * 32 + lane;  // row of this CTA == TMEM lane
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint32_t pfull_cl[2] = {map_rank(&bars->p_full[0], 0), map_rank(&bars->p_full[1], 0)};
    uint32_t g = 0;
    int nitem = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int k = cluster_item(r, G, c);
      if (k >= p.n_items) break;
      const Item it = make_item(p, k);
      const int pos = it.t0 + (int)rank * p.P + row / p.hq;
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
          // a piece is visible in full for most rows (every compressed tile, all but the
          // last piece of the raw tile): the masks are only applied where some lane needs them
          const int c0 = q * 32;
          if (__all_sync(0xffffffffu, c0 >= vlo && c0 + 32 <= vhi)) {
#pragma unroll
            for (int e = 0; e < 32; ++e) mx[e & 7] = fmaxf(mx[e & 7], __uint_as_float(cur[e]));
          } else if (!__all_sync(0xffffffffu, c0 >= vhi || c0 + 32 <= vlo)) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const bool in = (uint32_t)(c0 + e - vlo) < vlen;
              mx[e & 7] = fmaxf(mx[e & 7], in ? __uint_as_float(cur[e]) : -INFINITY);
            }
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
        // written over the score columns: 16-key group k of the tile keeps hi in columns
        // [16k, 16k+8) and lo in [16k+8, 16k+16), so piece q (keys 32q .. 32q+31) lands on
        // its own columns, already read
        float ps[4] = {0.f, 0.f, 0.f, 0.f};
        tmem_ld32(s_addr, cur);
        tmem_wait_ld();
#pragma unroll 1
        for (int q = 0; q < npieces; ++q) {
          if (q + 1 < npieces) tmem_ld32(s_addr + (q + 1) * 32, nxt);
          uint32_t pk[32];
          const int c0 = q * 32;
          if (__all_sync(0xffffffffu, c0 >= vlo && c0 + 32 <= vhi)) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const float p0 = fast_exp2(fmaf(__uint_as_float(cur[2 * e]), p.scale_log2, -base));
              const float p1 =
                  fast_exp2(fmaf(__uint_as_float(cur[2 * e + 1]), p.scale_log2, -base));
              split_bf16x2(p0, p1, pk[(e & 8) * 2 + (e & 7)], pk[(e & 8) * 2 + 8 + (e & 7)]);
              ps[e & 3] += p0 + p1;
            }
          } else if (__all_sync(0xffffffffu, c0 >= vhi || c0 + 32 <= vlo)) {
#pragma unroll
            for (int e = 0; e < 32; ++e) pk[e] = 0u;
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int cc = c0 + 2 * e;
              const bool in0 = (uint32_t)(cc - vlo) < vlen;
              const bool in1 = (uint32_t)(cc + 1 - vlo) < vlen;
              const float p0 =
                  in0 ? fast_exp2(fmaf(__uint_as_float(cur[2 * e]), p.scale_log2, -base)) : 0.f;
              const float p1 =
                  in1 ? fast_exp2(fmaf(__uint_as_float(cur[2 * e + 1]), p.scale_log2, -base))
                      : 0.f;
              split_bf16x2(p0, p1, pk[(e & 8) * 2 + (e & 7)], pk[(e & 8) * 2 + 8 + (e & 7)]);
              ps[e & 3] += p0 + p1;
            }
          }
          tmem_st32(s_addr + q * 32, pk);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) cur[e] = nxt[e];
        }
        l = l * alpha + (ps[0] + ps[1]) + (ps[2] + ps[3]);
        m = ref;
        // P.V(gg - 1) must be complete before O is rescaled. Without a rescale its completion
        // is observed after P(gg) is handed over, so P.V(gg) queues behind it on the tensor
        // pipe. Each of the two o_done barriers (tile parity) has its phases consumed in
        // order, and P.V(gg + 1), its next phase, cannot start before P(gg + 1) is handed over,
        // so every parity wait is exact.
        const bool rescale_o = __any_sync(0xffffffffu, rescale) && j > 0;
        if (rescale_o) {
          if (!(ok = mbar_wait(&bars->o_done[(gg - 1) & 1], ((gg - 1) >> 1) & 1, abort))) break;
          tc_fence_after();
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
        if (lane == 0) mbar_arrive_cl(pfull_cl[sb]);
        if (!rescale_o && gg > 0) {
          if (!(ok = mbar_wait(&bars->o_done[(gg - 1) & 1], ((gg - 1) >> 1) & 1, abort))) break;
        }
      }
      g += it.ntiles;
      ++nitem;
    }
    if (!ok) raise_timeout(p, bars, 4);
  } else if (warp >= 6 && warp < 10) {
    // ------------------------------------------------------------------ epilogue
    // O half / l (* gate) -> bf16 for this CTA's rows, overlapping the next item's softmax
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
    const uint64_t pol_stream = policy_evict_first();
    const uint32_t ofree_cl = map_rank(&bars->o_free, 0);
    int nitem = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int k = cluster_item(r, G, c);
      if (k >= p.n_items) break;
      const Item it = make_item(p, k);
      const int pos = it.t0 + (int)rank * p.P + row / p.hq;
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
      // 32-column pieces; the next piece's TMEM (and gate) loads are in flight while this
      // one is scaled, rounded and stored. O is handed back to the UMMA warp as soon as the
      // last piece is in registers.
      uint32_t cur[32], nxt[32];
      uint4 gcur[4], gnxt[4];
      tmem_ld32(o_addr, cur);
      if (gp) {
#pragma unroll
        for (int w = 0; w < 4; ++w) gcur[w] = ld_stream_hint(gp + w * 8, pol_stream);
      }
      tmem_wait_ld();
#pragma unroll 1
      for (int q = 0; q < kDH / 32; ++q) {
        const bool more = q + 1 < kDH / 32;
        if (more) {
          tmem_ld32(o_addr + (q + 1) * 32, nxt);
          if (gp) {
#pragma unroll
            for (int w = 0; w < 4; ++w)
              gnxt[w] = ld_stream_hint(gp + (q + 1) * 32 + w * 8, pol_stream);
          }
        }
        float o[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(cur[e]) * inv;
        if (gp) {
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gcur[w]);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(g2[e]);
              o[w * 8 + 2 * e] *= f.x;
              o[w * 8 + 2 * e + 1] *= f.y;
            }
          }
        }
        if (row_valid) {
          uint32_t pk[16];
#pragma unroll
          for (int w = 0; w < 16; ++w) pk[w] = pack_bf16x2(o[2 * w], o[2 * w + 1]);
          if (p.o32) {
            st_stream_hint32(op + q * 32, pk, pol_stream);
            st_stream_hint32(op + q * 32 + 16, pk + 8, pol_stream);
          } else {
#pragma unroll
            for (int w = 0; w < 4; ++w)
              st_stream_hint(op + q * 32 + w * 8,
                             make_uint4(pk[4 * w], pk[4 * w + 1], pk[4 * w + 2], pk[4 * w + 3]),
                             pol_stream);
          }
        }
        if (more) {
          tmem_wait_ld();
          if (q + 2 == kDH / 32) {
            // every TMEM read of this warp has completed
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cl(ofree_cl);
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) cur[e] = nxt[e];
#pragma unroll
          for (int w = 0; w < 4; ++w) gcur[w] = gnxt[w];
        }
      }
      ++nitem;
    }
    if (!ok) raise_timeout(p, bars, 5);
  }

  // both CTAs leave together: the leader's UMMAs (which read the peer's shared memory and
  // write its TMEM) have drained before either CTA passes this point. After a time-out the
  // leader first waits for the loads still in flight into either CTA (drain_loads); the
  // peer cannot pass the cluster barrier before the leader arrives.
  tc_fence_before();
  __syncthreads();
  if (leader && threadIdx.x == 0 && *abort) drain_loads(p, bars, G, c);
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// Clusters of two that fit on the device at once (one CTA per SM); 0 if the query fails.
int resident_pairs(cudaLaunchConfig_t cfg) {
  static PerDevice<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  int n = 0;
  if (cache.get(dev, &n)) return n;
  if (cudaOccupancyMaxActiveClusters(&n, (const void*)prefill_pair_kernel, &cfg) != cudaSuccess)
    return 0;
  if (n > 0) cache.put(dev, n);
  return n;
}

}  // namespace

bool prefill_pair_supported(const hca_desc& d, const hca_cache& c) {
  if (d.dtype != HCA_BF16 || d.head_dim != kD || d.hkv != 1) return false;
  // 2 P positions per pair row tile; the union window of 2 P - 1 + W keys must fit one
  // 128-key raw tile plus the 16-key one, so P <= 8
  if (d.hq < 16 || d.hq > 128 || (128 % d.hq) != 0) return false;
  if (d.window < 1 || d.window > 128 || d.block < 1) return false;
  if (c.page_entries % kBN != 0) return false;
  // TMA row coordinates and row indices are 32-bit; the peer's Q rows of the last pair row
  // tile may start up to 2 P positions past the end
  if (((int64_t)d.batch * d.seqlen + 2 * kBM) * d.hq >= (int64_t(1) << 31)) return false;
  if ((int64_t)c.num_pages * c.page_entries >= (int64_t(1) << 31)) return false;
  if (d.gate) {
    const uintptr_t ga = reinterpret_cast<uintptr_t>(d.gate);
    if (ga % 16 || d.gate_strides[0] % 8 || d.gate_strides[1] % 8 || d.gate_strides[2] % 8)
      return false;
  }
  return true;
}

cudaError_t launch_prefill_pair(const hca_desc& d, const void* Q, const void* K, const void* V,
                                const hca_cache& c, void* O, float* lse, int32_t* dbg_mask,
                                const PrefillRange& r, cudaStream_t s) {
  Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t rowsQ = (uint64_t)d.batch * d.seqlen * d.hq;
  const uint64_t rowsK = (uint64_t)d.batch * r.kv_len;
  const uint64_t rowsC = (uint64_t)c.num_pages * c.page_entries;
  cudaError_t e;
  if ((e = encode_bf16_chunks(&p.tmQ, Q, rowsQ, kBM, 2)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmK, K, rowsK, kBN / 2, 4)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmV, V, rowsK, kBN, 2)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmK8, K, rowsK, 8, kNCh)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmV16, V, rowsK, 16, 2)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmKc, c.kc_pool, rowsC, kBN / 2, 4)) != cudaSuccess) return e;
  if ((e = encode_bf16_chunks(&p.tmVc, c.vc_pool, rowsC, kBN, 2)) != cudaSuccess) return e;
  p.O = static_cast<__nv_bfloat16*>(O);
  p.o32 = (reinterpret_cast<uintptr_t>(O) % 32) == 0 ? 1 : 0;
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
  p.n_pt = (d.seqlen + 2 * p.P - 1) / (2 * p.P);
  p.n_items = 2 * d.batch * p.n_pt;
  p.scale_log2 = d.scale * 1.4426950408889634f;
  if (p.n_items == 0) return cudaSuccess;
  static PerDevice<int> smem_limit_set;
  if ((e = set_smem_limit_once(smem_limit_set, (const void*)prefill_pair_kernel, (int)kSmemBytes)) !=
      cudaSuccess)
    return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(2, 1, 1);
  int pairs = resident_pairs(cfg);
  if (pairs <= 0) pairs = device_sm_count() / 2;
  const int G = min(p.n_items / 2, pairs);  // pair row tiles (pairs of items) per launch
  cfg.gridDim = dim3(2 * G, 1, 1);
  e = cudaLaunchKernelEx(&cfg, prefill_pair_kernel, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace hca
