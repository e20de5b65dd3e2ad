// decode_keys.cuh -- the key list of one decode query and its cut into splits and tiles,
// shared by the 16-bit and the 8-bit decode kernels.
//
// The query is the newest token t = ctx_len - 1 of a sequence ([news 二.1] in
// include/hca.h). Its keys are the visible compressed entries j < n_c(t) (of which a call
// takes [e0, e1)), then the raw window when the call includes it. The list is walked in
// tiles of 128 keys: compressed tiles of 128 entries from e0 (only the one holding e1 - 1
// may be shorter), then one ring tile; `nsplit` splits take contiguous runs of tiles.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "sm100.cuh"

namespace hca {
namespace dkeys {

constexpr int kTN = 128;  // keys per tile (compressed or ring)

enum { kCompressed = 0, kRing = 1 };

struct Seq {
  int t, nc;      // query position, visible compressed entries
  int e0, e1;     // compressed entries of the call's part, [e0, e1)
  int nct, total, j0, j1;  // tiles [j0, j1) belong to this split
};

struct Tile {
  int kind, key0, n;
};

__device__ __forceinline__ int round16(int x) { return (x + 15) & ~15; }

// P: any parameter block with ctx_len, n_entries, seqlen, W, block, PE, max_pages, e0, e1
// and with_ring; the sequence's key list is cut into nsplit splits.
template <typename P>
__device__ __forceinline__ Seq make_seq_n(const P& p, int b, int split, int nsplit) {
  Seq s;
  // ctx_len is clamped into [1, seqlen]: the host sized the splits (and with them the TMEM
  // columns a split's scores take) for seqlen
  const int ctx = p.ctx_len[b];
  s.t = min(max(ctx, 1), p.seqlen) - 1;
  int x = s.t + 1 - p.W;
  int nc = x < 0 ? 0 : x / p.block;
  s.nc = min(nc, min(p.n_entries[b], p.max_pages * p.PE));
  s.e0 = min(p.e0, s.nc);
  s.e1 = max(s.e0, min(p.e1, s.nc));
  s.nct = (s.e1 - s.e0 + kTN - 1) / kTN;
  s.total = s.nct + (p.with_ring ? 1 : 0);
  const int tps = (s.total + nsplit - 1) / nsplit;
  s.j0 = min(s.total, split * tps);
  s.j1 = min(s.total, s.j0 + tps);
  return s;
}

template <typename P>
__device__ __forceinline__ Seq make_seq(const P& p, int b, int split) {
  return make_seq_n(p, b, split, p.nsplit);
}

template <typename P>
__device__ __forceinline__ Tile tile_of(const P& p, const Seq& s, int j) {
  Tile t;
  if (j < s.nct) {
    t.kind = kCompressed;
    t.key0 = s.e0 + j * kTN;
    t.n = min(kTN, round16(s.e1 - t.key0));
  } else {
    t.kind = kRing;
    t.key0 = 0;
    t.n = round16(p.W);
  }
  return t;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t row, int32_t chunk,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(row), "r"(chunk),
      "l"(policy)
      : "memory");
}

// The new token's row (one KV head of 512 bf16 values: 64 16-byte units) into ring slot
// t % W of sequence b, written by the calling thread, followed by a proxy fence so that the
// bulk-tensor loads this thread issues afterwards read it. P: a parameter block with W.
template <typename P>
__device__ __forceinline__ void append_ring_row(const P& p, const uint4* src, uint4* ring, int b,
                                                int t) {
  const int64_t slot = t % p.W;
  const uint4* s = src + (int64_t)b * 64;
  uint4* d = ring + ((int64_t)b * p.W + slot) * 64;
#pragma unroll 8
  for (int i = 0; i < 64; ++i) d[i] = s[i];
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

}  // namespace dkeys
}  // namespace hca
