// The packed key sequence of a query block's work list, shared by the
// tensor-core attention kernels (forward and backward).
//
// Method: the "decoupled block-tile" design in the abstract of "PSA: Pyramid
// Sparse Attention for Efficient Video Understanding and Generation": a query
// block's kept KV blocks are 64, 32, 16 or 8 pooled rows depending on their
// level; the work list orders them by level (then block index), and
// consecutive entries are packed into fixed 128-key tiles.  Sizes are powers
// of two in decreasing order, so no entry crosses a tile edge.
#pragma once

#include "psa_internal.cuh"

namespace psa {
namespace tile {

constexpr int kTileKeys = 128;           // keys per packed tile
constexpr int kListCache = 1024;         // work-list entries staged in shared memory

// Per query block: entry counts per level give where each level starts in
// the entry list (f1..f4) and in the packed key sequence (b1..b4).  Kept in
// scalars (no arrays) so that lookups by a run-time level stay in registers.
struct RowWork {
  int f1, f2, f3, f4;       // first entry of level 1, 2, 3; number of entries
  int b1, b2, b3, b4;       // first packed key of level 1, 2, 3; number of keys
  int tiles;
};

__device__ __forceinline__ RowWork row_work(int4 c) {
  RowWork w;
  w.f1 = c.x;
  w.f2 = w.f1 + c.y;
  w.f3 = w.f2 + c.z;
  w.f4 = w.f3 + c.w;
  w.b1 = 64 * c.x;
  w.b2 = w.b1 + 32 * c.y;
  w.b3 = w.b2 + 16 * c.z;
  w.b4 = w.b3 + 8 * c.w;
  w.tiles = (w.b4 + kTileKeys - 1) / kTileKeys;
  return w;
}

__device__ __forceinline__ int sel4(int l, int a0, int a1, int a2, int a3) {
  return l == 0 ? a0 : (l == 1 ? a1 : (l == 2 ? a2 : a3));
}

// The entries of tile t, one per lane: lane i takes the tile's first entry + i.
// Entries never cross a tile edge, so the lanes inside the tile form a prefix.
struct TileEntry {
  bool in_tile;
  int j, l, R, r0;          // KV block, level, sub-block rows, first row in the tile
};

__device__ __forceinline__ TileEntry tile_entry(const RowWork& w, const int* lrow,
                                                const int* lcache, int t, int lane) {
  // first entry of tile t: packed offset 128*t is always an entry boundary
  const int off0 = t * kTileKeys;
  const int l0 = (off0 >= w.b1) + (off0 >= w.b2) + (off0 >= w.b3);
  const int e = sel4(l0, 0, w.f1, w.f2, w.f3) + ((off0 - sel4(l0, 0, w.b1, w.b2, w.b3)) >> (6 - l0)) +
                lane;
  TileEntry te;
  const int l = (e >= w.f1) + (e >= w.f2) + (e >= w.f3);
  te.l = l;
  te.R = 64 >> l;
  const int off = sel4(l, 0, w.b1, w.b2, w.b3) + ((e - sel4(l, 0, w.f1, w.f2, w.f3)) << (6 - l));
  te.in_tile = e < w.f4 && off < (t + 1) * kTileKeys;
  te.r0 = off - t * kTileKeys;
  te.j = te.in_tile ? (e < kListCache ? lcache[e] : __ldg(lrow + e)) : 0;
  return te;
}

// The query blocks (items, (b * Hq + h) * Nq + a) a persistent CTA c of G
// processes, band by band: band j holds positions [j G, j G + G).  Without
// causality every row costs about the same, and CTA c takes position j G + c
// = the item itself, so that consecutive CTAs work on consecutive query
// blocks of a head while its K/V stay in L2.  Causally, row a keeps about
// a + 1 blocks' worth of keys: positions are dealt in a snake (band j goes
// c or G - 1 - c alternately) and position p is query block Nq - 1 - p / BH
// of head p % BH, so every band holds rows of about the same length and the
// bands go from the longest rows to the shortest.  Every role of a CTA walks
// the same sequence.
struct Schedule {
  int G, c, n, Nq, BH;
  bool causal;
  __device__ __forceinline__ int bands() const { return (n + G - 1) / G; }
  // the item of band j, or -1 where the band has none for this CTA
  __device__ __forceinline__ int item(int j) const {
    if (!causal) {
      const int k = j * G + c;
      return k < n ? k : -1;
    }
    const int pos = j * G + ((j & 1) ? G - 1 - c : c);
    if (pos >= n) return -1;
    return (pos % BH) * Nq + (Nq - 1 - pos / BH);
  }
};

__device__ __forceinline__ Schedule make_schedule(int n_items, int Nq, bool causal) {
  Schedule s;
  s.G = gridDim.x;
  s.c = blockIdx.x;
  s.n = n_items;
  s.Nq = Nq;
  s.BH = n_items / Nq;
  s.causal = causal;
  return s;
}

}  // namespace tile
}  // namespace psa
