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

}  // namespace tile
}  // namespace psa
