// Pyramid attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// bf16 inputs, fp32 accumulation, 128-row query blocks, d in {64, 128}.  A
// 64-row query block runs in the same 128-row tiles with rows 64-127 dead (no
// softmax, no stores): half the tensor work is wasted, against a CUDA-core
// kernel.
//
// Method: adaptive pyramid attention (top168.com article on PSA, component
// three: one probability distribution over all kept keys) with the paper's
// "decoupled block-tile" idea (abstract of "PSA: Pyramid Sparse Attention for
// Efficient Video Understanding and Generation"): the logical KV block of 64
// tokens is decoupled from the hardware tile.  A query block's kept blocks are
// 64, 32, 16 or 8 pooled rows depending on their level; the work list orders
// them by level, and consecutive entries are packed into fixed 128-key tiles
// (sizes are powers of two in decreasing order, so no entry crosses a tile).
// Each pooled key's logit gets + log2(c) (c = tokens it averages) so that it
// carries their softmax mass.
//
// Persistent CTAs (one per SM) walk the query blocks; 12 warps:
//   warp 0     TMA producer for Q and K: Q once per query block; per tile, one
//              2-D box per sub-block and 64-column half (the box height is the
//              level's sub-block height), plus the tile's key bias table.
//   warp 2     TMA producer for V, the same boxes into the V ring.
//   warp 1     TMEM allocator and single-thread tcgen05.mma issuer.
//   warps 4-7, 8-11   softmax, one warpgroup per stream.
// A query block's tiles alternate between two streams (even tiles, odd
// tiles), each with its own S buffer and O accumulator in TMEM and its own
// online softmax state, merged once at the end of the block (the two partial
// softmaxes over disjoint key sets combine exactly).  The warpgroups never
// wait for each other inside a block, so one computes exponentials while the
// other waits for or loads its scores, and the tensor pipe always has the
// other stream's QK^T or PV to run.  Per stream s and tile t (t = s mod 2):
//   S_s = Q K_t^T (SS form; Q and K in shared memory),
//   softmax(t): P_t = exp2(S_s * scale + bias - m_s), written over S_s (bf16),
//   O_s += P_t V_t (TS form, P from TMEM), then QK^T of tile t + 2 into S_s
//   (the in-order tensor pipe finishes PV(t) before it overwrites P_t).  At
//   d = 64 the products of keys [0, 64) are issued once their P is written,
//   while the softmax computes the exponentials of keys [64, 128).
// Each row's logits get + log2(c) of the pooled key's token count; the
// running maximum is rescaled lazily (only when it grows by more than 2^8).
// TMEM columns: S_0 [0,128) S_1 [128,256) O_0 [256,256+d) O_1 [256+d,256+2d).
// Every mbarrier wait is bounded: on expiry the kernel records a timeout in
// the workspace error word and winds down without trapping.
#include "psa_internal.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include "sm100_ptx.cuh"
#include "tile_walk.cuh"
#include "tma_host.cuh"

namespace psa {
namespace {

using namespace ptx;
using namespace tile;

constexpr int kBM = 128;                 // query rows per CTA
constexpr int kBN = kTileKeys;           // keys per packed tile
constexpr int kStreams = 2;              // softmax warpgroups, one per stream of tiles
constexpr int kVWarp = 2;                // the V producer
constexpr int kSoftWarp0 = 4;            // first softmax warp (warpgroup aligned)
constexpr int kThreads = 128 + 128 * kStreams;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;     // lazy rescale threshold (factor 256)

template <int D>
struct Cfg {
  static constexpr int HALVES = D / 64;
  static constexpr int KSTAGES = D == 128 ? 3 : 6;   // K ring (freed when QK^T completes)
  static constexpr int VSTAGES = D == 128 ? 2 : 4;   // V ring (freed when PV completes)
  static constexpr int MSTAGES = 4;                  // per-tile bias / position tables
  static constexpr int HALF = kBN * 128;             // bytes of one 64-column half tile
  static constexpr int Q_BYTES = kBM * D * 2;
  static constexpr int KV_BYTES = kBN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KSTAGES * KV_BYTES;
  static constexpr int OFF_META = OFF_V + VSTAGES * KV_BYTES;   // per table: bias[128], kpos[128]
  static constexpr int META_BYTES = 128 + 1024;                // chunk biases, flag, per-key tables
  static constexpr int OFF_BAR = OFF_META + MSTAGES * META_BYTES;
  static constexpr int OFF_XCH = OFF_BAR + 512;                 // stream 0's (max, sum): [2][128][2]
  static constexpr int OFF_LIST = OFF_XCH + 2 * 128 * 8;        // the query block's work list
  static constexpr int SMEM = OFF_LIST + 2 * kListCache * 4 + 1024;   // two list copies + slack
};

struct __align__(64) TcParams {
  CUtensorMap tq;
  CUtensorMap tk[kLevels];
  CUtensorMap tv[kLevels];
  const int* list;
  const int4* counts;
  __nv_bfloat16* O;
  float* lse;
  int* err;
  int Hq, Hkv, N, Nq, Nk, causal, n_rows;
  int qb;                                   // query rows per block: 128, or 64 (rows 64-127 dead)
  float scale_log2;
};

// ---- packed fp32 pairs (sm_100 f32x2 instructions) and the exp2 polynomial

__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 2^x for a pair x <= 0 on the FMA pipes, so that only part of a tile's
// exponentials queue on the transcendental unit.  Cody-Waite style: x is
// clamped to >= -126, split as n + f with n = round(x) (the 1.5 * 2^23
// addition rounds to an integer held in the low mantissa bits) and f in
// [-1/2, 1/2]; 2^f is a degree-3 polynomial whose coefficients were fitted
// here for the least maximum relative error on that interval (7.5e-5, far
// below the bf16 rounding of P); 2^n is added into the exponent field.
// Inputs of -inf give 2^-126 rather than 0, so a row counts as holding keys
// only once its running maximum is finite.
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& y0, float& y1) {
  constexpr float kMagic = 12582912.0f;                    // 1.5 * 2^23
  constexpr float c0 = 0.9999280571937561f, c1 = 0.6932609677314758f;
  constexpr float c2 = 0.2426111400127411f, c3 = 0.0551716685295105f;
  const uint64_t X = f2pack(fmaxf(x0, -126.f), fmaxf(x1, -126.f));
  const uint64_t T = fadd2(X, f2pack(kMagic, kMagic));
  const uint64_t N = fadd2(T, f2pack(-kMagic, -kMagic));
  const uint64_t F = ffma2(N, f2pack(-1.f, -1.f), X);
  uint64_t P = ffma2(F, f2pack(c3, c3), f2pack(c2, c2));
  P = ffma2(P, F, f2pack(c1, c1));
  P = ffma2(P, F, f2pack(c0, c0));
  float p0, p1, t0, t1;
  f2unpack(P, p0, p1);
  f2unpack(T, t0, t1);
  y0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// How many of every 8 exponential pairs of a softmax tile take the FMA-pipe
// polynomial above, the rest the transcendental unit (MUFU).
constexpr int kPolyPairs = 0;

// Items (query blocks) of this CTA: the bands of tile::Schedule (round robin
// over consecutive query blocks of a head, for L2 reuse of its K/V; causally,
// longest rows first, dealt in a snake so that the CTAs' loads even out).

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<D>;
  // At d = 64 the softmax outlasts a tile's products, and the first half of
  // PV overlapping the second half of the exponentials shortens each
  // stream's chain (measured 5% faster on the CogVideoX shape); at d = 128
  // the extra store wait in the softmax costs more than the overlap gains.
  constexpr bool kSplitPV = D == 64;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  constexpr int KS = C::KSTAGES, VS = C::VSTAGES, MS = C::MSTAGES;
  constexpr int B_QFULL = 0, B_QEMPTY = 1;
  constexpr int B_KFULL = 2, B_KEMPTY = B_KFULL + KS;
  constexpr int B_VFULL = B_KEMPTY + KS, B_VEMPTY = B_VFULL + VS;
  constexpr int B_MFULL = B_VEMPTY + VS, B_MEMPTY = B_MFULL + MS;
  constexpr int B_SFULL = B_MEMPTY + MS, B_PHALF = B_SFULL + kStreams;
  constexpr int B_PFULL = B_PHALF + kStreams;
  constexpr int B_OFULL = B_PFULL + kStreams, B_OFREE = B_OFULL + 1;
  constexpr int B_FINAL = B_OFREE + 1, B_XFULL = B_FINAL + 1, NBARS = B_XFULL + 8;
  static_assert(NBARS * 8 + 16 <= 512, "barrier area");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.n_rows;
  const Schedule sched = make_schedule(n_items, p.Nq, p.causal != 0);

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_QEMPTY), 1);                     // the block's last QK^T completed
    for (int s = 0; s < KS; ++s) { mbar_init(bar(B_KFULL + s), 1); mbar_init(bar(B_KEMPTY + s), 1); }
    for (int s = 0; s < VS; ++s) { mbar_init(bar(B_VFULL + s), 1); mbar_init(bar(B_VEMPTY + s), 1); }
    for (int s = 0; s < MS; ++s) { mbar_init(bar(B_MFULL + s), 32); mbar_init(bar(B_MEMPTY + s), 4); }
    for (int i = 0; i < kStreams; ++i) {
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_PHALF + i), 128);             // P of keys [0, 64) written (d = 64)
      mbar_init(bar(B_PFULL + i), 128);             // P of all keys written
    }
    mbar_init(bar(B_OFULL), 1);                      // the block's last PV completed
    mbar_init(bar(B_OFREE), 128);                    // both accumulators read out (warpgroup 1)
    mbar_init(bar(B_FINAL), 1);
    for (int i = 0; i < 8; ++i) mbar_init(bar(B_XFULL + i), 32);   // [block parity][quad]: (max, sum) handed over
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // Zero the K/V rings once: rows of a partial last tile are never loaded, and
  // their (masked, P = 0) products must not meet NaN bit patterns.
  {
    uint4* kv = reinterpret_cast<uint4*>(smem + C::OFF_K);
    const int n16 = (C::OFF_META - C::OFF_K) / 16;
    for (int i = threadIdx.x; i < n16; i += kThreads) kv[i] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S_s [128 s, 128 s + 128) (P_t written over it as bf16 pairs),
  // O_s [256 + D s, 256 + D s + D)
  const uint32_t T_S = tmem, T_O = tmem + 256;

  if (warp == 0) {
    // ---------------------------------------------------- K / Q producer
    int gk = 0, iq = 0;
    bool ok = true;
    for (int jb = 0; ok && jb < sched.bands(); ++jb) {
      const int item = sched.item(jb);
      if (item < 0) continue;
      const RowWork w = row_work(p.counts[item]);
      const int T = w.tiles;
      if (T == 0) continue;
      const int qa = item % p.Nq, bhq = item / p.Nq;
      const int bhk = (bhq / p.Hq) * p.Hkv + (bhq % p.Hq) / (p.Hq / p.Hkv);
      const int* lrow = p.list + (long long)item * p.Nk;
      // stage the work list (first kListCache entries) once per query block
      int* lcache = reinterpret_cast<int*>(smem + C::OFF_LIST);
      const int n_ent = min(w.f4, kListCache);
      __syncwarp();
      for (int i = lane; i < n_ent; i += 32) lcache[i] = __ldg(lrow + i);
      __syncwarp();
      TileEntry cur = tile_entry(w, lrow, lcache, 0, lane);
      if (iq > 0 && !warp_wait(bar(B_QEMPTY), (iq - 1) & 1, abort_flag, p.err)) { ok = false; break; }   // smem Q free
      if (lane == 0) {
        mbar_expect_tx(bar(B_QFULL), C::Q_BYTES);
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_3d(sbase + C::OFF_Q + h * (kBM * 128), &p.tq, bar(B_QFULL), h * 64,
                      qa * p.qb, bhq);
      }
      ++iq;
      for (int t = 0; t < T; ++t) {
        // the next tile's list entries are loaded before this tile's waits
        const TileEntry nxt = t + 1 < T ? tile_entry(w, lrow, lcache, t + 1, lane) : cur;
        {
          // K of tile t, and its per-key bias / position table
          const int s = gk % KS, ms = gk % MS;
          if (gk >= KS && !warp_wait(bar(B_KEMPTY + s), ((gk / KS) + 1) & 1, abort_flag, p.err)) { ok = false; break; }
          if (gk >= MS && !warp_wait(bar(B_MEMPTY + ms), ((gk / MS) + 1) & 1, abort_flag, p.err)) { ok = false; break; }
          const int n_in = __popc(__ballot_sync(0xffffffffu, cur.in_tile));
          // every entry fills exactly its R rows, so the tile carries
          // min(128, keys - 128 t) keys
          const int bytes = min(kBN, w.b4 - t * kBN) * D * 2;
          // Per-key bias table of this tile.  Usually every key of an 8-key
          // chunk has bias = its level (log2 of the pool factor), so 16 chunk
          // values describe the tile, read off the level boundaries of the
          // packed key sequence.  Tiles holding the ragged last KV block
          // (partial groups, rows past the end) or, causally, a block that
          // straddles the diagonal (token positions) get a full per-key table.
          unsigned char* mt_base = smem + C::OFF_META + ms * C::META_BYTES;
          float* cbias = reinterpret_cast<float*>(mt_base);                 // [16]
          int* mflag = reinterpret_cast<int*>(mt_base + 64);
          float* mbias = reinterpret_cast<float*>(mt_base + 128);           // [128]
          int* mpos = reinterpret_cast<int*>(mt_base + 128 + 512);          // [128]
          const bool special = cur.in_tile && (cur.j == p.Nk - 1 ||
                               (p.causal && cur.l == 0 &&
                                (cur.j + 1) * 64 - 1 >= qa * p.qb));
          const bool slow = __any_sync(0xffffffffu, special);
          if (!slow) {
            if (lane < 16) {
              const int off = t * kBN + 8 * lane;
              const int lvl = (off >= w.b1) + (off >= w.b2) + (off >= w.b3);
              cbias[lane] = off < w.b4 ? (float)lvl : -INFINITY;
            }
            if (lane == 16) *mflag = 0;
          } else {
            const int col = 4 * lane;
            int owner = 0;
            for (int i = 1; i < n_in; ++i)
              if (__shfl_sync(0xffffffffu, cur.r0, i) <= col) owner = i;
            const int oj = __shfl_sync(0xffffffffu, cur.j, owner);
            const int ol = __shfl_sync(0xffffffffu, cur.l, owner);
            const int oR = __shfl_sync(0xffffffffu, cur.R, owner);
            const int or0 = __shfl_sync(0xffffffffu, cur.r0, owner);
            const bool live = n_in > 0 && col < or0 + oR;   // false past the last entry
            float bias[4];
            int kpos[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int g = oj * oR + (col + c - or0);
              const int tok = g << ol;
              const int cnt = min(1 << ol, p.N - tok);
              bias[c] = !live || cnt <= 0 ? -INFINITY : (cnt == (1 << ol) ? (float)ol : log2f((float)cnt));
              kpos[c] = (live && p.causal && ol == 0) ? tok : INT_MIN;
            }
            reinterpret_cast<float4*>(mbias)[lane] = make_float4(bias[0], bias[1], bias[2], bias[3]);
            reinterpret_cast<int4*>(mpos)[lane] = make_int4(kpos[0], kpos[1], kpos[2], kpos[3]);
            if (lane == 0) *mflag = 1;
          }
          mbar_arrive(bar(B_MFULL + ms));           // each lane releases its own table writes
          if (lane == 0) mbar_expect_tx(bar(B_KFULL + s), bytes);
          __syncwarp();
          if (cur.in_tile) {
            const uint32_t kdst = sbase + C::OFF_K + s * C::KV_BYTES + cur.r0 * 128;
            for (int h = 0; h < C::HALVES; ++h)
              tma_load_3d(kdst + h * C::HALF, &p.tk[cur.l], bar(B_KFULL + s), h * 64,
                          cur.j * cur.R, bhk);
          }
          ++gk;
        }
        cur = nxt;
      }
    }
  } else if (warp == kVWarp) {
    // ------------------------------------------------------------ V producer
    int gv = 0;
    bool ok = true;
    for (int jb = 0; ok && jb < sched.bands(); ++jb) {
      const int item = sched.item(jb);
      if (item < 0) continue;
      const RowWork w = row_work(p.counts[item]);
      const int T = w.tiles;
      if (T == 0) continue;
      const int bhq = item / p.Nq;
      const int bhk = (bhq / p.Hq) * p.Hkv + (bhq % p.Hq) / (p.Hq / p.Hkv);
      const int* lrow = p.list + (long long)item * p.Nk;
      int* lcache = reinterpret_cast<int*>(smem + C::OFF_LIST + kListCache * 4);
      const int n_ent = min(w.f4, kListCache);
      __syncwarp();
      for (int i = lane; i < n_ent; i += 32) lcache[i] = __ldg(lrow + i);
      __syncwarp();
      TileEntry cur = tile_entry(w, lrow, lcache, 0, lane);
      for (int t = 0; t < T; ++t) {
        const TileEntry nxt = t + 1 < T ? tile_entry(w, lrow, lcache, t + 1, lane) : cur;
        const int s = gv % VS;
        if (gv >= VS && !warp_wait(bar(B_VEMPTY + s), ((gv / VS) + 1) & 1, abort_flag, p.err)) { ok = false; break; }
        const int bytes = min(kBN, w.b4 - t * kBN) * D * 2;
        if (lane == 0) mbar_expect_tx(bar(B_VFULL + s), bytes);
        __syncwarp();
        if (cur.in_tile) {
          const uint32_t vdst = sbase + C::OFF_V + s * C::KV_BYTES + cur.r0 * 128;
          for (int h = 0; h < C::HALVES; ++h)
            tma_load_3d(vdst + h * C::HALF, &p.tv[cur.l], bar(B_VFULL + s), h * 64,
                        cur.j * cur.R, bhk);
        }
        ++gv;
        cur = nxt;
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_QK = idesc_bf16(kBM, kBN, false);
      constexpr uint32_t ID_PV = idesc_bf16(kBM, D, true);
      const uint64_t qdesc0 = sdesc(sbase + C::OFF_Q, 16, 1024);
      const uint64_t kdesc0 = sdesc(sbase + C::OFF_K, 16, 1024);
      const uint64_t vdesc0 = sdesc(sbase + C::OFF_V, C::HALF, 1024);
      bool ok = true;
      int np[kStreams] = {0, 0};             // PVs issued per stream
      // S_s = Q K^T of the tile with global index u (K stage u % KS)
      auto issue_qk = [&](int u, int st) -> bool {
        const int s = u % KS;
        if (!wait_bar(bar(B_KFULL + s), (u / KS) & 1, abort_flag, p.err)) return false;
        tc_fence_after();
        // descriptors advance by adding the byte offset / 16 to the start-address field
        const uint64_t kd = kdesc0 + (uint64_t)((s * C::KV_BYTES) >> 4);
        const uint32_t dS = T_S + st * 128;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          constexpr uint32_t kHalfStep = C::HALF >> 4;   // same layout for Q and K halves
          const uint64_t off = (uint64_t)((k >> 2) * kHalfStep + (k & 3) * 2);
          mma_ss(dS, qdesc0 + off, kd + off, ID_QK, k > 0 ? 1u : 0u);
        }
        mma_commit(bar(B_SFULL + st));
        mma_commit(bar(B_KEMPTY + s));
        return true;
      };
      // O_s += P V of the tile with global index u; P was written over S_s.
      // With kSplitPV the products of keys [0, 64) start as soon as the
      // softmax has written their P, while it computes the rest.
      auto issue_pv = [&](int u, int st, bool first) -> bool {
        const int s = u % VS;
        if (!wait_bar(bar(B_VFULL + s), (u / VS) & 1, abort_flag, p.err)) return false;
        const uint64_t vd = vdesc0 + (uint64_t)((s * C::KV_BYTES) >> 4);
        const uint32_t dP = T_S + st * 128;
        const uint32_t dO = T_O + st * D;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (half == 0 || kSplitPV) {
            const int b = (kSplitPV && half == 0) ? B_PHALF : B_PFULL;
            if (!wait_bar(bar(b + st), np[st] & 1, abort_flag, p.err)) return false;
            tc_fence_after();
          }
#pragma unroll
          for (int k = 4 * half; k < 4 * half + 4; ++k)
            mma_ts(dO, dP + k * 8, vd + (uint64_t)(k * (2048 >> 4)), ID_PV,
                   (first && k == 0) ? 0u : 1u);
        }
        ++np[st];
        mma_commit(bar(B_VEMPTY + s));
        return true;
      };
      // Per query block: QK(0), QK(1); then for each tile t: PV(t), QK(t + 2).
      int g = 0, iq = 0;
      for (int jb = 0; ok && jb < sched.bands(); ++jb) {
      const int item = sched.item(jb);
      if (item < 0) continue;
        const int T = row_work(p.counts[item]).tiles;
        if (T == 0) continue;
        if (!wait_bar(bar(B_QFULL), iq & 1, abort_flag, p.err)) { ok = false; break; }
        for (int t = 0; ok && t < 2 && t < T; ++t) {
          ok = issue_qk(g + t, t);
          if (ok && t == T - 1) mma_commit(bar(B_QEMPTY));   // the block's last QK^T
        }
        // both accumulators of the previous block have been read out
        if (ok && iq > 0 && !wait_bar(bar(B_OFREE), (iq - 1) & 1, abort_flag, p.err)) ok = false;
        ++iq;
        for (int t = 0; ok && t < T; ++t) {
          ok = issue_pv(g + t, t & 1, t < 2);
          if (ok && t + 2 < T) {
            ok = issue_qk(g + t + 2, t & 1);
            if (ok && t + 2 == T - 1) mma_commit(bar(B_QEMPTY));
          }
        }
        if (!ok) break;
        mma_commit(bar(B_OFULL));
        g += T;
      }
      // drain: every MMA issued so far completes before TMEM is released
      mma_commit(bar(B_FINAL));
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(bar(B_FINAL), 0) && global_ns() - t0 < kTimeoutNs) {
      }
    }
  } else if (warp >= kSoftWarp0) {
    // --------------------------------------------------------------- softmax
    // Warpgroup st owns stream st: tiles t = st, st + 2, ... of every query
    // block.  Thread = query row r of the block (TMEM lane r).  The row's
    // scores of a tile are read from S_st twice: pass 1 (all 128 at once)
    // takes the tile maximum, pass 2 the exponentials, 64 keys at a time.  At the end of the block
    // warpgroup 0 hands its stream's (max, sum) to warpgroup 1, which merges
    // the two streams and writes O, while warpgroup 0 starts the next block.
    const int st = (warp - kSoftWarp0) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const bool dead = r >= p.qb;             // warp-uniform (qb is 64 or 128)
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t T_Ss = T_S + st * 128 + lane_off;
    float* xch = reinterpret_cast<float*>(smem + C::OFF_XCH);   // [block parity][128][max, sum]
    const float sc = p.scale_log2;
    const uint64_t sc2 = f2pack(sc, sc);
    int g = 0, ns = 0, nb = 0;               // tiles before this block, stream tiles, blocks with work
    bool ok = true;
    for (int jb = 0; jb < sched.bands(); ++jb) {
      const int item = sched.item(jb);
      if (item < 0) continue;
      const int T = row_work(p.counts[item]).tiles;
      const int qa = item % p.Nq, bhq = item / p.Nq;
      const int qpos = qa * p.qb + r;
      float m = -INFINITY, lsum = 0.f;
      for (int t = st; t < T; t += 2, ++ns) {
        const int gt = g + t, ms = gt % MS;
        ok = ok && warp_wait(bar(B_SFULL + st), ns & 1, abort_flag, p.err) &&
             warp_wait(bar(B_MFULL + ms), (gt / MS) & 1, abort_flag, p.err);
        if (!ok) continue;
        tc_fence_after();
        if (dead) {
          // rows past a 64-row query block (whole warps): no softmax, no
          // stores; their P rows are never read into a live row of O
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(B_MEMPTY + ms));
          tc_fence_before();
          if (kSplitPV) mbar_arrive(bar(B_PHALF + st));
          mbar_arrive(bar(B_PFULL + st));
          continue;
        }
        const unsigned char* mt_base = smem + C::OFF_META + ms * C::META_BYTES;
        const bool slow = *reinterpret_cast<const int*>(mt_base + 64) != 0;
        const float* cb = reinterpret_cast<const float*>(mt_base);            // [16] chunk biases
        const float* mbias = reinterpret_cast<const float*>(mt_base + 128);   // [128]
        const int* mpos = reinterpret_cast<const int*>(mt_base + 128 + 512);  // [128]
        // scaled, biased (and causally masked) logits of keys [h*64, h*64+64)
        auto logits = [&](float (&x)[64], int h) {
          tmem_ldn<64>(T_Ss + 64 * h, reinterpret_cast<uint32_t*>(x));
          tmem_ld_wait();
          reg_fence<64>(reinterpret_cast<uint32_t*>(x));
          if (!slow) {
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const float b = cb[8 * h + (c >> 3)];
              f2unpack(ffma2(f2pack(x[c], x[c + 1]), sc2, f2pack(b, b)), x[c], x[c + 1]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
              const float4 b4 = *reinterpret_cast<const float4*>(mbias + 64 * h + c);
              f2unpack(ffma2(f2pack(x[c], x[c + 1]), sc2, f2pack(b4.x, b4.y)), x[c], x[c + 1]);
              f2unpack(ffma2(f2pack(x[c + 2], x[c + 3]), sc2, f2pack(b4.z, b4.w)), x[c + 2], x[c + 3]);
              if (p.causal) {
                const int4 k4 = *reinterpret_cast<const int4*>(mpos + 64 * h + c);
                if (qpos < k4.x) x[c] = -INFINITY;
                if (qpos < k4.y) x[c + 1] = -INFINITY;
                if (qpos < k4.z) x[c + 2] = -INFINITY;
                if (qpos < k4.w) x[c + 3] = -INFINITY;
              }
            }
          }
        };
        // pass 1: the tile's row maximum.  In the common case every key of an
        // 8-key chunk has the same bias, so the chunk's largest dot product
        // gives its largest logit.
        float mt = -INFINITY;
        if (!slow) {
          uint32_t v[128];
          tmem_ldn<64>(T_Ss, v);
          tmem_ldn<64>(T_Ss + 64, v + 64);
          tmem_ld_wait();
          reg_fence<128>(v);
          float mc[16];
#pragma unroll
          for (int c = 0; c < 128; c += 8) {
            const float mx = fmax3(fmax3(__uint_as_float(v[c]), __uint_as_float(v[c + 1]), __uint_as_float(v[c + 2])),
                                   fmax3(__uint_as_float(v[c + 3]), __uint_as_float(v[c + 4]), __uint_as_float(v[c + 5])),
                                   fmaxf(__uint_as_float(v[c + 6]), __uint_as_float(v[c + 7])));
            mc[c >> 3] = fmaf(mx, sc, cb[c >> 3]);   // -inf bias: the chunk holds no keys
          }
          mt = fmax3(fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]), fmax3(mc[6], mc[7], mc[8])),
                     fmax3(mc[9], mc[10], mc[11]), fmax3(mc[12], mc[13], fmaxf(mc[14], mc[15])));
        } else {
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {
            float x[64];
            logits(x, h);
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int c = 0; c < 64; c += 4) {
              mx0 = fmax3(mx0, x[c], x[c + 1]);
              mx1 = fmax3(mx1, x[c + 2], x[c + 3]);
            }
            mt = fmaxf(mt, fmaxf(mx0, mx1));
          }
        }
        const float m_new = fmaxf(m, mt);
        const bool need = m_new > m + kRescaleLog2;     // false while both are -inf
        if (__any_sync(0xffffffffu, need)) {
          const float m_use = need ? m_new : m;
          const float factor = need ? ex2(m - m_use) : 1.f;   // 0 when m = -inf
          if (t >= 2) {
            // O_st is quiescent: PV(t - 2) completed before S(t) was committed
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(T_O + st * D + lane_off + c0, o);
              tmem_ld_wait();
              reg_fence<32>(o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
              tmem_st32(T_O + st * D + lane_off + c0, o);
            }
          }
          lsum *= factor;
          m = m_use;
        }
        // pass 2: P = exp2(logit - m) as bf16 pairs, written over S_st
        const float m_base = m == -INFINITY ? 0.f : m;
        const uint64_t nm2 = f2pack(-m_base, -m_base);
        uint64_t acc0 = f2pack(0.f, 0.f), acc1 = acc0;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          float x[64];
          logits(x, h);
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            float d0, d1, p0, p1;
            f2unpack(fadd2(f2pack(x[c], x[c + 1]), nm2), d0, d1);
            if (((c >> 1) & 7) < kPolyPairs) {
              exp2_poly2(d0, d1, p0, p1);
            } else {
              p0 = ex2(d0);
              p1 = ex2(d1);
            }
            if ((c >> 1) & 1) acc1 = fadd2(acc1, f2pack(p0, p1));
            else acc0 = fadd2(acc0, f2pack(p0, p1));
            __nv_bfloat162 hh = __floats2bfloat162_rn(p0, p1);
            pk[c / 2] = *reinterpret_cast<uint32_t*>(&hh);
          }
          // P columns [32 h, 32 h + 32) overwrite logits this thread has read
          tmem_stn<32>(T_Ss + 32 * h, pk);
          if (kSplitPV && h == 0) {
            // P of keys [0, 64) is complete: their products may start
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(bar(B_PHALF + st));
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_MEMPTY + ms));   // bias table read
        float a0, a1, a2, a3;
        f2unpack(acc0, a0, a1);
        f2unpack(acc1, a2, a3);
        lsum += (a0 + a1) + (a2 + a3);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL + st));
      }
      // ---- end of the query block.  Warpgroup 0 hands its (max, sum) to
      // warpgroup 1 through shared memory and an mbarrier per warp, and goes
      // on to the next block's first tile; warpgroup 1 merges the two streams
      // and writes the whole row of O and the LSE.  The buffer and barrier
      // alternate by block parity: warpgroup 0 reaches the end of block
      // nb + 2 only after the issuer has seen block nb's accumulators
      // released, i.e. after warpgroup 1 read block nb's values.
      const int xid = nb & 1;
      float* xb = xch + xid * (128 * 2);
      const uint32_t xbar = bar(B_XFULL + 4 * xid + quad);
      if (st == 0) {
        if (T > 0) {
          xb[r * 2] = m;
          xb[r * 2 + 1] = lsum;
          mbar_arrive(xbar);
          ++nb;
        }
        g += T;
        continue;
      }
      float m0 = -INFINITY, l0 = 0.f;
      if (T > 0) {
        ok = ok && warp_wait(xbar, (nb >> 1) & 1, abort_flag, p.err);
        m0 = xb[r * 2];
        l0 = xb[r * 2 + 1];
      }
      const float M = fmaxf(m0, m);
      const bool keys = M > -INFINITY;                  // the row kept at least one key
      const float f0 = m0 > -INFINITY ? ex2(m0 - M) : 0.f;
      const float f1 = m > -INFINITY ? ex2(m - M) : 0.f;
      const float L = l0 * f0 + lsum * f1;
      const float inv = keys ? 1.f / L : 0.f;
      const bool row_ok = !dead && qpos < p.N;
      __nv_bfloat16* dst = p.O + ((long long)bhq * p.N + qpos) * D;
      const bool have_o = T > 0 && __all_sync(0xffffffffu, ok) &&
                          warp_wait(bar(B_OFULL), nb & 1, abort_flag, p.err);
      if (have_o) tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        float o[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0.f;
        if (have_o) {
#pragma unroll
          for (int i = 0; i < kStreams; ++i) {
            if (i < T) {                     // stream i holds tiles
              uint32_t u[32];
              tmem_ldn<32>(T_O + i * D + lane_off + c0, u);
              tmem_ld_wait();
              reg_fence<32>(u);
              const float fi = i == 0 ? f0 : f1;
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = fmaf(__uint_as_float(u[k]), fi, o[k]);
            }
          }
        }
        if (row_ok) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            __nv_bfloat162 hh = __floats2bfloat162_rn(o[2 * i] * inv, o[2 * i + 1] * inv);
            pk[i] = *reinterpret_cast<uint32_t*>(&hh);
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (row_ok && p.lse)
        p.lse[(long long)bhq * p.N + qpos] = keys ? (M + log2f(L)) * kLn2 : -INFINITY;
      if (T > 0) {
        // the accumulators may be overwritten by the next block's PVs
        tc_fence_before();
        mbar_arrive(bar(B_OFREE));
        ++nb;
      }
      g += T;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512)
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side

// 3-D bf16 map over [heads, rows, D] (D contiguous), box {64, box_rows, 1},
// 128-byte swizzle; rows past `rows` read as zero.
bool encode_map(CUtensorMap* m, const void* base, int D, long long rows, int heads, int box_rows) {
  return encode_map_3d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, D, rows, heads, 64, box_rows);
}

template <int D>
cudaError_t launch_tc_typed(const TcParams& prm, int rows, cudaStream_t st) {
  const int smem = Cfg<D>::SMEM;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = rows < sms ? rows : sms;   // persistent: one CTA per SM
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // A plain launch: in this persistent kernel a grid-dependency wait
  // measured 12 to 18 us slower per call (Wan-1.3B, Qwen2.5-VL shapes).
  attn_tc_kernel<D><<<grid, kThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace

bool attention_tc_supported(const psa_params_t& p) {
  return p.dtype == PSA_BF16 && (p.q_blk == 128 || p.q_blk == 64) && p.kv_blk == 64 &&
         (p.d == 64 || p.d == 128);
}

cudaError_t launch_attention_tc(const psa_params_t& p, const Layout& L, float scale,
                                const void* Q, const void* K, const void* V, char* ws,
                                void* O, float* lse, cudaStream_t st) {
  TcParams prm;
  memset(&prm, 0, sizeof(prm));
  const int BHq = p.B * p.Hq, BHk = p.B * p.Hkv;
  bool ok = encode_map(&prm.tq, Q, p.d, p.N, BHq, kBM);
  for (int l = 0; l < kLevels && ok; ++l) {
    const void* kb = l == 0 ? K : (const void*)(ws + L.kp[l]);
    const void* vb = l == 0 ? V : (const void*)(ws + L.vp[l]);
    ok = encode_map(&prm.tk[l], kb, p.d, (long long)L.rows[l], BHk, 64 >> l) &&
         encode_map(&prm.tv[l], vb, p.d, (long long)L.rows[l], BHk, 64 >> l);
  }
  if (!ok) return cudaErrorInvalidValue;
  prm.list = (const int*)(ws + L.list);
  prm.counts = (const int4*)(ws + L.counts);
  prm.O = (__nv_bfloat16*)O;
  prm.lse = lse;
  prm.err = (int*)(ws + L.err);
  prm.Hq = p.Hq; prm.Hkv = p.Hkv; prm.N = p.N; prm.Nq = L.Nq; prm.Nk = L.Nk;
  prm.causal = p.causal;
  prm.n_rows = BHq * L.Nq;
  prm.qb = p.q_blk;
  prm.scale_log2 = scale * kLog2e;
  return p.d == 128 ? launch_tc_typed<128>(prm, prm.n_rows, st)
                    : launch_tc_typed<64>(prm, prm.n_rows, st);
}

}  // namespace psa
