// Gradient of pyramid attention on the 5th-generation tensor cores (tcgen05 +
// TMEM + TMA), bf16 inputs, fp32 accumulation, 128-row query blocks (64-row
// blocks as 128-row tiles whose rows 64-127 have P = dS = 0), d in
// {64, 128}.
//
// Method: the chain rule through adaptive pyramid attention (top168.com
// article on PSA, component three: one softmax over every kept key, a pooled
// key carrying the mass of the c tokens it averages) with the level map held
// fixed; the formulas are in bwd_internal.cuh.  The query block's keys are
// walked in the packed 128-key tiles of the forward pass (the "decoupled
// block-tile" design of the PSA abstract), so each tile mixes sub-blocks of
// several KV blocks and levels.
//
// Persistent CTAs (one per SM) walk the query blocks; 12 warps:
//   warp 0     TMA producer for Q and dO (once per query block) and K; per
//              tile, one 2-D box per sub-block and 64-column half, plus the
//              tile's per-key table (log2 c bias, causal position, gradient
//              destination: level and pooled row).
//   warp 2     TMA producer for V.
//   warp 1     TMEM allocator and single-thread tcgen05.mma issuer.
//   warps 4-11 two compute warpgroups: warpgroup h takes keys [64h, 64h+64)
//              of each query row for P and dS, and columns [h d/2, h d/2 + d/2)
//              of each key row in the epilogue.
// Per tile t:
//   MMA1   S = Q K_t^T, dP = dO V_t^T        (SS, K-major operands)
//   compute P = exp2(S s log2e + log2 c - lse log2e), dS = P (dP - D),
//          both written to shared memory as bf16 [query][key], 128B-swizzled
//   MMA2   dQ += dS K_t                      (A K-major, B MN-major; TMEM)
//          dV_t = P^T dO, dK_t = dS^T Q      (A read transposed: MN-major)
//   epilogue  per key row: dK_t * s and dV_t added into the fp32 gradient
//          of the key's level and pooled row (vector atomics; a pooled row
//          is shared by every query block that keeps it)
// At the end of the query block dQ * s is read from TMEM and stored.
// TMEM columns: S / dK_t [0, 128), dP [128, 256), dQ [256, 256 + d),
// dV_t [384, 384 + d).  dP of the next tile of a block is issued as soon as
// the softmax has read this tile's, so it overlaps this tile's epilogue.
// Every mbarrier wait is bounded: on expiry the kernel records a timeout in
// the workspace error word and winds down without trapping.
#include "bwd_internal.cuh"

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
constexpr int kVWarp = 2;
constexpr int kCompWarp0 = 4;
constexpr int kThreads = 384;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
struct BCfg {
  static constexpr int HALVES = D / 64;
  static constexpr int STAGES = D == 128 ? 1 : 2;     // K ring and V ring
  static constexpr int MSTAGES = 2;                   // per-tile key tables
  static constexpr int HALF = 128 * 128;              // one 64-column half of a 128-row tile
  static constexpr int T_BYTES = 128 * D * 2;         // a Q, dO, K or V tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = OFF_Q + T_BYTES;
  static constexpr int OFF_P = OFF_DO + T_BYTES;      // P  [128 queries][128 keys] bf16
  static constexpr int OFF_DS = OFF_P + 2 * HALF;     // dS [128 queries][128 keys] bf16
  static constexpr int OFF_K = OFF_DS + 2 * HALF;
  static constexpr int OFF_V = OFF_K + STAGES * T_BYTES;
  static constexpr int OFF_META = OFF_V + STAGES * T_BYTES;
  static constexpr int META_BYTES = 3 * 512;          // bias f32, kpos i32, dst i32, [128] each
  static constexpr int OFF_BAR = OFF_META + MSTAGES * META_BYTES;
  static constexpr int OFF_LIST = OFF_BAR + 256;      // work-list copies of warps 0 and 2
  static constexpr int SMEM = OFF_LIST + 2 * kListCache * 4 + 1024;
};

struct __align__(64) BwdTcParams {
  CUtensorMap tq, tdo;
  CUtensorMap tk[kLevels];
  CUtensorMap tv[kLevels];
  const int* list;
  const int4* counts;
  const float* lse;
  const float* delta;
  float* dk[kLevels];
  float* dv[kLevels];
  long long rows[kLevels];
  __nv_bfloat16* dQ;
  int* err;
  int Hq, Hkv, N, Nq, Nk, causal, n_rows;
  int qb;                                   // query rows per block: 128, or 64 (rows 64-127 dead)
  float scale, scale_log2;
};

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// packed fp32 pairs (sm_100 f32x2 instructions)
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

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_bwd_tc_kernel(const __grid_constant__ BwdTcParams p) {
  using C = BCfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  constexpr int KS = C::STAGES, MS = C::MSTAGES;
  constexpr int B_QFULL = 0, B_QEMPTY = 1;
  constexpr int B_KFULL = 2, B_KEMPTY = B_KFULL + KS;
  constexpr int B_VFULL = B_KEMPTY + KS, B_VEMPTY = B_VFULL + KS;
  constexpr int B_MFULL = B_VEMPTY + KS, B_MEMPTY = B_MFULL + MS;
  constexpr int B_SFULL = B_MEMPTY + MS, B_PFULL = B_SFULL + 1;
  constexpr int B_GFULL = B_PFULL + 1, B_TFREE = B_GFULL + 1;
  constexpr int B_DQFREE = B_TFREE + 1, B_FINAL = B_DQFREE + 1, NBARS = B_FINAL + 1;
  static_assert(NBARS * 8 + 16 <= 256, "barrier area");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.n_rows;
  const Schedule sched = make_schedule(n_items, p.Nq, p.causal != 0);

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_QEMPTY), 1);                 // the block's last MMA2 completed
    for (int s = 0; s < KS; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_KEMPTY + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_VEMPTY + s), 1);
    }
    for (int s = 0; s < MS; ++s) {
      mbar_init(bar(B_MFULL + s), 32);           // every producer lane wrote its keys
      mbar_init(bar(B_MEMPTY + s), 8);           // every compute warp is done with it
    }
    mbar_init(bar(B_SFULL), 1);
    mbar_init(bar(B_PFULL), 256);
    mbar_init(bar(B_GFULL), 1);
    mbar_init(bar(B_TFREE), 256);
    mbar_init(bar(B_DQFREE), 256);
    mbar_init(bar(B_FINAL), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // Zero the K/V rings once: rows of a partial last tile are never loaded, and
  // their (P = 0, dS = 0) products must not meet NaN bit patterns.
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
  const uint32_t T_S = tmem, T_DP = tmem + 128, T_DQ = tmem + 256, T_DV = tmem + 384;

  if (warp == 0 || warp == kVWarp) {
    // ----------------------------------------- producers: Q, dO, K (warp 0); V (warp 2)
    const bool kprod = warp == 0;
    int gk = 0, iq = 0;
    bool ok = true;
    int* lcache = reinterpret_cast<int*>(smem + C::OFF_LIST + (kprod ? 0 : kListCache * 4));
    for (int jb = 0; ok && jb < sched.bands(); ++jb) {
      const int item = sched.item(jb);
      if (item < 0) continue;
      const RowWork w = row_work(p.counts[item]);
      const int T = w.tiles;
      if (T == 0) continue;
      const int qa = item % p.Nq, bhq = item / p.Nq;
      const int bhk = (bhq / p.Hq) * p.Hkv + (bhq % p.Hq) / (p.Hq / p.Hkv);
      const int* lrow = p.list + (long long)item * p.Nk;
      const int n_ent = min(w.f4, kListCache);
      __syncwarp();
      for (int i = lane; i < n_ent; i += 32) lcache[i] = __ldg(lrow + i);
      __syncwarp();
      TileEntry cur = tile_entry(w, lrow, lcache, 0, lane);
      if (kprod) {
        if (iq > 0 && !warp_wait(bar(B_QEMPTY), (iq - 1) & 1, abort_flag, p.err)) { ok = false; break; }
        if (lane == 0) {
          mbar_expect_tx(bar(B_QFULL), 2 * C::T_BYTES);
          for (int h = 0; h < C::HALVES; ++h) {
            tma_load_3d(sbase + C::OFF_Q + h * C::HALF, &p.tq, bar(B_QFULL), h * 64, qa * p.qb, bhq);
            tma_load_3d(sbase + C::OFF_DO + h * C::HALF, &p.tdo, bar(B_QFULL), h * 64, qa * p.qb, bhq);
          }
        }
        ++iq;
      }
      for (int t = 0; t < T; ++t) {
        const TileEntry nxt = t + 1 < T ? tile_entry(w, lrow, lcache, t + 1, lane) : cur;
        const int s = gk % KS;
        const int b_full = kprod ? B_KFULL : B_VFULL, b_empty = kprod ? B_KEMPTY : B_VEMPTY;
        if (gk >= KS && !warp_wait(bar(b_empty + s), ((gk / KS) + 1) & 1, abort_flag, p.err)) { ok = false; break; }
        if (kprod) {
          // the tile's per-key table; lane i covers keys [4i, 4i + 4), which
          // never straddle two sub-blocks (every sub-block has >= 8 rows)
          const int ms = gk % MS;
          if (gk >= MS && !warp_wait(bar(B_MEMPTY + ms), ((gk / MS) + 1) & 1, abort_flag, p.err)) { ok = false; break; }
          unsigned char* mt = smem + C::OFF_META + ms * C::META_BYTES;
          const int n_in = __popc(__ballot_sync(0xffffffffu, cur.in_tile));
          const int col = 4 * lane;
          int owner = 0;
          for (int i = 1; i < n_in; ++i)
            if (__shfl_sync(0xffffffffu, cur.r0, i) <= col) owner = i;
          const int oj = __shfl_sync(0xffffffffu, cur.j, owner);
          const int ol = __shfl_sync(0xffffffffu, cur.l, owner);
          const int oR = __shfl_sync(0xffffffffu, cur.R, owner);
          const int or0 = __shfl_sync(0xffffffffu, cur.r0, owner);
          const bool live = n_in > 0 && col < or0 + oR;
          float bias[4];
          int kpos[4], dst[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int g = oj * oR + (col + c - or0);
            const int tok = g << ol;
            const int cnt = min(1 << ol, p.N - tok);
            const bool key = live && cnt > 0;
            bias[c] = !key ? -INFINITY : (cnt == (1 << ol) ? (float)ol : log2f((float)cnt));
            kpos[c] = (key && p.causal && ol == 0) ? tok : INT_MIN;
            dst[c] = key ? ((ol << 24) | g) : -1;
          }
          reinterpret_cast<float4*>(mt)[lane] = make_float4(bias[0], bias[1], bias[2], bias[3]);
          reinterpret_cast<int4*>(mt + 512)[lane] = make_int4(kpos[0], kpos[1], kpos[2], kpos[3]);
          reinterpret_cast<int4*>(mt + 1024)[lane] = make_int4(dst[0], dst[1], dst[2], dst[3]);
          mbar_arrive(bar(B_MFULL + ms));       // each lane releases its own table writes
        }
        const int bytes = min(kBN, w.b4 - t * kBN) * D * 2;
        if (lane == 0) mbar_expect_tx(bar(b_full + s), bytes);
        __syncwarp();
        if (cur.in_tile) {
          const uint32_t dst = sbase + (kprod ? C::OFF_K : C::OFF_V) + s * C::T_BYTES + cur.r0 * 128;
          const CUtensorMap* map = kprod ? &p.tk[cur.l] : &p.tv[cur.l];
          for (int h = 0; h < C::HALVES; ++h)
            tma_load_3d(dst + h * C::HALF, map, bar(b_full + s), h * 64, cur.j * cur.R, bhk);
        }
        ++gk;
        cur = nxt;
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_S = idesc_bf16(kBM, kBN, false);          // S, dP
      constexpr uint32_t ID_DQ = idesc_bf16(kBM, D, true);            // dQ += dS K
      constexpr uint32_t ID_KV = idesc_bf16(kBN, D, true, true);      // dV = P^T dO, dK = dS^T Q
      // K-major views (K = the 64-column halves of d, or of the 128 keys)
      const uint64_t q_k = sdesc(sbase + C::OFF_Q, 16, 1024);
      const uint64_t do_k = sdesc(sbase + C::OFF_DO, 16, 1024);
      const uint64_t k_k = sdesc(sbase + C::OFF_K, 16, 1024);
      const uint64_t v_k = sdesc(sbase + C::OFF_V, 16, 1024);
      const uint64_t ds_k = sdesc(sbase + C::OFF_DS, 16, 1024);
      // MN-major views: 64-element chunks along M or N HALF bytes apart,
      // 8-row groups along K 1024 bytes apart
      const uint64_t k_mn = sdesc(sbase + C::OFF_K, C::HALF, 1024);
      const uint64_t q_mn = sdesc(sbase + C::OFF_Q, C::HALF, 1024);
      const uint64_t do_mn = sdesc(sbase + C::OFF_DO, C::HALF, 1024);
      const uint64_t p_mn = sdesc(sbase + C::OFF_P, C::HALF, 1024);
      const uint64_t ds_mn = sdesc(sbase + C::OFF_DS, C::HALF, 1024);
      constexpr uint32_t kHalfStep = C::HALF >> 4;
      constexpr uint32_t kRow16 = (16 * 128) >> 4;   // 16 rows along K of an MN-major view
      bool ok = true;
      int u = 0, iq = 0;
      for (int jb = 0; ok && jb < sched.bands(); ++jb) {
      const int item = sched.item(jb);
      if (item < 0) continue;
        const int T = row_work(p.counts[item]).tiles;
        if (T == 0) continue;
        if (!wait_bar(bar(B_QFULL), iq & 1, abort_flag, p.err)) { ok = false; break; }
        // dP of a tile is issued as soon as its region is free: after the
        // softmax of the previous tile of the block has read dP (dV_t has
        // its own columns), so it runs while that tile's epilogue reads
        // dK_t / dV_t; S waits for the epilogue, since dK_t shares its columns
        bool dp_issued = false;
        auto issue_dp = [&](int uu) -> bool {
          const int sv = uu % KS;
          if (!wait_bar(bar(B_VFULL + sv), (uu / KS) & 1, abort_flag, p.err)) return false;
          tc_fence_after();
          const uint64_t stv = (uint64_t)((sv * C::T_BYTES) >> 4);
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t off = (uint64_t)((k >> 2) * kHalfStep + (k & 3) * 2);
            mma_ss(T_DP, do_k + off, v_k + stv + off, ID_S, k > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_VEMPTY + sv));
          return true;
        };
        for (int t = 0; ok && t < T; ++t, ++u) {
          const int s = u % KS;
          const uint64_t stage = (uint64_t)((s * C::T_BYTES) >> 4);
          if (!dp_issued && !issue_dp(u)) { ok = false; break; }
          ok = wait_bar(bar(B_KFULL + s), (u / KS) & 1, abort_flag, p.err) &&
               (u == 0 || wait_bar(bar(B_TFREE), (u - 1) & 1, abort_flag, p.err));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint64_t off = (uint64_t)((k >> 2) * kHalfStep + (k & 3) * 2);
            mma_ss(T_S, q_k + off, k_k + stage + off, ID_S, k > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_SFULL));                    // S and dP of tile u
          ok = wait_bar(bar(B_PFULL), u & 1, abort_flag, p.err) &&
               (t > 0 || iq == 0 || wait_bar(bar(B_DQFREE), (iq - 1) & 1, abort_flag, p.err));
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < kBN / 16; ++k) {
            const uint64_t koff = (uint64_t)((k >> 2) * kHalfStep + (k & 3) * 2);
            mma_ss(T_DQ, ds_k + koff, k_mn + stage + (uint64_t)(k * kRow16), ID_DQ,
                   (t > 0 || k > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int k = 0; k < kBM / 16; ++k) {
            const uint64_t roff = (uint64_t)(k * kRow16);
            mma_ss(T_DV, p_mn + roff, do_mn + roff, ID_KV, k > 0 ? 1u : 0u);
            mma_ss(T_S, ds_mn + roff, q_mn + roff, ID_KV, k > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_GFULL));
          mma_commit(bar(B_KEMPTY + s));
          if (t == T - 1) mma_commit(bar(B_QEMPTY));
          // the next tile's dP (the softmax of this tile has read dP: PFULL)
          dp_issued = t + 1 < T;
          if (dp_issued && !issue_dp(u + 1)) { ok = false; break; }
        }
        ++iq;
      }
      // drain: every MMA issued so far completes before TMEM is released
      mma_commit(bar(B_FINAL));
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(bar(B_FINAL), 0) && global_ns() - t0 < kTimeoutNs) {
      }
    }
  } else if (warp >= kCompWarp0) {
    // --------------------------------------------------------------- compute
    constexpr int DH = D / 2;
    const int h = (warp - kCompWarp0) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float sl2 = p.scale_log2;
    int u = 0;
    bool ok = true;
    for (int jb = 0; jb < sched.bands(); ++jb) {
      const int item = sched.item(jb);
      if (item < 0) continue;
      const int T = row_work(p.counts[item]).tiles;
      const int qa = item % p.Nq, bhq = item / p.Nq;
      const int bhk = (bhq / p.Hq) * p.Hkv + (bhq % p.Hq) / (p.Hq / p.Hkv);
      const int qpos = qa * p.qb + r;
      // rows past a 64-row query block are dead: P = dS = 0 (so they add
      // nothing to dK, dV), no dQ store
      const bool valid = r < p.qb && qpos < p.N;
      const long long qrow = (long long)bhq * p.N + qpos;
      const float lse2 = valid && T > 0 ? p.lse[qrow] * kLog2e : -INFINITY;
      const float Di = valid && T > 0 ? p.delta[qrow] : 0.f;
      const bool live = lse2 > -INFINITY;      // the row kept a key (false for NaN too)
      for (int t = 0; t < T; ++t, ++u) {
        const int ms = u % MS;
        ok = ok && warp_wait(bar(B_SFULL), u & 1, abort_flag, p.err) &&
             warp_wait(bar(B_MFULL + ms), (u / MS) & 1, abort_flag, p.err);
        if (!ok) continue;
        tc_fence_after();
        const unsigned char* mt = smem + C::OFF_META + ms * C::META_BYTES;
        const float* mbias = reinterpret_cast<const float*>(mt);
        const int* mpos = reinterpret_cast<const int*>(mt + 512);
        const int* mdst = reinterpret_cast<const int*>(mt + 1024);
        {
          // P and dS of keys [64h, 64h + 64) of row r, 32 keys at a time:
          // x = S * scale * log2e + (log2 c - lse * log2e) in pairs, P = exp2(x)
          // (a -inf bias, no key, gives 0), dS = P (dP - D), written to half h
          // of the P / dS tiles (128-byte swizzle: 16-byte chunk index XOR row
          // mod 8).  A row that kept no key (or lies past N) writes zeros.
          const uint64_t sl2x2 = f2pack(sl2, sl2), nl2 = f2pack(-lse2, -lse2);
          const uint64_t nd2 = f2pack(-Di, -Di), zero2 = f2pack(0.f, 0.f);
          const uint32_t rowb = (uint32_t)(h * C::HALF + r * 128);
#pragma unroll 1
          for (int q = 0; q < 2; ++q) {
            uint32_t sv[32], gv[32];
            tmem_ld32(T_S + lane_off + 64 * h + 32 * q, sv);
            tmem_ld32(T_DP + lane_off + 64 * h + 32 * q, gv);
            tmem_ld_wait();
            reg_fence<32>(sv);
            reg_fence<32>(gv);
            uint32_t pk[16], xk[16];
            if (live) {
#pragma unroll
              for (int c = 0; c < 32; c += 4) {
                const int k = 64 * h + 32 * q + c;
                const float4 b4 = *reinterpret_cast<const float4*>(mbias + k);
                float x[4], pp[4], xx[4];
                f2unpack(ffma2(f2pack(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sl2x2,
                               fadd2(f2pack(b4.x, b4.y), nl2)), x[0], x[1]);
                f2unpack(ffma2(f2pack(__uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3])), sl2x2,
                               fadd2(f2pack(b4.z, b4.w), nl2)), x[2], x[3]);
                if (p.causal) {
                  const int4 k4 = *reinterpret_cast<const int4*>(mpos + k);
                  if (qpos < k4.x) x[0] = -INFINITY;
                  if (qpos < k4.y) x[1] = -INFINITY;
                  if (qpos < k4.z) x[2] = -INFINITY;
                  if (qpos < k4.w) x[3] = -INFINITY;
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) pp[i] = ex2(x[i]);
#pragma unroll
                for (int i = 0; i < 4; i += 2) {
                  const uint64_t gd = fadd2(f2pack(__uint_as_float(gv[c + i]), __uint_as_float(gv[c + i + 1])), nd2);
                  f2unpack(ffma2(f2pack(pp[i], pp[i + 1]), gd, zero2), xx[i], xx[i + 1]);
                }
                pk[c / 2] = pack_bf16(pp[0], pp[1]);
                pk[c / 2 + 1] = pack_bf16(pp[2], pp[3]);
                xk[c / 2] = pack_bf16(xx[0], xx[1]);
                xk[c / 2 + 1] = pack_bf16(xx[2], xx[3]);
              }
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) pk[i] = xk[i] = 0u;
            }
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const uint32_t o = rowb + (uint32_t)(((4 * q + cc) ^ (r & 7)) << 4);
              st_shared_v4(sbase + C::OFF_P + o, pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
              st_shared_v4(sbase + C::OFF_DS + o, xk[4 * cc], xk[4 * cc + 1], xk[4 * cc + 2], xk[4 * cc + 3]);
            }
          }
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // visible to the tensor core
        tc_fence_before();
        mbar_arrive(bar(B_PFULL));
        ok = warp_wait(bar(B_GFULL), u & 1, abort_flag, p.err);
        if (!ok) continue;
        tc_fence_after();
        {
          // epilogue: key r of the tile, columns [h DH, h DH + DH)
          uint32_t kv[DH], vv[DH];
          tmem_ldn<DH>(T_S + lane_off + h * DH, kv);
          tmem_ldn<DH>(T_DV + lane_off + h * DH, vv);
          tmem_ld_wait();
          reg_fence<DH>(kv);
          reg_fence<DH>(vv);
          tc_fence_before();
          mbar_arrive(bar(B_TFREE));               // dK_t, dV_t read: S and dV_t may be overwritten
          // Each key row's DH columns go to its level's fp32 accumulator row.
          // Added one row per thread, a warp's vector atomics would touch 32
          // rows each; instead the warp stages its 32 rows in shared memory,
          // then adds them a row per NC lanes, so that every atomic
          // instruction covers whole rows: about twice the reduction
          // throughput.  The staging area is the 4 KB of P rows and the 4 KB
          // of dS rows that this warp itself writes for the next tile (the
          // MMAs of this tile have finished reading them; no other warp
          // writes there).  dK_t (times the scale) first, then dV_t, through
          // the same area.  Chunk c of row R sits at 16-byte position
          // c ^ (R mod NC): conflict-free both ways.
          constexpr int NC = DH / 4;             // 16-byte chunks per row: 16 (d=128), 8 (d=64)
          constexpr int RPI = 32 / NC;           // rows per warp instruction: 2 or 4
          constexpr int ROWB = NC * 16;          // staged bytes per row
          constexpr int RPP = 4096 / ROWB;       // rows per 4 KB piece: 16 (d=128), 32 (d=64)
          const uint32_t own = (uint32_t)(h * C::HALF + quad * 4096);
          auto staged = [&](int R, int c) -> uint32_t {
            return sbase + (R < RPP ? C::OFF_P : C::OFF_DS) + own + (uint32_t)((R % RPP) * ROWB) +
                   (uint32_t)((c ^ (R & (NC - 1))) << 4);
          };
          const float s = p.scale;
#pragma unroll
          for (int which = 0; which < 2; ++which) {
            const uint32_t* x = which == 0 ? kv : vv;
            const float f = which == 0 ? s : 1.f;
#pragma unroll
            for (int c = 0; c < NC; ++c)
              st_shared_v4(staged(lane, c),
                           __float_as_uint(__uint_as_float(x[4 * c]) * f),
                           __float_as_uint(__uint_as_float(x[4 * c + 1]) * f),
                           __float_as_uint(__uint_as_float(x[4 * c + 2]) * f),
                           __float_as_uint(__uint_as_float(x[4 * c + 3]) * f));
            __syncwarp();
            float* const* acc = which == 0 ? p.dk : p.dv;
            const int c = lane % NC;
#pragma unroll 4
            for (int k = 0; k < 32 / RPI; ++k) {
              const int R = k * RPI + lane / NC;
              const int dst = mdst[quad * 32 + R];
              if (dst >= 0) {
                const int l = dst >> 24;
                float4 v4;
                asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                             : "=f"(v4.x), "=f"(v4.y), "=f"(v4.z), "=f"(v4.w)
                             : "r"(staged(R, c)));
                float* g = acc[l] + ((long long)bhk * p.rows[l] + (dst & 0xffffff)) * D + h * DH + 4 * c;
                atomicAdd(reinterpret_cast<float4*>(g), v4);
              }
            }
            __syncwarp();                        // the slot is read before it is rewritten
          }
          if (lane == 0) mbar_arrive(bar(B_MEMPTY + ms));   // key table read
        }
      }
      // ---- end of the query block: dQ of row r, columns [h DH, h DH + DH)
      if (T > 0 && !__all_sync(0xffffffffu, ok)) continue;
      uint32_t dq[DH];
      if (T > 0) {
        tmem_ldn<DH>(T_DQ + lane_off + h * DH, dq);
        tmem_ld_wait();
        reg_fence<DH>(dq);
        tc_fence_before();
        mbar_arrive(bar(B_DQFREE));
      } else {
#pragma unroll
        for (int i = 0; i < DH; ++i) dq[i] = 0u;
      }
      if (valid) {
        uint4* d4 = reinterpret_cast<uint4*>(p.dQ + qrow * D + h * DH);
        const float s = p.scale;
#pragma unroll
        for (int i = 0; i < DH; i += 8)
          d4[i / 8] = make_uint4(
              pack_bf16(__uint_as_float(dq[i]) * s, __uint_as_float(dq[i + 1]) * s),
              pack_bf16(__uint_as_float(dq[i + 2]) * s, __uint_as_float(dq[i + 3]) * s),
              pack_bf16(__uint_as_float(dq[i + 4]) * s, __uint_as_float(dq[i + 5]) * s),
              pack_bf16(__uint_as_float(dq[i + 6]) * s, __uint_as_float(dq[i + 7]) * s));
      }
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

// 3-D bf16 map over [heads, rows, D] (D contiguous), box {64, box_rows, 1},
// 128-byte swizzle; rows past `rows` read as zero.
bool encode_map(CUtensorMap* m, const void* base, int D, long long rows, int heads, int box_rows) {
  return encode_map_3d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, D, rows, heads, 64, box_rows);
}

template <int D>
cudaError_t launch_typed(const BwdTcParams& prm, cudaStream_t st) {
  const int smem = BCfg<D>::SMEM;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = prm.n_rows < sms ? prm.n_rows : sms;   // persistent: one CTA per SM
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // a plain launch, as the forward attention kernel (see there)
  attn_bwd_tc_kernel<D><<<grid, kThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace

bool attention_bwd_tc_supported(const psa_params_t& p) {
  return p.dtype == PSA_BF16 && (p.q_blk == 128 || p.q_blk == 64) && p.kv_blk == 64 &&
         (p.d == 64 || p.d == 128);
}

cudaError_t launch_attention_bwd_tc(const psa_params_t& p, const Layout& L, const BwdLayout& B,
                                    const BwdArgs& a, cudaStream_t st) {
  BwdTcParams prm;
  memset(&prm, 0, sizeof(prm));
  const int BHq = p.B * p.Hq, BHk = p.B * p.Hkv;
  bool ok = encode_map(&prm.tq, a.Q, p.d, p.N, BHq, kBM) &&
            encode_map(&prm.tdo, a.dO, p.d, p.N, BHq, kBM);
  for (int l = 0; l < kLevels && ok; ++l) {
    const void* kb = l == 0 ? a.K : (const void*)(a.ws + L.kp[l]);
    const void* vb = l == 0 ? a.V : (const void*)(a.ws + L.vp[l]);
    ok = encode_map(&prm.tk[l], kb, p.d, (long long)L.rows[l], BHk, 64 >> l) &&
         encode_map(&prm.tv[l], vb, p.d, (long long)L.rows[l], BHk, 64 >> l);
  }
  if (!ok) return cudaErrorInvalidValue;
  prm.list = (const int*)(a.ws + L.list);
  prm.counts = (const int4*)(a.ws + L.counts);
  prm.lse = a.lse;
  prm.delta = reinterpret_cast<const float*>(a.bws + B.delta);
  for (int l = 0; l < kLevels; ++l) {
    prm.dk[l] = reinterpret_cast<float*>(a.bws + B.dk[l]);
    prm.dv[l] = reinterpret_cast<float*>(a.bws + B.dv[l]);
    prm.rows[l] = (long long)L.rows[l];
  }
  prm.dQ = (__nv_bfloat16*)a.dQ;
  prm.err = (int*)(a.ws + L.err);
  prm.Hq = p.Hq; prm.Hkv = p.Hkv; prm.N = p.N; prm.Nq = L.Nq; prm.Nk = L.Nk;
  prm.causal = p.causal;
  prm.n_rows = BHq * L.Nq;
  prm.qb = p.q_blk;
  prm.scale = a.scale;
  prm.scale_log2 = a.scale * kLog2e;
  return p.d == 128 ? launch_typed<128>(prm, st) : launch_typed<64>(prm, st);
}

}  // namespace psa
