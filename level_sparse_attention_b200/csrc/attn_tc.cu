// Pyramid attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA),
// bf16 inputs, fp32 accumulation, 128-row query blocks, d in {64, 128}.
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
// CTA = one (batch, query head, 128-row query block), 6 warps:
//   warp 0     TMA producer: Q once; per tile, one 2-D box per sub-block and
//              64-column half for K and for V (the box height is the level's
//              sub-block height), plus a per-key bias / position table.
//   warp 1     TMEM allocator and single-thread tcgen05.mma issuer:
//              S[t%2] = Q K_t^T (SS form), then O += P_t V_t with P read from
//              TMEM (TS form); commits signal the softmax and free stages.
//   warps 2-5  softmax: one query row per thread (TMEM lane = row), online
//              softmax in log2 units, P written back to TMEM as bf16, lazy O
//              rescale (only when the running max grows by more than 2^8),
//              epilogue O / lse.
// TMEM columns: S0 [0,128) S1 [128,256) P0 [256,320) P1 [320,384) O [384,384+d).
// Every mbarrier wait is bounded: on expiry the kernel records a timeout in
// the workspace error word and winds down without trapping.
#include "psa_internal.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace psa {
namespace {

constexpr int kBM = 128;                 // query rows per CTA
constexpr int kBN = 128;                 // keys per packed tile
constexpr int kThreads = 192;
constexpr uint64_t kTimeoutNs = 2000000000ull;
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
  static constexpr int OFF_BAR = OFF_META + MSTAGES * 1024;
  static constexpr int SMEM = OFF_BAR + 512 + 1024;             // + slack for 1024 alignment
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
  float scale_log2;
};

// ------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait on phase `parity` of `bar`.  Returns false when the CTA is
// winding down (this or another role timed out).
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (global_ns() - t0 > kTimeoutNs) {
      *abort_flag = 1;
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
}

// All lanes wait; the warp proceeds only if every lane saw the phase.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          int* err) {
  const bool ok = wait_bar(bar, parity, abort_flag, err);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (tcgen05 format: start >> 4
// in bits 0-13, leading byte offset >> 4 in 16-29, stride byte offset >> 4 in
// 32-45, version 1 in bits 46-47, layout type 2 = SWIZZLE_128B in bits 61-63).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, A K-major,
// B K-major (QK^T) or MN-major (PV), shape M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                       uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

#define PSA_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                  "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define PSA_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                  "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 consecutive TMEM columns of this warp's 32 lanes -> 32 registers per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : PSA_R8(0), PSA_R8(8), PSA_R8(16), PSA_R8(24)
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      PSA_W8(0), PSA_W8(8), PSA_W8(16), PSA_W8(24)
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// Ties registers written by tcgen05.ld to the preceding wait::ld so that no
// use is scheduled above it.
template <int N>
__device__ __forceinline__ void reg_fence(uint32_t* r) {
#pragma unroll
  for (int i = 0; i < N; ++i) asm volatile("" : "+r"(r[i]));
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------ work list

struct RowWork {
  int first[kLevels + 1];   // entry index where level l starts (first[4] = entries)
  int base[kLevels + 1];    // packed key offset where level l starts (base[4] = keys)
  int tiles;
};

__device__ __forceinline__ RowWork row_work(int4 c) {
  RowWork w;
  const int n[kLevels] = {c.x, c.y, c.z, c.w};
  w.first[0] = 0;
  w.base[0] = 0;
  for (int l = 0; l < kLevels; ++l) {
    w.first[l + 1] = w.first[l] + n[l];
    w.base[l + 1] = w.base[l] + n[l] * (64 >> l);
  }
  w.tiles = (w.base[kLevels] + kBN - 1) / kBN;
  return w;
}

// The entries of tile t, one per lane: lane i takes entry e0 + i.  Entries
// never cross a tile edge, so the lanes inside the tile form a prefix.
struct TileEntry {
  bool in_tile;
  int j, l, R, r0;          // KV block, level, sub-block rows, first row in the tile
};

__device__ __forceinline__ TileEntry tile_entry(const RowWork& w, const int* lrow, int e0, int t,
                                                int lane) {
  TileEntry te;
  const int e = e0 + lane;
  int l = 0;
  while (l < kLevels - 1 && e >= w.first[l + 1]) ++l;
  te.l = l;
  te.R = 64 >> l;
  const int off = w.base[l] + (e - w.first[l]) * te.R;
  te.in_tile = e < w.first[kLevels] && off < (t + 1) * kBN;
  te.r0 = off - t * kBN;
  te.j = te.in_tile ? __ldg(lrow + e) : 0;
  return te;
}

// Items (query blocks) of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
// Consecutive CTAs take consecutive query blocks of the same head, so the
// head's K/V and pyramid stay in L2 while its query blocks are processed.

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<D>;
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
  constexpr int B_SFULL = B_MEMPTY + MS, B_PFULL = B_SFULL + 2, B_ODONE = B_PFULL + 2;
  constexpr int B_FINAL = B_ODONE + 2, NBARS = B_FINAL + 1;
  static_assert(NBARS * 8 + 16 <= 512, "barrier area");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NBARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.n_rows;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    mbar_init(bar(B_QEMPTY), 1);
    for (int s = 0; s < KS; ++s) { mbar_init(bar(B_KFULL + s), 1); mbar_init(bar(B_KEMPTY + s), 1); }
    for (int s = 0; s < VS; ++s) { mbar_init(bar(B_VFULL + s), 1); mbar_init(bar(B_VEMPTY + s), 1); }
    for (int s = 0; s < MS; ++s) { mbar_init(bar(B_MFULL + s), 1); mbar_init(bar(B_MEMPTY + s), 4); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_PFULL + i), 128);
      mbar_init(bar(B_ODONE + i), 1);
    }
    mbar_init(bar(B_FINAL), 1);
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
  const uint32_t T_S = tmem, T_P = tmem + 256, T_O = tmem + 384;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int gk = 0, gv = 0, iq = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
      const RowWork w = row_work(p.counts[item]);
      const int T = w.tiles;
      if (T == 0) continue;
      const int qa = item % p.Nq, bhq = item / p.Nq;
      const int bhk = (bhq / p.Hq) * p.Hkv + (bhq % p.Hq) / (p.Hq / p.Hkv);
      const int* lrow = p.list + (long long)item * p.Nk;
      if (iq > 0 && !warp_wait(bar(B_QEMPTY), (iq - 1) & 1, abort_flag, p.err)) { ok = false; break; }
      if (lane == 0) {
        mbar_expect_tx(bar(B_QFULL), C::Q_BYTES);
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_3d(sbase + C::OFF_Q + h * (kBM * 128), &p.tq, bar(B_QFULL), h * 64,
                      qa * kBM, bhq);
      }
      ++iq;
      int ek = 0, ev = 0;
      for (int t = 0; t <= T; ++t) {
        if (t < T) {
          // K of tile t, and its per-key bias / position table
          const int s = gk % KS, ms = gk % MS;
          if (gk >= KS && !warp_wait(bar(B_KEMPTY + s), ((gk / KS) + 1) & 1, abort_flag, p.err)) { ok = false; break; }
          if (gk >= MS && !warp_wait(bar(B_MEMPTY + ms), ((gk / MS) + 1) & 1, abort_flag, p.err)) { ok = false; break; }
          const TileEntry te = tile_entry(w, lrow, ek, t, lane);
          const unsigned ballot = __ballot_sync(0xffffffffu, te.in_tile);
          const int n_in = __popc(ballot);
          int bytes = te.in_tile ? te.R * D * 2 : 0;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, o);
          // table: lane covers columns 4*lane .. 4*lane+3 (inside one 8-column chunk)
          const int col = 4 * lane;
          int owner = 0;
          for (int i = 1; i < n_in; ++i)
            if (__shfl_sync(0xffffffffu, te.r0, i) <= col) owner = i;
          const int oj = __shfl_sync(0xffffffffu, te.j, owner);
          const int ol = __shfl_sync(0xffffffffu, te.l, owner);
          const int oR = __shfl_sync(0xffffffffu, te.R, owner);
          const int or0 = __shfl_sync(0xffffffffu, te.r0, owner);
          const bool live = n_in > 0 && col < or0 + oR;   // false past the last entry
          float bias[4];
          int kpos[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const long long g = (long long)oj * oR + (col + c - or0);
            const long long tok = g << ol;
            const int cnt = (int)min((long long)(1 << ol), (long long)p.N - tok);
            bias[c] = !live || cnt <= 0 ? -INFINITY : (cnt == (1 << ol) ? (float)ol : log2f((float)cnt));
            kpos[c] = (live && p.causal && ol == 0) ? (int)tok : INT_MIN;
          }
          float* mb = reinterpret_cast<float*>(smem + C::OFF_META + ms * 1024);
          reinterpret_cast<float4*>(mb)[lane] = make_float4(bias[0], bias[1], bias[2], bias[3]);
          reinterpret_cast<int4*>(mb + kBN)[lane] = make_int4(kpos[0], kpos[1], kpos[2], kpos[3]);
          __threadfence_block();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(bar(B_MFULL + ms));
            mbar_expect_tx(bar(B_KFULL + s), bytes);
          }
          __syncwarp();
          if (te.in_tile) {
            const uint32_t kdst = sbase + C::OFF_K + s * C::KV_BYTES + te.r0 * 128;
            for (int h = 0; h < C::HALVES; ++h)
              tma_load_3d(kdst + h * C::HALF, &p.tk[te.l], bar(B_KFULL + s), h * 64, te.j * te.R, bhk);
          }
          ek += n_in;
          ++gk;
        }
        if (t >= 1) {
          // V of tile t - 1
          const int s = gv % VS;
          if (gv >= VS && !warp_wait(bar(B_VEMPTY + s), ((gv / VS) + 1) & 1, abort_flag, p.err)) { ok = false; break; }
          const TileEntry te = tile_entry(w, lrow, ev, t - 1, lane);
          const int n_in = __popc(__ballot_sync(0xffffffffu, te.in_tile));
          int bytes = te.in_tile ? te.R * D * 2 : 0;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, o);
          if (lane == 0) mbar_expect_tx(bar(B_VFULL + s), bytes);
          __syncwarp();
          if (te.in_tile) {
            const uint32_t vdst = sbase + C::OFF_V + s * C::KV_BYTES + te.r0 * 128;
            for (int h = 0; h < C::HALVES; ++h)
              tma_load_3d(vdst + h * C::HALF, &p.tv[te.l], bar(B_VFULL + s), h * 64, te.j * te.R, bhk);
          }
          ev += n_in;
          ++gv;
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID_QK = idesc_bf16(kBM, kBN, false);
      constexpr uint32_t ID_PV = idesc_bf16(kBM, D, true);
      bool ok = true;
      auto issue_pv = [&](int u, bool first) -> bool {
        const int s = u % VS, bb = u & 1;
        if (!wait_bar(bar(B_PFULL + bb), (u >> 1) & 1, abort_flag, p.err)) return false;
        if (!wait_bar(bar(B_VFULL + s), (u / VS) & 1, abort_flag, p.err)) return false;
        tc_fence_after();
        const uint32_t vb = sbase + C::OFF_V + s * C::KV_BYTES;
#pragma unroll
        for (int k = 0; k < kBN / 16; ++k)
          mma_ts(T_O, T_P + bb * 64 + k * 8, sdesc(vb + k * 2048, C::HALF, 1024), ID_PV,
                 (first && k == 0) ? 0u : 1u);
        mma_commit(bar(B_ODONE + bb));
        mma_commit(bar(B_VEMPTY + s));
        return true;
      };
      int g = 0, iq = 0;
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
        const int T = row_work(p.counts[item]).tiles;
        if (T == 0) continue;
        if (!wait_bar(bar(B_QFULL), iq & 1, abort_flag, p.err)) { ok = false; break; }
        ++iq;
        for (int t = 0; t < T; ++t) {
          const int gk = g + t, s = gk % KS, bb = gk & 1;
          if (!wait_bar(bar(B_KFULL + s), (gk / KS) & 1, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kb = sbase + C::OFF_K + s * C::KV_BYTES;
          const uint32_t qb = sbase + C::OFF_Q;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t koff = (k >> 2) * C::HALF + (k & 3) * 32;
            const uint32_t qoff = (k >> 2) * (kBM * 128) + (k & 3) * 32;
            mma_ss(T_S + bb * 128, sdesc(qb + qoff, 16, 1024), sdesc(kb + koff, 16, 1024), ID_QK,
                   k > 0 ? 1u : 0u);
          }
          mma_commit(bar(B_SFULL + bb));
          mma_commit(bar(B_KEMPTY + s));
          if (t == T - 1) mma_commit(bar(B_QEMPTY));
          if (t >= 1 && !issue_pv(gk - 1, t == 1)) { ok = false; break; }
        }
        if (!ok || !issue_pv(g + T - 1, T == 1)) { ok = false; break; }
        g += T;
      }
      // drain: every MMA issued so far completes before TMEM is released
      mma_commit(bar(B_FINAL));
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(bar(B_FINAL), 0) && global_ns() - t0 < kTimeoutNs) {
      }
    }
  } else {
    // --------------------------------------------------------------- softmax
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    int g = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
      const int T = row_work(p.counts[item]).tiles;
      const int qa = item % p.Nq, bhq = item / p.Nq;
      const int qpos = qa * kBM + r;
      float m = -INFINITY, lsum = 0.f;
      for (int t = 0; ok && t < T; ++t) {
        const int gt = g + t, bb = gt & 1, ms = gt % MS;
        if (!warp_wait(bar(B_SFULL + bb), (gt >> 1) & 1, abort_flag, p.err) ||
            !warp_wait(bar(B_MFULL + ms), (gt / MS) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* mbias = reinterpret_cast<const float*>(smem + C::OFF_META + ms * 1024);
        const int* mpos = reinterpret_cast<const int*>(mbias + kBN);
        float x[kBN];
#pragma unroll
        for (int c0 = 0; c0 < kBN; c0 += 32)
          tmem_ld32(T_S + bb * 128 + lane_off + c0, reinterpret_cast<uint32_t*>(x + c0));
        tmem_ld_wait();
        reg_fence<kBN>(reinterpret_cast<uint32_t*>(x));
        float mt = -INFINITY;
#pragma unroll
        for (int c = 0; c < kBN; c += 4) {
          const float4 b4 = *reinterpret_cast<const float4*>(mbias + c);
          x[c] = fmaf(x[c], p.scale_log2, b4.x);
          x[c + 1] = fmaf(x[c + 1], p.scale_log2, b4.y);
          x[c + 2] = fmaf(x[c + 2], p.scale_log2, b4.z);
          x[c + 3] = fmaf(x[c + 3], p.scale_log2, b4.w);
          if (p.causal) {
            const int4 k4 = *reinterpret_cast<const int4*>(mpos + c);
            if (qpos < k4.x) x[c] = -INFINITY;
            if (qpos < k4.y) x[c + 1] = -INFINITY;
            if (qpos < k4.z) x[c + 2] = -INFINITY;
            if (qpos < k4.w) x[c + 3] = -INFINITY;
          }
          mt = fmaxf(mt, fmaxf(fmaxf(x[c], x[c + 1]), fmaxf(x[c + 2], x[c + 3])));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_MEMPTY + ms));
        const float m_new = fmaxf(m, mt);
        const bool need = m_new > m + kRescaleLog2;     // false while both are -inf
        if (__any_sync(0xffffffffu, need)) {
          const float m_use = need ? m_new : m;
          const float factor = need ? ex2(m - m_use) : 1.f;   // 0 when m = -inf
          if (t > 0) {
            if (!warp_wait(bar(B_ODONE + ((gt - 1) & 1)), ((gt - 1) >> 1) & 1, abort_flag, p.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(T_O + lane_off + c0, o);
              tmem_ld_wait();
              reg_fence<32>(o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * factor);
              tmem_st32(T_O + lane_off + c0, o);
            }
          }
          lsum *= factor;
          m = m_use;
        }
        const float m_base = m == -INFINITY ? 0.f : m;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float p0 = ex2(x[h * 64 + c] - m_base);
            const float p1 = ex2(x[h * 64 + c + 1] - m_base);
            lsum += p0 + p1;
            __nv_bfloat162 hh = __floats2bfloat162_rn(p0, p1);
            pk[c / 2] = *reinterpret_cast<uint32_t*>(&hh);
          }
          tmem_st32(T_P + bb * 64 + lane_off + h * 32, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(B_PFULL + bb));
      }
      // epilogue of this query block
      const bool row_ok = qpos < p.N;
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      __nv_bfloat16* dst = p.O + ((long long)bhq * p.N + qpos) * D;
      const bool have_o = __all_sync(0xffffffffu, ok) && T > 0 &&
                          warp_wait(bar(B_ODONE + ((g + T - 1) & 1)), ((g + T - 1) >> 1) & 1,
                                    abort_flag, p.err);
      if (have_o) tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t o[32];
        if (have_o) {
          tmem_ld32(T_O + lane_off + c0, o);
          tmem_ld_wait();
          reg_fence<32>(o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        if (row_ok) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            __nv_bfloat162 hh = __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * inv,
                                                      __uint_as_float(o[2 * i + 1]) * inv);
            pk[i] = *reinterpret_cast<uint32_t*>(&hh);
          }
          uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        }
      }
      if (row_ok && p.lse)
        p.lse[(long long)bhq * p.N + qpos] = lsum > 0.f ? (m + log2f(lsum)) * kLn2 : -INFINITY;
      g += T;
      if (!ok) break;
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

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 3-D bf16 map over [heads, rows, D] (D contiguous), box {64, box_rows, 1},
// 128-byte swizzle; rows past `rows` read as zero.
bool encode_map(CUtensorMap* m, const void* base, int D, long long rows, int heads, int box_rows) {
  auto fn = get_encode();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)heads};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  const cuuint32_t box[3] = {64u, (cuuint32_t)box_rows, 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
  attn_tc_kernel<D><<<grid, kThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace

bool attention_tc_supported(const psa_params_t& p) {
  return p.dtype == PSA_BF16 && p.q_blk == 128 && p.kv_blk == 64 && (p.d == 64 || p.d == 128);
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
  prm.scale_log2 = scale * kLog2e;
  return p.d == 128 ? launch_tc_typed<128>(prm, prm.n_rows, st)
                    : launch_tc_typed<64>(prm, prm.n_rows, st);
}

}  // namespace psa
