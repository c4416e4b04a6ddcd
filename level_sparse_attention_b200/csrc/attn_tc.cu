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
  static constexpr int STAGES = D == 128 ? 2 : 4;
  static constexpr int HALF = kBN * 128;            // bytes of one 64-column half tile
  static constexpr int Q_BYTES = kBM * D * 2;
  static constexpr int KV_BYTES = kBN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_META = OFF_V + STAGES * KV_BYTES;    // per stage: bias[128], kpos[128]
  static constexpr int OFF_BAR = OFF_META + STAGES * 1024;
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
  int Hq, Hkv, N, Nq, Nk, causal;
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

// ------------------------------------------------------------------ kernel

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  // barrier slots
  const int B_QFULL = 0, B_KFULL = 1, B_VFULL = 1 + C::STAGES, B_EMPTY = 1 + 2 * C::STAGES;
  const int B_SFULL = 1 + 3 * C::STAGES, B_PFULL = B_SFULL + 2, B_ODONE = B_PFULL + 2;
  const int B_FINAL = B_ODONE + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + B_FINAL + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row_id = blockIdx.x;                 // (b*Hq + hq) * Nq + qa
  const int qa = row_id % p.Nq;
  const int bhq = row_id / p.Nq;
  const int b = bhq / p.Hq, hq = bhq % p.Hq;
  const int bhk = b * p.Hkv + hq / (p.Hq / p.Hkv);
  const RowWork w = row_work(p.counts[row_id]);
  const int T = w.tiles;

  if (threadIdx.x == 0) {
    mbar_init(bar(B_QFULL), 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(bar(B_KFULL + s), 1);
      mbar_init(bar(B_VFULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_PFULL + i), 128);
      mbar_init(bar(B_ODONE + i), 1);
    }
    mbar_init(bar(B_FINAL), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // Zero the K/V stages once: rows of a partial last tile are never loaded, and
  // their (masked, P = 0) products must not meet NaN bit patterns.
  {
    uint4* kv = reinterpret_cast<uint4*>(smem + C::OFF_K);
    const int n16 = (2 * C::STAGES * C::KV_BYTES) / 16;
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
    if (T > 0) {
      if (lane == 0) {
        mbar_expect_tx(bar(B_QFULL), C::Q_BYTES);
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_3d(sbase + C::OFF_Q + h * (kBM * 128), &p.tq, bar(B_QFULL), h * 64,
                      qa * kBM, bhq);
      }
      const int* lrow = p.list + (long long)row_id * p.Nk;
      int e_next = 0;
      for (int t = 0; t < T; ++t) {
        const int s = t % C::STAGES;
        if (t >= C::STAGES &&
            !warp_wait(bar(B_EMPTY + s), ((t / C::STAGES) + 1) & 1, abort_flag, p.err))
          break;
        float* mbias = reinterpret_cast<float*>(smem + C::OFF_META + s * 1024);
        int* mpos = reinterpret_cast<int*>(mbias + kBN);
        const int e = e_next + lane;
        int l = 0;
        while (l < kLevels - 1 && e >= w.first[l + 1]) ++l;
        const int R = 64 >> l;
        const int off = w.base[l] + (e - w.first[l]) * R;
        const bool in_tile = e < w.first[kLevels] && off < (t + 1) * kBN;
        int j = 0, r0 = 0;
        if (in_tile) {
          j = lrow[e];
          r0 = off - t * kBN;
          const long long g0 = (long long)j * R;      // first level-l row of block j
          for (int rr = 0; rr < R; ++rr) {
            const long long g = g0 + rr;
            const long long tok = g << l;
            const int cg = (int)min((long long)(1 << l), (long long)p.N - tok);
            mbias[r0 + rr] = cg > 0 ? log2f((float)cg) : -INFINITY;
            mpos[r0 + rr] = (p.causal && l == 0) ? (int)tok : INT_MIN;
          }
        }
        const unsigned ballot = __ballot_sync(0xffffffffu, in_tile);
        const int n_in = __popc(ballot);
        if (t == T - 1) {      // keys after the last entry: no key
          for (int c = w.base[kLevels] - t * kBN + lane; c < kBN; c += 32) {
            if (c >= 0) {
              mbias[c] = -INFINITY;
              mpos[c] = INT_MIN;
            }
          }
        }
        int bytes = in_tile ? R * D * 2 : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) bytes += __shfl_xor_sync(0xffffffffu, bytes, o);
        __threadfence_block();
        __syncwarp();
        if (lane == 0) {
          mbar_expect_tx(bar(B_KFULL + s), bytes);
          mbar_expect_tx(bar(B_VFULL + s), bytes);
        }
        __syncwarp();
        if (in_tile) {
          const uint32_t kdst = sbase + C::OFF_K + s * C::KV_BYTES + r0 * 128;
          const uint32_t vdst = sbase + C::OFF_V + s * C::KV_BYTES + r0 * 128;
          for (int h = 0; h < C::HALVES; ++h)
            tma_load_3d(kdst + h * C::HALF, &p.tk[l], bar(B_KFULL + s), h * 64, j * R, bhk);
          for (int h = 0; h < C::HALVES; ++h)
            tma_load_3d(vdst + h * C::HALF, &p.tv[l], bar(B_VFULL + s), h * 64, j * R, bhk);
        }
        e_next += n_in;
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0 && T > 0) {
      constexpr uint32_t ID_QK = idesc_bf16(kBM, kBN, false);
      constexpr uint32_t ID_PV = idesc_bf16(kBM, D, true);
      bool ok = wait_bar(bar(B_QFULL), 0, abort_flag, p.err);
      auto issue_pv = [&](int u) -> bool {
        const int s = u % C::STAGES, bb = u & 1;
        if (!wait_bar(bar(B_PFULL + bb), (u >> 1) & 1, abort_flag, p.err)) return false;
        if (!wait_bar(bar(B_VFULL + s), (u / C::STAGES) & 1, abort_flag, p.err)) return false;
        tc_fence_after();
        const uint32_t vb = sbase + C::OFF_V + s * C::KV_BYTES;
#pragma unroll
        for (int k = 0; k < kBN / 16; ++k)
          mma_ts(T_O, T_P + bb * 64 + k * 8, sdesc(vb + k * 2048, C::HALF, 1024), ID_PV,
                 (u > 0 || k > 0) ? 1u : 0u);
        mma_commit(bar(B_ODONE + bb));
        mma_commit(bar(B_EMPTY + s));
        return true;
      };
      for (int t = 0; ok && t < T; ++t) {
        const int s = t % C::STAGES, bb = t & 1;
        if (!wait_bar(bar(B_KFULL + s), (t / C::STAGES) & 1, abort_flag, p.err)) { ok = false; break; }
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
        if (t >= 1 && !issue_pv(t - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(T - 1);
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
    const int qpos = qa * kBM + r;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    float m = -INFINITY, lsum = 0.f;
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int s = t % C::STAGES, bb = t & 1;
      if (!warp_wait(bar(B_SFULL + bb), (t >> 1) & 1, abort_flag, p.err) ||
          !warp_wait(bar(B_KFULL + s), (t / C::STAGES) & 1, abort_flag, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* mbias = reinterpret_cast<const float*>(smem + C::OFF_META + s * 1024);
      const int* mpos = reinterpret_cast<const int*>(mbias + kBN);
      float x[kBN];
#pragma unroll
      for (int c0 = 0; c0 < kBN; c0 += 32)
        tmem_ld32(T_S + bb * 128 + lane_off + c0, reinterpret_cast<uint32_t*>(x + c0));
      tmem_ld_wait();
      reg_fence<kBN>(reinterpret_cast<uint32_t*>(x));
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN; ++c) {
        float v = fmaf(x[c], p.scale_log2, mbias[c]);
        if (p.causal && qpos < mpos[c]) v = -INFINITY;
        x[c] = v;
        mt = fmaxf(mt, v);
      }
      const float m_new = fmaxf(m, mt);
      const bool need = m_new > m + kRescaleLog2;     // false while both are -inf
      if (__any_sync(0xffffffffu, need)) {
        const float m_use = need ? m_new : m;
        const float factor = need ? exp2f(m - m_use) : 1.f;   // 0 when m = -inf
        if (t > 0) {
          if (!warp_wait(bar(B_ODONE + ((t - 1) & 1)), ((t - 1) >> 1) & 1, abort_flag, p.err)) {
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
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int c = 0; c < kBN; c += 2) {
        const float p0 = exp2f(x[c] - m_base);
        const float p1 = exp2f(x[c + 1] - m_base);
        lsum += p0 + p1;
        __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
        pk[c / 2] = *reinterpret_cast<uint32_t*>(&h);
      }
      tmem_st32(T_P + bb * 64 + lane_off, pk);
      tmem_st32(T_P + bb * 64 + lane_off + 32, pk + 32);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_PFULL + bb));
    }
    // epilogue
    const bool row_ok = qpos < p.N;
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    __nv_bfloat16* dst = p.O + ((long long)bhq * p.N + qpos) * D;
    const bool have_o = __all_sync(0xffffffffu, ok) && T > 0 &&
                        warp_wait(bar(B_ODONE + ((T - 1) & 1)), ((T - 1) >> 1) & 1, abort_flag,
                                  p.err);
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
          __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(o[2 * i]) * inv,
                                                   __uint_as_float(o[2 * i + 1]) * inv);
          pk[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        uint4* d4 = reinterpret_cast<uint4*>(dst + c0);
#pragma unroll
        for (int i = 0; i < 4; ++i) d4[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
    if (row_ok && p.lse)
      p.lse[(long long)bhq * p.N + qpos] = lsum > 0.f ? (m + log2f(lsum)) * kLn2 : -INFINITY;
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
cudaError_t launch_tc_typed(const TcParams& prm, int grid, cudaStream_t st) {
  const int smem = Cfg<D>::SMEM;
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
  prm.scale_log2 = scale * kLog2e;
  const int grid = BHq * L.Nq;
  return p.d == 128 ? launch_tc_typed<128>(prm, grid, st) : launch_tc_typed<64>(prm, grid, st);
}

}  // namespace psa
