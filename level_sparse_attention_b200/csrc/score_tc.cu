// Block logits on the tensor cores in split precision.
//
// Method: multi-level mask generation (top168.com article on PSA, component
// two: levels follow the importance of query-key block pairs).  The block
// logit of query block a and KV block j is z = logsumexp over j's level-3
// pooled keys g of (s * q_bar_a . K3_g + ln c_g); the dot products form one
// GEMM per head, C = Q_bar [Nq x d] . K3 [rows3 x d]^T.
//
// The level map is compared bit for bit with an fp64 reference, so C must be
// fp32-accurate.  Each fp32 operand x arrives split (by the kernels that
// produce it) into a tf32 head h (x with its low 13 mantissa bits cleared)
// and the remainder l = x - h; C accumulates h_q h_k + h_q l_k + l_q h_k in
// fp32 on tcgen05 (kind::tf32), which leaves an error of about 2^-20
// relative to sum |q_i k_i|, close to a plain fp32 dot product (the dropped
// l_q l_k term is below that).
//
// Persistent CTAs, one per SM, walk tiles of 128 query blocks x 256 level-3
// keys (32 KV blocks):
//   warp 0      TMA producer: per 32-wide slice of the head dimension, four
//               boxes (query-mean head and tail, 128 x 32; key head and tail,
//               256 x 32) into a 2-stage ring of 96 KB stages, 128-byte
//               swizzled, which is the K-major layout the MMA descriptors
//               describe;
//   warp 1      MMA issuer: 12 MMAs of 128 x 256 x 8 per slice into one of two
//               TMEM accumulators (256 columns each), so that a tile's
//               epilogue overlaps the next tile's MMAs;
//   warps 2-9   epilogue: one query block per thread (TMEM lane), two warps
//               per lane quadrant taking half of the tile's keys each;
//               logsumexp of every KV block's 8 keys in packed f32x2 math,
//               staged per warp in shared memory and written as 64-byte row
//               runs.
#include "sm100_ptx.cuh"
#include "tma_host.cuh"

#include <string.h>

namespace psa {
namespace {

using namespace ptx;

constexpr int kTM = 128;                 // query blocks per tile
constexpr int kTN = 256;                 // level-3 keys per tile (32 KV blocks)
constexpr int kKC = 32;                  // head-dim elements per slice (128 bytes of fp32)
constexpr int kStages = 2;
constexpr int kEpiWarps = 8;             // 2 per TMEM lane quadrant
constexpr int kThr = 64 + 32 * kEpiWarps;   // producer, MMA, epilogue
constexpr int kATile = kTM * kKC * 4;    // 16 KB
constexpr int kBTile = kTN * kKC * 4;    // 32 KB
constexpr int kStage = 2 * kATile + 2 * kBTile;   // A head, A tail, B head, B tail: 96 KB
constexpr int kEpiCols = kTN / 2;        // keys per epilogue warp
constexpr int kZPitch = kEpiCols / 8 + 1;   // 16 blocks + 1 (bank spread)
constexpr int kOffZ = kStages * kStage;
constexpr int kZBytes = kEpiWarps * 32 * kZPitch * 4;   // 32 rows per epilogue warp
constexpr int kOffBar = kOffZ + kZBytes;
constexpr int kSmem = kOffBar + 256 + 1024;       // + barriers, + 1024-byte alignment slack

// barrier indices
constexpr int B_FULL = 0;                // + stage
constexpr int B_EMPTY = B_FULL + kStages;
constexpr int B_TFULL = B_EMPTY + kStages;   // + accumulator
constexpr int B_TEMPTY = B_TFULL + 2;
constexpr int B_FINAL = B_TEMPTY + 2;
constexpr int kBars = B_FINAL + 1;

struct ScoreParams {
  CUtensorMap qh, ql;                    // [B*Hq, Nq, D] fp32
  CUtensorMap kh, kl;                    // [B*Hkv, rows3, D] fp32
  float* zlog;
  int* err;
  int Hq, Hkv, N, Nq, Nk;
  int m_tiles, n_tiles, n_items;
  float scale;
};

__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
  // D fp32, A and B tf32, both K-major
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}

__device__ __forceinline__ uint64_t f2pack(float a, float b) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(uint64_t v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
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
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

struct Tile {
  int bhq, bhk, m0, n0;
};
__device__ __forceinline__ Tile tile_of(const ScoreParams& p, int item) {
  Tile t;
  const int nt = item % p.n_tiles;
  const int rest = item / p.n_tiles;
  const int mt = rest % p.m_tiles;
  t.bhq = rest / p.m_tiles;
  const int b = t.bhq / p.Hq, hq = t.bhq % p.Hq;
  t.bhk = b * p.Hkv + hq / (p.Hq / p.Hkv);
  t.m0 = mt * kTM;
  t.n0 = nt * kTN;
  return t;
}

template <int D>
__global__ void __launch_bounds__(kThr, 1) score_tc_kernel(const __grid_constant__ ScoreParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NC = D / kKC;            // slices per tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(B_TFULL + b), 1);
      mbar_init(bar(B_TEMPTY + b), kEpiWarps);   // one arrival per epilogue warp
    }
    mbar_init(bar(B_FINAL), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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
  pdl_trigger();
  pdl_wait();                               // query means and level-3 keys are complete

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.qh)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.ql)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.kh)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.kl)) : "memory");
      int it = 0;                        // slices issued
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x) {
        const Tile t = tile_of(p, item);
        for (int kc = 0; kc < NC; ++kc) {
          const int s = it % kStages;
          if (it >= kStages &&
              !wait_bar(bar(B_EMPTY + s), ((it / kStages) + 1) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          const uint32_t dst = sbase + s * kStage;
          const uint32_t fb = bar(B_FULL + s);
          mbar_expect_tx(fb, kStage);
          tma_load_3d(dst, &p.qh, fb, kc * kKC, t.m0, t.bhq);
          tma_load_3d(dst + kATile, &p.ql, fb, kc * kKC, t.m0, t.bhq);
          tma_load_3d(dst + 2 * kATile, &p.kh, fb, kc * kKC, t.n0, t.bhk);
          tma_load_3d(dst + 2 * kATile + kBTile, &p.kl, fb, kc * kKC, t.n0, t.bhk);
          ++it;
        }
      }
      // no copy may still be in flight when the CTA exits: wait (bounded)
      // for the last slices issued; phases already consumed pass at once
      for (int k = it - kStages; k < it; ++k) {
        if (k < 0) continue;
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(bar(B_FULL + k % kStages), (k / kStages) & 1) &&
               global_ns() - t0 < kTimeoutNs) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t ID = idesc_tf32(kTM, kTN);
      int it = 0, tl = 0;                // slices consumed, tiles of this CTA
      bool ok = true;
      for (int item = blockIdx.x; ok && item < p.n_items; item += gridDim.x, ++tl) {
        const int b = tl & 1;
        if (tl >= 2 && !wait_bar(bar(B_TEMPTY + b), ((tl >> 1) + 1) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + b * kTN;
        for (int kc = 0; kc < NC; ++kc, ++it) {
          const int s = it % kStages;
          if (!wait_bar(bar(B_FULL + s), (it / kStages) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = sbase + s * kStage;
          const uint64_t ah = sdesc(sb, 16, 1024), al = sdesc(sb + kATile, 16, 1024);
          const uint64_t bh = sdesc(sb + 2 * kATile, 16, 1024);
          const uint64_t bl = sdesc(sb + 2 * kATile + kBTile, 16, 1024);
#pragma unroll
          for (int ks = 0; ks < kKC / 8; ++ks) {      // 8 tf32 = 32 bytes per MMA
            const uint64_t o = (uint64_t)(ks * 2);     // +32 bytes in the start-address field
            mma_tf32(acc, ah + o, bh + o, ID, (kc > 0 || ks > 0) ? 1u : 0u);
            mma_tf32(acc, ah + o, bl + o, ID, 1u);
            mma_tf32(acc, al + o, bh + o, ID, 1u);
          }
          mma_commit(bar(B_EMPTY + s));             // stage free once these MMAs complete
        }
        if (!ok) break;
        mma_commit(bar(B_TFULL + b));               // accumulator b holds the tile
      }
      // drain: every MMA issued so far completes before TMEM is released
      mma_commit(bar(B_FINAL));
      const uint64_t t0 = global_ns();
      while (!mbar_try_wait(bar(B_FINAL), 0) && global_ns() - t0 < kTimeoutNs) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp w reads TMEM lane quadrant w % 4 (query blocks m0 + 32 (w % 4) +
    // lane) and key half (w - 2) / 4 of the tile
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    float* zs = reinterpret_cast<float*>(smem + kOffZ) + (warp - 2) * 32 * kZPitch;
    const float sl2 = p.scale * 1.4426950408889634f;      // > 0
    const uint64_t sl2x2 = f2pack(sl2, sl2);
    int tl = 0;
    for (int item = blockIdx.x; item < p.n_items; item += gridDim.x, ++tl) {
      const int b = tl & 1;
      if (!warp_wait(bar(B_TFULL + b), (tl >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      const Tile t = tile_of(p, item);
      const int j0 = t.n0 / 8 + half * (kEpiCols / 8);    // first KV block of this warp
      const uint32_t taddr = tmem + b * kTN + half * kEpiCols + ((uint32_t)(quad * 32) << 16);
#pragma unroll 1
      for (int c0 = 0; c0 < kEpiCols; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(taddr + c0, v);
        tmem_ld_wait();
        reg_fence<32>(v);
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
          const int j = j0 + (c0 >> 3) + blk;
          const uint32_t* u = v + blk * 8;
          float z;
          if ((j + 1) * 64 <= p.N) {
            // 8 full groups: logit = sl2 * dot + log2 8; the block maximum of
            // the dots gives the shift, exp2(sl2 * (dot - max)) the terms
            const float m = fmax3(fmax3(__uint_as_float(u[0]), __uint_as_float(u[1]), __uint_as_float(u[2])),
                                  fmax3(__uint_as_float(u[3]), __uint_as_float(u[4]), __uint_as_float(u[5])),
                                  fmaxf(__uint_as_float(u[6]), __uint_as_float(u[7])));
            const uint64_t nm = f2pack(-sl2 * m, -sl2 * m);
            uint64_t acc = f2pack(0.f, 0.f);
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
              float e0, e1;
              f2unpack(ffma2(f2pack(__uint_as_float(u[c]), __uint_as_float(u[c + 1])), sl2x2, nm), e0, e1);
              acc = fadd2(acc, f2pack(ex2(e0), ex2(e1)));
            }
            float a0, a1;
            f2unpack(acc, a0, a1);
            z = (fmaf(sl2, m, 3.f) + lg2(a0 + a1)) * 0.6931471805599453f;
          } else {
            // ragged or missing groups at the end of the sequence
            float lg[8], mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const int cnt = min(8, p.N - (j * 8 + c) * 8);
              lg[c] = cnt > 0 ? fmaf(sl2, __uint_as_float(u[c]), log2f((float)cnt)) : -INFINITY;
              mx = fmaxf(mx, lg[c]);
            }
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) sum += ex2(lg[c] - mx);   // ex2(-inf) = 0
            z = (mx + lg2(sum)) * 0.6931471805599453f;
          }
          zs[lane * kZPitch + (c0 >> 3) + blk] = z;
        }
      }
      // accumulator b may be overwritten once every epilogue warp has read it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_TEMPTY + b));
      // this warp's 32 query blocks x 16 KV blocks: lanes 0-15 write row r,
      // lanes 16-31 row r + 1, each a 64-byte run
      const int j = j0 + (lane & 15);
#pragma unroll 4
      for (int r = 0; r < 32; r += 2) {
        const int rr = r + (lane >> 4);
        const int qa = t.m0 + quad * 32 + rr;
        if (qa < p.Nq && j < p.Nk)
          p.zlog[((long long)t.bhq * p.Nq + qa) * p.Nk + j] = zs[rr * kZPitch + (lane & 15)];
      }
      __syncwarp();
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

}  // namespace

cudaError_t launch_score(const psa_params_t& p, const Layout& L, float scale, char* ws,
                         cudaStream_t st) {
  ScoreParams prm;
  memset(&prm, 0, sizeof(prm));
  const int BHq = p.B * p.Hq, BHk = p.B * p.Hkv;
  const long long rows3 = (long long)L.rows[3];
  const CUtensorMapDataType f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  bool ok = encode_map_3d(&prm.qh, f32, 4, ws + L.qmh, p.d, L.Nq, BHq, kKC, kTM) &&
            encode_map_3d(&prm.ql, f32, 4, ws + L.qml, p.d, L.Nq, BHq, kKC, kTM) &&
            encode_map_3d(&prm.kh, f32, 4, ws + L.k3h, p.d, rows3, BHk, kKC, kTN) &&
            encode_map_3d(&prm.kl, f32, 4, ws + L.k3l, p.d, rows3, BHk, kKC, kTN);
  if (!ok) return cudaErrorInvalidValue;
  prm.zlog = (float*)(ws + L.zlog);
  prm.err = (int*)(ws + L.err);
  prm.Hq = p.Hq; prm.Hkv = p.Hkv; prm.N = p.N; prm.Nq = L.Nq; prm.Nk = L.Nk;
  prm.m_tiles = (L.Nq + kTM - 1) / kTM;
  prm.n_tiles = (int)((rows3 + kTN - 1) / kTN);
  const long long items = (long long)BHq * prm.m_tiles * prm.n_tiles;
  if (items > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  prm.n_items = (int)items;
  prm.scale = scale;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = prm.n_items < sms ? prm.n_items : sms;   // persistent: one CTA per SM
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    return launch_dependent(kern, dim3(grid), dim3(kThr), kSmem, st, prm);
  };
  return p.d == 128 ? go(score_tc_kernel<128>) : go(score_tc_kernel<64>);
}

}  // namespace psa
