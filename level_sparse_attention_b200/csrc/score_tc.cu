// Block logits on the tensor cores in split precision.
//
// Method: multi-level mask generation (top168.com article on PSA, component
// two: levels follow the importance of query-key block pairs).  The block
// logit of query block a and KV block j is z = logsumexp over j's level-3
// pooled keys g of (s * q_bar_a . K3_g + ln c_g); the dot products form one
// GEMM per head, C = Q_bar [Nq x d] . K3 [rows3 x d]^T.
//
// The level map is compared bit for bit with an fp64 reference, so C must be
// fp32-accurate.  Each fp32 operand x is split into a tf32 head h (x with its
// low 13 mantissa bits cleared) and the tf32 part of the remainder l = x - h;
// C accumulates h_q h_k + h_q l_k + l_q h_k in fp32 on tcgen05 (kind::tf32),
// which leaves an error of about 2^-20 relative to sum |q_i k_i|, close to a
// plain fp32 dot product (the dropped l_q l_k term is below that).
//
// CTA tile: 128 query blocks x 256 keys (32 KV blocks), fp32 accumulator in
// TMEM (256 columns).  The head dimension is staged 32 elements at a time (one
// 128-byte swizzle row of fp32) into four shared tiles (A head/tail, B
// head/tail), double-buffered; 12 MMAs of 128x256x8 per stage.  The epilogue
// reads each query block's row of the accumulator and writes the logsumexp
// of every KV block's 8 keys.
#include "sm100_ptx.cuh"

namespace psa {
namespace {

using namespace ptx;

constexpr int kTM = 128;                 // query blocks per tile
constexpr int kTN = 256;                 // level-3 keys per tile
constexpr int kKC = 32;                  // head-dim elements per stage
constexpr int kThr = 256;
constexpr int kATile = kTM * kKC * 4;    // 16 KB
constexpr int kBTile = kTN * kKC * 4;    // 32 KB
constexpr int kStage = 2 * kATile + 2 * kBTile;   // A head, A tail, B head, B tail
constexpr int kOffBar = 2 * kStage;
constexpr int kSmem = kOffBar + 256 + 1024;

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

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// head / tail split of four fp32 values
__device__ __forceinline__ void split4(const float4 x, float4& h, float4& l) {
  auto hd = [](float v) { return __uint_as_float(__float_as_uint(v) & 0xffffe000u); };
  h = make_float4(hd(x.x), hd(x.y), hd(x.z), hd(x.w));
  l = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
}

template <int D>
__global__ void __launch_bounds__(kThr, 1)
    score_tc_kernel(MaskArgs a, int m_tiles, int n_tiles, const float* __restrict__ qmean,
                    const float* __restrict__ k3f, float* __restrict__ zlog, int* err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };   // 0,1: stage MMAs done; 2: all done

  int id = blockIdx.x;
  const int nt = id % n_tiles; id /= n_tiles;
  const int mt = id % m_tiles;
  const int bhq = id / m_tiles;
  const int b = bhq / a.Hq, hq = bhq % a.Hq;
  const int bhk = b * a.Hkv + hq / (a.Hq / a.Hkv);
  const long long rows3 = ((long long)a.N + 7) / 8;
  const int m0 = mt * kTM;
  const long long n0 = (long long)nt * kTN;
  const float* Ag = qmean + (long long)bhq * a.Nq * D;
  const float* Bg = k3f + (long long)bhk * rows3 * D;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < 3; ++i) mbar_init(bar(i), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(256)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Stage head-dim slice kc of the A (query-block means) and B (level-3 keys)
  // tiles, split into tf32 head and tail, in the 128-byte swizzled K-major
  // layout the MMA descriptors describe (16-byte chunk c of row r lands at
  // chunk c ^ (r & 7)).  The slice is first loaded into registers (all loads
  // in flight together), then split and stored.
  constexpr int NA = kTM * (kKC / 4) / kThr;     // float4 per thread: 4
  constexpr int NB = kTN * (kKC / 4) / kThr;     // 8
  float4 ra[NA], rb[NB];
  auto load = [&](int kc) {
#pragma unroll
    for (int k = 0; k < NA; ++k) {
      const int i = tid + k * kThr, r = i >> 3, c = i & 7;
      ra[k] = (m0 + r < a.Nq)
                  ? __ldg(reinterpret_cast<const float4*>(Ag + (long long)(m0 + r) * D + kc * kKC + c * 4))
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < NB; ++k) {
      const int i = tid + k * kThr, r = i >> 3, c = i & 7;
      rb[k] = (n0 + r < rows3)
                  ? __ldg(reinterpret_cast<const float4*>(Bg + (n0 + r) * D + kc * kKC + c * 4))
                  : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store = [&](int buf) {
    unsigned char* sb = smem + buf * kStage;
#pragma unroll
    for (int k = 0; k < NA; ++k) {
      const int i = tid + k * kThr, r = i >> 3, c = i & 7;
      float4 h, l;
      split4(ra[k], h, l);
      const int off = r * 128 + ((c ^ (r & 7)) << 4);
      *reinterpret_cast<float4*>(sb + off) = h;
      *reinterpret_cast<float4*>(sb + kATile + off) = l;
    }
#pragma unroll
    for (int k = 0; k < NB; ++k) {
      const int i = tid + k * kThr, r = i >> 3, c = i & 7;
      float4 h, l;
      split4(rb[k], h, l);
      const int off = r * 128 + ((c ^ (r & 7)) << 4);
      *reinterpret_cast<float4*>(sb + 2 * kATile + off) = h;
      *reinterpret_cast<float4*>(sb + 2 * kATile + kBTile + off) = l;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  };

  constexpr int NC = D / kKC;
  constexpr uint32_t ID = idesc_tf32(kTM, kTN);
  bool ok = true;
  load(0);
  store(0);
  tc_fence_before();
  __syncthreads();
  for (int kc = 0; kc < NC; ++kc) {
    const int buf = kc & 1;
    if (tid == 0 && ok) {
      tc_fence_after();
      const uint32_t sb = sbase + buf * kStage;
      const uint64_t ah = sdesc(sb, 16, 1024), al = sdesc(sb + kATile, 16, 1024);
      const uint64_t bh = sdesc(sb + 2 * kATile, 16, 1024);
      const uint64_t bl = sdesc(sb + 2 * kATile + kBTile, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < kKC / 8; ++ks) {        // 8 tf32 = 32 bytes per MMA
        const uint64_t o = (uint64_t)(ks * 2);       // +32 bytes in the start-address field
        mma_tf32(tmem, ah + o, bh + o, ID, (kc > 0 || ks > 0) ? 1u : 0u);
        mma_tf32(tmem, ah + o, bl + o, ID, 1u);
        mma_tf32(tmem, al + o, bh + o, ID, 1u);
      }
      mma_commit(bar(buf));
    }
    if (kc + 1 < NC) {
      const int nb = (kc + 1) & 1;
      load(kc + 1);                 // in flight while the MMAs of slice kc run
      if (kc >= 1) ok = ok && wait_bar(bar(nb), ((kc - 1) >> 1) & 1, abort_flag, err);
      if (ok) store(nb);
      tc_fence_before();
      ok = __syncthreads_and(ok);
    }
  }
  if (tid == 0) mma_commit(bar(2));
  ok = ok && wait_bar(bar(2), 0, abort_flag, err);
  tc_fence_after();

  // Epilogue: warps 0-3 hold TMEM lane quadrants 0-3 = query blocks m0 + row.
  // Logsumexp in log2 units (exact for the pooled-count term log2 8 = 3 of
  // full groups), block logits staged through shared memory (the staging
  // tiles are free now) so that each warp then writes whole 128-byte runs of
  // a query block's row.
  constexpr int kZPitch = kTN / 8 + 1;                    // 32 blocks + 1 (bank spread)
  float* zs = reinterpret_cast<float*>(smem);             // [kTM][kZPitch]
  const float sl2 = a.scale * 1.4426950408889634f;
  if (warp < 4 && __all_sync(0xffffffffu, ok)) {
    const int row = warp * 32 + lane;
    const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
    for (int c0 = 0; c0 < kTN; c0 += 32) {
      uint32_t v[32];
      tmem_ld32(taddr + c0, v);
      tmem_ld_wait();
      reg_fence<32>(v);
#pragma unroll
      for (int blk = 0; blk < 4; ++blk) {
        const long long j = n0 / 8 + (c0 >> 3) + blk;
        const bool tail = (j + 1) * 64 > a.N;               // ragged or missing groups
        float lg[8], mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const long long g = j * 8 + c;
          float l2c = 3.f;                                  // log2 8
          if (tail) {
            const long long cnt = min(8LL, (long long)a.N - g * 8);
            l2c = cnt > 0 ? log2f((float)cnt) : -INFINITY;
          }
          lg[c] = l2c == -INFINITY ? -INFINITY : fmaf(sl2, __uint_as_float(v[blk * 8 + c]), l2c);
          mx = fmaxf(mx, lg[c]);
        }
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < 8; ++c) sum += ex2(lg[c] - mx);   // ex2(-inf) = 0
        zs[row * kZPitch + (c0 >> 3) + blk] = (mx + lg2(sum)) * 0.6931471805599453f;
      }
    }
  }
  ok = __syncthreads_and(ok);
  if (ok) {
    // 8 warps x (one row of 32 blocks per step): coalesced 128-byte stores
    const long long j = n0 / 8 + lane;
    for (int row = warp; row < kTM; row += kThr / 32) {
      const int qa = m0 + row;
      if (qa < a.Nq && j < a.Nk) zlog[((long long)bhq * a.Nq + qa) * a.Nk + j] = zs[row * kZPitch + lane];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(256)
                 : "memory");
  }
}

}  // namespace

cudaError_t launch_score(const psa_params_t& p, const Layout& L, float scale, char* ws,
                         cudaStream_t st) {
  const MaskArgs a = make_mask_args(p, L, scale);
  const int m_tiles = (L.Nq + kTM - 1) / kTM;
  const int n_tiles = (int)((L.rows[3] + kTN - 1) / kTN);
  const long long grid = (long long)p.B * p.Hq * m_tiles * n_tiles;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const float* qm = (const float*)(ws + L.qmean);
  const float* k3 = (const float*)(ws + L.k3f);
  float* z = (float*)(ws + L.zlog);
  int* err = (int*)(ws + L.err);
  cudaError_t e;
  if (p.d == 128) {
    e = cudaFuncSetAttribute(score_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    score_tc_kernel<128><<<(unsigned)grid, kThr, kSmem, st>>>(a, m_tiles, n_tiles, qm, k3, z, err);
  } else {
    e = cudaFuncSetAttribute(score_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    score_tc_kernel<64><<<(unsigned)grid, kThr, kSmem, st>>>(a, m_tiles, n_tiles, qm, k3, z, err);
  }
  return cudaGetLastError();
}

}  // namespace psa
