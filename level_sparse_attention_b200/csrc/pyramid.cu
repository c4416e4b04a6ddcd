// Pyramid KV construction: average pooling of K and V into levels 1..3
// (2x, 4x, 8x), plus the level-3 keys in fp32 for block scoring, stored as a
// tf32 head and the exact remainder (the split operands of the scoring GEMM).
//
// Method: top168.com article on PSA (arXiv:2512.04025), pyramid paragraph and
// component one — the bottom level is the original KV and each level above is
// an average-pooled, coarser copy; "Psa Pyramid Sparse Attention" (skillmd),
// Core Technique — levels 1/2/3 pool 2/4/8 tokens.  Pooled row g of level l is
// the mean of tokens [g*2^l, min((g+1)*2^l, N)).
//
// Pure streaming, HBM-bound: every thread owns one group of 8 tokens x 4
// columns of K or V, reads it with 8 vector loads (8 B each for bf16) issued
// before any arithmetic, and writes the 4 + 2 + 1 pooled rows it determines
// (and the fp32 level-3 row for K).  Consecutive threads take consecutive
// 4-column chunks of the same rows, so each warp load/store covers whole
// 128-byte lines.  Index math is shifts and masks on a 3-D grid.
#include "psa_internal.cuh"

#include <type_traits>

namespace psa {
namespace {

// Four consecutive columns: 8 bytes of bf16 or 16 bytes of fp32.
template <typename T> struct Vec4;
template <> struct Vec4<__nv_bfloat16> {
  uint2 raw;
  __device__ void load(const __nv_bfloat16* p) { raw = *reinterpret_cast<const uint2*>(p); }
  __device__ void to_f32(float* f) const {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
  }
  __device__ static void store(__nv_bfloat16* p, const float* f) {
    __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(f[2], f[3]);
    uint2 o;
    o.x = *reinterpret_cast<uint32_t*>(&a);
    o.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = o;
  }
};
template <> struct Vec4<float> {
  float4 raw;
  __device__ void load(const float* p) { raw = *reinterpret_cast<const float4*>(p); }
  __device__ void to_f32(float* f) const { f[0] = raw.x; f[1] = raw.y; f[2] = raw.z; f[3] = raw.w; }
  __device__ static void store(float* p, const float* f) {
    *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  }
};

struct PyrArgs {
  int BH, N, d;
  int chunk_shift;               // log2(d / 4): 4-column chunks per row
  int groups;                    // ceil(N / 8)
  int rows1, rows2, rows3;
  int Nk;                        // KV blocks per head (cosine constraint)
  float theta;                   // cosine-similarity threshold
};

// mean of the first `n` of the summed values: sum / n (n = 1..8); exact for
// powers of two, correctly rounded otherwise.
__device__ __forceinline__ float mean_of(float sum, int n) {
  return (n & (n - 1)) == 0 ? sum * (1.0f / (float)n) : __fdiv_rn(sum, (float)n);
}

// 4 resident CTAs per SM for bf16 (64 registers, no spills): 32 warps per
// SM, each thread with 8 loads in flight.
template <typename T> struct PyrOcc { static constexpr int kMinBlocks = 4; };
template <> struct PyrOcc<float> { static constexpr int kMinBlocks = 2; };

// Pools one group of 8 tokens x 4 columns held in `raw` (rows past `valid`
// unused).  FULL: all 8 tokens lie inside N, every count is a power of two and
// every mean a multiplication; otherwise counts come from `valid`.
template <bool FULL, typename T>
__device__ __forceinline__ void pool_group(const Vec4<T>* raw, int valid, T* p1, T* p2, T* p3,
                                           float* pf, float* pl, int d) {
  // rows are consumed pairwise: each level-1 row is stored as soon as its
  // two tokens are summed, each level-2 row as soon as its two level-1 sums
  // are, so that few sums are live at once
  float s2[4], s3[4], m[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float x0[4], x1[4], s1[4];
    if (FULL || 2 * q < valid) raw[2 * q].to_f32(x0);
    else
#pragma unroll
      for (int e = 0; e < 4; ++e) x0[e] = 0.f;
    if (FULL || 2 * q + 1 < valid) raw[2 * q + 1].to_f32(x1);
    else
#pragma unroll
      for (int e = 0; e < 4; ++e) x1[e] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) s1[e] = x0[e] + x1[e];
    const int n1 = FULL ? 2 : min(2, valid - 2 * q);
    if (n1 > 0) {
#pragma unroll
      for (int e = 0; e < 4; ++e) m[e] = FULL ? s1[e] * 0.5f : mean_of(s1[e], n1);
      Vec4<T>::store(p1 + (size_t)q * d, m);
    }
    if ((q & 1) == 0) {
#pragma unroll
      for (int e = 0; e < 4; ++e) s2[e] = s1[e];
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) s2[e] += s1[e];
      const int h = q >> 1;
      const int n2 = FULL ? 4 : min(4, valid - 4 * h);
      if (n2 > 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) m[e] = FULL ? s2[e] * 0.25f : mean_of(s2[e], n2);
        Vec4<T>::store(p2 + (size_t)h * d, m);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) s3[e] = h == 0 ? s2[e] : s3[e] + s2[e];
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) m[e] = FULL ? s3[e] * 0.125f : mean_of(s3[e], valid);
  Vec4<T>::store(p3, m);
  if (pf) {                           // level-3 key in fp32 as tf32 head + exact tail
    float h[4], l[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      h[e] = tf32_head(m[e]);
      l[e] = m[e] - h[e];
    }
    Vec4<float>::store(pf, h);
    Vec4<float>::store(pl, l);
  }
}

// Cosine-similarity constraint on the pyramid levels, fused into the K pass.
//
// The top168.com article on PSA (ablations) names a cosine-similarity
// constraint on mask generation and its gain, without defining it.  The
// library's reading: every pooled row of level l >= 1 merges two rows of
// level l - 1 (token ranges [2g f, (2g+1) f) and [(2g+1) f, (2g+2) f) with
// f = 2^(l-1), cut at N); the merge is similar when the cosine of the two
// halves' mean keys is >= theta (an empty or zero half passes).  KV block j
// may be represented at level l when every merge at levels 1..l inside it is
// similar; the assignment lowers kept levels above that.
//
// Every merge lies inside one 8-token group, which the pyramid's threads
// already hold (d / 4 threads of 4 columns each).  A group's 7 merges (4 at
// level 1, 2 at level 2, 1 at level 3) need 21 partial sums (a . b, |a|^2,
// |b|^2 of the halves' sums, which point the same way as their means); each
// thread forms them over its 4 columns, the CTA adds them up per group in
// shared memory, and the 8 groups of a KV block decide its largest level
// (a CTA of 256 threads holds whole KV blocks: 1 for d = 128, 2 for d = 64).
constexpr int kSimSums = 21;

template <typename T>
__device__ __forceinline__ void merge_sums(const Vec4<T>* raw, int valid, float* part) {
  float x[8][4];
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    if (t < valid) raw[t].to_f32(x[t]);
    else
#pragma unroll
      for (int e = 0; e < 4; ++e) x[t][e] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < kSimSums; ++i) part[i] = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float s2[4], s4[2];
#pragma unroll
    for (int q = 0; q < 4; ++q) {             // level 1: tokens 2q | 2q + 1
      const float u = x[2 * q][c], w = x[2 * q + 1][c];
      part[3 * q] = fmaf(u, w, part[3 * q]);
      part[3 * q + 1] = fmaf(u, u, part[3 * q + 1]);
      part[3 * q + 2] = fmaf(w, w, part[3 * q + 2]);
      s2[q] = u + w;
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {             // level 2: tokens 4q, 4q+1 | 4q+2, 4q+3
      const float u = s2[2 * q], w = s2[2 * q + 1];
      part[12 + 3 * q] = fmaf(u, w, part[12 + 3 * q]);
      part[13 + 3 * q] = fmaf(u, u, part[13 + 3 * q]);
      part[14 + 3 * q] = fmaf(w, w, part[14 + 3 * q]);
      s4[q] = u + w;
    }
    part[18] = fmaf(s4[0], s4[1], part[18]);  // level 3: tokens 0..3 | 4..7
    part[19] = fmaf(s4[0], s4[0], part[19]);
    part[20] = fmaf(s4[1], s4[1], part[20]);
  }
}

// The K CTA's groups.  A group's G = d / 4 threads are G consecutive lanes (a
// whole warp at d = 128, half a warp at d = 64).  Their 21 partial sums
// (padded to 32) are added across the group by a reduce-scatter: at each step
// a lane keeps the half of its values that its lane bit selects and adds its
// partner's copy of that half, so that lane i of the group ends with the sums
// of values i (and 16 + i when G = 16).  The group's values go to shared
// memory, the group's first lane takes its largest allowed level, and after
// one barrier each KV block takes the minimum over its 8 groups.
template <int G, typename T>
__device__ __forceinline__ void similarity_blocks(const Vec4<T>* raw, int valid, const PyrArgs& a,
                                                  int bh, int8_t* maxlev, int iter) {
  __shared__ float s_sum[16][32];                  // per group of the CTA
  __shared__ int s_lv[2][16];                      // double-buffered by head iteration
  constexpr int NG = 256 / G;                      // groups per CTA: 8 or 16
  const int tid = threadIdx.x, lane = tid & 31;
  const int gl = tid / G;                          // group of this thread in the CTA
  const int li = tid % G;                          // lane inside the group
  float part[32];
  merge_sums(raw, valid, part);
#pragma unroll
  for (int i = kSimSums; i < 32; ++i) part[i] = 0.f;
  if constexpr (G == 32) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const bool upper = lane & o;
#pragma unroll
      for (int i = 0; i < o; ++i) {
        const float send = upper ? part[i] : part[i + o];
        const float keep = upper ? part[i + o] : part[i];
        part[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    s_sum[gl][li] = part[0];
  } else {
    // two 16-value halves, each reduce-scattered over the 16 lanes
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) {
      const bool upper = lane & o;
#pragma unroll
      for (int hh = 0; hh < 2; ++hh)
#pragma unroll
        for (int i = 0; i < o; ++i) {
          const float send = upper ? part[16 * hh + i] : part[16 * hh + i + o];
          const float keep = upper ? part[16 * hh + i + o] : part[16 * hh + i];
          part[16 * hh + i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    s_sum[gl][li] = part[0];
    s_sum[gl][16 + li] = part[16];
  }
  __syncwarp();
  const int g0 = (blockIdx.x * 256) / G;           // first group of the CTA
  if (li == 0) {
    const int nv = max(0, min(8, a.N - (g0 + gl) * 8));
    const float* f = s_sum[gl];
    // merge m: a . b = f[3m], |a|^2 = f[3m + 1], |b|^2 = f[3m + 2]; a zero half passes
    auto similar = [&](int m) {
      const float nn = f[3 * m + 1] * f[3 * m + 2];
      return nn == 0.f || f[3 * m] >= a.theta * sqrtf(nn);
    };
    bool ok1 = true, ok2 = true, ok3 = true;      // a merge exists when its second half has a token
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (2 * q + 1 < nv && !similar(q)) ok1 = false;
#pragma unroll
    for (int q = 0; q < 2; ++q)
      if (4 * q + 2 < nv && !similar(4 + q)) ok2 = false;
    if (4 < nv && !similar(6)) ok3 = false;
    s_lv[iter & 1][gl] = ok1 ? (ok2 ? (ok3 ? 3 : 2) : 1) : 0;
  }
  __syncthreads();
  if (tid < NG / 8) {
    const int j = g0 / 8 + tid;                      // KV block
    if (j < a.Nk) {
      int lv = 3;
#pragma unroll
      for (int k = 0; k < 8; ++k) lv = min(lv, s_lv[iter & 1][tid * 8 + k]);
      maxlev[(size_t)bh * a.Nk + j] = (int8_t)lv;
    }
  }
  // s_sum is rewritten by the next head only after every group of this one
  // has read its own row (__syncwarp above); s_lv alternates between heads
}

// grid: x = (groups << chunk_shift) / 256 rounded up, y = KV heads of all
// batches (strided), z = 0 for K, 1 for V.  SIM: the K CTAs also record each
// KV block's largest level under the cosine constraint (every thread of such
// a CTA takes its barriers, so none leaves early).
template <typename T, bool SIM>
__global__ void __launch_bounds__(256, SIM ? 3 : PyrOcc<T>::kMinBlocks)
pyramid_kernel(PyrArgs a, const T* __restrict__ K, const T* __restrict__ V, T* kp1, T* kp2,
               T* kp3, T* vp1, T* vp2, T* vp3, float* k3h, float* k3l, int8_t* maxlev) {
  pdl_trigger();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const bool is_v = blockIdx.z != 0;
  const bool live = i < (a.groups << a.chunk_shift);
  if constexpr (SIM) {
    if (!live && is_v) return;
  } else {
    if (!live) return;
  }
  const int c = i & ((1 << a.chunk_shift) - 1);
  const int g = i >> a.chunk_shift;
  // tokens of this group inside N (0 for a K thread past the end kept for the barriers)
  const int valid = SIM && !live ? 0 : min(8, a.N - g * 8);
  const T* base = is_v ? V : K;
  T* d1 = is_v ? vp1 : kp1;
  T* d2 = is_v ? vp2 : kp2;
  T* d3 = is_v ? vp3 : kp3;

  int it = 0;                                   // head iterations of this CTA
  for (int bh = blockIdx.y; bh < a.BH; bh += gridDim.y) {
    const T* src = base + ((size_t)bh * a.N + (size_t)g * 8) * a.d + c * 4;
    T* p1 = d1 + ((size_t)bh * a.rows1 + (size_t)g * 4) * a.d + c * 4;
    T* p2 = d2 + ((size_t)bh * a.rows2 + (size_t)g * 2) * a.d + c * 4;
    T* p3 = d3 + ((size_t)bh * a.rows3 + g) * a.d + c * 4;
    const size_t o3 = ((size_t)bh * a.rows3 + g) * a.d + c * 4;
    float* pf = is_v ? nullptr : k3h + o3;
    float* pl = is_v ? nullptr : k3l + o3;
    // all loads first, so that 8 are in flight per thread
    Vec4<T> raw[8];
    if (valid == 8) {
#pragma unroll
      for (int r = 0; r < 8; ++r) raw[r].load(src + (size_t)r * a.d);
      pool_group<true>(raw, 8, p1, p2, p3, pf, pl, a.d);
    } else if (!SIM || valid > 0) {
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < valid) raw[r].load(src + (size_t)r * a.d);
      pool_group<false>(raw, valid, p1, p2, p3, pf, pl, a.d);
    }
    if constexpr (SIM) {
      if (!is_v) {
        if (a.d == 128) similarity_blocks<32>(raw, valid, a, bh, maxlev, it);
        else similarity_blocks<16>(raw, valid, a, bh, maxlev, it);
      }
    }
    ++it;
  }
}

}  // namespace

cudaError_t launch_pyramid(const psa_params_t& p, const Layout& L, const void* K, const void* V,
                           char* ws, cudaStream_t st) {
  PyrArgs a;
  a.BH = p.B * p.Hkv;
  a.N = p.N;
  a.d = p.d;
  a.chunk_shift = p.d == 128 ? 5 : 4;     // d / 4 column chunks of 4 elements
  a.groups = (int)L.rows[3];
  a.rows1 = (int)L.rows[1];
  a.rows2 = (int)L.rows[2];
  a.rows3 = (int)L.rows[3];
  a.Nk = L.Nk;
  a.theta = p.sim_threshold;
  const int block = 256;
  const dim3 grid((unsigned)(((long long)a.groups << a.chunk_shift) + block - 1) / block,
                  (unsigned)min(a.BH, 65535), 2);
  const bool sim = p.sim_threshold > -1.f;
  int8_t* ml = (int8_t*)(ws + L.maxlev);
  auto go = [&](auto kern, auto* k, auto* v) -> cudaError_t {
    using T = std::remove_const_t<std::remove_pointer_t<decltype(k)>>;
    return launch_dependent(kern, grid, dim3(block), 0, st, a, k, v, (T*)(ws + L.kp[1]),
                            (T*)(ws + L.kp[2]), (T*)(ws + L.kp[3]), (T*)(ws + L.vp[1]),
                            (T*)(ws + L.vp[2]), (T*)(ws + L.vp[3]), (float*)(ws + L.k3h),
                            (float*)(ws + L.k3l), ml);
  };
  if (p.dtype == PSA_BF16) {
    using T = __nv_bfloat16;
    return sim ? go(pyramid_kernel<T, true>, (const T*)K, (const T*)V)
               : go(pyramid_kernel<T, false>, (const T*)K, (const T*)V);
  }
  return sim ? go(pyramid_kernel<float, true>, (const float*)K, (const float*)V)
             : go(pyramid_kernel<float, false>, (const float*)K, (const float*)V);
}

}  // namespace psa
