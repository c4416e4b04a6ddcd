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

// grid: x = (groups << chunk_shift) / 256 rounded up, y = KV heads of all
// batches (strided), z = 0 for K, 1 for V.
template <typename T>
__global__ void __launch_bounds__(256, PyrOcc<T>::kMinBlocks)
pyramid_kernel(PyrArgs a, const T* __restrict__ K, const T* __restrict__ V, T* kp1, T* kp2,
               T* kp3, T* vp1, T* vp2, T* vp3, float* k3h, float* k3l) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= (a.groups << a.chunk_shift)) return;
  const int c = i & ((1 << a.chunk_shift) - 1);
  const int g = i >> a.chunk_shift;
  const bool is_v = blockIdx.z != 0;
  const int valid = min(8, a.N - g * 8);   // tokens of this group inside N
  const T* base = is_v ? V : K;
  T* d1 = is_v ? vp1 : kp1;
  T* d2 = is_v ? vp2 : kp2;
  T* d3 = is_v ? vp3 : kp3;

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
    } else {
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < valid) raw[r].load(src + (size_t)r * a.d);
      pool_group<false>(raw, valid, p1, p2, p3, pf, pl, a.d);
    }
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
  const int block = 256;
  const dim3 grid((unsigned)(((long long)a.groups << a.chunk_shift) + block - 1) / block,
                  (unsigned)min(a.BH, 65535), 2);
  if (p.dtype == PSA_BF16) {
    using T = __nv_bfloat16;
    pyramid_kernel<T><<<grid, block, 0, st>>>(
        a, (const T*)K, (const T*)V, (T*)(ws + L.kp[1]), (T*)(ws + L.kp[2]), (T*)(ws + L.kp[3]),
        (T*)(ws + L.vp[1]), (T*)(ws + L.vp[2]), (T*)(ws + L.vp[3]), (float*)(ws + L.k3h),
        (float*)(ws + L.k3l));
  } else {
    pyramid_kernel<float><<<grid, block, 0, st>>>(
        a, (const float*)K, (const float*)V, (float*)(ws + L.kp[1]), (float*)(ws + L.kp[2]),
        (float*)(ws + L.kp[3]), (float*)(ws + L.vp[1]), (float*)(ws + L.vp[2]),
        (float*)(ws + L.vp[3]), (float*)(ws + L.k3h), (float*)(ws + L.k3l));
  }
  return cudaGetLastError();
}

}  // namespace psa
