// Pyramid KV construction: average pooling of K and V into levels 1..3
// (2x, 4x, 8x), plus the level-3 keys in fp32 for block scoring.
//
// Method: top168.com article on PSA (arXiv:2512.04025), pyramid paragraph and
// component one — the bottom level is the original KV and each level above is
// an average-pooled, coarser copy; "Psa Pyramid Sparse Attention" (skillmd),
// Core Technique — levels 1/2/3 pool 2/4/8 tokens.  Pooled row g of level l is
// the mean of tokens [g*2^l, min((g+1)*2^l, N)).
//
// Pure streaming, HBM-bound: every thread owns one group of 8 tokens x 8
// columns of K or V, reads it with 8 vector loads (16 B each for bf16), and
// writes the 4 + 2 + 1 pooled rows it determines (and the fp32 level-3 row for
// K).  Consecutive threads take consecutive 8-column chunks of the same rows,
// so each warp load/store covers whole 128-byte lines.
#include "psa_internal.cuh"

namespace psa {
namespace {

template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
  uint4 raw;
  __device__ void load(const __nv_bfloat16* p) { raw = *reinterpret_cast<const uint4*>(p); }
  __device__ void to_f32(float* f) const {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 v = __bfloat1622float2(h[i]);
      f[2 * i] = v.x;
      f[2 * i + 1] = v.y;
    }
  }
  __device__ static void store(__nv_bfloat16* p, const float* f) {
    uint4 o;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    *reinterpret_cast<uint4*>(p) = o;
  }
};
template <> struct Vec8<float> {
  float4 a, b;
  __device__ void load(const float* p) {
    a = reinterpret_cast<const float4*>(p)[0];
    b = reinterpret_cast<const float4*>(p)[1];
  }
  __device__ void to_f32(float* f) const {
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
  __device__ static void store(float* p, const float* f) {
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
};

struct PyrArgs {
  int BH, N, d, chunks;          // chunks = d / 8
  long long groups;              // ceil(N / 8)
  long long rows1, rows2, rows3;
};

// mean of the first `n` of the summed values: sum / n (n = 1..8); exact for
// powers of two, correctly rounded otherwise.
__device__ __forceinline__ float mean_of(float sum, int n) {
  return (n & (n - 1)) == 0 ? sum * (1.0f / (float)n) : __fdiv_rn(sum, (float)n);
}

template <typename T>
__global__ void __launch_bounds__(256) pyramid_kernel(PyrArgs a, const T* __restrict__ K,
                                                      const T* __restrict__ V, T* kp1, T* kp2,
                                                      T* kp3, T* vp1, T* vp2, T* vp3,
                                                      float* k3f) {
  const long long per_tensor = (long long)a.BH * a.groups * a.chunks;
  long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= 2 * per_tensor) return;
  const int tensor = idx >= per_tensor;   // 0 = K, 1 = V
  if (tensor) idx -= per_tensor;
  const int c = (int)(idx % a.chunks);
  const long long rest = idx / a.chunks;
  const long long g = rest % a.groups;
  const long long bh = rest / a.groups;

  const T* src = (tensor ? V : K) + (bh * a.N + g * 8) * a.d + c * 8;
  const int valid = min(8, a.N - (int)(g * 8));   // tokens of this group inside N

  float x[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r < valid) {
      Vec8<T> v;
      v.load(src + (long long)r * a.d);
      v.to_f32(x[r]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[r][e] = 0.f;
    }
  }
  // level 1: pairs (r, r+1)
  float s1[4][8], s2[2][8], s3[8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) s1[i][e] = x[2 * i][e] + x[2 * i + 1][e];
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) s2[i][e] = s1[2 * i][e] + s1[2 * i + 1][e];
#pragma unroll
  for (int e = 0; e < 8; ++e) s3[e] = s2[0][e] + s2[1][e];

  T* p1 = (tensor ? vp1 : kp1) + (bh * a.rows1 + g * 4) * a.d + c * 8;
  T* p2 = (tensor ? vp2 : kp2) + (bh * a.rows2 + g * 2) * a.d + c * 8;
  T* p3 = (tensor ? vp3 : kp3) + (bh * a.rows3 + g) * a.d + c * 8;
  float m[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int n = min(2, valid - 2 * i);
    if (n > 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = mean_of(s1[i][e], n);
      Vec8<T>::store(p1 + (long long)i * a.d, m);
    }
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int n = min(4, valid - 4 * i);
    if (n > 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = mean_of(s2[i][e], n);
      Vec8<T>::store(p2 + (long long)i * a.d, m);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = mean_of(s3[e], valid);
  Vec8<T>::store(p3, m);
  if (!tensor) Vec8<float>::store(k3f + (bh * a.rows3 + g) * a.d + c * 8, m);
}

}  // namespace

cudaError_t launch_pyramid(const psa_params_t& p, const Layout& L, const void* K, const void* V,
                           char* ws, cudaStream_t st) {
  PyrArgs a;
  a.BH = p.B * p.Hkv;
  a.N = p.N;
  a.d = p.d;
  a.chunks = p.d / 8;
  a.groups = (long long)L.rows[3];
  a.rows1 = (long long)L.rows[1];
  a.rows2 = (long long)L.rows[2];
  a.rows3 = (long long)L.rows[3];
  const long long threads = 2LL * a.BH * a.groups * a.chunks;
  const int block = 256;
  const long long grid = (threads + block - 1) / block;
  if (p.dtype == PSA_BF16) {
    using T = __nv_bfloat16;
    pyramid_kernel<T><<<(unsigned)grid, block, 0, st>>>(
        a, (const T*)K, (const T*)V, (T*)(ws + L.kp[1]), (T*)(ws + L.kp[2]), (T*)(ws + L.kp[3]),
        (T*)(ws + L.vp[1]), (T*)(ws + L.vp[2]), (T*)(ws + L.vp[3]), (float*)(ws + L.k3f));
  } else {
    pyramid_kernel<float><<<(unsigned)grid, block, 0, st>>>(
        a, (const float*)K, (const float*)V, (float*)(ws + L.kp[1]), (float*)(ws + L.kp[2]),
        (float*)(ws + L.kp[3]), (float*)(ws + L.vp[1]), (float*)(ws + L.vp[2]),
        (float*)(ws + L.vp[3]), (float*)(ws + L.k3f));
  }
  return cudaGetLastError();
}

}  // namespace psa
