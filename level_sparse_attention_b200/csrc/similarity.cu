// Cosine-similarity constraint on the pyramid levels.
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
// One CTA per (batch, KV head, KV block), one warp per 8-token group (every
// merge lies inside one group); lane = d/32 columns.  A group's 7 merges (4
// at level 1, 2 at level 2, 1 at level 3) need 21 partial sums (a . b,
// |a|^2, |b|^2), reduced across the warp by one reduce-scatter; the warps'
// results are combined per level with a block-wide AND.  The cosine is taken of the
// halves' sums (same direction as their means) in fp32.
#include "psa_internal.cuh"

namespace psa {
namespace {

// N consecutive elements (a lane's columns of one token) as fp32, one vector load.
template <int N> __device__ __forceinline__ void load_cols(const __nv_bfloat16* p, float* x) {
  if constexpr (N == 4) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
  } else {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    x[0] = a.x; x[1] = a.y;
  }
}
template <int N> __device__ __forceinline__ void load_cols(const float* p, float* x) {
  if constexpr (N == 4) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  } else {
    const float2 a = *reinterpret_cast<const float2*>(p);
    x[0] = a.x; x[1] = a.y;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) similarity_kernel(const T* __restrict__ K,
                                                         int8_t* __restrict__ maxlev, int N,
                                                         int Nk, float theta) {
  constexpr int CPL = D / 32;                  // columns per lane
  const long long item = blockIdx.x;           // (b * Hkv + h) * Nk + j
  const int j = (int)(item % Nk);
  const long long bh = item / Nk;
  const int lane = threadIdx.x & 31, g8 = threadIdx.x >> 5;
  const int t0 = j * 64 + g8 * 8;
  const int nv = max(0, min(8, N - t0));       // valid tokens of this warp's group
  bool ok1 = true, ok2 = true, ok3 = true;
  if (nv > 1) {                                // whole warp; a single token merges nothing
    const T* base = K + (bh * N + t0) * D + lane * CPL;
    float x[8][CPL];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (t < nv) {
        load_cols<CPL>(base + (long long)t * D, x[t]);
      } else {
#pragma unroll
        for (int c = 0; c < CPL; ++c) x[t][c] = 0.f;
      }
    }
    // halves of the 7 merges as sums of tokens: level 1 (2p | 2p+1),
    // level 2 (4q, 4q+1 | 4q+2, 4q+3), level 3 (0..3 | 4..7)
    float part[32];                            // 21 used, padded for the reduction below
#pragma unroll
    for (int i = 0; i < 32; ++i) part[i] = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      float s2[4], s4[2];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = x[2 * q][c], b = x[2 * q + 1][c];
        part[3 * q] = fmaf(a, b, part[3 * q]);
        part[3 * q + 1] = fmaf(a, a, part[3 * q + 1]);
        part[3 * q + 2] = fmaf(b, b, part[3 * q + 2]);
        s2[q] = a + b;
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const float a = s2[2 * q], b = s2[2 * q + 1];
        part[12 + 3 * q] = fmaf(a, b, part[12 + 3 * q]);
        part[13 + 3 * q] = fmaf(a, a, part[13 + 3 * q]);
        part[14 + 3 * q] = fmaf(b, b, part[14 + 3 * q]);
        s4[q] = a + b;
      }
      part[18] = fmaf(s4[0], s4[1], part[18]);
      part[19] = fmaf(s4[0], s4[0], part[19]);
      part[20] = fmaf(s4[1], s4[1], part[20]);
    }
    // reduce-scatter across the warp: at each step a lane keeps the half of
    // its values that its lane bit selects and adds its partner's copy of
    // that half; at the end lane i holds the warp's sum of value i (31
    // shuffles for all 32 values)
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
    // merge m: a . b on lane 3m, |a|^2 and |b|^2 on lanes 3m + 1, 3m + 2;
    // cos >= theta, with a zero half passing
    const float na = __shfl_down_sync(0xffffffffu, part[0], 1);
    const float nb = __shfl_down_sync(0xffffffffu, part[0], 2);
    const float nn = na * nb;
    const unsigned sim = __ballot_sync(0xffffffffu, nn == 0.f || part[0] >= theta * sqrtf(nn));
    auto similar = [&](int m) { return (sim >> (3 * m)) & 1u; };
    // merge m exists when its second half holds a token
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (2 * q + 1 < nv && !similar(q)) ok1 = false;
#pragma unroll
    for (int q = 0; q < 2; ++q)
      if (4 * q + 2 < nv && !similar(4 + q)) ok2 = false;
    if (4 < nv && !similar(6)) ok3 = false;
  }
  ok1 = __syncthreads_and(ok1);
  ok2 = __syncthreads_and(ok2);
  ok3 = __syncthreads_and(ok3);
  if (threadIdx.x == 0) maxlev[item] = (int8_t)(ok1 ? (ok2 ? (ok3 ? 3 : 2) : 1) : 0);
}

template <typename T, int D>
cudaError_t similarity_typed(const psa_params_t& p, const Layout& L, const void* K, char* ws,
                             cudaStream_t st) {
  const long long n_items = (long long)p.B * p.Hkv * L.Nk;
  similarity_kernel<T, D><<<(unsigned)n_items, 256, 0, st>>>(
      (const T*)K, (int8_t*)(ws + L.maxlev), p.N, L.Nk, p.sim_threshold);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_similarity(const psa_params_t& p, const Layout& L, const void* K, char* ws,
                              cudaStream_t st) {
  if (p.dtype == PSA_BF16)
    return p.d == 128 ? similarity_typed<__nv_bfloat16, 128>(p, L, K, ws, st)
                      : similarity_typed<__nv_bfloat16, 64>(p, L, K, ws, st);
  return p.d == 128 ? similarity_typed<float, 128>(p, L, K, ws, st)
                    : similarity_typed<float, 64>(p, L, K, ws, st);
}

}  // namespace psa
