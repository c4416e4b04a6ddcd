// The two bandwidth-bound stages around the attention gradient:
//   bwd_prep_kernel   D_i = dO_i . O_i per query row (fp32), and zeroes the
//                     per-level fp32 gradient accumulators;
//   bwd_unpool_kernel dK[t] = sum_l dK_l[t >> l] / c_l(t) (and the same for
//                     V): the adjoint of the mean pooling that built the
//                     pyramid (top168.com article on PSA, pyramid levels
//                     average-pooled from the original KV), written in the
//                     input dtype.
#include "bwd_internal.cuh"

namespace psa {
namespace {

// 8 consecutive elements as fp32.
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    x[2 * i] = f.x;
    x[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float* p, float (&x)[8]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ void store4(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t*>(&a);
  u.y = *reinterpret_cast<uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}
__device__ __forceinline__ void store4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }

// D/8 threads per row, 8 elements each; then a grid-stride zero fill.
template <typename T, int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const T* __restrict__ O,
                                                       const T* __restrict__ dO,
                                                       float* __restrict__ delta,
                                                       long long n_rows, float4* zero,
                                                       long long n_zero4) {
  constexpr int TPR = D / 8;
  pdl_trigger();
  pdl_wait();
  const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long row = gtid / TPR;
  const int part = (int)(gtid % TPR);
  float acc = 0.f;
  if (row < n_rows) {
    float o[8], g[8];
    load8(O + row * D + part * 8, o);
    load8(dO + row * D + part * 8, g);
#pragma unroll
    for (int i = 0; i < 8; ++i) acc = fmaf(o[i], g[i], acc);
  }
#pragma unroll
  for (int m = 1; m < TPR; m <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if (row < n_rows && part == 0) delta[row] = acc;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = gtid; i < n_zero4; i += stride) zero[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

struct UnpoolArgs {
  const float* dk[kLevels];
  const float* dv[kLevels];
  long long rows[kLevels];
  int N;
  long long n_items;          // B * Hkv * N * D / 4
};

// One thread per 4 columns of one token, for both K and V.
template <typename T, int D>
__global__ void __launch_bounds__(256) bwd_unpool_kernel(UnpoolArgs a, T* __restrict__ dK,
                                                         T* __restrict__ dV) {
  pdl_trigger();
  pdl_wait();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.n_items) return;
  constexpr int C4 = D / 4;
  const int c = (int)(i % C4) * 4;
  const long long tok = i / C4;              // (b * Hkv + h) * N + t
  const int t = (int)(tok % a.N);
  const long long bh = tok / a.N;
  float4 k = *reinterpret_cast<const float4*>(a.dk[0] + tok * D + c);
  float4 v = *reinterpret_cast<const float4*>(a.dv[0] + tok * D + c);
#pragma unroll
  for (int l = 1; l < kLevels; ++l) {
    const int g = t >> l;
    const int cnt = min(1 << l, a.N - (g << l));
    const float w = 1.0f / (float)cnt;       // exact for the full groups (powers of two)
    const long long off = (bh * a.rows[l] + g) * D + c;
    const float4 kl = *reinterpret_cast<const float4*>(a.dk[l] + off);
    const float4 vl = *reinterpret_cast<const float4*>(a.dv[l] + off);
    k.x = fmaf(kl.x, w, k.x); k.y = fmaf(kl.y, w, k.y); k.z = fmaf(kl.z, w, k.z); k.w = fmaf(kl.w, w, k.w);
    v.x = fmaf(vl.x, w, v.x); v.y = fmaf(vl.y, w, v.y); v.z = fmaf(vl.z, w, v.z); v.w = fmaf(vl.w, w, v.w);
  }
  store4(dK + tok * D + c, k);
  store4(dV + tok * D + c, v);
}

template <typename T, int D>
cudaError_t prep_typed(const psa_params_t& p, const BwdLayout& B, const BwdArgs& a,
                       cudaStream_t st) {
  const long long n_rows = (long long)p.B * p.Hq * p.N;
  const long long threads = n_rows * (D / 8);
  const long long blocks = (threads + 255) / 256;
  float4* zero = reinterpret_cast<float4*>(a.bws + B.acc_begin);
  const long long n_zero4 = (long long)((B.total - B.acc_begin) / 16);
  return launch_dependent(bwd_prep_kernel<T, D>, dim3((unsigned)blocks), dim3(256), 0, st,
                          (const T*)a.O, (const T*)a.dO, reinterpret_cast<float*>(a.bws + B.delta),
                          n_rows, zero, n_zero4);
}

template <typename T, int D>
cudaError_t unpool_typed(const psa_params_t& p, const BwdLayout& B, const BwdArgs& a,
                         cudaStream_t st) {
  UnpoolArgs u;
  for (int l = 0; l < kLevels; ++l) {
    u.dk[l] = reinterpret_cast<const float*>(a.bws + B.dk[l]);
    u.dv[l] = reinterpret_cast<const float*>(a.bws + B.dv[l]);
    u.rows[l] = (long long)cdiv(p.N, (size_t)1 << l);
  }
  u.N = p.N;
  u.n_items = (long long)p.B * p.Hkv * p.N * (D / 4);
  const long long blocks = (u.n_items + 255) / 256;
  return launch_dependent(bwd_unpool_kernel<T, D>, dim3((unsigned)blocks), dim3(256), 0, st, u,
                          (T*)a.dK, (T*)a.dV);
}

}  // namespace

cudaError_t launch_bwd_prep(const psa_params_t& p, const BwdLayout& B, const BwdArgs& a,
                            cudaStream_t st) {
  if (p.dtype == PSA_BF16)
    return p.d == 128 ? prep_typed<__nv_bfloat16, 128>(p, B, a, st)
                      : prep_typed<__nv_bfloat16, 64>(p, B, a, st);
  return p.d == 128 ? prep_typed<float, 128>(p, B, a, st) : prep_typed<float, 64>(p, B, a, st);
}

cudaError_t launch_bwd_unpool(const psa_params_t& p, const BwdLayout& B, const BwdArgs& a,
                              cudaStream_t st) {
  if (p.dtype == PSA_BF16)
    return p.d == 128 ? unpool_typed<__nv_bfloat16, 128>(p, B, a, st)
                      : unpool_typed<__nv_bfloat16, 64>(p, B, a, st);
  return p.d == 128 ? unpool_typed<float, 128>(p, B, a, st) : unpool_typed<float, 64>(p, B, a, st);
}

}  // namespace psa
