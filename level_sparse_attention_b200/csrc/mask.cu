// Multi-level mask generation: query-block means, block logits against the
// level-3 pooled keys, per-query-block softmax, ranking and threshold cuts.
//
// Method: top168.com article on PSA (arXiv:2512.04025), component two (levels
// are allocated from the importance of query-key block pairs) and the ablation
// paragraph (threshold-based allocation beats quantile-based); abstract of
// "PSA: Pyramid Sparse Attention for Efficient Video Understanding and
// Generation" (lower pooling levels for critical KV blocks, higher ones for
// the rest).  How a query block is summarised, how the 8 level-3 keys of a KV
// block become one logit, and how masses become levels are readings of this
// implementation: q_bar = mean of the valid rows; z_j = logsumexp_g(s q_bar.K3_g
// + ln c_g); P = softmax_j(z); rank by P descending (ties to the lower j); a
// block ranked r takes the smallest level l with C_r < tau_l, C_r the mass of
// the blocks ranked before it, else it is pruned.
//
// Three launches:
//   qmean_kernel   one CTA per query block; streams Q once (HBM-bound).
//   score_kernel   lanes = 32 query blocks of one head, q_bar in registers;
//                  chunks of level-3 keys staged in shared memory, read as
//                  broadcast 16-byte loads, 8 independent FMA chains per lane.
//   assign_kernel  one CTA per query block: softmax, bitonic sort of packed
//                  (P, index) keys in shared memory, scan, cut, overrides, and
//                  the work list (KV block indices grouped by level).
#include "psa_internal.cuh"

namespace psa {
namespace {

// -------------------------------------------------------------- q means

template <typename T>
__global__ void __launch_bounds__(256) qmean_kernel(MaskArgs a, const T* __restrict__ Q,
                                                    float* __restrict__ qmean) {
  const int row = blockIdx.x;               // (b*Hq + h) * Nq + qa
  const int qa = row % a.Nq;
  const long long bh = row / a.Nq;
  const int lo = qa * a.q_blk;
  const int n = min(a.q_blk, a.N - lo);
  const int chunks = a.d / 8;
  const int parts = blockDim.x / chunks;    // row slices summed by separate threads
  const int c = threadIdx.x % chunks;
  const int part = threadIdx.x / chunks;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const T* base = Q + (bh * a.N + lo) * a.d + c * 8;
  for (int r = part; r < n; r += parts) {
    const T* src = base + (long long)r * a.d;
    if constexpr (sizeof(T) == 2) {
      const uint4 raw = *reinterpret_cast<const uint4*>(src);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 v = __bfloat1622float2(h[i]);
        acc[2 * i] += v.x;
        acc[2 * i + 1] += v.y;
      }
    } else {
      const float4 u = reinterpret_cast<const float4*>(src)[0];
      const float4 w = reinterpret_cast<const float4*>(src)[1];
      acc[0] += u.x; acc[1] += u.y; acc[2] += u.z; acc[3] += u.w;
      acc[4] += w.x; acc[5] += w.y; acc[6] += w.z; acc[7] += w.w;
    }
  }
  __shared__ float red[256 * 8];
#pragma unroll
  for (int e = 0; e < 8; ++e) red[threadIdx.x * 8 + e] = acc[e];
  __syncthreads();
  if (part == 0) {
    for (int q = 1; q < parts; ++q)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += red[(q * chunks + c) * 8 + e];
    float* dst = qmean + (long long)row * a.d + c * 8;
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[e] = __fdiv_rn(acc[e], (float)n);
  }
}

// -------------------------------------------------------------- scoring

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

constexpr int kScoreChunk = 8;       // KV blocks staged per step (one per warp)

// Lanes = 32 query blocks of one head (q_bar in registers); the CTA walks a
// range of KV blocks in chunks of 8, staging the chunk's 64 level-3 keys in
// shared memory (cp.async, double-buffered).  Warp w scores KV block w of the
// chunk: its 8 keys are read as broadcast 16-byte shared loads, 8 independent
// FMA chains per lane.
template <int D>
__global__ void __launch_bounds__(256) score_kernel(MaskArgs a, int splits,
                                                    const float* __restrict__ qmean,
                                                    const float* __restrict__ k3f,
                                                    float* __restrict__ zlog) {
  extern __shared__ __align__(16) float ks[];        // [2][kScoreChunk * 8][D]
  constexpr int KEYS = kScoreChunk * 8;
  const int groups = (a.Nq + 31) / 32;
  int id = blockIdx.x;
  const int split = id % splits; id /= splits;
  const int grp = id % groups;
  const int bhq = id / groups;
  const int b = bhq / a.Hq, hq = bhq % a.Hq;
  const int bhk = b * a.Hkv + hq / (a.Hq / a.Hkv);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int qa = grp * 32 + lane;
  const bool active = qa < a.Nq;

  float q[D];
  const float* qsrc = qmean + ((long long)bhq * a.Nq + (active ? qa : 0)) * D;
#pragma unroll
  for (int c = 0; c < D; c += 4) {
    const float4 v = *reinterpret_cast<const float4*>(qsrc + c);
    q[c] = v.x; q[c + 1] = v.y; q[c + 2] = v.z; q[c + 3] = v.w;
  }
  const long long rows3 = ((long long)a.N + 7) / 8;
  const float* kbase = k3f + (long long)bhk * rows3 * D;
  const int per = (a.Nk + splits - 1) / splits;
  const int j0 = split * per, j1 = min(a.Nk, j0 + per);
  const int n_chunks = j1 > j0 ? (j1 - j0 + kScoreChunk - 1) / kScoreChunk : 0;

  auto stage = [&](int ci, int buf) {
    const long long g0 = (long long)(j0 + ci * kScoreChunk) * 8;
    float* dst = ks + (size_t)buf * KEYS * D;
    for (int i = threadIdx.x; i < KEYS * D / 4; i += blockDim.x) {
      const int key = i / (D / 4), c4 = i % (D / 4);
      if (g0 + key < rows3) cp_async16(dst + key * D + c4 * 4, kbase + (g0 + key) * D + c4 * 4);
    }
    cp_async_commit();
  };
  if (n_chunks > 0) stage(0, 0);
  for (int ci = 0; ci < n_chunks; ++ci) {
    if (ci + 1 < n_chunks) {
      stage(ci + 1, (ci + 1) & 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int j = j0 + ci * kScoreChunk + warp;
    if (j < j1) {
      const float* kb = ks + (size_t)(ci & 1) * KEYS * D + warp * 8 * D;
      const long long g0 = (long long)j * 8;
      const int ng = (int)min(8LL, rows3 - g0);
      float acc[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) acc[g] = 0.f;
#pragma unroll
      for (int c = 0; c < D; c += 4) {
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float4 v = *reinterpret_cast<const float4*>(kb + g * D + c);
          acc[g] = fmaf(q[c], v.x, acc[g]);
          acc[g] = fmaf(q[c + 1], v.y, acc[g]);
          acc[g] = fmaf(q[c + 2], v.z, acc[g]);
          acc[g] = fmaf(q[c + 3], v.w, acc[g]);
        }
      }
      float lg[8], mx = -INFINITY;
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const int cnt = min(8, a.N - (int)(g0 + g) * 8);
        lg[g] = g < ng ? a.scale * acc[g] + logf((float)cnt) : -INFINITY;
        mx = fmaxf(mx, lg[g]);
      }
      float s = 0.f;
#pragma unroll
      for (int g = 0; g < 8; ++g)
        if (g < ng) s += expf(lg[g] - mx);
      if (active) zlog[((long long)bhq * a.Nq + qa) * a.Nk + j] = mx + logf(s);
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------ assignment

__device__ __forceinline__ int block_sum_int(int v, int* red) {
  // returns the exclusive prefix of v over threads and writes the total to red[32]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    int t = lane < nw ? red[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) red[lane] = t - (lane < nw ? red[lane] : 0);   // exclusive warp offsets
    if (lane == nw - 1) red[32] = t;
  }
  __syncthreads();
  const int excl = red[warp] + x - v;
  __syncthreads();
  return excl;
}

__device__ __forceinline__ float block_sum_float_excl(float v, float* red, float* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) red[warp] = x;
  __syncthreads();
  if (warp == 0) {
    const int nw = blockDim.x >> 5;
    float t = lane < nw ? red[lane] : 0.f;
    const float own = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) red[lane] = t - own;
    if (lane == nw - 1) red[32] = t;
  }
  __syncthreads();
  const float excl = red[warp] + (x - v);
  if (total) *total = red[32];
  __syncthreads();
  return excl;
}

// Writes the work list of one query block from its level row `lev` (shared):
// KV block indices at level 0, then 1, 2, 3, each in increasing index order.
__device__ void emit_list(const int8_t* lev, int Nk, int* __restrict__ list_row,
                          int4* __restrict__ count_row, int* red) {
  const int per = (Nk + blockDim.x - 1) / blockDim.x;
  const int j0 = threadIdx.x * per;
  int base = 0;
  int cnt[kLevels];
  for (int l = 0; l < kLevels; ++l) {
    int mine = 0;
    for (int j = j0; j < min(Nk, j0 + per); ++j) mine += lev[j] == l;
    const int excl = block_sum_int(mine, red);
    const int total = red[32];
    __syncthreads();
    int pos = base + excl;
    for (int j = j0; j < min(Nk, j0 + per); ++j)
      if (lev[j] == l) list_row[pos++] = j;
    cnt[l] = total;
    base += total;
  }
  if (threadIdx.x == 0) *count_row = make_int4(cnt[0], cnt[1], cnt[2], cnt[3]);
}

__global__ void __launch_bounds__(256) assign_kernel(MaskArgs a, int n2,
                                                     const float* __restrict__ zlog,
                                                     int8_t* __restrict__ map_ws,
                                                     int8_t* __restrict__ map_user,
                                                     float* __restrict__ mass_user,
                                                     int* __restrict__ list,
                                                     int4* __restrict__ counts) {
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned long long* key = reinterpret_cast<unsigned long long*>(smem);   // [n2]
  int8_t* lev = reinterpret_cast<int8_t*>(key + n2);                          // [Nk]
  __shared__ float redf[33];
  __shared__ int redi[33];

  const int row = blockIdx.x;
  const int qa = row % a.Nq;
  const int q_lo = qa * a.q_blk;
  const int q_hi = min(a.N, q_lo + a.q_blk) - 1;
  const int nvis = a.causal ? min(a.Nk, q_hi / a.kv_blk + 1) : a.Nk;
  const float* z = zlog + (long long)row * a.Nk;

  // softmax over the visible blocks
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < nvis; j += blockDim.x) mx = fmaxf(mx, z[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((threadIdx.x & 31) == 0) redf[threadIdx.x >> 5] = mx;
  __syncthreads();
  mx = -INFINITY;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, redf[w]);
  __syncthreads();
  float part = 0.f;
  for (int j = threadIdx.x; j < nvis; j += blockDim.x) part += expf(z[j] - mx);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((threadIdx.x & 31) == 0) redf[threadIdx.x >> 5] = part;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += redf[w];
  __syncthreads();
  const float inv = 1.0f / tot;

  for (int i = threadIdx.x; i < n2; i += blockDim.x) {
    unsigned long long k = 0ull;
    if (i < nvis) {
      const float p = expf(z[i] - mx) * inv;
      k = ((unsigned long long)__float_as_uint(p) << 32) | (0xffffffffu - (unsigned)i);
    }
    key[i] = k;
  }
  for (int j = threadIdx.x; j < a.Nk; j += blockDim.x) lev[j] = -1;
  __syncthreads();

  // bitonic sort, descending: P high, then lower index first
  for (int k = 2; k <= n2; k <<= 1) {
    for (int s = k >> 1; s > 0; s >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int ixj = i ^ s;
        if (ixj > i) {
          const unsigned long long u = key[i], v = key[ixj];
          const bool desc = (i & k) == 0;
          if (desc ? (u < v) : (u > v)) { key[i] = v; key[ixj] = u; }
        }
      }
      __syncthreads();
    }
  }

  // exclusive running mass in rank order, then the threshold cut
  const int per = (n2 + blockDim.x - 1) / blockDim.x;
  const int r0 = threadIdx.x * per;
  float mine = 0.f;
  for (int r = r0; r < min(nvis, r0 + per); ++r) mine += __uint_as_float((unsigned)(key[r] >> 32));
  float c = block_sum_float_excl(mine, redf, nullptr);
  for (int r = r0; r < min(nvis, r0 + per); ++r) {
    const float p = __uint_as_float((unsigned)(key[r] >> 32));
    const int j = (int)(0xffffffffu - (unsigned)(key[r] & 0xffffffffu));
    int l = -1;
#pragma unroll
    for (int t = kLevels - 1; t >= 0; --t)
      if (c < a.tau[t]) l = t;
    lev[j] = (int8_t)l;
    c += p;
  }
  __syncthreads();
  // overrides: causal diagonal -> 0, forced prefix -> 0 (visible blocks only)
  for (int j = threadIdx.x; j < nvis; j += blockDim.x) {
    const bool strad = a.causal && (min((j + 1) * a.kv_blk, a.N) - 1 >= q_lo);
    const bool forced = j * a.kv_blk < a.forced_prefix_tokens;
    if (strad || forced) lev[j] = 0;
  }
  __syncthreads();
  int8_t* mrow = map_ws + (long long)row * a.Nk;
  for (int j = threadIdx.x; j < a.Nk; j += blockDim.x) {
    mrow[j] = lev[j];
    if (map_user) map_user[(long long)row * a.Nk + j] = lev[j];
    if (mass_user) mass_user[(long long)row * a.Nk + j] = j < nvis ? expf(z[j] - mx) * inv : 0.f;
  }
  emit_list(lev, a.Nk, list + (long long)row * a.Nk, counts + row, redi);
}

__global__ void __launch_bounds__(256) map_to_list_kernel(MaskArgs a,
                                                          const int8_t* __restrict__ map,
                                                          int* __restrict__ list,
                                                          int4* __restrict__ counts) {
  extern __shared__ __align__(16) unsigned char smem[];
  int8_t* lev = reinterpret_cast<int8_t*>(smem);
  __shared__ int redi[33];
  const int row = blockIdx.x;
  for (int j = threadIdx.x; j < a.Nk; j += blockDim.x) {
    const int8_t v = map[(long long)row * a.Nk + j];
    lev[j] = (v >= 0 && v < kLevels) ? v : (int8_t)-1;
  }
  __syncthreads();
  emit_list(lev, a.Nk, list + (long long)row * a.Nk, counts + row, redi);
}

int next_pow2(int x) {
  int n = 1;
  while (n < x) n <<= 1;
  return n;
}

}  // namespace

cudaError_t launch_qmean(const psa_params_t& p, const Layout& L, const void* Q, char* ws,
                         cudaStream_t st) {
  const MaskArgs a = make_mask_args(p, L, 0.f);
  const int grid = p.B * p.Hq * L.Nq;
  float* qm = (float*)(ws + L.qmean);
  if (p.dtype == PSA_BF16)
    qmean_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(a, (const __nv_bfloat16*)Q, qm);
  else
    qmean_kernel<float><<<grid, 256, 0, st>>>(a, (const float*)Q, qm);
  return cudaGetLastError();
}

cudaError_t launch_score(const psa_params_t& p, const Layout& L, float scale, char* ws,
                         cudaStream_t st) {
  const MaskArgs a = make_mask_args(p, L, scale);
  const int groups = (L.Nq + 31) / 32;
  const int base = p.B * p.Hq * groups;
  int splits = (4 * 148 + base - 1) / base;
  splits = splits < 1 ? 1 : (splits > L.Nk ? L.Nk : splits);
  const dim3 grid(base * splits);
  const float* qm = (const float*)(ws + L.qmean);
  const float* k3 = (const float*)(ws + L.k3f);
  float* z = (float*)(ws + L.zlog);
  const size_t smem = (size_t)2 * kScoreChunk * 8 * p.d * sizeof(float);
  cudaError_t e;
  if (p.d == 128) {
    e = cudaFuncSetAttribute(score_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    score_kernel<128><<<grid, 256, smem, st>>>(a, splits, qm, k3, z);
  } else {
    e = cudaFuncSetAttribute(score_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    score_kernel<64><<<grid, 256, smem, st>>>(a, splits, qm, k3, z);
  }
  return cudaGetLastError();
}

cudaError_t launch_assign(const psa_params_t& p, const Layout& L, float scale, char* ws,
                          int8_t* user_map, float* block_mass, cudaStream_t st) {
  const MaskArgs a = make_mask_args(p, L, scale);
  const int n2 = next_pow2(L.Nk);
  const size_t smem = (size_t)n2 * 8 + align256(L.Nk);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(assign_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  assign_kernel<<<p.B * p.Hq * L.Nq, 256, smem, st>>>(
      a, n2, (const float*)(ws + L.zlog), (int8_t*)(ws + L.map), user_map, block_mass,
      (int*)(ws + L.list), (int4*)(ws + L.counts));
  return cudaGetLastError();
}

cudaError_t launch_map_to_list(const psa_params_t& p, const Layout& L, const int8_t* map,
                               char* ws, cudaStream_t st) {
  const MaskArgs a = make_mask_args(p, L, 0.f);
  map_to_list_kernel<<<p.B * p.Hq * L.Nq, 256, align256(L.Nk), st>>>(
      a, map, (int*)(ws + L.list), (int4*)(ws + L.counts));
  return cudaGetLastError();
}

}  // namespace psa
