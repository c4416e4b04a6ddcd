// Pyramid attention on CUDA cores (fp32 FMA): the path for fp32 inputs (the
// tensor-core kernel takes bf16 with 64- and 128-row query blocks).
//
// Method: adaptive pyramid attention (top168.com article on PSA, component
// three: the probability distribution stays consistent).  Row i of query block
// a takes one softmax over every key it keeps: for block j at level l >= 0 the
// level-l pooled rows of block j, each with logit s * q_i . K_l[g] + ln c_g, so
// a pooled key carries the mass of the c_g tokens it averages.  Causal blocks
// straddling the diagonal are level 0 and mask keys after the row.
//
// One CTA per (batch, query head, query block); D/32 threads per query row,
// each holding 32 of the row's q and o values in registers.  The work list is
// packed into 64-key tiles (entries are sorted by level, so a 64/32/16/8-row
// sub-block never crosses a tile edge); a tile's keys and values are staged in
// shared memory as fp32 together with a per-key log2(c) bias and position.
#include "psa_internal.cuh"

namespace psa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kTileKeys = 64;

struct SimtArgs {
  int B, Hq, Hkv, N, q_blk, Nq, Nk, causal;
  float scale_log2;
  long long rows[kLevels];
  const void* klev[kLevels];
  const void* vlev[kLevels];
};

template <typename T, int D>
__global__ void __launch_bounds__(512) attn_simt_kernel(SimtArgs a, const T* __restrict__ Q,
                                                        const int* __restrict__ list,
                                                        const int4* __restrict__ counts,
                                                        T* __restrict__ O,
                                                        float* __restrict__ lse) {
  constexpr int TPR = D / 32;          // threads per query row
  constexpr int F4 = 32 / 4;           // float4 groups per thread
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;                      // [kTileKeys][D]
  float* Vs = Ks + kTileKeys * D;      // [kTileKeys][D]
  float* bias = Vs + kTileKeys * D;    // [kTileKeys] log2 c, -inf = no key
  int* kpos = reinterpret_cast<int*>(bias + kTileKeys);   // [kTileKeys] token position or INT_MIN
  pdl_wait();

  const int row = blockIdx.x;          // (b*Hq + hq) * Nq + qa
  const int qa = row % a.Nq;
  const int bhq = row / a.Nq;
  const int b = bhq / a.Hq, hq = bhq % a.Hq;
  const int bhk = b * a.Hkv + hq / (a.Hq / a.Hkv);
  const int r = threadIdx.x / TPR, t = threadIdx.x % TPR;
  const int qpos = qa * a.q_blk + r;
  const bool valid_row = r < a.q_blk && qpos < a.N;

  float4 q4[F4], o4[F4];
#pragma unroll
  for (int i = 0; i < F4; ++i) {
    const int c = (i * TPR + t) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (valid_row) {
      const T* src = Q + ((long long)bhq * a.N + qpos) * D + c;
      v = make_float4(to_f32(src[0]), to_f32(src[1]), to_f32(src[2]), to_f32(src[3]));
    }
    q4[i] = v;
    o4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float m = -INFINITY, lsum = 0.f;

  const int4 cnt = counts[row];
  const int n_ent[kLevels] = {cnt.x, cnt.y, cnt.z, cnt.w};
  const int* lrow = list + (long long)row * a.Nk;
  int total_keys = 0;
  for (int l = 0; l < kLevels; ++l) total_keys += n_ent[l] * (64 >> l);
  const int n_tiles = (total_keys + kTileKeys - 1) / kTileKeys;

  int e_next = 0, lvl = 0, lvl_first = 0;   // entry cursor
  for (int tile = 0; tile < n_tiles; ++tile) {
    __syncthreads();
    // stage the tile: walk the entries that fall inside it
    int filled = 0;
    int e = e_next, l = lvl, lf = lvl_first;
    while (filled < kTileKeys) {
      while (l < kLevels && e - lf >= n_ent[l]) { lf += n_ent[l]; ++l; }
      if (l >= kLevels) break;
      const int R = 64 >> l;
      const int j = lrow[e];
      const long long row0 = (long long)j * R;
      const T* kl = reinterpret_cast<const T*>(a.klev[l]) + ((long long)bhk * a.rows[l]) * D;
      const T* vl = reinterpret_cast<const T*>(a.vlev[l]) + ((long long)bhk * a.rows[l]) * D;
      for (int idx = threadIdx.x; idx < R * D; idx += blockDim.x) {
        const int rr = idx / D, c = idx % D;
        const long long g = row0 + rr;
        const bool ok = g < a.rows[l];
        Ks[(filled + rr) * D + c] = ok ? to_f32(kl[g * D + c]) : 0.f;
        Vs[(filled + rr) * D + c] = ok ? to_f32(vl[g * D + c]) : 0.f;
      }
      for (int rr = threadIdx.x; rr < R; rr += blockDim.x) {
        const long long g = row0 + rr;
        const long long first_tok = g << l;
        const int cg = (int)min((long long)(1 << l), (long long)a.N - first_tok);
        bias[filled + rr] = (g < a.rows[l] && cg > 0) ? log2f((float)cg) : -INFINITY;
        kpos[filled + rr] = (a.causal && l == 0) ? (int)first_tok : INT_MIN;
      }
      filled += R;
      ++e;
    }
    for (int k = filled + threadIdx.x; k < kTileKeys; k += blockDim.x) {
      bias[k] = -INFINITY;
      kpos[k] = INT_MIN;
      for (int c = 0; c < D; ++c) { Ks[k * D + c] = 0.f; Vs[k * D + c] = 0.f; }
    }
    e_next = e; lvl = l; lvl_first = lf;
    __syncthreads();

    // scores, 16 keys at a time, online softmax in log2 units
    for (int k0 = 0; k0 < kTileKeys; k0 += 16) {
      float x[16];
      float cmax = -INFINITY;
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        const float* kr = Ks + (k0 + kk) * D;
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < F4; ++i) {
          const float4 kv = *reinterpret_cast<const float4*>(kr + (i * TPR + t) * 4);
          acc = fmaf(q4[i].x, kv.x, acc);
          acc = fmaf(q4[i].y, kv.y, acc);
          acc = fmaf(q4[i].z, kv.z, acc);
          acc = fmaf(q4[i].w, kv.w, acc);
        }
#pragma unroll
        for (int o = 1; o < TPR; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        float v = fmaf(acc, a.scale_log2, bias[k0 + kk]);
        if (qpos < kpos[k0 + kk]) v = -INFINITY;
        x[kk] = v;
        cmax = fmaxf(cmax, v);
      }
      const float m_new = fmaxf(m, cmax);
      if (m_new == -INFINITY) continue;              // nothing kept yet
      const float corr = exp2f(m - m_new);           // 0 when m = -inf
      lsum *= corr;
#pragma unroll
      for (int i = 0; i < F4; ++i) {
        o4[i].x *= corr; o4[i].y *= corr; o4[i].z *= corr; o4[i].w *= corr;
      }
      m = m_new;
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        const float p = exp2f(x[kk] - m);
        lsum += p;
        const float* vr = Vs + (k0 + kk) * D;
#pragma unroll
        for (int i = 0; i < F4; ++i) {
          const float4 vv = *reinterpret_cast<const float4*>(vr + (i * TPR + t) * 4);
          o4[i].x = fmaf(p, vv.x, o4[i].x);
          o4[i].y = fmaf(p, vv.y, o4[i].y);
          o4[i].z = fmaf(p, vv.z, o4[i].z);
          o4[i].w = fmaf(p, vv.w, o4[i].w);
        }
      }
    }
  }

  if (!valid_row) return;
  const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
  T* dst = O + ((long long)bhq * a.N + qpos) * D;
#pragma unroll
  for (int i = 0; i < F4; ++i) {
    const int c = (i * TPR + t) * 4;
    dst[c] = from_f32<T>(o4[i].x * inv);
    dst[c + 1] = from_f32<T>(o4[i].y * inv);
    dst[c + 2] = from_f32<T>(o4[i].z * inv);
    dst[c + 3] = from_f32<T>(o4[i].w * inv);
  }
  if (lse && t == 0)
    lse[(long long)bhq * a.N + qpos] = lsum > 0.f ? (m + log2f(lsum)) * kLn2 : -INFINITY;
}

template <typename T, int D>
cudaError_t launch_simt_typed(const SimtArgs& a, int q_blk, int grid, const void* Q,
                              const char* ws, const Layout& L, void* O, float* lse,
                              cudaStream_t st) {
  const int threads = q_blk * (D / 32);
  const size_t smem = (size_t)2 * kTileKeys * D * 4 + kTileKeys * 8;
  cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_dependent(attn_simt_kernel<T, D>, dim3(grid), dim3(threads), smem, st, a,
                          (const T*)Q, (const int*)(ws + L.list), (const int4*)(ws + L.counts),
                          (T*)O, lse);
}

}  // namespace

cudaError_t launch_attention_simt(const psa_params_t& p, const Layout& L, float scale,
                                  const void* Q, const void* K, const void* V, const char* ws,
                                  void* O, float* lse, cudaStream_t st) {
  SimtArgs a;
  a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv; a.N = p.N; a.q_blk = p.q_blk;
  a.Nq = L.Nq; a.Nk = L.Nk; a.causal = p.causal;
  a.scale_log2 = scale * kLog2e;
  for (int l = 0; l < kLevels; ++l) {
    a.rows[l] = (long long)L.rows[l];
    a.klev[l] = l == 0 ? K : (const void*)(ws + L.kp[l]);
    a.vlev[l] = l == 0 ? V : (const void*)(ws + L.vp[l]);
  }
  const int grid = p.B * p.Hq * L.Nq;
  if (p.dtype == PSA_BF16) {
    if (p.d == 128) return launch_simt_typed<__nv_bfloat16, 128>(a, p.q_blk, grid, Q, ws, L, O, lse, st);
    return launch_simt_typed<__nv_bfloat16, 64>(a, p.q_blk, grid, Q, ws, L, O, lse, st);
  }
  if (p.d == 128) return launch_simt_typed<float, 128>(a, p.q_blk, grid, Q, ws, L, O, lse, st);
  return launch_simt_typed<float, 64>(a, p.q_blk, grid, Q, ws, L, O, lse, st);
}

}  // namespace psa
