// Gradient of pyramid attention on CUDA cores (fp32 FMA): the path for fp32
// inputs (the tensor-core kernel takes bf16 with 64- and 128-row query
// blocks).  The gradient is the chain rule through the forward pass of adaptive
// pyramid attention (top168.com article on PSA, component three) with the
// level map held fixed; see bwd_internal.cuh for the formulas.
//
// One CTA per (batch, query head, query block), D/32 threads per query row.
// The work list is packed into 64-key tiles as in the forward kernel; a
// tile's pooled keys and values are staged in shared memory as fp32 with a
// per-key log2(c) bias, causal position and gradient destination (level and
// pooled row).  Per tile:
//   1. threads by row: P_ik = exp2(s log2e q_i.k + log2 c - lse_i log2e),
//      dX_ik = P_ik (dO_i . v_k - D_i); dQ_i += dX_ik k in registers; P and
//      dX go to shared memory;
//   2. threads by (key, column): dK_l[g] += s sum_i dX_ik q_i and
//      dV_l[g] += sum_i P_ik dO_i over the block's rows, added atomically
//      into the fp32 accumulators of the key's level.
#include "bwd_internal.cuh"

namespace psa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kTileKeys = 64;

struct BwdSimtArgs {
  int B, Hq, Hkv, N, q_blk, Nq, Nk, causal;
  float scale, scale_log2;
  long long rows[kLevels];
  const void* klev[kLevels];
  const void* vlev[kLevels];
  float* dk[kLevels];
  float* dv[kLevels];
  const float* lse;
  const float* delta;
};

template <typename T, int D>
__global__ void __launch_bounds__(512) attn_bwd_simt_kernel(BwdSimtArgs a, const T* __restrict__ Q,
                                                            const T* __restrict__ dO,
                                                            const int* __restrict__ list,
                                                            const int4* __restrict__ counts,
                                                            T* __restrict__ dQ) {
  constexpr int TPR = D / 32;          // threads per query row
  constexpr int F4 = 32 / 4;           // float4 groups per thread
  extern __shared__ __align__(16) float sm[];
  float* Ks = sm;                                  // [kTileKeys][D]
  float* Vs = Ks + kTileKeys * D;                  // [kTileKeys][D]
  float* Ps = Vs + kTileKeys * D;                  // [q_blk][kTileKeys]
  float* Xs = Ps + a.q_blk * kTileKeys;            // [q_blk][kTileKeys]  dX
  pdl_wait();
  float* bias = Xs + a.q_blk * kTileKeys;          // [kTileKeys] log2 c, -inf = no key
  int* kpos = reinterpret_cast<int*>(bias + kTileKeys);   // token position or INT_MIN
  int* dst = kpos + kTileKeys;                     // (level << 24) | pooled row, or -1

  const int row = blockIdx.x;          // (b*Hq + hq) * Nq + qa
  const int qa = row % a.Nq;
  const int bhq = row / a.Nq;
  const int b = bhq / a.Hq, hq = bhq % a.Hq;
  const int bhk = b * a.Hkv + hq / (a.Hq / a.Hkv);
  const int r = threadIdx.x / TPR, t = threadIdx.x % TPR;
  const int qpos = qa * a.q_blk + r;
  const bool valid_row = qpos < a.N;
  const int n_rows = min(a.q_blk, a.N - qa * a.q_blk);

  float4 q4[F4], g4[F4], dq4[F4];
#pragma unroll
  for (int i = 0; i < F4; ++i) {
    const int c = (i * TPR + t) * 4;
    float4 qv = make_float4(0.f, 0.f, 0.f, 0.f), gv = qv;
    if (valid_row) {
      const T* qs = Q + ((long long)bhq * a.N + qpos) * D + c;
      const T* gs = dO + ((long long)bhq * a.N + qpos) * D + c;
      qv = make_float4(to_f32(qs[0]), to_f32(qs[1]), to_f32(qs[2]), to_f32(qs[3]));
      gv = make_float4(to_f32(gs[0]), to_f32(gs[1]), to_f32(gs[2]), to_f32(gs[3]));
    }
    q4[i] = qv;
    g4[i] = gv;
    dq4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float lse2 = valid_row ? a.lse[(long long)bhq * a.N + qpos] * kLog2e : -INFINITY;
  const float Di = valid_row ? a.delta[(long long)bhq * a.N + qpos] : 0.f;
  const bool live = lse2 > -INFINITY;  // the row kept a key (also false for NaN)

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
      const long long row0 = (long long)lrow[e] * R;
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
        const bool key = g < a.rows[l] && cg > 0;
        bias[filled + rr] = key ? log2f((float)cg) : -INFINITY;
        kpos[filled + rr] = (a.causal && l == 0) ? (int)first_tok : INT_MIN;
        dst[filled + rr] = key ? (int)(((long long)l << 24) | g) : -1;
      }
      filled += R;
      ++e;
    }
    for (int k = filled + threadIdx.x; k < kTileKeys; k += blockDim.x) {
      bias[k] = -INFINITY;
      kpos[k] = INT_MIN;
      dst[k] = -1;
      for (int c = 0; c < D; ++c) { Ks[k * D + c] = 0.f; Vs[k * D + c] = 0.f; }
    }
    e_next = e; lvl = l; lvl_first = lf;
    __syncthreads();

    // 1. P and dX by row; dQ in registers
    for (int k = 0; k < kTileKeys; ++k) {
      const float* kr = Ks + k * D;
      const float* vr = Vs + k * D;
      float sq = 0.f, sv = 0.f;
#pragma unroll
      for (int i = 0; i < F4; ++i) {
        const float4 kv = *reinterpret_cast<const float4*>(kr + (i * TPR + t) * 4);
        const float4 vv = *reinterpret_cast<const float4*>(vr + (i * TPR + t) * 4);
        sq = fmaf(q4[i].x, kv.x, sq); sq = fmaf(q4[i].y, kv.y, sq);
        sq = fmaf(q4[i].z, kv.z, sq); sq = fmaf(q4[i].w, kv.w, sq);
        sv = fmaf(g4[i].x, vv.x, sv); sv = fmaf(g4[i].y, vv.y, sv);
        sv = fmaf(g4[i].z, vv.z, sv); sv = fmaf(g4[i].w, vv.w, sv);
      }
#pragma unroll
      for (int o = 1; o < TPR; o <<= 1) {
        sq += __shfl_xor_sync(0xffffffffu, sq, o);
        sv += __shfl_xor_sync(0xffffffffu, sv, o);
      }
      float x = fmaf(sq, a.scale_log2, bias[k]);
      if (qpos < kpos[k]) x = -INFINITY;
      const float p = live ? exp2f(x - lse2) : 0.f;
      const float dx = p * (sv - Di);
#pragma unroll
      for (int i = 0; i < F4; ++i) {
        const float4 kv = *reinterpret_cast<const float4*>(kr + (i * TPR + t) * 4);
        dq4[i].x = fmaf(dx, kv.x, dq4[i].x); dq4[i].y = fmaf(dx, kv.y, dq4[i].y);
        dq4[i].z = fmaf(dx, kv.z, dq4[i].z); dq4[i].w = fmaf(dx, kv.w, dq4[i].w);
      }
      if (t == 0) {
        Ps[r * kTileKeys + k] = p;
        Xs[r * kTileKeys + k] = dx;
      }
    }
    __syncthreads();

    // 2. dK_l, dV_l of the tile's keys: sums over the block's rows
    for (int idx = threadIdx.x; idx < kTileKeys * D; idx += blockDim.x) {
      const int k = idx / D, c = idx % D;
      const int dk = dst[k];
      if (dk < 0) continue;
      float ak = 0.f, av = 0.f;
      for (int rr = 0; rr < n_rows; ++rr) {
        const long long qrow = (long long)bhq * a.N + qa * a.q_blk + rr;
        ak = fmaf(Xs[rr * kTileKeys + k], to_f32(Q[qrow * D + c]), ak);
        av = fmaf(Ps[rr * kTileKeys + k], to_f32(dO[qrow * D + c]), av);
      }
      const int lv = dk >> 24;
      const long long off = ((long long)bhk * a.rows[lv] + (dk & 0xffffff)) * D + c;
      atomicAdd(a.dk[lv] + off, ak * a.scale);
      atomicAdd(a.dv[lv] + off, av);
    }
  }

  if (!valid_row) return;
  T* out = dQ + ((long long)bhq * a.N + qpos) * D;
#pragma unroll
  for (int i = 0; i < F4; ++i) {
    const int c = (i * TPR + t) * 4;
    out[c] = from_f32<T>(dq4[i].x * a.scale);
    out[c + 1] = from_f32<T>(dq4[i].y * a.scale);
    out[c + 2] = from_f32<T>(dq4[i].z * a.scale);
    out[c + 3] = from_f32<T>(dq4[i].w * a.scale);
  }
}

template <typename T, int D>
cudaError_t launch_bwd_simt_typed(const BwdSimtArgs& a, int grid, const Layout& L,
                                  const BwdArgs& x, cudaStream_t st) {
  const int threads = a.q_blk * (D / 32);
  const size_t smem = (size_t)2 * kTileKeys * D * 4 + (size_t)2 * a.q_blk * kTileKeys * 4 +
                      (size_t)kTileKeys * 12;
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_simt_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_dependent(attn_bwd_simt_kernel<T, D>, dim3(grid), dim3(threads), smem, st, a,
                          (const T*)x.Q, (const T*)x.dO, (const int*)(x.ws + L.list),
                          (const int4*)(x.ws + L.counts), (T*)x.dQ);
}

}  // namespace

cudaError_t launch_attention_bwd_simt(const psa_params_t& p, const Layout& L, const BwdLayout& B,
                                      const BwdArgs& x, cudaStream_t st) {
  BwdSimtArgs a;
  a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv; a.N = p.N; a.q_blk = p.q_blk;
  a.Nq = L.Nq; a.Nk = L.Nk; a.causal = p.causal;
  a.scale = x.scale;
  a.scale_log2 = x.scale * kLog2e;
  for (int l = 0; l < kLevels; ++l) {
    a.rows[l] = (long long)L.rows[l];
    a.klev[l] = l == 0 ? x.K : (const void*)(x.ws + L.kp[l]);
    a.vlev[l] = l == 0 ? x.V : (const void*)(x.ws + L.vp[l]);
    a.dk[l] = reinterpret_cast<float*>(x.bws + B.dk[l]);
    a.dv[l] = reinterpret_cast<float*>(x.bws + B.dv[l]);
  }
  a.lse = x.lse;
  a.delta = reinterpret_cast<const float*>(x.bws + B.delta);
  const int grid = p.B * p.Hq * L.Nq;
  if (p.dtype == PSA_BF16) {
    if (p.d == 128) return launch_bwd_simt_typed<__nv_bfloat16, 128>(a, grid, L, x, st);
    return launch_bwd_simt_typed<__nv_bfloat16, 64>(a, grid, L, x, st);
  }
  if (p.d == 128) return launch_bwd_simt_typed<float, 128>(a, grid, L, x, st);
  return launch_bwd_simt_typed<float, 64>(a, grid, L, x, st);
}

}  // namespace psa
