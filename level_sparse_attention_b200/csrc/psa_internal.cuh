// Internal definitions shared by the PSA kernels and the C-ABI layer:
// workspace layout, launch descriptions, small device helpers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/psa.h"

namespace psa {

constexpr int kLevels = 4;
constexpr int kMaxNk = 8192;          // KV blocks per query block row (N <= 524288 at 64)
constexpr int kErrTimeout = 1;        // bits in the device error word: a wait ran out,
constexpr int kErrLevelMap = 2;       // a caller's level map was corrected,
constexpr int kErrListBounds = 4;     // (debug builds) a work list failed its bounds check

inline __host__ __device__ size_t cdiv(size_t a, size_t b) { return (a + b - 1) / b; }
inline __host__ __device__ size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Byte offsets of everything kept in the caller's workspace.
struct Layout {
  size_t err;                 // int32 device error word (+ padding)
  size_t kp[kLevels];         // pooled keys, level 1..3 (index 0 unused)
  size_t vp[kLevels];         // pooled values, level 1..3
  // fp32 operands of the block-logit GEMM, each split into a tf32 head (low
  // 13 mantissa bits clear) and the exact remainder: x = head + tail
  size_t k3h, k3l;            // level-3 keys [B, Hkv, ceil(N/8), d]
  size_t qmh, qml;            // query-block means [B, Hq, Nq, d]
  size_t zlog;                // block logits fp32 [B, Hq, Nq, Nk]
  size_t map;                 // internal level map int8 [B, Hq, Nq, Nk]
  size_t maxlev;              // int8 [B, Hkv, Nk]: largest level the cosine constraint allows
  size_t counts;              // int4 per query block: entries at level 0..3
  size_t list;                // int32 [B, Hq, Nq, Nk]: KV block indices, by level then index
  size_t total;
  size_t rows[kLevels];       // rows per head of each level
  int Nq, Nk;
};

inline __host__ __device__ Layout make_layout(const psa_params_t& p) {
  Layout L;
  const size_t es = p.dtype == PSA_BF16 ? 2 : 4;
  size_t off = 0;
  L.err = off;
  off += 256;
  L.Nq = (int)cdiv(p.N, p.q_blk);
  L.Nk = (int)cdiv(p.N, p.kv_blk);
  for (int l = 0; l < kLevels; ++l) L.rows[l] = cdiv(p.N, (size_t)1 << l);
  L.kp[0] = L.vp[0] = 0;
  for (int l = 1; l < kLevels; ++l) {
    const size_t bytes = align256((size_t)p.B * p.Hkv * L.rows[l] * p.d * es);
    L.kp[l] = off; off += bytes;
    L.vp[l] = off; off += bytes;
  }
  const size_t k3_bytes = align256((size_t)p.B * p.Hkv * L.rows[3] * p.d * 4);
  L.k3h = off; off += k3_bytes;
  L.k3l = off; off += k3_bytes;
  const size_t rowsq = (size_t)p.B * p.Hq * L.Nq;
  L.qmh = off; off += align256(rowsq * p.d * 4);
  L.qml = off; off += align256(rowsq * p.d * 4);
  L.zlog = off; off += align256(rowsq * L.Nk * 4);
  L.map = off; off += align256(rowsq * L.Nk);
  L.maxlev = off; off += align256((size_t)p.B * p.Hkv * L.Nk);
  L.counts = off; off += align256(rowsq * 16);
  L.list = off; off += align256(rowsq * L.Nk * 4);
  L.total = off;
  return L;
}

// Launch description passed by value to the mask-stage kernels.
struct MaskArgs {
  int B, Hq, Hkv, N, d, q_blk, kv_blk, Nq, Nk;
  int causal, forced_prefix_tokens;
  int assign;                 // psa_assign_t
  float sim_threshold;        // cosine constraint; <= -1: off
  float scale;
  float tau[kLevels];
};

inline MaskArgs make_mask_args(const psa_params_t& p, const Layout& L, float scale) {
  MaskArgs a;
  a.B = p.B; a.Hq = p.Hq; a.Hkv = p.Hkv; a.N = p.N; a.d = p.d;
  a.q_blk = p.q_blk; a.kv_blk = p.kv_blk; a.Nq = L.Nq; a.Nk = L.Nk;
  a.causal = p.causal; a.forced_prefix_tokens = p.forced_prefix_tokens;
  a.assign = (int)p.assign;
  a.sim_threshold = p.sim_threshold;
  a.scale = scale;
  for (int l = 0; l < kLevels; ++l) a.tau[l] = p.tau[l];
  return a;
}

// ----------------------------------------------------------------- device

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// tf32 head of x (low 13 mantissa bits cleared) and the exact remainder.
__device__ __forceinline__ float tf32_head(float x) {
  return __uint_as_float(__float_as_uint(x) & 0xffffe000u);
}

// Programmatic dependent launch.  The short kernels of the library (pyramid,
// query means, block logits, assignment, list kernels, the backward's prep and
// unpool) are launched so that they may be scheduled before the kernel ahead
// of them on the stream has finished (launch_dependent below), and call
// pdl_wait() before their first global-memory access: that returns once the
// previous grid has completed and its writes are visible, so ordering is
// exactly that of plain launches, while the launch itself, and a kernel's
// set-up of shared memory, barriers and TMEM, overlap the previous kernel's
// tail.  They call pdl_trigger() once started, so that the next kernel's CTAs
// are scheduled as their own retire.  Outside such a launch both are no-ops.
// The persistent attention kernels (forward and backward) are plain launches:
// a grid-dependency wait in them measured slower.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                    cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg;
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

}  // namespace psa

// Host-side launchers implemented in the kernel files.
namespace psa {
// The pyramid of K and V; with sim_threshold > -1 also each KV block's largest
// level under the cosine constraint (same launch, from the same loads of K).
cudaError_t launch_pyramid(const psa_params_t& p, const Layout& L, const void* K, const void* V,
                           char* ws, cudaStream_t st);
cudaError_t launch_qmean(const psa_params_t& p, const Layout& L, const void* Q, char* ws,
                         cudaStream_t st);
cudaError_t launch_score(const psa_params_t& p, const Layout& L, float scale, char* ws,
                         cudaStream_t st);
cudaError_t launch_assign(const psa_params_t& p, const Layout& L, float scale, char* ws,
                          int8_t* user_map, float* block_mass, cudaStream_t st);
cudaError_t launch_map_to_list(const psa_params_t& p, const Layout& L, const int8_t* map,
                               char* ws, cudaStream_t st);
// Debug builds (PSA_DEBUG): checks every work list before it is walked; a
// no-op otherwise.
cudaError_t launch_list_check(const psa_params_t& p, const Layout& L, char* ws, cudaStream_t st);
cudaError_t launch_attention_simt(const psa_params_t& p, const Layout& L, float scale,
                                  const void* Q, const void* K, const void* V, const char* ws,
                                  void* O, float* lse, cudaStream_t st);
bool attention_tc_supported(const psa_params_t& p);
cudaError_t launch_attention_tc(const psa_params_t& p, const Layout& L, float scale,
                                const void* Q, const void* K, const void* V, char* ws,
                                void* O, float* lse, cudaStream_t st);
}  // namespace psa
