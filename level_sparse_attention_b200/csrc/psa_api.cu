// C ABI of the PSA forward pass (declared in include/psa.h): host-side
// validation, workspace layout and the launch order of the kernels.
#include <math.h>
#include <string.h>

#include "bwd_internal.cuh"
#include "psa_internal.cuh"

namespace psa {
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// lse and block_mass are written one float at a time
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

psa_status_t validate(const psa_params_t* p) {
  if (!p) return PSA_ERR_INVALID_ARG;
  if (p->B <= 0 || p->Hq <= 0 || p->Hkv <= 0 || p->N <= 0 || p->d <= 0) return PSA_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return PSA_ERR_INVALID_ARG;
  if (p->dtype != PSA_F32 && p->dtype != PSA_BF16) return PSA_ERR_INVALID_ARG;
  if (p->n_levels != kLevels) return PSA_ERR_UNSUPPORTED;
  for (int l = 0; l < kLevels; ++l)
    if (p->pool[l] != (1 << l)) return PSA_ERR_UNSUPPORTED;
  for (int l = 0; l < kLevels; ++l) {
    if (!(p->tau[l] > 0.f && p->tau[l] <= 1.f)) return PSA_ERR_INVALID_ARG;   // also rejects NaN
    if (l > 0 && p->tau[l] < p->tau[l - 1]) return PSA_ERR_INVALID_ARG;
  }
  if (!(p->scale >= 0.f) || isinf(p->scale)) return PSA_ERR_INVALID_ARG;
  if (p->causal != 0 && p->causal != 1) return PSA_ERR_INVALID_ARG;
  if (p->assign != PSA_ASSIGN_THRESHOLD && p->assign != PSA_ASSIGN_QUANTILE) return PSA_ERR_INVALID_ARG;
  if (p->forced_prefix_tokens < 0) return PSA_ERR_INVALID_ARG;
  if (!(p->sim_threshold <= 1.f)) return PSA_ERR_INVALID_ARG;             // also rejects NaN
  if (p->d != 64 && p->d != 128) return PSA_ERR_UNSUPPORTED;
  if (p->kv_blk != 64) return PSA_ERR_UNSUPPORTED;
  if (p->q_blk != 64 && p->q_blk != 128) return PSA_ERR_UNSUPPORTED;
  if (cdiv(p->N, p->kv_blk) > (size_t)kMaxNk) return PSA_ERR_UNSUPPORTED;
  const long long heads = (long long)p->B * p->Hq;
  if (heads * (long long)cdiv(p->N, p->q_blk) > 0x7fffffffLL) return PSA_ERR_UNSUPPORTED;
  if ((long long)p->B * p->Hq > 0x7fffffffLL / 2) return PSA_ERR_UNSUPPORTED;
  return PSA_OK;
}

float scale_of(const psa_params_t* p) {
  return p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
}

psa_status_t check_ws(const psa_params_t* p, const void* ws, size_t bytes, Layout* L) {
  *L = make_layout(*p);
  if (!ws) return PSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return PSA_ERR_MISALIGNED;
  if (bytes < L->total) return PSA_ERR_WORKSPACE_TOO_SMALL;
  return PSA_OK;
}

psa_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? PSA_OK : PSA_ERR_CUDA; }

psa_status_t check_ptrs(std::initializer_list<const void*> required) {
  for (const void* q : required) {
    if (!q) return PSA_ERR_INVALID_ARG;
    if (!aligned16(q)) return PSA_ERR_MISALIGNED;
  }
  return PSA_OK;
}

psa_status_t run_pyramid(const psa_params_t* p, const Layout& L, const void* K, const void* V,
                         void* ws, cudaStream_t st) {
  return from_cuda(launch_pyramid(*p, L, K, V, (char*)ws, st));
}

psa_status_t run_mask(const psa_params_t* p, const Layout& L, const void* Q, void* ws,
                      int8_t* map, float* mass, cudaStream_t st) {
  const float s = scale_of(p);
  psa_status_t r = from_cuda(launch_qmean(*p, L, Q, (char*)ws, st));
  if (r == PSA_OK) r = from_cuda(launch_score(*p, L, s, (char*)ws, st));
  if (r == PSA_OK) r = from_cuda(launch_assign(*p, L, s, (char*)ws, map, mass, st));
  return r;
}

psa_status_t run_attention(const psa_params_t* p, const Layout& L, const void* Q, const void* K,
                           const void* V, void* ws, const int8_t* map, void* O, float* lse,
                           cudaStream_t st) {
  const float s = scale_of(p);
  if (map) {
    psa_status_t r = from_cuda(launch_map_to_list(*p, L, map, (char*)ws, st));
    if (r != PSA_OK) return r;
  }
  if (psa_status_t r = from_cuda(launch_list_check(*p, L, (char*)ws, st)); r != PSA_OK) return r;
  if (attention_tc_supported(*p))
    return from_cuda(launch_attention_tc(*p, L, s, Q, K, V, (char*)ws, O, lse, st));
  return from_cuda(launch_attention_simt(*p, L, s, Q, K, V, (const char*)ws, O, lse, st));
}

}  // namespace
}  // namespace psa

using namespace psa;

extern "C" {

size_t psa_workspace_size(const psa_params_t* params) {
  if (validate(params) != PSA_OK) return 0;
  return make_layout(*params).total;
}

psa_status_t psa_build_pyramid(const psa_params_t* params, const void* K, const void* V,
                               void* workspace, size_t workspace_bytes, void* stream) {
  psa_status_t r = validate(params);
  if (r != PSA_OK) return r;
  Layout L;
  if ((r = check_ws(params, workspace, workspace_bytes, &L)) != PSA_OK) return r;
  if ((r = check_ptrs({K, V})) != PSA_OK) return r;
  return run_pyramid(params, L, K, V, workspace, (cudaStream_t)stream);
}

psa_status_t psa_score_and_mask(const psa_params_t* params, const void* Q, void* workspace,
                                size_t workspace_bytes, int8_t* level_map, float* block_mass,
                                void* stream) {
  psa_status_t r = validate(params);
  if (r != PSA_OK) return r;
  Layout L;
  if ((r = check_ws(params, workspace, workspace_bytes, &L)) != PSA_OK) return r;
  if ((r = check_ptrs({Q})) != PSA_OK) return r;
  if (block_mass && !aligned4(block_mass)) return PSA_ERR_MISALIGNED;
  return run_mask(params, L, Q, workspace, level_map, block_mass, (cudaStream_t)stream);
}

psa_status_t psa_attention_fwd(const psa_params_t* params, const void* Q, const void* K,
                               const void* V, void* workspace, size_t workspace_bytes,
                               const int8_t* level_map, void* O, float* lse, void* stream) {
  psa_status_t r = validate(params);
  if (r != PSA_OK) return r;
  Layout L;
  if ((r = check_ws(params, workspace, workspace_bytes, &L)) != PSA_OK) return r;
  if ((r = check_ptrs({Q, K, V, O})) != PSA_OK) return r;
  if (lse && !aligned4(lse)) return PSA_ERR_MISALIGNED;
  return run_attention(params, L, Q, K, V, workspace, level_map, O, lse, (cudaStream_t)stream);
}

psa_status_t psa_forward(const psa_params_t* params, const void* Q, const void* K, const void* V,
                         void* O, float* lse, int8_t* level_map, void* workspace,
                         size_t workspace_bytes, void* stream) {
  psa_status_t r = validate(params);
  if (r != PSA_OK) return r;
  Layout L;
  if ((r = check_ws(params, workspace, workspace_bytes, &L)) != PSA_OK) return r;
  if ((r = check_ptrs({Q, K, V, O})) != PSA_OK) return r;
  if (lse && !aligned4(lse)) return PSA_ERR_MISALIGNED;
  cudaStream_t st = (cudaStream_t)stream;
  if ((r = run_pyramid(params, L, K, V, workspace, st)) != PSA_OK) return r;
  if ((r = run_mask(params, L, Q, workspace, level_map, nullptr, st)) != PSA_OK) return r;
  return run_attention(params, L, Q, K, V, workspace, nullptr, O, lse, st);
}

size_t psa_backward_workspace_size(const psa_params_t* params) {
  if (validate(params) != PSA_OK) return 0;
  return make_bwd_layout(*params).total;
}

psa_status_t psa_backward(const psa_params_t* params, const void* Q, const void* K, const void* V,
                          const void* O, const float* lse, const void* dO,
                          const int8_t* level_map, void* workspace, size_t workspace_bytes,
                          void* bwd_workspace, size_t bwd_workspace_bytes, void* dQ, void* dK,
                          void* dV, void* stream) {
  psa_status_t r = validate(params);
  if (r != PSA_OK) return r;
  Layout L;
  if ((r = check_ws(params, workspace, workspace_bytes, &L)) != PSA_OK) return r;
  if ((r = check_ptrs({Q, K, V, O, dO, dQ, dK, dV})) != PSA_OK) return r;
  if (!lse || !bwd_workspace) return PSA_ERR_INVALID_ARG;
  if (!aligned4(lse) || (reinterpret_cast<uintptr_t>(bwd_workspace) & 255u) != 0)
    return PSA_ERR_MISALIGNED;
  const BwdLayout B = make_bwd_layout(*params);
  if (bwd_workspace_bytes < B.total) return PSA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = (cudaStream_t)stream;
  BwdArgs a;
  a.Q = Q; a.K = K; a.V = V; a.O = O; a.dO = dO; a.lse = lse;
  a.dQ = dQ; a.dK = dK; a.dV = dV;
  a.ws = (char*)workspace;
  a.bws = (char*)bwd_workspace;
  a.scale = scale_of(params);
  if ((r = run_pyramid(params, L, K, V, workspace, st)) != PSA_OK) return r;
  if (level_map && (r = from_cuda(launch_map_to_list(*params, L, level_map, (char*)workspace, st))) != PSA_OK)
    return r;
  if ((r = from_cuda(launch_list_check(*params, L, (char*)workspace, st))) != PSA_OK) return r;
  if ((r = from_cuda(launch_bwd_prep(*params, B, a, st))) != PSA_OK) return r;
  r = from_cuda(attention_bwd_tc_supported(*params) ? launch_attention_bwd_tc(*params, L, B, a, st)
                                                    : launch_attention_bwd_simt(*params, L, B, a, st));
  if (r != PSA_OK) return r;
  return from_cuda(launch_bwd_unpool(*params, B, a, st));
}

psa_status_t psa_check_device(const psa_params_t* params, void* workspace, size_t workspace_bytes,
                              void* stream) {
  psa_status_t r = validate(params);
  if (r != PSA_OK) return r;
  Layout L;
  if ((r = check_ws(params, workspace, workspace_bytes, &L)) != PSA_OK) return r;
  cudaStream_t st = (cudaStream_t)stream;
  int host_err = 0;
  int* dev_err = (int*)((char*)workspace + L.err);
  if (cudaMemcpyAsync(&host_err, dev_err, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return PSA_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PSA_ERR_CUDA;
  if (host_err != 0) {
    if (cudaMemsetAsync(dev_err, 0, sizeof(int), st) != cudaSuccess) return PSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return PSA_ERR_CUDA;
    if (host_err & kErrTimeout) return PSA_ERR_DEVICE_TIMEOUT;
    return (host_err & kErrListBounds) ? PSA_ERR_DEVICE_BOUNDS : PSA_ERR_LEVEL_MAP;
  }
  return PSA_OK;
}

int psa_debug_build(void) {
#ifdef PSA_DEBUG
  return 1;
#else
  return 0;
#endif
}

const char* psa_status_string(psa_status_t status) {
  switch (status) {
    case PSA_OK: return "ok";
    case PSA_ERR_INVALID_ARG: return "invalid argument";
    case PSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case PSA_ERR_MISALIGNED: return "device pointer misaligned (Q/K/V/O 16-byte, lse/mass 4-byte, workspace 256-byte)";
    case PSA_ERR_WORKSPACE_TOO_SMALL: return "workspace smaller than psa_workspace_size()";
    case PSA_ERR_CUDA: return "CUDA error";
    case PSA_ERR_DEVICE_TIMEOUT: return "a kernel gave up waiting on the device (timeout)";
    case PSA_ERR_DEVICE_BOUNDS: return "a work list in the workspace failed the debug build's "
                                       "bounds check (its query block was skipped)";
    case PSA_ERR_LEVEL_MAP: return "a caller's level map broke the contract and was corrected "
                                   "(values outside -1..3 pruned; causal: future blocks pruned, "
                                   "diagonal blocks at level 0)";
  }
  return "unknown status";
}

}  // extern "C"
