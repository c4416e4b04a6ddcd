// Backward pass of pyramid attention: scratch layout and the launchers of its
// kernels.
//
// The gradient follows the forward pass of adaptive pyramid attention
// (top168.com article on PSA, component three) by the chain rule, with the
// level map held fixed and the ln c bias a constant:
//   D_i      = dO_i . O_i
//   P_ig     = exp(s q_i . K_l[g] + ln c_g - lse_i)
//   dX_ig    = P_ig (dO_i . V_l[g] - D_i)
//   dQ_i     = s sum_g dX_ig K_l[g]
//   dK_l[g] += s sum_i dX_ig q_i,   dV_l[g] += sum_i P_ig dO_i
// and each pooled row's gradient, divided by its token count c_g, goes to
// every token it averages (the adjoint of mean pooling).
#pragma once

#include "psa_internal.cuh"

namespace psa {

// Byte offsets in the caller's backward scratch.
struct BwdLayout {
  size_t delta;               // fp32 [B, Hq, N]: D_i = dO_i . O_i
  size_t dk[kLevels];         // fp32 [B, Hkv, rows_l, d]: gradient of level l's keys
  size_t dv[kLevels];         // fp32 [B, Hkv, rows_l, d]
  size_t acc_begin, total;    // [acc_begin, total): the accumulators, zeroed per call
};

inline BwdLayout make_bwd_layout(const psa_params_t& p) {
  BwdLayout L;
  size_t off = 0;
  L.delta = off;
  off += align256((size_t)p.B * p.Hq * p.N * 4);
  L.acc_begin = off;
  for (int l = 0; l < kLevels; ++l) {
    const size_t bytes = align256((size_t)p.B * p.Hkv * cdiv(p.N, (size_t)1 << l) * p.d * 4);
    L.dk[l] = off; off += bytes;
    L.dv[l] = off; off += bytes;
  }
  L.total = off;
  return L;
}

// Everything the gradient kernels read or write.
struct BwdArgs {
  const void *Q, *K, *V, *O, *dO;
  const float* lse;
  void *dQ, *dK, *dV;
  char* ws;                   // forward workspace: pyramid levels, work list, error word
  char* bws;                  // backward scratch
  float scale;
};

cudaError_t launch_bwd_prep(const psa_params_t& p, const BwdLayout& B, const BwdArgs& a,
                            cudaStream_t st);
cudaError_t launch_bwd_unpool(const psa_params_t& p, const BwdLayout& B, const BwdArgs& a,
                              cudaStream_t st);
cudaError_t launch_attention_bwd_simt(const psa_params_t& p, const Layout& L, const BwdLayout& B,
                                      const BwdArgs& a, cudaStream_t st);
bool attention_bwd_tc_supported(const psa_params_t& p);
cudaError_t launch_attention_bwd_tc(const psa_params_t& p, const Layout& L, const BwdLayout& B,
                                    const BwdArgs& a, cudaStream_t st);

}  // namespace psa
