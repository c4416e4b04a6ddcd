// The forward pass from host buffers: host -> device copies, the forward
// pass and the device -> host copy of O pipelined by head group, so that the
// copies of one group overlap the kernels of another.
//
// Every (batch, head) of the forward pass is independent (the pyramid, the
// mask and the attention of a head read only that head's Q and its KV head),
// so head groups can be computed one after another on their own slices.  A
// group is a contiguous range of query heads together with the KV heads they
// read: whole GQA groups when there are at least as many KV heads as groups,
// else an even split of each KV head's query heads.
#include <string.h>

#include <vector>

#include "psa_internal.cuh"

namespace psa {
namespace {

// Query heads [q0, q1) and KV heads [kv0, kv1) of group g of G; false if the
// split is impossible (see the file comment).
bool head_group(int Hq, int Hkv, int g, int G, int* q0, int* q1, int* kv0, int* kv1) {
  if (G < 1 || g < 0 || g >= G || Hq % Hkv) return false;
  const int grp = Hq / Hkv;
  if (Hkv >= G) {
    *kv0 = (int)((long long)g * Hkv / G);
    *kv1 = (int)((long long)(g + 1) * Hkv / G);
    *q0 = *kv0 * grp;
    *q1 = *kv1 * grp;
    return true;
  }
  if (G % Hkv) return false;
  const int per = G / Hkv;
  if (per > grp) return false;
  const int kv = g / per, i = g % per;
  *kv0 = kv;
  *kv1 = kv + 1;
  *q0 = kv * grp + i * grp / per;
  *q1 = kv * grp + (i + 1) * grp / per;
  return true;
}

struct Events {
  std::vector<cudaEvent_t> ev;
  ~Events() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);   // released once their work completes
  }
  cudaEvent_t make() {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    ev.push_back(e);
    return e;
  }
};

}  // namespace
}  // namespace psa

extern "C" psa_status_t psa_forward_host(const psa_params_t* params, const void* Q_host,
                                         const void* K_host, const void* V_host, void* O_host,
                                         float* lse_host, void* Q_dev, void* K_dev, void* V_dev,
                                         void* O_dev, float* lse_dev, void* workspace,
                                         size_t workspace_bytes, int head_groups, void* stream,
                                         void* h2d_stream, void* d2h_stream) {
  using namespace psa;
  if (!params) return PSA_ERR_INVALID_ARG;
  if (psa_workspace_size(params) == 0) return PSA_ERR_INVALID_ARG;   // validates params
  if (!Q_host || !K_host || !V_host || !O_host || !Q_dev || !K_dev || !V_dev || !O_dev)
    return PSA_ERR_INVALID_ARG;
  if ((lse_host == nullptr) != (lse_dev == nullptr)) return PSA_ERR_INVALID_ARG;
  if (!h2d_stream || !d2h_stream || h2d_stream == stream || d2h_stream == stream ||
      h2d_stream == d2h_stream)
    return PSA_ERR_INVALID_ARG;
  if (head_groups < 1) return PSA_ERR_INVALID_ARG;
  if (workspace_bytes < psa_workspace_size(params)) return PSA_ERR_WORKSPACE_TOO_SMALL;
  const psa_params_t& p = *params;
  int q0, q1, kv0, kv1;
  for (int g = 0; g < head_groups; ++g)
    if (!head_group(p.Hq, p.Hkv, g, head_groups, &q0, &q1, &kv0, &kv1) || q1 <= q0)
      return PSA_ERR_INVALID_ARG;

  cudaStream_t st = (cudaStream_t)stream, hs = (cudaStream_t)h2d_stream,
               ds = (cudaStream_t)d2h_stream;
  const size_t es = p.dtype == PSA_BF16 ? 2 : 4;
  const size_t head_bytes = (size_t)p.N * p.d * es;
  auto off = [&](const void* base, size_t bytes) {
    return static_cast<const char*>(base) + bytes;
  };
  auto offw = [&](void* base, size_t bytes) { return static_cast<char*>(base) + bytes; };
  Events E;
  // the copies must not overwrite device buffers that earlier work on the
  // caller's stream may still read
  cudaEvent_t ev_start = E.make();
  if (!ev_start || cudaEventRecord(ev_start, st) != cudaSuccess ||
      cudaStreamWaitEvent(hs, ev_start, 0) != cudaSuccess)
    return PSA_ERR_CUDA;
  for (int b = 0; b < p.B; ++b) {
    int kv_copied = 0;                                  // KV heads of batch b already on the device
    for (int g = 0; g < head_groups; ++g) {
      head_group(p.Hq, p.Hkv, g, head_groups, &q0, &q1, &kv0, &kv1);
      const size_t qo = ((size_t)b * p.Hq + q0) * head_bytes, qn = (size_t)(q1 - q0) * head_bytes;
      const size_t ko = ((size_t)b * p.Hkv + kv0) * head_bytes;
      // host -> device: this group's queries and the KV heads not copied yet
      if (cudaMemcpyAsync(offw(Q_dev, qo), off(Q_host, qo), qn, cudaMemcpyHostToDevice, hs) !=
          cudaSuccess)
        return PSA_ERR_CUDA;
      const int k_from = kv0 > kv_copied ? kv0 : kv_copied;
      if (kv1 > k_from) {
        const size_t ka = ((size_t)b * p.Hkv + k_from) * head_bytes;
        const size_t kn = (size_t)(kv1 - k_from) * head_bytes;
        if (cudaMemcpyAsync(offw(K_dev, ka), off(K_host, ka), kn, cudaMemcpyHostToDevice, hs) !=
                cudaSuccess ||
            cudaMemcpyAsync(offw(V_dev, ka), off(V_host, ka), kn, cudaMemcpyHostToDevice, hs) !=
                cudaSuccess)
          return PSA_ERR_CUDA;
        kv_copied = kv1;
      }
      cudaEvent_t ev_in = E.make(), ev_out = E.make();
      if (!ev_in || !ev_out || cudaEventRecord(ev_in, hs) != cudaSuccess ||
          cudaStreamWaitEvent(st, ev_in, 0) != cudaSuccess)
        return PSA_ERR_CUDA;
      // the group's forward pass on the caller's stream
      psa_params_t gp = p;
      gp.B = 1;
      gp.Hq = q1 - q0;
      gp.Hkv = kv1 - kv0;
      const size_t lo = ((size_t)b * p.Hq + q0) * (size_t)p.N;
      psa_status_t r = psa_forward(&gp, off(Q_dev, qo), off(K_dev, ko), off(V_dev, ko),
                                   offw(O_dev, qo), lse_dev ? lse_dev + lo : nullptr, nullptr,
                                   workspace, workspace_bytes, stream);
      if (r != PSA_OK) return r;
      if (cudaEventRecord(ev_out, st) != cudaSuccess ||
          cudaStreamWaitEvent(ds, ev_out, 0) != cudaSuccess)
        return PSA_ERR_CUDA;
      // device -> host: the group's outputs
      if (cudaMemcpyAsync(offw(O_host, qo), off(O_dev, qo), qn, cudaMemcpyDeviceToHost, ds) !=
          cudaSuccess)
        return PSA_ERR_CUDA;
      if (lse_dev &&
          cudaMemcpyAsync(lse_host + lo, lse_dev + lo, (size_t)(q1 - q0) * p.N * sizeof(float),
                          cudaMemcpyDeviceToHost, ds) != cudaSuccess)
        return PSA_ERR_CUDA;
    }
  }
  // the caller's stream completes after the last copy back
  cudaEvent_t ev_end = E.make();
  if (!ev_end || cudaEventRecord(ev_end, ds) != cudaSuccess ||
      cudaStreamWaitEvent(st, ev_end, 0) != cudaSuccess)
    return PSA_ERR_CUDA;
  return PSA_OK;
}
