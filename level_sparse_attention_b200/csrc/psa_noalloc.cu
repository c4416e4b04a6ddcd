// psa_forward_noalloc: the whole PSA forward pass without any device
// allocation, for callers that are not allowed to allocate.
//
// Some callers of this library cannot call cudaMalloc (or ask torch for a
// buffer) at the moment they run the forward pass: a host framework that
// plans all device memory ahead of time and hands a plugin only its inputs
// and outputs, or a latency-sensitive loop in which the implicit device-wide
// synchronisation of cudaMalloc / cudaFree is not acceptable.  For them the
// scratch memory that psa_forward normally takes from the caller's workspace
// (pooled K/V levels, level-3 keys, query means, block logits, level map, work
// list, error word) lives instead in one file-scope device array of fixed size.
//
// The array is kStaticScratchBytes (32 MiB) and is held on every GPU that
// loads this library until the process exits.  Problems whose
// psa_workspace_size() exceeds it are rejected.  All calls share the one
// array: two calls that overlap on the GPU (different streams, or different
// host threads without ordering) race on it and give wrong results.
#include <mutex>

#include "psa_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

// The scratch itself.  Host code must never pass `g_scratch` to a kernel: on
// the host that name is only a stand-in for the symbol, not a device address.
// Its device address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device, looked up on the first
// call for that device (which must therefore not run inside a stream capture).
psa_status_t scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return PSA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return PSA_OK;
}

}  // namespace

extern "C" psa_status_t psa_forward_noalloc(const psa_params_t* params, const void* Q,
                                            const void* K, const void* V, void* O, float* lse,
                                            int8_t* level_map, void* stream) {
  const size_t need = psa_workspace_size(params);
  if (need == 0)   // invalid parameters: let psa_forward report which check failed
    return psa_forward(params, Q, K, V, O, lse, level_map, nullptr, 0, stream);
  if (need > kStaticScratchBytes) return PSA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  psa_status_t st = scratch_address(&scratch);
  if (st != PSA_OK) return st;
  // The array keeps the previous call's contents.  Every region is rewritten
  // before it is read except the sticky device error word, which starts at 0.
  const psa::Layout L = psa::make_layout(*params);
  if (cudaMemsetAsync(static_cast<char*>(scratch) + L.err, 0, sizeof(int),
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return PSA_ERR_CUDA;
  return psa_forward(params, Q, K, V, O, lse, level_map, scratch, kStaticScratchBytes, stream);
}
