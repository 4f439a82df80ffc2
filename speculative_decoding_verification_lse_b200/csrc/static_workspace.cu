// static_workspace.cu -- sv_verify_static: the verification step without any
// device allocation, for callers that must not allocate.
//
// Its scratch is a fixed array in the library's own device memory (below), so
// no call allocates or frees anything: the array is created when the CUDA
// runtime loads this library's device code onto a GPU, and every GPU that loads
// the library keeps it (SV_STATIC_WORKSPACE_BYTES) until the process exits.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "specverify.h"
#include "sv_common.cuh"

namespace sv {

// Sets the message sv_last_error returns and passes the code through (api.cu).
int set_last_error(int code, const char* msg);
// sv_verify_ex's host-side argument checks (api.cu).
int check_args(const void* target_logits, const void* draft_logits, const int32_t* draft_tokens,
               int B, int D_max, int V, int dtype, float temperature, int mode,
               const int32_t* out_tokens, const int32_t* out_accept_len, const sv_params& prm);

namespace {

constexpr size_t kStaticBytes = SV_STATIC_WORKSPACE_BYTES;

// The shared scratch of every sv_verify_static call on a device.  In host code
// this name is only a stand-in for the device array: the kernels get its device
// address, looked up once per device.
__device__ __align__(256) unsigned char g_static_ws[kStaticBytes];

std::mutex g_mu;
std::vector<void*> g_addr;  // per device: device address of g_static_ws, or nullptr

// Device address of the array on device `dev` (the current device); the first
// call on a device looks it up.
int static_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  if ((int)g_addr.size() <= dev) g_addr.resize(dev + 1, nullptr);
  if (!g_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_ws);
    if (e != cudaSuccess) {
      char buf[256];
      snprintf(buf, sizeof buf, "cudaGetSymbolAddress(static workspace): %s", cudaGetErrorString(e));
      return set_last_error(SV_ERR_CUDA, buf);
    }
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return SV_OK;
}

}  // namespace
}  // namespace sv

extern "C" int sv_verify_static(const void* target_logits, const void* draft_logits,
                                const int32_t* draft_tokens, const int32_t* row_D, int B,
                                int D_max, int V, int dtype, float temperature, int mode,
                                uint64_t seed, int32_t* out_tokens, int32_t* out_accept_len,
                                const sv_params* p) {
  using namespace sv;
  sv_params q;
  memset(&q, 0, sizeof q);
  if (p) q = *p;
  // sv_verify_ex's argument checks first, so that invalid calls get its error codes
  {
    const int rc = check_args(target_logits, draft_logits, draft_tokens, B, D_max, V, dtype,
                              temperature, mode, out_tokens, out_accept_len, q);
    if (rc != SV_OK) return rc;
  }
  const size_t need = sv_workspace_bytes(B, D_max, V, dtype);
  if (need > kStaticBytes) {
    char buf[256];
    snprintf(buf, sizeof buf,
             "sv_verify_static: B=%d, D_max=%d, V=%d need %zu bytes of scratch, more than its "
             "fixed %zu; use sv_verify_ex with a workspace",
             B, D_max, V, need, (size_t)kStaticBytes);
    return set_last_error(SV_ERR_UNSUPPORTED, buf);
  }
  int dev = 0;
  const cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return set_last_error(SV_ERR_CUDA, cudaGetErrorString(e));
  void* ws = nullptr;
  const int rc = static_address(dev, &ws);
  if (rc != SV_OK) return rc;
  q.workspace = ws;
  q.workspace_bytes = kStaticBytes;
  return sv_verify_ex(target_logits, draft_logits, draft_tokens, row_D, B, D_max, V, dtype,
                      temperature, mode, seed, out_tokens, out_accept_len, &q);
}
