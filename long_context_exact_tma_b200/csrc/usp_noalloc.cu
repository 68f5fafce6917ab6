// usp_noalloc.cu -- usp_attn_bwd_noalloc: the attention backward for callers
// that cannot allocate a workspace. Its scratch is a static device array of
// this file; the call runs the regular usp_attn_bwd path on that array.
#include <stddef.h>

#include <mutex>

#include "../../include/usp.h"
#include "usp_internal.h"

namespace {

// The scratch itself. Host code must not use this name as an address: on the
// host it is only a stand-in for the device symbol, so the device address is
// looked up with cudaGetSymbolAddress once per device (below).
__device__ __align__(256) unsigned char g_bwd_scratch[USP_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// The device address of the scratch on the current device, looked up once per
// device (with that device current) and kept for the life of the process.
int scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return usp::record_error(USP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return usp::record_error(USP_ERR_UNSUPPORTED, "usp_attn_bwd_noalloc: device index %d >= %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (e != cudaSuccess || p == nullptr)
      return usp::record_error(USP_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return USP_OK;
}

}  // namespace

extern "C" int usp_attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* out, const float* lse,
                                    const void* dO, void* dQ, float* dK, float* dV, int B, int S, int Hq, int Hkv,
                                    int D, int causal, int P_u, int P_r, void* stream) {
  const size_t need = usp_attn_workspace_size(B, S, Hq, Hkv, D, causal, P_u, P_r, USP_MODE_FUSED, 1);
  if (need == 0)  // a shape the backward does not support: the regular entry point reports why
    return usp_attn_bwd(q, k, v, out, lse, dO, dQ, dK, dV, B, S, Hq, Hkv, D, causal, P_u, P_r, nullptr, 0, stream);
  if (need > USP_NOALLOC_SCRATCH_BYTES)
    return usp::record_error(USP_ERR_WORKSPACE,
                             "usp_attn_bwd_noalloc: this problem needs %zu bytes of scratch but the static scratch "
                             "holds %zu; call usp_attn_bwd with a workspace instead",
                             need, static_cast<size_t>(USP_NOALLOC_SCRATCH_BYTES));
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != USP_OK) return rc;
  // usp_attn_bwd clears the status word; its prepare step rewrites the LSE and
  // Delta tables in full (padding rows included), so stale contents never leak.
  return usp_attn_bwd(q, k, v, out, lse, dO, dQ, dK, dV, B, S, Hq, Hkv, D, causal, P_u, P_r, scratch,
                      USP_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" int usp_attn_bwd_noalloc_status(int* site, void* stream) {
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != USP_OK) return rc;
  return usp_workspace_status(scratch, site, stream);
}
