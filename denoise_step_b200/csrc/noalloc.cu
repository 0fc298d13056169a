// pl_ref_attention_noalloc: reference attention without a caller-supplied
// workspace, for callers that cannot allocate device memory.
//
// The scratch this call needs (the fused Q/K/V projection, the bank K/V
// projection and the attention output before Wo) lives in one file-scope
// device array of fixed size. Every GPU that loads this library reserves that
// array for as long as the process runs.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/pl.h"

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(PL_NOALLOC_SCRATCH_BYTES);

// In host code this name is only a stand-in for the device array; its device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device, looked up once per device
// and kept: a cudaDeviceReset between calls would leave it stale (pl.h says
// none may come between calls).
pl_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PL_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return PL_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return PL_ECUDA;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return PL_OK;
}

}  // namespace

extern "C" pl_status pl_ref_attention_noalloc(const void* hidden, const void* w_qkv,
                                              const void* w_o, const void* const* bank_feats,
                                              int n_bank, int frames, int n, int c, int heads,
                                              void* out, void* stream) {
  size_t need = 0;
  const pl_status v = pl_ref_attention_workspace_bytes(frames, n, c, n_bank, &need);
  if (v != PL_OK) return v;
  if (need > kScratchBytes) return PL_ENOMEM;
  void* scratch = nullptr;
  const pl_status s = scratch_for_current_device(&scratch);
  if (s != PL_OK) return s;
  // Nothing in the scratch has to start at zero: each region is written in
  // full by this call before it is read.
  return pl_ref_attention(hidden, w_qkv, w_o, bank_feats, n_bank, frames, n, c, heads, out,
                          scratch, kScratchBytes, stream);
}
