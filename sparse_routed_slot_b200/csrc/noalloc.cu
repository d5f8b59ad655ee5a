// noalloc.cu -- rsm_forward_noalloc: the chunked prefill for callers that cannot allocate.
//
// Some callers may not allocate device memory at all: code that runs inside a CUDA graph being
// captured (a cudaMalloc there breaks the capture), allocators that own every byte of the device
// and hand none out, or embedded runtimes with a fixed memory plan. rsm_forward needs a caller-
// provided workspace when it splits a long sequence into segments; this entry point instead
// takes that scratch from a fixed array compiled into the library, so the caller passes only the
// inputs and outputs.
//
// The array lives in device global memory for as long as the library is loaded, on every GPU
// that loads it. All calls share it; it keeps whatever the last call left there, and every word
// the kernels read from it is written earlier in the same call, so nothing needs clearing. Two
// calls whose GPU work overlaps in time (different streams, or different host threads on one
// device) race on the array and must not be issued.
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device. The host-side symbol is only a
// handle; the address is looked up once per device, with that device current.
rsm_status scratch_address(void** out) {
  char msg[192];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "rsm_forward_noalloc: cudaGetDevice: %s", cudaGetErrorString(e));
    return rsm::report_error(RSM_ERR_CUDA, msg);
  }
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(msg, sizeof(msg), "rsm_forward_noalloc: device ordinal %d is beyond %d", dev, kMaxDevices);
    return rsm::report_error(RSM_ERR_UNSUPPORTED, msg);
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      snprintf(msg, sizeof(msg), "rsm_forward_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      return rsm::report_error(RSM_ERR_CUDA, msg);
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return RSM_OK;
}

}  // namespace

extern "C" {

size_t rsm_forward_noalloc_max_scratch(void) { return kNoAllocScratchBytes; }

rsm_status rsm_forward_noalloc(const rsm_forward_args* args, void* stream) {
  if (!args) return rsm::report_error(RSM_ERR_INVALID_ARG, "rsm_forward_noalloc: args must not be NULL");
  rsm_forward_args a = *args;
  a.workspace = nullptr;
  a.workspace_bytes = 0;
  const size_t need = rsm_forward_workspace_size(&a);
  if (need == (size_t)-1) return rsm_forward(&a, stream);  // reports the argument error
  if (need > kNoAllocScratchBytes) {
    // Too many (b,h) streams times segments for the fixed array: refuse rather than allocate.
    char msg[192];
    snprintf(msg, sizeof(msg),
             "rsm_forward_noalloc: these sizes need %zu bytes of scratch, more than the built-in %zu",
             need, kNoAllocScratchBytes);
    return rsm::report_error(RSM_ERR_WORKSPACE, msg);
  }
  if (need > 0) {
    void* p = nullptr;
    const rsm_status s = scratch_address(&p);
    if (s != RSM_OK) return s;
    a.workspace = p;
    a.workspace_bytes = kNoAllocScratchBytes;
  }
  return rsm_forward(&a, stream);
}

}  // extern "C"
