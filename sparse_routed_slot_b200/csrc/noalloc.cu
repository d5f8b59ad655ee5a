// noalloc.cu -- rsm_forward_noalloc: the chunked prefill for callers that cannot allocate.
//
// Some callers may not allocate device memory at all: code that runs inside a CUDA graph being
// captured (a cudaMalloc there breaks the capture), allocators that own every byte of the device
// and hand none out, or embedded runtimes with a fixed memory plan. rsm_forward's tensor-core
// path needs a caller-provided workspace (the routing records of every token, 144 bytes per
// token and head for K <= 16, and the segment states when a long sequence is split); this entry
// point instead takes that scratch from a fixed array compiled into the library, so the caller
// passes only the inputs and outputs.
//
// The array lives in device global memory for as long as the library is loaded, on every GPU
// that loads it. All calls share it; it keeps whatever the last call left there, and every word
// the kernels read from it is written earlier in the same call, so nothing needs clearing. Two
// calls whose GPU work overlaps in time (different streams, or different host threads on one
// device) race on the array and must not be issued.
#include <cuda.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// The array's device address per device, with the unique id of the CUDA context it was looked up
// in: a device reset creates a new context in which the array may sit elsewhere, so a changed id
// means the address is looked up again.
struct ScratchAddr {
  void* ptr = nullptr;
  unsigned long long ctx_id = 0;
};
ScratchAddr g_scratch_addr[kMaxDevices];
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 when the driver cannot tell).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx) get_id(ctx, &id);
  return id;
}

// Device address of the scratch array on the current device. The host-side symbol is only a
// handle; the address is looked up with the device current, once per device and context.
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
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchAddr& s = g_scratch_addr[dev];
  if (!s.ptr || ctx == 0 || s.ctx_id != ctx) {  // id 0: no current context yet, or no driver query
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      snprintf(msg, sizeof(msg), "rsm_forward_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      return rsm::report_error(RSM_ERR_CUDA, msg);
    }
    s.ptr = p;
    s.ctx_id = ctx ? ctx : current_context_id();  // the lookup made the device's context current
  }
  *out = s.ptr;
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
