// capi.cu -- the extern "C" entry points of librsm (declared in include/rsm.h).
//
// Every entry point validates its arguments on the host and returns an error before launching
// anything; launch failures map to RSM_ERR_CUDA with the CUDA error text in rsm_last_error().
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

namespace rsm {
__device__ unsigned int g_device_status = 0u;
}  // namespace rsm

namespace {

thread_local char g_err[512] = "";

rsm_status fail(rsm_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

rsm_status cuda_fail(cudaError_t e, const char* where) {
  return fail(RSM_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pow2_slots(int M) { return M == 32 || M == 64 || M == 128 || M == 256; }

bool valid_router(rsm_router r) {
  return r == RSM_ROUTER_SIGMOID || r == RSM_ROUTER_SOFTMAX || r == RSM_ROUTER_SIGMOID_NORM ||
         r == RSM_ROUTER_SOFTMAX_NORM;
}

// Shared size checks. Returns RSM_OK or an error with g_err set.
rsm_status check_sizes(int M, int K, int Dv) {
  if (M < 1 || K < 1 || Dv < 1) return fail(RSM_ERR_INVALID_ARG, "M, K and Dv must be >= 1");
  if (K > M) return fail(RSM_ERR_INVALID_ARG, "K (%d) must not exceed M (%d)", K, M);
  if (!pow2_slots(M)) return fail(RSM_ERR_UNSUPPORTED, "M must be 32, 64, 128 or 256 (got %d)", M);
  if (Dv > 256 || Dv % 4 != 0)
    return fail(RSM_ERR_UNSUPPORTED, "Dv must be a multiple of 4 in [4, 256] (got %d)", Dv);
  return RSM_OK;
}

#define RSM_REQUIRE_PTR(p, name)                                                  \
  do {                                                                            \
    if (!(p)) return fail(RSM_ERR_INVALID_ARG, "%s must not be NULL", name);       \
    if (!aligned16(p)) return fail(RSM_ERR_INVALID_ARG, "%s must be 16-byte aligned", name); \
  } while (0)
#define RSM_OPTIONAL_PTR(p, name)                                                 \
  do {                                                                            \
    if ((p) && !aligned16(p)) return fail(RSM_ERR_INVALID_ARG, "%s must be 16-byte aligned", name); \
  } while (0)

rsm_status check_forward(const rsm_forward_args* a) {
  if (!a) return fail(RSM_ERR_INVALID_ARG, "args must not be NULL");
  if (a->B < 0 || a->T < 0 || a->H < 0) return fail(RSM_ERR_INVALID_ARG, "B, T, H must be >= 0");
  rsm_status s = check_sizes(a->M, a->K, a->Dv);
  if (s != RSM_OK) return s;
  if (a->qkv_dtype != RSM_F32 && a->qkv_dtype != RSM_BF16)
    return fail(RSM_ERR_INVALID_ARG, "unknown qkv_dtype %d", (int)a->qkv_dtype);
  if (a->decay != RSM_DECAY_HEAD && a->decay != RSM_DECAY_SLOT)
    return fail(RSM_ERR_INVALID_ARG, "unknown decay %d", (int)a->decay);
  if (a->path != RSM_PATH_AUTO && a->path != RSM_PATH_SIMT && a->path != RSM_PATH_TENSOR)
    return fail(RSM_ERR_INVALID_ARG, "unknown path %d", (int)a->path);
  if (!valid_router(a->router)) return fail(RSM_ERR_INVALID_ARG, "unknown router %d", (int)a->router);
  if ((int64_t)a->B * a->H > (int64_t)0x7fffffff)
    return fail(RSM_ERR_UNSUPPORTED, "B*H too large");
  const bool tokens = (int64_t)a->B * a->T * a->H > 0;
  if (tokens) {
    RSM_REQUIRE_PTR(a->q, "q");
    RSM_REQUIRE_PTR(a->k, "k");
    RSM_REQUIRE_PTR(a->v, "v");
    RSM_REQUIRE_PTR(a->logits, "logits");
    RSM_REQUIRE_PTR(a->f, "f");
    RSM_REQUIRE_PTR(a->o, "o");
  }
  RSM_OPTIONAL_PTR(a->H0, "H0");
  RSM_OPTIONAL_PTR(a->HT, "HT");
  RSM_OPTIONAL_PTR(a->idx_out, "idx_out");
  RSM_OPTIONAL_PTR(a->score_out, "score_out");
  RSM_OPTIONAL_PTR(a->slot_counts, "slot_counts");
  if (a->path == RSM_PATH_TENSOR && !rsm::prefill_tc_supported(*a))
    return fail(RSM_ERR_UNSUPPORTED,
                "the tensor-core path needs bf16 q/k/v, M = Dv = 128 and K <= 32");
  return RSM_OK;
}

bool use_tensor_path(const rsm_forward_args& a) {
  if (a.path == RSM_PATH_SIMT) return false;
  if (a.path == RSM_PATH_TENSOR) return true;
  return rsm::prefill_tc_supported(a);
}

}  // namespace

namespace rsm {
ProfileEvents& profile_events() {
  static thread_local ProfileEvents pe;
  return pe;
}
cudaError_t profile_mark(cudaStream_t stream) {
  ProfileEvents& pe = profile_events();
  if (!pe.events || pe.next >= pe.n) return cudaSuccess;
  return cudaEventRecord(static_cast<cudaEvent_t>(pe.events[pe.next++]), stream);
}
// Records a failure message for rsm_last_error() from other translation units of the library.
rsm_status report_error(rsm_status s, const char* msg) { return fail(s, "%s", msg); }
}  // namespace rsm

extern "C" {

const char* rsm_status_string(rsm_status s) {
  switch (s) {
    case RSM_OK: return "RSM_OK";
    case RSM_ERR_INVALID_ARG: return "RSM_ERR_INVALID_ARG";
    case RSM_ERR_UNSUPPORTED: return "RSM_ERR_UNSUPPORTED";
    case RSM_ERR_CUDA: return "RSM_ERR_CUDA";
    case RSM_ERR_NONFINITE: return "RSM_ERR_NONFINITE";
    case RSM_ERR_WORKSPACE: return "RSM_ERR_WORKSPACE";
    case RSM_ERR_TIMEOUT: return "RSM_ERR_TIMEOUT";
  }
  return "RSM_ERR_UNKNOWN";
}

const char* rsm_last_error(void) { return g_err; }

int rsm_version(void) { return 100; }

rsm_status rsm_route_ex(const float* logits, int64_t rows, int M, int K, rsm_router router, int flags,
                        int32_t* idx_out, float* score_out, void* stream) {
  g_err[0] = 0;
  if (rows < 0) return fail(RSM_ERR_INVALID_ARG, "rows must be >= 0");
  rsm_status s = check_sizes(M, K, 4);
  if (s != RSM_OK) return s;
  if (!valid_router(router)) return fail(RSM_ERR_INVALID_ARG, "unknown router %d", (int)router);
  if (rows == 0) return RSM_OK;
  RSM_REQUIRE_PTR(logits, "logits");
  RSM_REQUIRE_PTR(idx_out, "idx_out");
  RSM_OPTIONAL_PTR(score_out, "score_out");
  cudaError_t e = rsm::launch_route(logits, rows, M, K, idx_out, score_out, (int)router,
                                    (flags & RSM_FLAG_VALIDATE) ? 1 : 0, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RSM_OK : cuda_fail(e, "rsm_route launch");
}

rsm_status rsm_route(const float* logits, int64_t rows, int M, int K, int32_t* idx_out,
                     float* score_out, void* stream) {
  return rsm_route_ex(logits, rows, M, K, RSM_ROUTER_SIGMOID, 0, idx_out, score_out, stream);
}

size_t rsm_forward_workspace_size(const rsm_forward_args* a) {
  if (check_forward(a) != RSM_OK) return (size_t)-1;
  return use_tensor_path(*a) ? rsm::prefill_tc_workspace_bytes(*a) : 0;
}

int rsm_forward_selected_path(const rsm_forward_args* a) {
  if (check_forward(a) != RSM_OK) return -1;
  return use_tensor_path(*a) ? RSM_PATH_TENSOR : RSM_PATH_SIMT;
}

int rsm_forward_kernel_launches(const rsm_forward_args* a) {
  if (check_forward(a) != RSM_OK) return -1;
  if ((int64_t)a->B * a->H == 0 || a->T == 0) return 0;
  return use_tensor_path(*a) ? rsm::prefill_tc_launches(*a) : 1;
}

rsm_status rsm_forward(const rsm_forward_args* a, void* stream) {
  g_err[0] = 0;
  rsm_status s = check_forward(a);
  if (s != RSM_OK) return s;
  const bool tc = use_tensor_path(*a);
  const size_t need = tc ? rsm::prefill_tc_workspace_bytes(*a) : 0;
  if (need > 0) {
    if (!a->workspace || a->workspace_bytes < need)
      return fail(RSM_ERR_WORKSPACE, "workspace of %zu bytes required (got %zu)", need,
                  a->workspace ? a->workspace_bytes : (size_t)0);
    if ((reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
      return fail(RSM_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  }
  if ((int64_t)a->B * a->H == 0) return RSM_OK;
  if (a->T == 0) {
    // No tokens: the final state is the initial state.
    if (a->HT) {
      const size_t bytes = (size_t)a->B * a->H * a->M * a->Dv * sizeof(float);
      cudaError_t e = a->H0 ? (a->H0 == a->HT ? cudaSuccess
                                              : cudaMemcpyAsync(a->HT, a->H0, bytes, cudaMemcpyDeviceToDevice,
                                                                static_cast<cudaStream_t>(stream)))
                            : cudaMemsetAsync(a->HT, 0, bytes, static_cast<cudaStream_t>(stream));
      if (e != cudaSuccess) return cuda_fail(e, "rsm_forward (T=0)");
    }
    return RSM_OK;
  }
  rsm::ProfileEvents& pe = rsm::profile_events();
  if (pe.events) {
    const int need = (tc ? rsm::prefill_tc_launches(*a) : 1) + 1;
    if (pe.n < need) return fail(RSM_ERR_INVALID_ARG, "%d profiling events needed (set: %d)", need, pe.n);
    pe.next = 0;
  }
  cudaError_t e = rsm::profile_mark(static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess)
    e = tc ? rsm::launch_prefill_tc(*a, static_cast<cudaStream_t>(stream))
           : rsm::launch_prefill_simt(*a, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess && !tc) e = rsm::profile_mark(static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RSM_OK : cuda_fail(e, tc ? "rsm_forward (tensor path)" : "rsm_forward (simt path)");
}

rsm_status rsm_forward_set_profile_events(void* const* events, int n_events) {
  g_err[0] = 0;
  if (events && n_events < 1) return fail(RSM_ERR_INVALID_ARG, "n_events must be >= 1");
  rsm::ProfileEvents& pe = rsm::profile_events();
  pe.events = n_events > 0 ? events : nullptr;
  pe.n = pe.events ? n_events : 0;
  pe.next = 0;
  return RSM_OK;
}

rsm_status rsm_decode_step(const rsm_decode_args* a, void* stream) {
  g_err[0] = 0;
  if (!a) return fail(RSM_ERR_INVALID_ARG, "args must not be NULL");
  if (a->B < 0 || a->H < 0) return fail(RSM_ERR_INVALID_ARG, "B, H must be >= 0");
  rsm_status s = check_sizes(a->M, a->K, a->Dv);
  if (s != RSM_OK) return s;
  if (a->qkv_dtype != RSM_F32 && a->qkv_dtype != RSM_BF16)
    return fail(RSM_ERR_INVALID_ARG, "unknown qkv_dtype %d", (int)a->qkv_dtype);
  if (a->decay != RSM_DECAY_HEAD && a->decay != RSM_DECAY_SLOT)
    return fail(RSM_ERR_INVALID_ARG, "unknown decay %d", (int)a->decay);
  if (!valid_router(a->router)) return fail(RSM_ERR_INVALID_ARG, "unknown router %d", (int)a->router);
  if ((int64_t)a->B * a->H == 0) return RSM_OK;
  if ((int64_t)a->B * a->H > (int64_t)0x7fffffff) return fail(RSM_ERR_UNSUPPORTED, "B*H too large");
  RSM_REQUIRE_PTR(a->q, "q");
  RSM_REQUIRE_PTR(a->k, "k");
  RSM_REQUIRE_PTR(a->v, "v");
  RSM_REQUIRE_PTR(a->logits, "logits");
  RSM_REQUIRE_PTR(a->f, "f");
  RSM_REQUIRE_PTR(a->state, "state");
  RSM_REQUIRE_PTR(a->o, "o");
  RSM_OPTIONAL_PTR(a->idx_out, "idx_out");
  RSM_OPTIONAL_PTR(a->score_out, "score_out");
  RSM_OPTIONAL_PTR(a->slot_counts, "slot_counts");
  cudaError_t e = rsm::launch_decode(*a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RSM_OK : cuda_fail(e, "rsm_decode_step launch");
}

static rsm_status check_backward(const rsm_backward_args* a) {
  if (!a) return fail(RSM_ERR_INVALID_ARG, "args must not be NULL");
  if (a->B < 0 || a->T < 0 || a->H < 0) return fail(RSM_ERR_INVALID_ARG, "B, T, H must be >= 0");
  rsm_status s = check_sizes(a->M, a->K, a->Dv);
  if (s != RSM_OK) return s;
  if (a->qkv_dtype != RSM_F32 && a->qkv_dtype != RSM_BF16)
    return fail(RSM_ERR_INVALID_ARG, "unknown qkv_dtype %d", (int)a->qkv_dtype);
  if (a->decay != RSM_DECAY_HEAD && a->decay != RSM_DECAY_SLOT)
    return fail(RSM_ERR_INVALID_ARG, "unknown decay %d", (int)a->decay);
  if (!valid_router(a->router)) return fail(RSM_ERR_INVALID_ARG, "unknown router %d", (int)a->router);
  if (a->router != RSM_ROUTER_SIGMOID)
    return fail(RSM_ERR_UNSUPPORTED, "the backward supports the sigmoid router only");
  if ((int64_t)a->M * a->Dv > 24576)
    return fail(RSM_ERR_UNSUPPORTED, "the backward keeps the state in shared memory: M*Dv <= 24576 (got %d)",
                a->M * a->Dv);
  if ((int64_t)a->B * a->H > (int64_t)0x7fffffff) return fail(RSM_ERR_UNSUPPORTED, "B*H too large");
  if ((int64_t)a->B * a->T * a->H > 0) {
    RSM_REQUIRE_PTR(a->q, "q");
    RSM_REQUIRE_PTR(a->k, "k");
    RSM_REQUIRE_PTR(a->v, "v");
    RSM_REQUIRE_PTR(a->logits, "logits");
    RSM_REQUIRE_PTR(a->f, "f");
  }
  RSM_OPTIONAL_PTR(a->H0, "H0");
  RSM_OPTIONAL_PTR(a->dO, "dO");
  RSM_OPTIONAL_PTR(a->dHT, "dHT");
  RSM_OPTIONAL_PTR(a->dq, "dq");
  RSM_OPTIONAL_PTR(a->dk, "dk");
  RSM_OPTIONAL_PTR(a->dv, "dv");
  RSM_OPTIONAL_PTR(a->dlogits, "dlogits");
  RSM_OPTIONAL_PTR(a->df, "df");
  RSM_OPTIONAL_PTR(a->dH0, "dH0");
  return RSM_OK;
}

size_t rsm_backward_workspace_size(const rsm_backward_args* a) {
  if (check_backward(a) != RSM_OK) return (size_t)-1;
  if ((int64_t)a->B * a->T * a->H == 0) return 0;
  return rsm::backward_workspace_bytes(*a);
}

rsm_status rsm_backward(const rsm_backward_args* a, void* stream) {
  g_err[0] = 0;
  rsm_status s = check_backward(a);
  if (s != RSM_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((int64_t)a->B * a->H == 0) return RSM_OK;
  if (a->T == 0) {
    // no tokens: dL/dH0 = dL/dH_T
    if (a->dH0) {
      const size_t bytes = (size_t)a->B * a->H * a->M * a->Dv * sizeof(float);
      cudaError_t e = a->dHT ? cudaMemcpyAsync(a->dH0, a->dHT, bytes, cudaMemcpyDeviceToDevice, st)
                             : cudaMemsetAsync(a->dH0, 0, bytes, st);
      if (e != cudaSuccess) return cuda_fail(e, "rsm_backward (T=0)");
    }
    return RSM_OK;
  }
  const size_t need = rsm::backward_workspace_bytes(*a);
  if (!a->workspace || a->workspace_bytes < need)
    return fail(RSM_ERR_WORKSPACE, "workspace of %zu bytes required (got %zu)", need,
                a->workspace ? a->workspace_bytes : (size_t)0);
  if ((reinterpret_cast<uintptr_t>(a->workspace) & 255u) != 0)
    return fail(RSM_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  cudaError_t e = rsm::launch_backward(*a, st);
  return e == cudaSuccess ? RSM_OK : cuda_fail(e, "rsm_backward launch");
}

rsm_status rsm_get_device_status(void* stream) {
  g_err[0] = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "rsm_get_device_status sync");
  unsigned int word = 0, zero = 0;
  e = cudaMemcpyFromSymbolAsync(&word, rsm::g_device_status, sizeof(word), 0, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(rsm::g_device_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "rsm_get_device_status copy");
  if (word & (1u << RSM_ERR_TIMEOUT)) return fail(RSM_ERR_TIMEOUT, "a bounded device wait expired");
  if (word & (1u << RSM_ERR_NONFINITE)) return fail(RSM_ERR_NONFINITE, "validation found a non-finite logit or f, or f > 0");
  return RSM_OK;
}

}  // extern "C"
