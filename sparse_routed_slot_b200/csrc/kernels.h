// kernels.h -- launch functions of the librsm kernels (internal; the public ABI is rsm.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "rsm.h"

namespace rsm {

cudaError_t launch_route(const float* logits, int64_t rows, int M, int K, int32_t* idx_out,
                         float* score_out, int router, int validate, cudaStream_t stream);

// Routing records for the tensor prefill (route_rec.cu, M = 128, K <= 32) over rows given as
// [B, T, H]: route_record_bytes(K) bytes per row, rows in [B, H, T] order; also the ranked
// indices and scores in the input row order when idx_out / score_out are not null.
bool route_records_supported(int M, int K);
int route_record_bytes(int K);
cudaError_t launch_route_records(const float* logits, const float* f, const void* k, int64_t B, int64_t T,
                                 int64_t H, int M, int K, int decay_slot, int router, int validate,
                                 unsigned char* rec, int32_t* idx_out, float* score_out, int32_t* counts,
                                 cudaStream_t stream);

// Adds the per-slot selection counts of routing records ([pairs, T] rows) to counts[pairs][128].
cudaError_t launch_record_counts(const unsigned char* rec, int64_t pairs, int64_t T, int K, int32_t* counts,
                                 cudaStream_t stream);

cudaError_t launch_decode(const rsm_decode_args& a, cudaStream_t stream);

// Gradients on CUDA cores (backward.cu).
size_t backward_smem_bytes(int M, int K, int Dv);
size_t backward_workspace_bytes(const rsm_backward_args& a);
cudaError_t launch_backward(const rsm_backward_args& a, cudaStream_t stream);

// CUDA-core fp32 chunked prefill (any supported size).
cudaError_t launch_prefill_simt(const rsm_forward_args& a, cudaStream_t stream);
size_t prefill_simt_smem_bytes(int M, int Dv);

// tcgen05 tensor-core chunked prefill. `supported` tells whether the shape/dtype can run there.
bool prefill_tc_supported(const rsm_forward_args& a);
size_t prefill_tc_workspace_bytes(const rsm_forward_args& a);
int prefill_tc_launches(const rsm_forward_args& a);  // kernel launches of one call
cudaError_t launch_prefill_tc(const rsm_forward_args& a, cudaStream_t stream);

// Profiling events of the calling host thread (rsm_forward_set_profile_events): when set, launch
// functions record event i after their i-th kernel (event 0 before the first).
struct ProfileEvents {
  void* const* events = nullptr;
  int n = 0;
  int next = 0;
};
ProfileEvents& profile_events();
// Records the next profiling event on `stream` (no-op when none are set).
cudaError_t profile_mark(cudaStream_t stream);

// Sets the message rsm_last_error() returns on this host thread; returns `s`.
rsm_status report_error(rsm_status s, const char* msg);

}  // namespace rsm
