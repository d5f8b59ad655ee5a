// prefill_tc.cu -- tcgen05/TMEM tensor-core chunked prefill (rsm_forward, RSM_PATH_TENSOR).
#include "common.cuh"
#include "kernels.h"

namespace rsm {

bool prefill_tc_supported(const rsm_forward_args&) { return false; }
size_t prefill_tc_workspace_bytes(const rsm_forward_args&) { return 0; }
cudaError_t launch_prefill_tc(const rsm_forward_args&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace rsm
