// route.cu -- standalone TopK routing of router logits (rsm_route).
//
// One warp per row of M logits, rows strided over a grid sized to the SM count. Each lane holds
// M/32 contiguous logits; the selection is warp_topk (common.cuh). Output per row: the K selected
// slot indices in rank order (logit desc, index asc) and their router scores (sigmoid or softmax,
// optionally normalised over the selection; warp_router_scores).
#include "common.cuh"
#include "kernels.h"

namespace rsm {

template <int M>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int64_t rows,
                                                    int K, int32_t* __restrict__ idx_out,
                                                    float* __restrict__ score_out, int router, int validate) {
  constexpr int E = M / 32;
  const int lane = threadIdx.x & 31;
  const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows;
       row += warps) {
    float x[E];
    load_row_logits<M>(logits + row * M, lane, x);
    if (validate) {
      bool bad = false;
#pragma unroll
      for (int e = 0; e < E; ++e) bad |= !finite_f32(x[e]);
      if (__any_sync(kFull, bad) && lane == 0) raise_status(RSM_ERR_NONFINITE);
    }
    int32_t* io = idx_out + row * K;
    float* so = score_out ? score_out + row * K : nullptr;
    int rank[E];
    const uint32_t sel = warp_topk<M>(x, K, lane, [&](int r, int slot, int e) {
      io[r] = slot;
      set_rank<E>(rank, e, r);
    });
    if (so) {
      float sc[E];
      warp_router_scores<E>(x, sel, router, sc);
#pragma unroll
      for (int e = 0; e < E; ++e)
        if ((sel >> e) & 1u) so[rank[e]] = sc[e];
    }
  }
}

cudaError_t launch_route(const float* logits, int64_t rows, int M, int K, int32_t* idx_out,
                         float* score_out, int router, int validate, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int sms = device_sm_count();
  const int64_t want = (rows + 7) / 8;
  const int grid = (int)(want < (int64_t)sms * 8 ? want : (int64_t)sms * 8);
  switch (M) {
    case 32: route_kernel<32><<<grid, 256, 0, stream>>>(logits, rows, K, idx_out, score_out, router, validate); break;
    case 64: route_kernel<64><<<grid, 256, 0, stream>>>(logits, rows, K, idx_out, score_out, router, validate); break;
    case 128: route_kernel<128><<<grid, 256, 0, stream>>>(logits, rows, K, idx_out, score_out, router, validate); break;
    case 256: route_kernel<256><<<grid, 256, 0, stream>>>(logits, rows, K, idx_out, score_out, router, validate); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace rsm
