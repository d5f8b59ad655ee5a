// decode.cu -- one generation step per (b,h) (rsm_decode_step).
//
// Persistent CTAs (three per SM) walk the (b,h) items. Each item's fp32 state H [M, Dv] streams
// through shared memory in blocks of rows fetched by bulk asynchronous copies into two buffers:
// while one block is processed, the next block -- of this item or of the next item -- is already
// in flight, so the copies never wait for the arithmetic. Warp 0 runs the TopK routing of an item
// and prepares the decay and write weight of each selected slot while that item's first block is
// still arriving. Every thread applies the sparse update to the rows it covers, writes back only
// the selected rows, and accumulates o = sum_i q_i H'[i,:] over all M rows.
// Bytes per (b,h): M*Dv*4 read + K*Dv*4 written + the token's inputs.
//
// Thread layout: CG = Dv/4 column groups of float4 by RG = floor(256/CG) row groups; thread
// (rg, cg) covers rows rg, rg+RG, ... of column group cg (a warp reads whole 512-byte rows).
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rsm {

namespace {

constexpr int kDecodeThreads = 256;
constexpr int kBlockBytes = 32 * 1024;  // state rows per bulk copy (one of two buffers)
constexpr int kCtasPerSm = 3;

RSM_DEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          tc::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
      : "memory");
}

template <int M, typename TIn>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(rsm_decode_args a) {
  constexpr int E = M / 32;
  const int Dv = a.Dv, K = a.K;
  const int CG = Dv >> 2;
  const int RG = kDecodeThreads / CG;
  const int rows_blk = min(M, kBlockBytes / (Dv * 4));  // rows per block
  const int nblk = (M + rows_blk - 1) / rows_blk;        // blocks per item
  const int tid = threadIdx.x;
  const int cg = tid % CG, rg = tid / CG;
  const bool active = rg < RG;  // threads past CG*RG only help with the small loads
  const int64_t items = (int64_t)a.B * a.H;

  extern __shared__ __align__(128) unsigned char dsm[];
  auto buf = [&](uint32_t j) { return reinterpret_cast<float*>(dsm + (j & 1) * kBlockBytes); };
  __shared__ float s_a[M], s_w[M], s_q[M];
  __shared__ unsigned char s_sel[M];
  __shared__ __align__(16) float s_v[256];
  __shared__ __align__(16) float s_red[kDecodeThreads * 4];
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int s_abort;

  if (tid == 0) {
    tc::mbar_init(&bar[0], 1);
    tc::mbar_init(&bar[1], 1);
    tc::fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();

  // The CTA's blocks form one stream: (item, block) in order. Block j goes to buffer j & 1.
  auto issue = [&](int64_t item, int blk, uint32_t j) {
    const int r0 = blk * rows_blk;
    const int rows = min(rows_blk, M - r0);
    const uint32_t bytes = (uint32_t)(rows * Dv * 4);
    tc::mbar_arrive_expect_tx(&bar[j & 1], bytes);
    bulk_load(buf(j), a.state + (item * M + r0) * (int64_t)Dv, bytes, &bar[j & 1]);
  };
  uint32_t j_issue = 0, j_use = 0;  // blocks issued / consumed by this CTA
  int64_t nx_item = blockIdx.x;
  int nx_blk = 0;
  auto issue_next = [&]() {
    if (nx_item < items) {
      issue(nx_item, nx_blk, j_issue++);
      if (++nx_blk == nblk) {
        nx_blk = 0;
        nx_item += gridDim.x;
      }
    }
  };
  if (tid == 0) {
    issue_next();
    issue_next();
  }

  for (int64_t pair = blockIdx.x; pair < items; pair += gridDim.x) {
    float* state = a.state + pair * (int64_t)M * Dv;
    // 1. small inputs and the routing of this item (its first block is in flight)
    const TIn* q = reinterpret_cast<const TIn*>(a.q) + pair * M;
    const TIn* k = reinterpret_cast<const TIn*>(a.k) + pair * M;
    const TIn* v = reinterpret_cast<const TIn*>(a.v) + pair * Dv;
    for (int i = tid; i < M; i += blockDim.x) s_q[i] = In<TIn>::ld(q + i);
    for (int d = tid; d < Dv; d += blockDim.x) s_v[d] = In<TIn>::ld(v + d);
    if (tid < 32) {
      const int lane = tid;
      float x[E];
      load_row_logits<M>(a.logits + pair * M, lane, x);
      float fv[E];
#pragma unroll
      for (int e = 0; e < E; ++e)
        fv[e] = (a.decay == RSM_DECAY_SLOT) ? a.f[pair * M + lane * E + e] : a.f[pair];
      if (a.flags & RSM_FLAG_VALIDATE) {
        bool bad = false;
#pragma unroll
        for (int e = 0; e < E; ++e) bad |= !finite_f32(x[e]) || !finite_f32(fv[e]) || fv[e] > 0.f;
        if (__any_sync(kFull, bad) && lane == 0) raise_status(RSM_ERR_NONFINITE);
      }
      int32_t* io = a.idx_out ? a.idx_out + pair * K : nullptr;
      float* so = a.score_out ? a.score_out + pair * K : nullptr;
      const uint32_t sel = warp_topk<M>(x, K, lane, [&](int r, int slot, int e) {
        if (io) io[r] = slot;
        if (so) so[r] = sigmoid_f32(x[e]);
      });
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int i = lane * E + e;
        if (sel & (1u << e)) {
          const float lam = sigmoid_f32(x[e]) * fv[e];  // log of the decay, <= 0
          s_sel[i] = 1;
          s_a[i] = expf(lam);
          s_w[i] = In<TIn>::ld(k + i) * (-expm1f(lam));  // k_i * (1 - a_i)
        } else {
          s_sel[i] = 0;
          s_a[i] = 1.f;
          s_w[i] = 0.f;
        }
      }
    }
    __syncthreads();

    // 2. blocks of rows: sparse update of the selected rows, read over all rows
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 vv = active ? reinterpret_cast<const float4*>(s_v)[cg] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int blk = 0; blk < nblk; ++blk) {
      const uint32_t j = j_use++;
      if (!tc::mbar_wait(&bar[j & 1], (j >> 1) & 1)) {
        if (tid == 0) {
          s_abort = 1;
          raise_status(RSM_ERR_TIMEOUT);
        }
      }
      const float* sb = buf(j);
      const int r0 = blk * rows_blk;
      const int rows = min(rows_blk, M - r0);
      if (active) {
        for (int rr = rg; rr < rows; rr += RG) {
          const int r = r0 + rr;
          float4 hv = reinterpret_cast<const float4*>(sb + rr * Dv)[cg];
          if (s_sel[r]) {
            const float ar = s_a[r], wr = s_w[r];
            hv.x = fmaf(ar, hv.x, wr * vv.x);
            hv.y = fmaf(ar, hv.y, wr * vv.y);
            hv.z = fmaf(ar, hv.z, wr * vv.z);
            hv.w = fmaf(ar, hv.w, wr * vv.w);
            reinterpret_cast<float4*>(state + (int64_t)r * Dv)[cg] = hv;
          }
          const float qr = s_q[r];
          acc.x = fmaf(qr, hv.x, acc.x);
          acc.y = fmaf(qr, hv.y, acc.y);
          acc.z = fmaf(qr, hv.z, acc.z);
          acc.w = fmaf(qr, hv.w, acc.w);
        }
      }
      __syncthreads();             // the buffer is consumed ...
      if (tid == 0) issue_next();  // ... and refilled with the stream's next block
    }
    if (active) reinterpret_cast<float4*>(s_red)[rg * CG + cg] = acc;
    __syncthreads();

    // 3. reduce over the row groups
    for (int d = tid; d < Dv; d += blockDim.x) {
      float s = 0.f;
      for (int g = 0; g < RG; ++g) s += s_red[g * Dv + d];
      a.o[pair * Dv + d] = s;
    }
    __syncthreads();  // small shared arrays are reused by the next item
    if (s_abort) break;
  }
  // a copy still in flight (only after an abort) must land before the CTA leaves
  if (tid == 0) {
    while (j_use < j_issue) {
      const uint32_t j = j_use++;
      tc::mbar_wait(&bar[j & 1], (j >> 1) & 1);
    }
  }
}

int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

template <int M>
cudaError_t launch_m(const rsm_decode_args& a, cudaStream_t stream) {
  const int smem = 2 * kBlockBytes;
  const int64_t items = (int64_t)a.B * a.H;
  const unsigned grid = (unsigned)std::min<int64_t>(items, (int64_t)sm_count() * kCtasPerSm);
  cudaError_t e;
  if (a.qkv_dtype == RSM_BF16) {
    e = cudaFuncSetAttribute(decode_kernel<M, __nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    decode_kernel<M, __nv_bfloat16><<<grid, kDecodeThreads, smem, stream>>>(a);
  } else {
    e = cudaFuncSetAttribute(decode_kernel<M, float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    decode_kernel<M, float><<<grid, kDecodeThreads, smem, stream>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const rsm_decode_args& a, cudaStream_t stream) {
  if ((int64_t)a.B * a.H == 0) return cudaSuccess;
  switch (a.M) {
    case 32: return launch_m<32>(a, stream);
    case 64: return launch_m<64>(a, stream);
    case 128: return launch_m<128>(a, stream);
    case 256: return launch_m<256>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rsm
