// decode.cu -- one generation step per (b,h) (rsm_decode_step).
//
// Persistent CTAs (three per SM) walk the (b,h) items. For each item the fp32 state H [M, Dv] is
// fetched with one bulk asynchronous copy into shared memory (in row blocks of at most 64 KB);
// while it is in flight, warp 0 runs the TopK routing of the token and prepares the decay and
// write weight of each selected slot. Then every thread applies the sparse update to the rows it
// covers, writes back only the selected rows, and accumulates o = sum_i q_i H'[i,:] over all M
// rows. Bytes per (b,h): M*Dv*4 read + K*Dv*4 written + the token's inputs. With three CTAs per
// SM, one CTA's copy overlaps the others' routing and arithmetic.
//
// Thread layout: CG = Dv/4 column groups of float4 by RG = floor(256/CG) row groups; thread
// (rg, cg) covers rows rg, rg+RG, ... of column group cg (a warp reads whole 512-byte rows).
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rsm {

namespace {

constexpr int kDecodeThreads = 256;
constexpr int kStageBytes = 64 * 1024;  // state rows fetched per bulk copy
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
  const int rows_per_stage = min(M, kStageBytes / (Dv * 4));
  const int tid = threadIdx.x;
  const int cg = tid % CG, rg = tid / CG;
  const bool active = rg < RG;  // threads past CG*RG only help with the small loads
  const int64_t items = (int64_t)a.B * a.H;

  extern __shared__ __align__(128) unsigned char dsm[];
  float* s_state = reinterpret_cast<float*>(dsm);  // [rows_per_stage][Dv]
  __shared__ float s_a[M], s_w[M], s_q[M];
  __shared__ unsigned char s_sel[M];
  __shared__ __align__(16) float s_v[256];
  __shared__ __align__(16) float s_red[kDecodeThreads * 4];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_abort;

  if (tid == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();
  uint32_t phase = 0;

  for (int64_t pair = blockIdx.x; pair < items; pair += gridDim.x) {
    float* state = a.state + pair * (int64_t)M * Dv;
    // 1. first block of state rows in flight
    if (tid == 0) {
      const int rows = min(rows_per_stage, M);
      tc::mbar_arrive_expect_tx(&bar, (uint32_t)(rows * Dv * 4));
      bulk_load(s_state, state, (uint32_t)(rows * Dv * 4), &bar);
    }
    // 2. small inputs
    const TIn* q = reinterpret_cast<const TIn*>(a.q) + pair * M;
    const TIn* k = reinterpret_cast<const TIn*>(a.k) + pair * M;
    const TIn* v = reinterpret_cast<const TIn*>(a.v) + pair * Dv;
    for (int i = tid; i < M; i += blockDim.x) s_q[i] = In<TIn>::ld(q + i);
    for (int d = tid; d < Dv; d += blockDim.x) s_v[d] = In<TIn>::ld(v + d);
    // 3. routing, decay and write weights of the selected slots (warp 0)
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

    // 4. sparse update of the selected rows, read over all rows, one block of rows at a time
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 vv = active ? reinterpret_cast<const float4*>(s_v)[cg] : make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r0 = 0; r0 < M; r0 += rows_per_stage) {
      if (r0 > 0) {
        __syncthreads();  // everyone is done with the previous block
        if (tid == 0) {
          const int rows = min(rows_per_stage, M - r0);
          tc::mbar_arrive_expect_tx(&bar, (uint32_t)(rows * Dv * 4));
          bulk_load(s_state, state + (int64_t)r0 * Dv, (uint32_t)(rows * Dv * 4), &bar);
        }
      }
      if (!tc::mbar_wait(&bar, phase & 1)) {
        if (tid == 0) {
          s_abort = 1;
          raise_status(RSM_ERR_TIMEOUT);
        }
      }
      ++phase;
      const int rows = min(rows_per_stage, M - r0);
      if (active) {
        for (int rr = rg; rr < rows; rr += RG) {
          const int r = r0 + rr;
          float4 hv = reinterpret_cast<const float4*>(s_state + rr * Dv)[cg];
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
    }
    if (active) reinterpret_cast<float4*>(s_red)[rg * CG + cg] = acc;
    __syncthreads();

    // 5. reduce over the row groups
    for (int d = tid; d < Dv; d += blockDim.x) {
      float s = 0.f;
      for (int g = 0; g < RG; ++g) s += s_red[g * Dv + d];
      a.o[pair * Dv + d] = s;
    }
    __syncthreads();  // shared buffers are reused by the next item
    if (s_abort) break;
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
  const int rows = std::min(M, kStageBytes / (a.Dv * 4));
  const int smem = rows * a.Dv * 4;
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
