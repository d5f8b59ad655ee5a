// decode.cu -- one generation step per (b,h) (rsm_decode_step).
//
// Per (b,h) one CTA streams the fp32 state H [M, Dv] once: the TopK routing of the token (one
// warp) runs while the state rows are already in flight; then every thread applies the sparse
// decay and write to the selected rows it holds, writes back only those rows, and accumulates
// o = sum_i q_i H'[i,:] over all M rows. Bytes per (b,h): M*Dv*4 read + K*Dv*4 written + inputs.
//
// Thread layout: CG = Dv/4 column groups of float4 (coalesced 16-byte accesses along a row) by
// RG = floor(256/CG) row groups; thread (rg, cg) owns rows rg, rg+RG, ... of column group cg.
#include "common.cuh"
#include "kernels.h"

namespace rsm {

namespace {

constexpr int kDecodeThreads = 256;
constexpr int kRowsInFlight = 16;  // float4 rows a thread loads before it needs the routing

template <int M, typename TIn>
__global__ void __launch_bounds__(kDecodeThreads) decode_kernel(rsm_decode_args a) {
  constexpr int E = M / 32;
  const int Dv = a.Dv, K = a.K;
  const int CG = Dv >> 2;
  const int RG = kDecodeThreads / CG;
  const int tid = threadIdx.x;
  const int cg = tid % CG, rg = tid / CG;
  const int64_t pair = blockIdx.x;  // flattened (b,h)

  __shared__ float s_a[M], s_w[M], s_q[M];
  __shared__ unsigned char s_sel[M];
  __shared__ __align__(16) float s_v[256];
  __shared__ __align__(16) float s_red[kDecodeThreads * 4];

  float* state = a.state + pair * (int64_t)M * Dv;
  const bool active = rg < RG;  // threads past CG*RG only help with the small loads

  // 1. issue the first rows' state loads (independent of the routing)
  float4 h[kRowsInFlight];
#pragma unroll
  for (int j = 0; j < kRowsInFlight; ++j) {
    const int r = rg + j * RG;
    if (active && r < M) h[j] = __ldcs(reinterpret_cast<const float4*>(state + (int64_t)r * Dv) + cg);
  }

  // 2. small inputs to shared memory
  const TIn* q = reinterpret_cast<const TIn*>(a.q) + pair * M;
  const TIn* k = reinterpret_cast<const TIn*>(a.k) + pair * M;
  const TIn* v = reinterpret_cast<const TIn*>(a.v) + pair * Dv;
  for (int i = tid; i < M; i += blockDim.x) s_q[i] = In<TIn>::ld(q + i);
  for (int d = tid; d < Dv; d += blockDim.x) s_v[d] = In<TIn>::ld(v + d);

  // 3. routing, decay and write weights of the selected slots (warp 0)
  if (tid < 32) {
    const int lane = tid;
    const float* lg = a.logits + pair * M;
    float x[E];
    load_row_logits<M>(lg, lane, x);
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

  // 4. sparse update of the selected rows, read over all rows
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (active) {
    const float4 vv = reinterpret_cast<const float4*>(s_v)[cg];
    for (int base = 0; base < M; base += kRowsInFlight * RG) {
      if (base > 0) {
#pragma unroll
        for (int j = 0; j < kRowsInFlight; ++j) {
          const int r = base + rg + j * RG;
          if (r < M) h[j] = __ldcs(reinterpret_cast<const float4*>(state + (int64_t)r * Dv) + cg);
        }
      }
#pragma unroll
      for (int j = 0; j < kRowsInFlight; ++j) {
        const int r = base + rg + j * RG;
        if (r < M) {
          float4 hv = h[j];
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
    reinterpret_cast<float4*>(s_red)[rg * CG + cg] = acc;
  }
  __syncthreads();

  // 5. reduce over the row groups
  for (int d = tid; d < Dv; d += blockDim.x) {
    float s = 0.f;
    for (int g = 0; g < RG; ++g) s += s_red[g * Dv + d];
    a.o[pair * Dv + d] = s;
  }
}

template <int M>
cudaError_t launch_m(const rsm_decode_args& a, cudaStream_t stream) {
  const unsigned grid = (unsigned)((int64_t)a.B * a.H);
  if (a.qkv_dtype == RSM_BF16)
    decode_kernel<M, __nv_bfloat16><<<grid, kDecodeThreads, 0, stream>>>(a);
  else
    decode_kernel<M, float><<<grid, kDecodeThreads, 0, stream>>>(a);
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
