// backward.cu -- gradients of the RSM mixer (rsm_backward), on CUDA cores in fp32.
//
// Reverse-mode differentiation of the recurrence (Raven README "How Raven Works"; the sigmoid
// router), with G = dL/dH per (b,h) and, per token t from the last to the first, selected slots
// i in S_t, a_i = e^{s_i f}, w_i = (1 - a_i) k_i:
//   read o_t = sum_i q_i H_t[i]:       dq_t[i] = do_t . H_t[i];   G[i] += q_i do_t  (every slot)
//   write H_t[i] = a_i H_{t-1}[i] + w_i v_t:
//     dv_t += w_i G[i];  dw_i = G[i] . v_t;  da_i = G[i] . H_{t-1}[i] - k_i dw_i;
//     dk_{t,i} = (1 - a_i) dw_i;  dlam_i = a_i da_i;  df += s_i dlam_i (per head; per slot: df_i);
//     dlogit_i = s_i (1 - s_i) f dlam_i;  then G[i] = a_i G[i]
//   unselected slots pass G unchanged and get no key or logit gradient (the TopK cut is
//   piecewise constant in the logits); dH0 = G after the first token.
//
// Launches: the routing of every row (rsm_route's kernel: slots and sigmoid scores into the
// workspace), then one CTA per (b,h) stream that runs
//   a forward sweep: the state in shared memory; before token t overwrites its K rows, they are
//     saved to a tape in the workspace ([pair][t][K][Dv] fp32);
//   a reverse sweep: the state and G in shared memory; each token's rows are put back from the
//     tape after its gradients are taken.
// Both sweeps are sequential over the tokens of a stream; the parallelism is over streams and,
// within a token, over slots and value columns.
#include "common.cuh"
#include "kernels.h"

namespace rsm {

namespace {

constexpr int kBwdThreads = 512;
constexpr int kBwdWarps = kBwdThreads / 32;

struct BwdSmem {
  int H, G, q, dO, v, dq, dk, dl, df, dv, ea, ew, es, ef, slot;  // float offsets (slot: int)
  int total;                                                     // bytes
};

__host__ __device__ inline BwdSmem bwd_layout(int M, int K, int Dv) {
  BwdSmem s;
  int o = 0;
  s.H = o; o += M * Dv;
  s.G = o; o += M * Dv;
  s.q = o; o += M;
  s.dO = o; o += Dv;
  s.v = o; o += Dv;
  s.dq = o; o += M;
  s.dk = o; o += M;
  s.dl = o; o += M;
  s.df = o; o += M;
  s.dv = o; o += Dv;
  s.ea = o; o += K;
  s.ew = o; o += K;
  s.es = o; o += K;
  s.ef = o; o += K;
  s.slot = o; o += K;
  s.total = o * 4;
  return s;
}

struct BwdParams {
  rsm_backward_args a;
  const int32_t* idx;  // [B*T*H, K] selected slots (rank order)
  const float* sc;     // [B*T*H, K] sigmoid scores
  float* tape;         // [pairs][T][K][Dv]
};

template <typename TIn>
RSM_DEV float ldin(const void* p, int64_t i) {
  return In<TIn>::ld(reinterpret_cast<const TIn*>(p) + i);
}

// Loads token `row`'s selected entries into shared memory: slot, score, f, decay a, weight w.
template <typename TIn>
RSM_DEV void load_entries(const BwdParams& P, int64_t row, const BwdSmem& L, float* sm) {
  const rsm_backward_args& a = P.a;
  int* slot = reinterpret_cast<int*>(sm + L.slot);
  for (int j = threadIdx.x; j < a.K; j += kBwdThreads) {
    const int i = P.idx[row * a.K + j];
    const float s = P.sc[row * a.K + j];
    const float f = a.decay == RSM_DECAY_SLOT ? a.f[row * a.M + i] : a.f[row];
    const float lam = s * f;
    slot[j] = i;
    sm[L.es + j] = s;
    sm[L.ef + j] = f;
    sm[L.ea + j] = expf(lam);
    sm[L.ew + j] = ldin<TIn>(a.k, row * a.M + i) * (-expm1f(lam));
  }
}

template <typename TIn>
__global__ void __launch_bounds__(kBwdThreads, 1) backward_kernel(const BwdParams P) {
  extern __shared__ __align__(16) float sm[];
  const rsm_backward_args& a = P.a;
  const int M = a.M, K = a.K, Dv = a.Dv, T = a.T, H = a.H;
  const BwdSmem L = bwd_layout(M, K, Dv);
  const int pair = blockIdx.x, b = pair / H, h = pair % H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* sH = sm + L.H;
  float* sG = sm + L.G;
  const int* slot = reinterpret_cast<const int*>(sm + L.slot);
  float* tape = P.tape + (int64_t)pair * T * K * Dv;

  for (int e = tid; e < M * Dv; e += kBwdThreads) sH[e] = a.H0 ? a.H0[(int64_t)pair * M * Dv + e] : 0.f;
  // ---------------------------------------------------------------- forward sweep with tape
  for (int t = 0; t < T; ++t) {
    const int64_t row = ((int64_t)b * T + t) * H + h;
    load_entries<TIn>(P, row, L, sm);
    for (int d = tid; d < Dv; d += kBwdThreads) sm[L.v + d] = ldin<TIn>(a.v, row * Dv + d);
    __syncthreads();
    for (int r = warp; r < K; r += kBwdWarps) {
      const int i = slot[r];
      const float ar = sm[L.ea + r], wr = sm[L.ew + r];
      float* Hi = sH + i * Dv;
      float* tp = tape + ((int64_t)t * K + r) * Dv;
      for (int d = lane; d < Dv; d += 32) {
        const float hv = Hi[d];
        tp[d] = hv;
        Hi[d] = fmaf(ar, hv, wr * sm[L.v + d]);
      }
    }
    __syncthreads();
  }
  // ---------------------------------------------------------------- reverse sweep
  for (int e = tid; e < M * Dv; e += kBwdThreads) sG[e] = a.dHT ? a.dHT[(int64_t)pair * M * Dv + e] : 0.f;
  for (int t = T - 1; t >= 0; --t) {
    const int64_t row = ((int64_t)b * T + t) * H + h;
    load_entries<TIn>(P, row, L, sm);
    for (int i = tid; i < M; i += kBwdThreads) {
      sm[L.q + i] = ldin<TIn>(a.q, row * M + i);
      sm[L.dk + i] = 0.f;
      sm[L.dl + i] = 0.f;
      sm[L.df + i] = 0.f;
    }
    for (int d = tid; d < Dv; d += kBwdThreads) {
      sm[L.dO + d] = a.dO ? a.dO[row * Dv + d] : 0.f;
      sm[L.v + d] = ldin<TIn>(a.v, row * Dv + d);
      sm[L.dv + d] = 0.f;
    }
    __syncthreads();
    // the read: dq from H_t, then G += q (x) do
    for (int i = warp; i < M; i += kBwdWarps) {
      float acc = 0.f;
      for (int d = lane; d < Dv; d += 32) acc = fmaf(sm[L.dO + d], sH[i * Dv + d], acc);
      acc = warp_sum_f(acc);
      if (lane == 0) sm[L.dq + i] = acc;
    }
    for (int e = tid; e < M * Dv; e += kBwdThreads) sG[e] = fmaf(sm[L.q + e / Dv], sm[L.dO + e % Dv], sG[e]);
    __syncthreads();
    // the writes of the selected slots (one warp per entry; the slots of a token are distinct)
    for (int r = warp; r < K; r += kBwdWarps) {
      const int i = slot[r];
      const float ar = sm[L.ea + r], wr = sm[L.ew + r], s = sm[L.es + r], f = sm[L.ef + r];
      float* Gi = sG + i * Dv;
      float* Hi = sH + i * Dv;
      const float* tp = tape + ((int64_t)t * K + r) * Dv;
      float dw = 0.f, dap = 0.f;
      for (int d = lane; d < Dv; d += 32) {
        const float g = Gi[d];
        dw = fmaf(g, sm[L.v + d], dw);
        dap = fmaf(g, tp[d], dap);
        atomicAdd(sm + L.dv + d, wr * g);
      }
      dw = warp_sum_f(dw);
      dap = warp_sum_f(dap);
      const float da = dap - ldin<TIn>(a.k, row * M + i) * dw;
      const float dlam = ar * da;
      if (lane == 0) {
        sm[L.dk + i] = (1.f - ar) * dw;
        sm[L.df + i] = s * dlam;
        sm[L.dl + i] = s * (1.f - s) * (f * dlam);
      }
      for (int d = lane; d < Dv; d += 32) {
        Gi[d] *= ar;
        Hi[d] = tp[d];
      }
    }
    __syncthreads();
    // this token's gradients out
    for (int i = tid; i < M; i += kBwdThreads) {
      if (a.dq) a.dq[row * M + i] = sm[L.dq + i];
      if (a.dk) a.dk[row * M + i] = sm[L.dk + i];
      if (a.dlogits) a.dlogits[row * M + i] = sm[L.dl + i];
      if (a.df && a.decay == RSM_DECAY_SLOT) a.df[row * M + i] = sm[L.df + i];
    }
    if (a.df && a.decay == RSM_DECAY_HEAD && warp == 0) {
      float acc = 0.f;
      for (int r = lane; r < K; r += 32) acc += sm[L.df + slot[r]];
      acc = warp_sum_f(acc);
      if (lane == 0) a.df[row] = acc;
    }
    if (a.dv)
      for (int d = tid; d < Dv; d += kBwdThreads) a.dv[row * Dv + d] = sm[L.dv + d];
    __syncthreads();
  }
  if (a.dH0)
    for (int e = tid; e < M * Dv; e += kBwdThreads) a.dH0[(int64_t)pair * M * Dv + e] = sG[e];
}

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

struct BwdWs {
  size_t idx, sc, tape, total;
};
BwdWs bwd_ws(const rsm_backward_args& a) {
  BwdWs w;
  const size_t rows = (size_t)a.B * a.T * a.H;
  w.idx = 0;
  w.sc = up256(rows * a.K * 4);
  w.tape = w.sc + up256(rows * a.K * 4);
  w.total = w.tape + up256(rows * (size_t)a.K * a.Dv * 4);
  return w;
}

}  // namespace

size_t backward_smem_bytes(int M, int K, int Dv) { return (size_t)bwd_layout(M, K, Dv).total; }

size_t backward_workspace_bytes(const rsm_backward_args& a) { return bwd_ws(a).total; }

cudaError_t launch_backward(const rsm_backward_args& a, cudaStream_t stream) {
  const BwdWs w = bwd_ws(a);
  char* ws = static_cast<char*>(a.workspace);
  BwdParams P;
  P.a = a;
  P.idx = reinterpret_cast<int32_t*>(ws + w.idx);
  P.sc = reinterpret_cast<float*>(ws + w.sc);
  P.tape = reinterpret_cast<float*>(ws + w.tape);
  const int64_t rows = (int64_t)a.B * a.T * a.H;
  cudaError_t e = launch_route(a.logits, rows, a.M, a.K, const_cast<int32_t*>(P.idx), const_cast<float*>(P.sc),
                               (int)RSM_ROUTER_SIGMOID, (a.flags & RSM_FLAG_VALIDATE) ? 1 : 0, stream);
  if (e != cudaSuccess) return e;
  const int smem = bwd_layout(a.M, a.K, a.Dv).total;
  const unsigned grid = (unsigned)((int64_t)a.B * a.H);
  if (a.qkv_dtype == RSM_BF16) {
    e = set_smem_limit<backward_kernel<__nv_bfloat16>>(smem);
    if (e == cudaSuccess) backward_kernel<__nv_bfloat16><<<grid, kBwdThreads, smem, stream>>>(P);
  } else {
    e = set_smem_limit<backward_kernel<float>>(smem);
    if (e == cudaSuccess) backward_kernel<float><<<grid, kBwdThreads, smem, stream>>>(P);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace rsm
