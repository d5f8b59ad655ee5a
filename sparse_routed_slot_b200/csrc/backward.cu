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
// Launches:
//   1. the routing of every row (rsm_route's kernel: slots and sigmoid scores into the workspace);
//   2. one record per token, in parallel: its K entries (slot, a, w, s, f, k) and its v, q and dO
//      rows in fp32, stored time-contiguous per (b,h) stream, so the sequential sweeps gather
//      nothing and fetch a token with one bulk copy;
//   3. one CTA per (b,h) stream that runs
//      a forward sweep: the state in shared memory; before token t overwrites its K rows, they are
//        saved to a tape in the workspace ([pair][t][K][Dv] fp32); one barrier per token;
//      a reverse sweep: the state and G in shared memory; each token's rows are put back from the
//        tape after its gradients are taken; three barriers per token.
// Both sweeps are sequential over the tokens of a stream, so they are bound by the latency of a
// token step, not by bandwidth. A token's record (and, when it fits, its tape rows) reaches shared
// memory through a ring of bulk copies issued R-1 tokens ahead by one thread; the reductions over
// the value columns use a few lanes per slot; the gradients are written straight from the threads
// that form them.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rsm {

namespace {

constexpr int kBwdThreads = 512;
constexpr int kBwdWarps = kBwdThreads / 32;
constexpr int kRingMax = 8;

// One selected entry of a token: decay a, write weight w, score s, decay rate f, key k, slot.
struct alignas(16) Entry {
  float a, w, s, f;
  float k;
  int slot;
  float pad0, pad1;
};

// Token record: [K] Entry, v [Dv], q [M], dO [Dv] (fp32); a multiple of 16 bytes (Dv % 4 == 0).
__host__ __device__ inline int rec_bytes(int M, int K, int Dv) { return K * 32 + (2 * Dv + M) * 4; }
__host__ __device__ inline int rec_v(int K) { return K * 32; }
__host__ __device__ inline int rec_q(int K, int Dv) { return K * 32 + Dv * 4; }
__host__ __device__ inline int rec_dO(int M, int K, int Dv) { return K * 32 + (Dv + M) * 4; }

// Shared memory: the state H and its gradient G, the per-entry df terms of a token, and a ring of
// R token slots (a record, then its tape rows when they travel through the ring).
struct BwdSmem {
  int H, G, dfe;  // float offsets
  int ring, slot; // byte offset of the ring, bytes per slot
  int total;      // bytes
};

__host__ __device__ inline BwdSmem bwd_layout(int M, int K, int Dv, int R, bool tape) {
  BwdSmem s;
  int o = 0;
  s.H = o; o += M * Dv;
  s.G = o; o += M * Dv;
  s.dfe = o; o += K;
  s.ring = ((o * 4) + 15) & ~15;
  s.slot = rec_bytes(M, K, Dv) + (tape ? K * Dv * 4 : 0);
  s.total = s.ring + R * s.slot;
  return s;
}

constexpr int kSmemLimit = 232448;  // dynamic shared memory per block on B200

struct BwdParams {
  rsm_backward_args a;
  const int32_t* idx;   // [B*T*H, K] selected slots (rank order)
  const float* sc;      // [B*T*H, K] sigmoid scores
  unsigned char* rec;   // [pairs][T] token records
  float* tape;          // [pairs][T][K][Dv]
  int tape_ring;        // the tape rows travel through the ring
};

template <typename TIn>
RSM_DEV float ldin(const void* p, int64_t i) {
  return In<TIn>::ld(reinterpret_cast<const TIn*>(p) + i);
}

// Token records: one warp per (pair, t).
template <typename TIn>
__global__ void __launch_bounds__(256) records_kernel(const BwdParams P) {
  const rsm_backward_args& a = P.a;
  const int M = a.M, K = a.K, Dv = a.Dv;
  const int lane = threadIdx.x & 31;
  const int64_t n = (int64_t)a.B * a.H * a.T;
  const int RB = rec_bytes(M, K, Dv);
  for (int64_t g = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; g < n;
       g += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int64_t pair = g / a.T;
    const int64_t t = g - pair * a.T;
    const int64_t b = pair / a.H, h = pair - b * a.H;
    const int64_t row = (b * a.T + t) * a.H + h;
    unsigned char* rp = P.rec + g * RB;
    for (int j = lane; j < K; j += 32) {
      const int i = P.idx[row * K + j];
      const float s = P.sc[row * K + j];
      const float f = a.decay == RSM_DECAY_SLOT ? a.f[row * M + i] : a.f[row];
      const float lam = s * f;
      const float kv = ldin<TIn>(a.k, row * M + i);
      float4* ep = reinterpret_cast<float4*>(rp + j * 32);
      ep[0] = make_float4(expf(lam), kv * (-expm1f(lam)), s, f);
      ep[1] = make_float4(kv, __int_as_float(i), 0.f, 0.f);
    }
    float* vr = reinterpret_cast<float*>(rp + rec_v(K));
    float* qr = reinterpret_cast<float*>(rp + rec_q(K, Dv));
    float* dr = reinterpret_cast<float*>(rp + rec_dO(M, K, Dv));
    for (int d = lane; d < Dv; d += 32) {
      vr[d] = ldin<TIn>(a.v, row * Dv + d);
      dr[d] = a.dO ? a.dO[row * Dv + d] : 0.f;
    }
    for (int i = lane; i < M; i += 32) qr[i] = ldin<TIn>(a.q, row * M + i);
  }
}

// One CTA per (b,h) stream; R token slots in the ring.
template <int R>
__global__ void __launch_bounds__(kBwdThreads, 1) backward_kernel(const BwdParams P) {
  extern __shared__ __align__(16) float sm[];
  __shared__ __align__(8) uint64_t bar[R];  // slot s: the copies of its current token landed
  __shared__ int s_abort;                    // a copy did not land in time: no more waits or copies
  const rsm_backward_args& a = P.a;
  const int M = a.M, K = a.K, Dv = a.Dv, T = a.T;
  const bool tape_ring = P.tape_ring != 0;
  const BwdSmem L = bwd_layout(M, K, Dv, R, tape_ring);
  const int RB = rec_bytes(M, K, Dv);
  const int pair = blockIdx.x, b = pair / a.H, h = pair % a.H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* sH = sm + L.H;
  float* sG = sm + L.G;
  unsigned char* ring = reinterpret_cast<unsigned char*>(sm) + L.ring;
  const unsigned char* rec = P.rec + (int64_t)pair * T * RB;
  float* tape = P.tape + (int64_t)pair * T * K * Dv;
  auto row_of = [&](int t) -> int64_t { return ((int64_t)b * T + t) * a.H + h; };
  auto slot_of = [&](int t) -> unsigned char* { return ring + (t % R) * L.slot; };

  volatile int* abort_flag = &s_abort;
  if (tid == 0) {
    for (int s = 0; s < R; ++s) tc::mbar_init(&bar[s], 1);
    tc::fence_mbar_init();
    s_abort = 0;
  }
  // token t's copies into its slot (thread 0): the record, or its first part (entries and v) in
  // the forward sweep, and the tape rows in the reverse sweep when they travel through the ring
  uint32_t pend = 0;  // thread 0: bit s set while slot s has copies in flight that no wait has seen
  // test flag: the first token's copy is withheld, so its wait (bounded to one poll) expires while
  // the copies of the tokens after it are in flight
  const bool stall_test = (a.flags & RSM_FLAG_TEST_STALL_ROUTING) != 0;
  auto issue = [&](int t, bool rev) {
    if (tid != 0 || t < 0 || t >= T || *abort_flag || (stall_test && t == 0 && !rev)) return;
    unsigned char* sl = slot_of(t);
    uint64_t* br = &bar[t % R];
    pend |= 1u << (t % R);
    const uint32_t rb = rev ? (uint32_t)RB : (uint32_t)rec_q(K, Dv);
    const uint32_t tb = (rev && tape_ring) ? (uint32_t)(K * Dv * 4) : 0u;
    tc::mbar_arrive_expect_tx(br, rb + tb);
    tc::bulk_load(sl, rec + (int64_t)t * RB, rb, br);
    if (tb) tc::bulk_load(sl + RB, tape + (int64_t)t * K * Dv, tb, br);
  };
  // bit s: parity of slot s's next completion (every thread counts alike). After an expired wait
  // the kernel stops copying and waiting, and the parity of a slot whose wait was skipped stays
  // that of its copies in flight, which thread 0 drains (bounded) before the CTA ends.
  uint32_t par = 0;
  // one poll under the test flag (the drain below keeps the normal bound)
  const uint32_t wait_limit = stall_test ? 1u : (1u << 22);
  // true when this thread has seen token t's copies land; a token is processed only when every
  // thread has (a CTA-wide AND at the barrier that follows), so no thread ever indexes with
  // entries from a slot that was not filled
  auto wait_slot = [&](int t) -> bool {
    const int s = t % R;
    if (*abort_flag) return false;
    if (!tc::mbar_wait(&bar[s], (par >> s) & 1u, wait_limit)) {
      *abort_flag = 1;
      raise_status(RSM_ERR_TIMEOUT);
      return false;
    }
    par ^= 1u << s;
    pend &= ~(1u << s);
    return true;
  };

  for (int e = tid; e < M * Dv; e += kBwdThreads) sH[e] = a.H0 ? a.H0[(int64_t)pair * M * Dv + e] : 0.f;
  __syncthreads();  // barriers initialised
  // ---------------------------------------------------------------- forward sweep with tape
  for (int j = 0; j < R - 1; ++j) issue(j, false);
  for (int t = 0; t < T; ++t) {
    // token t is in, and token t-1 is finished: its slot can be refilled
    const bool ok = __syncthreads_and(wait_slot(t)) != 0;
    issue(t + R - 1, false);
    if (!ok) continue;
    const unsigned char* sl = slot_of(t);
    const Entry* en = reinterpret_cast<const Entry*>(sl);
    const float* vr = reinterpret_cast<const float*>(sl + rec_v(K));
    for (int r = warp; r < K; r += kBwdWarps) {
      const int i = en[r].slot;
      const float ar = en[r].a, wr = en[r].w;
      float* Hi = sH + i * Dv;
      float* tp = tape + ((int64_t)t * K + r) * Dv;
      for (int d = lane; d < Dv; d += 32) {
        const float hv = Hi[d];
        tp[d] = hv;
        Hi[d] = fmaf(ar, hv, wr * vr[d]);
      }
    }
  }
  __syncthreads();  // the state and the tape are complete; every slot is free
  // ---------------------------------------------------------------- reverse sweep
  for (int e = tid; e < M * Dv; e += kBwdThreads) sG[e] = a.dHT ? a.dHT[(int64_t)pair * M * Dv + e] : 0.f;
  // phase A assignment: tps lanes per slot (M divides 512), float4 columns j, j + tps, ...
  const int tps = kBwdThreads / M;
  const int ai = tid / tps, aj = tid - ai * tps;
  const int dv4 = Dv / 4;
  for (int j = 0; j < R - 1; ++j) issue(T - 1 - j, true);
  for (int t = T - 1; t >= 0; --t) {
    const int64_t row = row_of(t);
    const bool ok = __syncthreads_and(wait_slot(t)) != 0;  // token t is in; token t+1 is finished
    issue(t - (R - 1), true);
    const unsigned char* sl = slot_of(t);
    const Entry* en = reinterpret_cast<const Entry*>(sl);
    const float* vr = reinterpret_cast<const float*>(sl + rec_v(K));
    const float* qr = reinterpret_cast<const float*>(sl + rec_q(K, Dv));
    const float4* dO4 = reinterpret_cast<const float4*>(sl + rec_dO(M, K, Dv));
    // ---- phase A: the read. dq_i = do . H_t[i] and G[i] += q_i do, slot i by tps lanes; the slot
    // gradients of the row start at zero (the selected entries overwrite theirs after the barrier)
    if (!ok) {
      // the token's copies did not land (an expired wait): no work, the barriers still match
    } else if (a.dO) {
      const float qi = qr[ai];
      const float4* H4 = reinterpret_cast<const float4*>(sH + ai * Dv);
      float4* G4 = reinterpret_cast<float4*>(sG + ai * Dv);
      float acc = 0.f;
      for (int c = aj; c < dv4; c += tps) {
        const float4 o = dO4[c], hv = H4[c];
        float4 g = G4[c];
        acc = fmaf(o.x, hv.x, fmaf(o.y, hv.y, fmaf(o.z, hv.z, fmaf(o.w, hv.w, acc))));
        g.x = fmaf(qi, o.x, g.x);
        g.y = fmaf(qi, o.y, g.y);
        g.z = fmaf(qi, o.z, g.z);
        g.w = fmaf(qi, o.w, g.w);
        G4[c] = g;
      }
      for (int o = tps >> 1; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
      if (aj == 0 && a.dq) a.dq[row * M + ai] = acc;
    } else if (a.dq && aj == 0) {
      a.dq[row * M + ai] = 0.f;
    }
    if (ok && aj == 0) {
      if (a.dk) a.dk[row * M + ai] = 0.f;
      if (a.dlogits) a.dlogits[row * M + ai] = 0.f;
      if (a.df && a.decay == RSM_DECAY_SLOT) a.df[row * M + ai] = 0.f;
    }
    __syncthreads();
    // ---- phase B: gradients of the selected entries (one warp per entry; a token's slots are
    // distinct), and dv_t = sum_r w_r G[i_r] by column (the last Dv threads)
    for (int r = warp; ok && r < K; r += kBwdWarps) {
      const Entry e = en[r];
      const float* Gi = sG + e.slot * Dv;
      const float* tp = tape_ring ? reinterpret_cast<const float*>(sl + RB) + r * Dv : tape + ((int64_t)t * K + r) * Dv;
      float dw = 0.f, dap = 0.f;
      for (int d = lane; d < Dv; d += 32) {
        const float g = Gi[d];
        dw = fmaf(g, vr[d], dw);
        dap = fmaf(g, tp[d], dap);
      }
      dw = warp_sum_f(dw);
      dap = warp_sum_f(dap);
      const float dlam = e.a * (dap - e.k * dw);
      if (lane == 0) {
        if (a.dk) a.dk[row * M + e.slot] = (1.f - e.a) * dw;
        if (a.dlogits) a.dlogits[row * M + e.slot] = e.s * (1.f - e.s) * (e.f * dlam);
        if (a.df && a.decay == RSM_DECAY_SLOT) a.df[row * M + e.slot] = e.s * dlam;
        sm[L.dfe + r] = e.s * dlam;
      }
    }
    if (ok && a.dv) {
      const int d = tid - (kBwdThreads - Dv);
      if (d >= 0) {
        float acc = 0.f;
        for (int r = 0; r < K; ++r) acc = fmaf(en[r].w, sG[en[r].slot * Dv + d], acc);
        a.dv[row * Dv + d] = acc;
      }
    }
    __syncthreads();
    // ---- phase C: G of the selected rows decays, their state rows go back to H_{t-1}; the
    // per-head df of the token out
    for (int r = warp; ok && r < K; r += kBwdWarps) {
      const int i = en[r].slot;
      const float ar = en[r].a;
      float* Gi = sG + i * Dv;
      float* Hi = sH + i * Dv;
      const float* tp = tape_ring ? reinterpret_cast<const float*>(sl + RB) + r * Dv : tape + ((int64_t)t * K + r) * Dv;
      for (int d = lane; d < Dv; d += 32) {
        Gi[d] *= ar;
        Hi[d] = tp[d];
      }
    }
    if (ok && a.df && a.decay == RSM_DECAY_HEAD && warp == kBwdWarps - 1) {
      float acc = 0.f;
      for (int r = lane; r < K; r += 32) acc += sm[L.dfe + r];
      acc = warp_sum_f(acc);
      if (lane == 0) a.df[row] = acc;
    }
  }
  __syncthreads();
  if (tid == 0 && pend) {  // only after an expired wait: no copy may land once the CTA is gone
    for (int sl = 0; sl < R; ++sl)
      if (pend & (1u << sl)) tc::mbar_wait(&bar[sl], (par >> sl) & 1u);
  }
  if (a.dH0)
    for (int e = tid; e < M * Dv; e += kBwdThreads) a.dH0[(int64_t)pair * M * Dv + e] = sG[e];
}

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

struct BwdWs {
  size_t idx, sc, rec, tape, total;
};
BwdWs bwd_ws(const rsm_backward_args& a) {
  BwdWs w;
  const size_t rows = (size_t)a.B * a.T * a.H;
  w.idx = 0;
  w.sc = up256(rows * a.K * 4);
  w.rec = w.sc + up256(rows * a.K * 4);
  w.tape = w.rec + up256(rows * (size_t)rec_bytes(a.M, a.K, a.Dv));
  w.total = w.tape + up256(rows * (size_t)a.K * a.Dv * 4);
  return w;
}

// Ring depth and tape placement for a shape: 8 slots with the tape, else 8 without it, else 2.
struct RingPlan {
  int R;
  bool tape;
  int smem;
};
RingPlan ring_plan(int M, int K, int Dv) {
  const int rs[3] = {kRingMax, kRingMax, 2};
  const bool tp[3] = {true, false, false};
  for (int c = 0; c < 3; ++c) {
    const int bytes = bwd_layout(M, K, Dv, rs[c], tp[c]).total;
    if (bytes <= kSmemLimit) return {rs[c], tp[c], bytes};
  }
  return {2, false, bwd_layout(M, K, Dv, 2, false).total};
}

template <int R>
cudaError_t run_sweep(const BwdParams& P, unsigned grid, int smem, cudaStream_t stream) {
  cudaError_t e = set_smem_limit<backward_kernel<R>>(smem);
  if (e == cudaSuccess) backward_kernel<R><<<grid, kBwdThreads, smem, stream>>>(P);
  return e;
}

}  // namespace

size_t backward_smem_bytes(int M, int K, int Dv) { return (size_t)ring_plan(M, K, Dv).smem; }

size_t backward_workspace_bytes(const rsm_backward_args& a) { return bwd_ws(a).total; }

cudaError_t launch_backward(const rsm_backward_args& a, cudaStream_t stream) {
  const BwdWs w = bwd_ws(a);
  char* ws = static_cast<char*>(a.workspace);
  BwdParams P;
  P.a = a;
  P.idx = reinterpret_cast<int32_t*>(ws + w.idx);
  P.sc = reinterpret_cast<float*>(ws + w.sc);
  P.rec = reinterpret_cast<unsigned char*>(ws + w.rec);
  P.tape = reinterpret_cast<float*>(ws + w.tape);
  const RingPlan rp = ring_plan(a.M, a.K, a.Dv);
  P.tape_ring = rp.tape ? 1 : 0;
  const int64_t rows = (int64_t)a.B * a.T * a.H;
  cudaError_t e = launch_route(a.logits, rows, a.M, a.K, const_cast<int32_t*>(P.idx), const_cast<float*>(P.sc),
                               (int)RSM_ROUTER_SIGMOID, (a.flags & RSM_FLAG_VALIDATE) ? 1 : 0, stream);
  if (e != cudaSuccess) return e;
  const unsigned rgrid = (unsigned)std::min<int64_t>((rows + 7) / 8, (int64_t)device_sm_count() * 8);
  if (a.qkv_dtype == RSM_BF16) records_kernel<__nv_bfloat16><<<rgrid, 256, 0, stream>>>(P);
  else records_kernel<float><<<rgrid, 256, 0, stream>>>(P);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((int64_t)a.B * a.H);
  e = rp.R == kRingMax ? run_sweep<kRingMax>(P, grid, rp.smem, stream) : run_sweep<2>(P, grid, rp.smem, stream);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace rsm
