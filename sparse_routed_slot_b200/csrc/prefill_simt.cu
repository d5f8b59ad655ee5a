// prefill_simt.cu -- chunked prefill on CUDA cores in fp32 (rsm_forward, RSM_PATH_SIMT).
//
// The fp32 path (1e-4 parity class) and the fallback for sizes the tensor-core path does not
// cover. One CTA owns one (b,h) stream and one tile of DT state columns, and walks the sequence
// in chunks of C = 32 tokens with its state tile resident in shared memory.
//
// Chunk algebra (paperlayer.ai summary, section A.5: chunkwise computation over T = n*C tokens),
// with g_{t,i} the cumulative log-decay of slot i from the chunk start through token t
// (g <= 0, non-increasing in t), w_{t,i} = k_{t,i} (1 - a_{t,i}) on the selected slots:
//   o_t   = (q_t * e^{g_t}) . H_start  +  sum_{s<=t} A_{t,s} v_s
//   A_{t,s} = sum_{i in S_s} q_{t,i} w_{s,i} e^{g_{t,i} - g_{s,i}}        (pairwise, sparse)
//   H_end = e^{g_C} * H_start + sum_s (w_s * e^{g_C - g_s}) (x) v_s
// Every exponential has a non-positive argument, so the path is exact in structure for any
// finite decay (no overflow, underflow only of terms that are truly negligible). Rows never
// selected in a chunk are skipped, so they keep their bits.
#include "common.cuh"
#include "kernels.h"

namespace rsm {

namespace {

constexpr int kC = 32;          // tokens per chunk
constexpr int kThreads = 1024;  // 32 warps: one routing row per warp, and latency hidden by width

// Value columns per CTA: 64 (32 at M = 256, for shared memory). It divides the thread count, as
// the register-blocked output and carry loops need; a narrower last tile is masked (DTe).
__host__ __device__ inline int simt_dt(int M, int /*Dv*/) { return M >= 256 ? 32 : 64; }
static_assert(kThreads % 64 == 0 && kThreads / 32 <= 32, "tile mapping: G = kThreads / DT groups <= kC");

struct SimtSmem {
  // float offsets into the dynamic shared buffer
  int g, q, qh, w, H, v, A, gC, D;
  int bytes_f;     // floats used by the above
  int sidx, touch; // byte offsets of the uint8 rank table and the int touch flags
  int total;       // bytes
};

__host__ __device__ inline SimtSmem simt_layout(int M, int DT) {
  SimtSmem s;
  int off = 0;
  s.g = off;  off += kC * M;
  s.q = off;  off += kC * M;
  s.qh = off; off += kC * M;
  s.w = off;  off += kC * M;
  s.H = off;  off += M * DT;
  s.v = off;  off += kC * DT;
  s.A = off;  off += kC * kC;
  s.gC = off; off += M;
  s.D = off;  off += M;
  s.bytes_f = off;
  int b = off * 4;
  s.touch = b; b += M * 4;
  s.sidx = b; b += kC * M;
  s.total = (b + 15) & ~15;
  return s;
}

template <int M, typename TIn>
__global__ void __launch_bounds__(kThreads) prefill_simt_kernel(rsm_forward_args a, int DT) {
  constexpr int E = M / 32;
  extern __shared__ __align__(16) unsigned char smem[];
  const SimtSmem L = simt_layout(M, DT);
  float* sf = reinterpret_cast<float*>(smem);
  float* s_g = sf + L.g;
  float* s_q = sf + L.q;
  float* s_qh = sf + L.qh;
  float* s_w = sf + L.w;
  float* s_H = sf + L.H;
  float* s_v = sf + L.v;
  float* s_A = sf + L.A;
  float* s_gC = sf + L.gC;
  float* s_D = sf + L.D;
  int* s_touch = reinterpret_cast<int*>(smem + L.touch);
  unsigned char* s_sidx = smem + L.sidx;

  const int T = a.T, H = a.H, K = a.K, Dv = a.Dv;
  const int pair = blockIdx.x;
  const int b = pair / H, h = pair % H;
  const int d0 = blockIdx.y * DT;
  const int DTe = min(DT, Dv - d0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool route_owner = blockIdx.y == 0;  // only one column tile writes the routing outputs
  const bool validate = (a.flags & RSM_FLAG_VALIDATE) && route_owner;

  const TIn* q = reinterpret_cast<const TIn*>(a.q);
  const TIn* k = reinterpret_cast<const TIn*>(a.k);
  const TIn* v = reinterpret_cast<const TIn*>(a.v);

  // initial state tile
  for (int p = tid; p < M * DT; p += kThreads) {
    const int i = p / DT, dd = p % DT;
    s_H[p] = (dd < DTe && a.H0) ? a.H0[((int64_t)pair * M + i) * Dv + d0 + dd] : 0.f;
  }

  float guess = __int_as_float(0x7fc00000);  // the warp's last threshold (none yet)
  for (int c0 = 0; c0 < T; c0 += kC) {
    const int nrows = min(kC, T - c0);
    for (int i = tid; i < M; i += kThreads) s_touch[i] = 0;
    __syncthreads();

    // --- routing, log-decay and write weights of the chunk's rows (one warp per row). Every load
    // of the chunk is issued before the ranking (this thread's value elements, and at M <= 128 the
    // row's q and k beside its logits), so the chunk waits on one memory round trip, not three.
    constexpr int kVRegs = kC * 64 / kThreads;  // value elements per thread at DT = 64
    constexpr bool kEarlyQK = E <= 4;
    constexpr bool kSetSelect = E <= 4;  // at M = 256 its registers would spill
    float vr[kVRegs];
#pragma unroll
    for (int j = 0; j < kVRegs; ++j) {
      const int p = tid + j * kThreads;
      const int t = p / DT, dd = p % DT;
      vr[j] = (p < kC * DT && t < nrows && dd < DTe)
                  ? In<TIn>::ld(v + (((int64_t)b * T + c0 + t) * H + h) * Dv + d0 + dd)
                  : 0.f;
    }
    for (int t = warp; t < kC; t += kThreads / 32) {
      if (t < nrows) {
        const int64_t row = ((int64_t)b * T + c0 + t) * H + h;
        float x[E];
        load_row_logits<M>(a.logits + row * M, lane, x);
        float fv[E], qv[E], kv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
          fv[e] = (a.decay == RSM_DECAY_SLOT) ? a.f[row * M + lane * E + e] : a.f[row];
          if (kEarlyQK) {
            qv[e] = In<TIn>::ld(q + row * M + lane * E + e);
            kv[e] = In<TIn>::ld(k + row * M + lane * E + e);
          }
        }
        if (validate) {
          bool bad = false;
#pragma unroll
          for (int e = 0; e < E; ++e) bad |= !finite_f32(x[e]) || !finite_f32(fv[e]) || fv[e] > 0.f;
          if (__any_sync(kFull, bad) && lane == 0) raise_status(RSM_ERR_NONFINITE);
        }
        int32_t* io = (route_owner && a.idx_out) ? a.idx_out + row * K : nullptr;
        float* so = (route_owner && a.score_out) ? a.score_out + row * K : nullptr;
        int32_t* cnt = (route_owner && a.slot_counts) ? a.slot_counts + (int64_t)pair * M : nullptr;
        int rank[E];
        uint32_t sel = 0u;
        // Without ranked outputs the entries' order is free: the exact TopK set from a threshold
        // search seeded with the warp's previous row, listed in slot order; the ranking tournament
        // when outputs want rank order, or when the search meets a tie at the cut
        bool listed = false;
        if (kSetSelect && !io && !so && K >= 2 && K < M && warp_select_guess<M>(x, K, guess, sel)) {
          const int n = __popc(sel);
          int before = n;  // inclusive scan of the lanes' counts
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, before, o);
            if (lane >= o) before += y;
          }
          int r = before - n;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            if (sel & (1u << e)) {
              const int slot = lane * E + e;
              s_sidx[t * M + r] = (unsigned char)slot;
              if (cnt) atomicAdd(cnt + slot, 1);
              set_rank<E>(rank, e, r);
              ++r;
            }
          }
          listed = true;
        }
        if (!listed)
          sel = warp_topk<M>(x, K, lane, [&](int r, int slot, int e) {
            s_sidx[t * M + r] = (unsigned char)slot;
            if (io) io[r] = slot;
            if (cnt) atomicAdd(cnt + slot, 1);
            set_rank<E>(rank, e, r);
          });
        float sc[E];
        warp_router_scores<E>(x, sel, a.router, sc);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = lane * E + e;
          s_q[t * M + i] = kEarlyQK ? qv[e] : In<TIn>::ld(q + row * M + i);
          if (sel & (1u << e)) {
            if (so) so[rank[e]] = sc[e];
            const float lam = sc[e] * fv[e];
            s_g[t * M + i] = lam;
            s_w[t * M + i] = (kEarlyQK ? kv[e] : In<TIn>::ld(k + row * M + i)) * (-expm1f(lam));
            s_touch[i] = 1;
          } else {
            s_g[t * M + i] = 0.f;
            s_w[t * M + i] = 0.f;
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = lane * E + e;
          s_q[t * M + i] = 0.f;
          s_g[t * M + i] = 0.f;
          s_w[t * M + i] = 0.f;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kVRegs; ++j) {
      const int p = tid + j * kThreads;
      if (p < kC * DT) s_v[p] = vr[j];
    }
    __syncthreads();

    // --- cumulative log-decay per slot (a prefix sum down the chunk), chunk decay
    bool strong = false;  // some slot decays by more than e^-80 in the chunk
    for (int i = tid; i < M; i += kThreads) {
      float g = 0.f;
      for (int t = 0; t < kC; ++t) {
        g += s_g[t * M + i];
        s_g[t * M + i] = g;
      }
      s_gC[i] = g;
      s_D[i] = expf(g);
      strong |= g < -80.f;
    }
    // A from start-referenced factors (below) unless a slot decays too strongly for e^{-g} to stay
    // finite; the entry table takes the raw q's memory, so K <= M/2
    const bool factored = !__syncthreads_or(strong) && 2 * K <= M;
    // --- q scaled to the chunk start, every element in parallel
    for (int p = tid; p < kC * M; p += kThreads) s_qh[p] = s_q[p] * expf(s_g[p]);
    float2* s_ent = reinterpret_cast<float2*>(s_q);  // [K][kC]: (slot, w e^{-g}) of entry r of token s
    if (factored) {
      __syncthreads();  // the raw q is consumed
      for (int p = tid; p < kC * K; p += kThreads) {
        const int r = p / kC, s = p - r * kC;
        int j = 0;
        float wh = 0.f;
        if (s < nrows) {
          j = s_sidx[s * M + r];
          wh = s_w[s * M + j] * expf(-s_g[s * M + j]);
        }
        s_ent[p] = make_float2(__int_as_float(j), wh);
      }
      __syncthreads();
    }

    // --- intra-chunk weights A[t][s], s <= t (sparse over the K slots written at s); each
    // thread carries its kC*kC/kThreads pairs together so that their exponentials overlap
    {
      constexpr int kPairs = kC * kC / kThreads;  // 1
      float acc[kPairs];
      int tt[kPairs], ss[kPairs];
#pragma unroll
      for (int k = 0; k < kPairs; ++k) {
        const int p = tid + k * kThreads;
        tt[k] = p / kC;
        ss[k] = p % kC;
        acc[k] = 0.f;
      }
      if (factored) {
        // A[t][s] = sum_r (q_{t,j} e^{g_{t,j}}) (w_{s,j} e^{-g_{s,j}}), j = slot of entry r of s
        for (int r = 0; r < K; ++r) {
#pragma unroll
          for (int k = 0; k < kPairs; ++k) {
            const int t = tt[k], s = ss[k];
            if (s <= t && t < nrows) {
              const float2 e = s_ent[r * kC + s];
              acc[k] = fmaf(s_qh[t * M + __float_as_int(e.x)], e.y, acc[k]);
            }
          }
        }
      } else {
        for (int r = 0; r < K; ++r) {
#pragma unroll
          for (int k = 0; k < kPairs; ++k) {
            const int t = tt[k], s = ss[k];
            if (s <= t && t < nrows) {
              const int j = s_sidx[s * M + r];
              acc[k] = fmaf(s_q[t * M + j] * s_w[s * M + j], expf(s_g[t * M + j] - s_g[s * M + j]), acc[k]);
            }
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kPairs; ++k) s_A[tid + k * kThreads] = acc[k];
    }
    __syncthreads();

    // --- outputs of the chunk for this column tile: thread (tp, cg) computes tokens 2tp, 2tp+1 x
    // columns 4cg..4cg+3, so each state row piece and value row piece it loads (16 bytes) serves
    // eight products
    {
      const int ncg = DT / 4;
      if (tid < (kC / 2) * ncg) {
        const int tp = tid / ncg, cg = tid - tp * ncg;
        const int t0 = 2 * tp;
        float4 o0 = make_float4(0.f, 0.f, 0.f, 0.f), o1 = o0;
#pragma unroll 4
        for (int i = 0; i < M; ++i) {
          const float4 hv = *reinterpret_cast<const float4*>(s_H + i * DT + 4 * cg);
          const float q0 = s_qh[t0 * M + i], q1 = s_qh[(t0 + 1) * M + i];
          o0.x = fmaf(q0, hv.x, o0.x); o0.y = fmaf(q0, hv.y, o0.y); o0.z = fmaf(q0, hv.z, o0.z); o0.w = fmaf(q0, hv.w, o0.w);
          o1.x = fmaf(q1, hv.x, o1.x); o1.y = fmaf(q1, hv.y, o1.y); o1.z = fmaf(q1, hv.z, o1.z); o1.w = fmaf(q1, hv.w, o1.w);
        }
#pragma unroll 4
        for (int s = 0; s <= t0; ++s) {
          const float4 vv = *reinterpret_cast<const float4*>(s_v + s * DT + 4 * cg);
          const float a0 = s_A[t0 * kC + s], a1 = s_A[(t0 + 1) * kC + s];
          o0.x = fmaf(a0, vv.x, o0.x); o0.y = fmaf(a0, vv.y, o0.y); o0.z = fmaf(a0, vv.z, o0.z); o0.w = fmaf(a0, vv.w, o0.w);
          o1.x = fmaf(a1, vv.x, o1.x); o1.y = fmaf(a1, vv.y, o1.y); o1.z = fmaf(a1, vv.z, o1.z); o1.w = fmaf(a1, vv.w, o1.w);
        }
        {  // s = t0 + 1 reaches token t0 + 1 only
          const float4 vv = *reinterpret_cast<const float4*>(s_v + (t0 + 1) * DT + 4 * cg);
          const float a1 = s_A[(t0 + 1) * kC + t0 + 1];
          o1.x = fmaf(a1, vv.x, o1.x); o1.y = fmaf(a1, vv.y, o1.y); o1.z = fmaf(a1, vv.z, o1.z); o1.w = fmaf(a1, vv.w, o1.w);
        }
        // Dv and the tile start are multiples of 4, so a column group is wholly inside or outside
        if (4 * cg < DTe) {
          float* op = a.o + (((int64_t)b * T + c0 + t0) * H + h) * Dv + d0 + 4 * cg;
          if (t0 < nrows) *reinterpret_cast<float4*>(op) = o0;
          if (t0 + 1 < nrows) *reinterpret_cast<float4*>(op + (int64_t)H * Dv) = o1;
        }
      }
    }
    // --- write weights carried to the chunk end (non-positive exponents)
    for (int p = tid; p < kC * M; p += kThreads) {
      const int t = p / M, i = p % M;
      const float w = s_w[p];
      if (w != 0.f) s_w[p] = w * expf(s_gC[i] - s_g[t * M + i]);
    }
    __syncthreads();

    // --- state carry; slots not selected in this chunk are left untouched. Thread (ig, cg)
    // updates slots 4ig..4ig+3 x columns 4cg..4cg+3: per token one 16-byte weight load and one
    // 16-byte value load serve sixteen products
    {
      const int ncg = DT / 4;
      for (int p = tid; p < (M / 4) * ncg; p += kThreads) {
        const int ig = p / ncg, cg = p - ig * ncg;
        float4 acc[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = 4 * ig + j;
          const float4 hv = *reinterpret_cast<const float4*>(s_H + i * DT + 4 * cg);
          const float d = s_D[i];
          acc[j] = make_float4(d * hv.x, d * hv.y, d * hv.z, d * hv.w);
        }
#pragma unroll 4
        for (int t = 0; t < kC; ++t) {
          const float4 vv = *reinterpret_cast<const float4*>(s_v + t * DT + 4 * cg);
          const float4 w4 = *reinterpret_cast<const float4*>(s_w + t * M + 4 * ig);
          const float wj[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[j].x = fmaf(wj[j], vv.x, acc[j].x);
            acc[j].y = fmaf(wj[j], vv.y, acc[j].y);
            acc[j].z = fmaf(wj[j], vv.z, acc[j].z);
            acc[j].w = fmaf(wj[j], vv.w, acc[j].w);
          }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = 4 * ig + j;
          if (s_touch[i]) *reinterpret_cast<float4*>(s_H + i * DT + 4 * cg) = acc[j];
        }
      }
    }
    __syncthreads();
  }

  if (a.HT) {
    for (int p = tid; p < M * DT; p += kThreads) {
      const int i = p / DT, dd = p % DT;
      if (dd < DTe) a.HT[((int64_t)pair * M + i) * Dv + d0 + dd] = s_H[p];
    }
  }
}

template <int M, typename TIn>
cudaError_t launch_simt(const rsm_forward_args& a, cudaStream_t stream) {
  const int DT = simt_dt(M, a.Dv);
  const SimtSmem L = simt_layout(M, DT);
  auto kern = prefill_simt_kernel<M, TIn>;
  cudaError_t e = set_smem_limit<prefill_simt_kernel<M, TIn>>(L.total);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)(a.B * a.H), (unsigned)((a.Dv + DT - 1) / DT));
  kern<<<grid, kThreads, L.total, stream>>>(a, DT);
  return cudaGetLastError();
}

template <int M>
cudaError_t launch_simt_m(const rsm_forward_args& a, cudaStream_t stream) {
  return a.qkv_dtype == RSM_BF16 ? launch_simt<M, __nv_bfloat16>(a, stream)
                                 : launch_simt<M, float>(a, stream);
}

}  // namespace

size_t prefill_simt_smem_bytes(int M, int Dv) { return (size_t)simt_layout(M, simt_dt(M, Dv)).total; }

cudaError_t launch_prefill_simt(const rsm_forward_args& a, cudaStream_t stream) {
  if (a.B * a.H == 0) return cudaSuccess;
  switch (a.M) {
    case 32: return launch_simt_m<32>(a, stream);
    case 64: return launch_simt_m<64>(a, stream);
    case 128: return launch_simt_m<128>(a, stream);
    case 256: return launch_simt_m<256>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rsm
