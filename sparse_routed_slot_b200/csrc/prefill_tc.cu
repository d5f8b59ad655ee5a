// prefill_tc.cu -- chunked prefill on the 5th-generation tensor cores (rsm_forward, tensor path).
//
// Shapes: M = 128 slots, Dv = 128, bf16 q/k/v, K <= 32, per-head or per-slot log-decay.
//
// Chunk algebra (paperlayer.ai summary of the Raven paper, section A.5: T = n*C chunks of C = 64
// tokens), for one (b,h) stream and one chunk, with g_{t,i} the cumulative log-decay of slot i from
// the chunk start through token t (g <= 0), w_{t,i} = k_{t,i} (1 - a_{t,i}) on the selected slots
// and 0 elsewhere, and the reference point of the exponentials at the chunk start:
//   Qh = q * e^{g}            (|Qh| <= |q|)
//   Wh = w * e^{-g}           (finite while every slot decays by less than e^-80 in the chunk)
//   S  = Qh Wh^T,  A = S masked to s <= t           (intra-chunk weights, read after write)
//   O  = Qh H_start + A V                            (chunk outputs)
//   H_end = e^{g_end} * (H_start + Wh^T V)           (carry; rows never selected are skipped)
// A chunk whose decay is stronger than that bound takes the exact path: A from pairwise sums
// with non-positive exponents and the carry with weights w * e^{g_end - g} (no overflow at all).
//
// Everything is fp32 in and out of the tensor cores: operands are rounded to nearest tf32 when
// they are written (kind::tf32) and products accumulate in fp32. The fp32 state lives in TMEM as
// H^T (lane = value column, column = slot); the carry accumulates into it directly, and a copy
// rounded to tf32 feeds the read of the next chunk as the A operand straight from TMEM.
//
// TMEM columns: [0,128) H^T, [128,256) H^T rounded to tf32, [256,320) O^T, [320,384) S (64-lane).
//
// Long sequences with few (b,h) streams are split into segments processed in parallel: a summary
// pass runs the state recurrence of each segment but the last from a zero state and stores
// (prod of chunk decays, end state); a scan combines them into the true start state of every
// segment; the main pass then runs every segment from its start state.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rsm {

namespace {

constexpr int kC = 64;        // tokens per chunk
constexpr int kM = 128;       // slots
constexpr int kDV = 128;      // value columns
constexpr int kKMax = 32;     // largest TopK on this path
constexpr int kThreads = 384; // 12 warps: WG0 slots, WG1 TMEM, WG2 values/issue
constexpr float kGMax = 80.f; // fast-path bound on the in-chunk decay (e^80 fits fp32/tf32)

constexpr int kColH = 0, kColHr = 128, kColO = 256, kColS = 320, kTmemCols = 512;

// Dynamic shared memory layout (offsets from a 1024-byte aligned base). Every operand tile is
// K-major in the swizzled format of tc.cuh (a tf32 operand cannot share one layout between the
// K-major and MN-major uses), so the token-contracted operands are stored transposed.
constexpr int kOffQ = 0;                       // Qh   [64 t][128 slot]
constexpr int kOffW = kOffQ + 32768;           // Wh   [64 s][128 slot]   (B of S)
constexpr int kOffWt = kOffW + 32768;          // Wh^T [128 slot][64 s]   (B of the carry)
constexpr int kOffVt = kOffWt + 32768;         // V^T  [128 dv][64 s]     (A of carry and intra)
constexpr int kOffRaw = kOffVt + 32768;        // q | k | v raw bf16 [64 x 128] each (TMA)
constexpr int kOffA = kOffRaw + 2 * 16384;     // A [64 t][64 s], over the raw v once it is converted
constexpr int kOffLam = kOffRaw + 3 * 16384;   // log-decay, then its running sum [64 x 128] fp32
constexpr int kOffSlam = kOffLam + 32768;      // log-decay of the selected slots [64 x kKMax]
constexpr int kOffSidx = kOffSlam + kC * kKMax * 4;  // selected slots [64 x kKMax] u8
constexpr int kOffSmall = kOffSidx + kC * kKMax;
constexpr int kSmallFloats = 2 * kM + 2 * kM + kM + kM;  // Dc[2], touch[2], Dseg, tseg
constexpr int kSmemBytes = kOffSmall + kSmallFloats * 4 + 1024;  // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Maps {
  CUtensorMap q, k, v;
};

struct Params {
  int B, T, H, K;
  int decay_slot;
  const float* logits;
  const float* f;
  const float* H0;
  float* o;
  float* HT;
  int32_t* idx_out;
  float* score_out;
  int validate;
  int nseg, seg_chunks;
  float* ws_state;  // [pairs][nseg][M][Dv]: slot 0 = start state, slot j+1 = summary of segment j
  float* ws_D;      // [pairs][nseg][M]
  int* ws_touch;    // [pairs][nseg][M]
};

RSM_DEV float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// Bounded mbarrier wait; on expiry records a timeout and raises the CTA abort flag.
RSM_DEV void wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (!tc::mbar_wait(bar, parity)) {
    *abort_flag = 1;
    raise_status(RSM_ERR_TIMEOUT);
  }
}

template <bool SUMMARY>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ Maps maps,
                                                                  const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* sQ = sm + kOffQ;
  unsigned char* sW = sm + kOffW;
  unsigned char* sWt = sm + kOffWt;
  unsigned char* sVt = sm + kOffVt;
  unsigned char* sA = sm + kOffA;
  const uint16_t* rq = reinterpret_cast<const uint16_t*>(sm + kOffRaw);
  const uint16_t* rk = rq + kC * kM;
  const uint16_t* rv = rk + kC * kM;
  float* sLam = reinterpret_cast<float*>(sm + kOffLam);
  float* sSlam = reinterpret_cast<float*>(sm + kOffSlam);
  unsigned char* sSidx = sm + kOffSidx;
  float* sDc = reinterpret_cast<float*>(sm + kOffSmall);   // [2][M]
  int* sTouch = reinterpret_cast<int*>(sDc + 2 * kM);       // [2][M]
  float* sDseg = reinterpret_cast<float*>(sTouch + 2 * kM); // [M]
  int* sTseg = reinterpret_cast<int*>(sDseg + kM);          // [M]

  __shared__ __align__(8) uint64_t bar_tma, bar_s, bar_o;
  __shared__ uint32_t s_tbase;
  __shared__ int s_fast, s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, wg = warp >> 2;
  const int T = p.T, H = p.H, K = p.K;
  const int pairs = p.B * H;
  const int segs_here = SUMMARY ? p.nseg - 1 : p.nseg;
  const int items = pairs * segs_here;
  const bool issuer = tid == 256;

  if (warp == 4) tc::tmem_alloc(&s_tbase, kTmemCols);
  if (tid == 0) {
    tc::mbar_init(&bar_tma, 1);
    tc::mbar_init(&bar_s, 1);
    tc::mbar_init(&bar_o, 1);
    tc::fence_mbar_init();
    s_abort = 0;
  }
  if (issuer) {
    tc::tma_prefetch_desc(&maps.q);
    tc::tma_prefetch_desc(&maps.k);
    tc::tma_prefetch_desc(&maps.v);
  }
  tc::tmem_fence_before();
  __syncthreads();
  tc::tmem_fence_after();
  const uint32_t tb = s_tbase;
  const uint32_t sub_lane = (uint32_t)((warp & 3) * 32);  // TMEM lanes this warp may access
  volatile int* abort_flag = &s_abort;

  uint32_t n_chunks = 0;  // chunks completed by this CTA (parity of bar_tma / bar_o)
  uint32_t n_tma = 0;     // tile loads issued (meaningful in the issuing thread)
  uint32_t n_s = 0;       // completions of bar_s
  bool fast_prev = true;

  for (int item = blockIdx.x; item < items && !s_abort; item += gridDim.x) {
    const int pair = item % pairs, seg = item / pairs;
    const int b = pair / H, h = pair % H;
    const int t0 = seg * p.seg_chunks * kC;
    const int t1 = min(T, t0 + p.seg_chunks * kC);
    const bool last_seg = seg == p.nseg - 1;

    // ---- start state into TMEM (WG1): H^T lane = value column, column = slot
    if (wg == 1) {
      const float* Hs = nullptr;
      if (!SUMMARY) Hs = p.nseg > 1 ? p.ws_state + ((int64_t)pair * p.nseg + seg) * kM * kDV
                                    : (p.H0 ? p.H0 + (int64_t)pair * kM * kDV : nullptr);
      const int dv = tid - 128;
#pragma unroll 1
      for (int c0 = 0; c0 < kM; c0 += 32) {
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = Hs ? Hs[(c0 + j) * kDV + dv] : 0.f;
        tc::tmem_st32(tc::tmem_addr(tb, sub_lane, kColH + c0), v);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = tc::to_tf32(v[j]);
        tc::tmem_st32(tc::tmem_addr(tb, sub_lane, kColHr + c0), v);
      }
      tc::tmem_wait_st();
    }
    if (SUMMARY && wg == 0) {
      sDseg[tid] = 1.f;
      sTseg[tid] = 0;
    }
    if (issuer) {
      ++n_tma;
      tc::mbar_arrive_expect_tx(&bar_tma, 3 * kC * kM * 2);
      tc::tma_load_4d(sm + kOffRaw, &maps.q, &bar_tma, 0, h, t0, b);
      tc::tma_load_4d(sm + kOffRaw + kC * kM * 2, &maps.k, &bar_tma, 0, h, t0, b);
      tc::tma_load_4d(sm + kOffRaw + 2 * kC * kM * 2, &maps.v, &bar_tma, 0, h, t0, b);
    }
    tc::tmem_fence_before();
    __syncthreads();
    tc::tmem_fence_after();
    fast_prev = true;

    for (int c0 = t0; c0 < t1; c0 += kC) {
      const int nrows = min(kC, t1 - c0);
      const int buf = n_chunks & 1;
      const bool first = c0 == t0;

      // ---- P0: routing of the chunk's rows (all warps, one row per warp at a time)
      if (tid == 0) s_fast = 1;
#pragma unroll 1
      for (int t = warp; t < kC; t += kThreads / 32) {
        float4* lrow = reinterpret_cast<float4*>(sLam + t * kM) + lane;
        if (t < nrows) {
          const int64_t row = ((int64_t)b * T + c0 + t) * H + h;
          float x[4];
          load_row_logits<kM>(p.logits + row * kM, lane, x);
          float fv[4];
          if (p.decay_slot) {
            const float4 t4 = reinterpret_cast<const float4*>(p.f + row * kM)[lane];
            fv[0] = t4.x; fv[1] = t4.y; fv[2] = t4.z; fv[3] = t4.w;
          } else {
            const float fs = p.f[row];
            fv[0] = fv[1] = fv[2] = fv[3] = fs;
          }
          if (p.validate) {
            bool bad = false;
#pragma unroll
            for (int e = 0; e < 4; ++e) bad |= !finite_f32(x[e]) || !finite_f32(fv[e]) || fv[e] > 0.f;
            if (__any_sync(kFull, bad) && lane == 0) raise_status(RSM_ERR_NONFINITE);
          }
          int32_t* io = (!SUMMARY && p.idx_out) ? p.idx_out + row * K : nullptr;
          float* so = (!SUMMARY && p.score_out) ? p.score_out + row * K : nullptr;
          float lam[4] = {0.f, 0.f, 0.f, 0.f};
          warp_topk<kM>(x, K, lane, [&](int r, int slot, int e) {
            const float s = sigmoid_f32(x[e]);
            lam[e] = s * fv[e];
            sSlam[t * kKMax + r] = lam[e];
            sSidx[t * kKMax + r] = (unsigned char)slot;
            if (io) io[r] = slot;
            if (so) so[r] = s;
          });
          *lrow = make_float4(lam[0], lam[1], lam[2], lam[3]);
        } else {
          *lrow = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      __syncthreads();

      // ---- P1: WG0 scans slots, WG1 applies the previous chunk's carry, WG2 converts V
      if (wg == 0 || wg == 2) {
        wait_or_abort(&bar_tma, n_chunks & 1, abort_flag);
        if (n_chunks > 0) wait_or_abort(&bar_o, (n_chunks - 1) & 1, abort_flag);
      }
      if (wg == 0) {
        const int i = tid;
        float g = 0.f;
        bool touched = false;
#pragma unroll 1
        for (int t4 = 0; t4 < kC; t4 += 4) {
          float wt[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int t = t4 + u;
            const float lam = sLam[t * kM + i];
            touched |= lam != 0.f;
            g += lam;
            sLam[t * kM + i] = g;
            const float w = bf16_to_f32(rk[t * kM + i]) * (-expm1f(lam));
            wt[u] = tc::to_tf32(w * expf(-g));
            if (!SUMMARY) {
              *reinterpret_cast<float*>(sW + tc::swz_offset(kC, t, i)) = wt[u];
              *reinterpret_cast<float*>(sQ + tc::swz_offset(kC, t, i)) =
                  tc::to_tf32(bf16_to_f32(rq[t * kM + i]) * expf(g));
            }
          }
          *reinterpret_cast<float4*>(sWt + tc::swz_offset(kM, i, t4)) = make_float4(wt[0], wt[1], wt[2], wt[3]);
        }
        const float D = expf(g);
        sDc[buf * kM + i] = D;
        sTouch[buf * kM + i] = touched;
        if (SUMMARY) {
          sDseg[i] *= D;
          sTseg[i] |= touched;
        }
        if (!(g >= -kGMax)) s_fast = 0;
        tc::fence_async_smem();
      } else if (wg == 1) {
        if (!first) {
          // previous chunk: the carry has landed in H; apply its decay (unless already applied on
          // the exact path) and refresh the rounded copy the read uses
          wait_or_abort(&bar_o, (n_chunks - 1) & 1, abort_flag);
          tc::tmem_fence_after();
          const float* Dp = sDc + (buf ^ 1) * kM;
          const int* Tp = sTouch + (buf ^ 1) * kM;
#pragma unroll 1
          for (int c = 0; c < kM; c += 32) {
            float hv[32];
            tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColH + c), hv);
            tc::tmem_wait_ld();
            if (fast_prev) {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (Tp[c + j]) hv[j] *= Dp[c + j];
              tc::tmem_st32(tc::tmem_addr(tb, sub_lane, kColH + c), hv);
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) hv[j] = tc::to_tf32(hv[j]);
            tc::tmem_st32(tc::tmem_addr(tb, sub_lane, kColHr + c), hv);
          }
          tc::tmem_wait_st();
        }
      } else {
        // V^T tile: row = value column, column = token (thread = value column; conflict-free stores)
        const int dv = tid - 256;
#pragma unroll 4
        for (int s4 = 0; s4 < kC; s4 += 4) {
          const float4 f4 = make_float4(bf16_to_f32(rv[(s4 + 0) * kDV + dv]), bf16_to_f32(rv[(s4 + 1) * kDV + dv]),
                                        bf16_to_f32(rv[(s4 + 2) * kDV + dv]), bf16_to_f32(rv[(s4 + 3) * kDV + dv]));
          *reinterpret_cast<float4*>(sVt + tc::swz_offset(kDV, dv, s4)) = f4;
        }
        tc::fence_async_smem();
      }
      tc::tmem_fence_before();
      __syncthreads();
      if (s_abort) break;
      const bool fast = s_fast != 0;

      // ---- exact path for a chunk with extreme decay (rare)
      if (!fast) {
        // carry weights w * e^{g_end - g} (every exponent <= 0)
        for (int e = tid; e < kC * kM; e += kThreads)
          *reinterpret_cast<float*>(sWt + tc::swz_offset(kM, e / kC, e % kC)) = 0.f;
        __syncthreads();
        for (int e = tid; e < nrows * K; e += kThreads) {
          const int t = e / K, r = e % K;
          const int i = sSidx[t * kKMax + r];
          const float w = bf16_to_f32(rk[t * kM + i]) * (-expm1f(sSlam[t * kKMax + r]));
          const float gend = sLam[(kC - 1) * kM + i];
          *reinterpret_cast<float*>(sWt + tc::swz_offset(kM, i, t)) = tc::to_tf32(w * expf(gend - sLam[t * kM + i]));
        }
        if (!SUMMARY) {
          // intra-chunk weights A[t][s] = sum_{i in S_s} q_ti w_si e^{g_ti - g_si}, s <= t
          for (int e = tid; e < kC * kC; e += kThreads) {
            const int t = e / kC, s = e % kC;
            float acc = 0.f;
            if (s <= t && t < nrows) {
              for (int r = 0; r < K; ++r) {
                const int i = sSidx[s * kKMax + r];
                const float w = bf16_to_f32(rk[s * kM + i]) * (-expm1f(sSlam[s * kKMax + r]));
                acc = fmaf(bf16_to_f32(rq[t * kM + i]) * w, expf(sLam[t * kM + i] - sLam[s * kM + i]), acc);
              }
            }
            *reinterpret_cast<float*>(sA + tc::swz_offset(kC, t, s)) = tc::to_tf32(acc);
          }
        }
        if (wg == 1) {
          // the exact-path carry uses end-referenced weights: decay the state first
          const float* Dc = sDc + buf * kM;
          const int* Tc = sTouch + buf * kM;
#pragma unroll 1
          for (int c = 0; c < kM; c += 32) {
            float hv[32];
            tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColH + c), hv);
            tc::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (Tc[c + j]) hv[j] *= Dc[c + j];
            tc::tmem_st32(tc::tmem_addr(tb, sub_lane, kColH + c), hv);
          }
          tc::tmem_wait_st();
          tc::tmem_fence_before();
        }
        tc::fence_async_smem();
        __syncthreads();
      }

      // ---- P2: tensor-core work of the chunk
      if (issuer) {
        tc::tmem_fence_after();
        const uint32_t q = tc::smem_u32(sQ), w = tc::smem_u32(sW), wt = tc::smem_u32(sWt),
                       vt = tc::smem_u32(sVt), a = tc::smem_u32(sA);
        if (!SUMMARY) {
          if (fast) {
#pragma unroll 1
            for (int j = 0; j < kM / 8; ++j) {  // S = Qh Wh^T
              const uint32_t off = (j >> 2) * (kC * 128) + (j & 3) * 32;
              tc::mma_tf32_ss(tb + kColS, tc::smem_desc(q + off, 16, 1024), tc::smem_desc(w + off, 16, 1024),
                              tc::idesc_tf32(64, kC, 0, 0), j > 0);
            }
            tc::mma_commit(&bar_s);
          }
#pragma unroll 1
          for (int j = 0; j < kM / 8; ++j) {  // O^T = H^T Qh^T (H^T read from TMEM)
            const uint32_t off = (j >> 2) * (kC * 128) + (j & 3) * 32;
            tc::mma_tf32_ts(tb + kColO, tb + kColHr + 8 * j, tc::smem_desc(q + off, 16, 1024),
                            tc::idesc_tf32(kDV, kC, 0, 0), j > 0);
          }
        }
#pragma unroll 1
        for (int j = 0; j < kC / 8; ++j) {  // H^T += V^T Wh (carry; H^T is not read by this chunk)
          const uint32_t off = (j >> 2) * (kM * 128) + (j & 3) * 32;
          tc::mma_tf32_ss(tb + kColH, tc::smem_desc(vt + off, 16, 1024), tc::smem_desc(wt + off, 16, 1024),
                          tc::idesc_tf32(kDV, kM, 0, 0), 1);
        }
        if (!SUMMARY && !fast) {
#pragma unroll 1
          for (int j = 0; j < kC / 8; ++j) {  // O^T += V^T A^T
            const uint32_t offa = (j >> 2) * (kC * 128) + (j & 3) * 32;
            const uint32_t offv = (j >> 2) * (kDV * 128) + (j & 3) * 32;
            tc::mma_tf32_ss(tb + kColO, tc::smem_desc(vt + offv, 16, 1024), tc::smem_desc(a + offa, 16, 1024),
                            tc::idesc_tf32(kDV, kC, 0, 0), 1);
          }
        }
        if (SUMMARY || !fast) tc::mma_commit(&bar_o);
      }

      if (!SUMMARY && fast) {
        // ---- P3: mask S into A (WG1; S rows t = 16*(warp%4) + lane at lanes 32*(warp%4) + lane)
        if (wg == 1) {
          wait_or_abort(&bar_s, n_s & 1, abort_flag);
          tc::tmem_fence_after();
          const int t = (warp & 3) * 16 + lane;
#pragma unroll 1
          for (int c = 0; c < kC; c += 32) {
            float sv[32];
            tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColS + c), sv);
            tc::tmem_wait_ld();
            if (lane < 16) {
#pragma unroll
              for (int j = 0; j < 32; j += 4) {
                const int s = c + j;
                float4 a4 = make_float4(s <= t ? tc::to_tf32(sv[j]) : 0.f, s + 1 <= t ? tc::to_tf32(sv[j + 1]) : 0.f,
                                        s + 2 <= t ? tc::to_tf32(sv[j + 2]) : 0.f, s + 3 <= t ? tc::to_tf32(sv[j + 3]) : 0.f);
                *reinterpret_cast<float4*>(sA + tc::swz_offset(kC, t, s)) = a4;
              }
            }
          }
          tc::fence_async_smem();
          tc::tmem_fence_before();
        }
        ++n_s;
        __syncthreads();
        if (s_abort) break;
        // ---- P4: O^T += V^T A^T
        if (issuer) {
          tc::tmem_fence_after();
          const uint32_t vt = tc::smem_u32(sVt), a = tc::smem_u32(sA);
#pragma unroll 1
          for (int j = 0; j < kC / 8; ++j) {
            const uint32_t offa = (j >> 2) * (kC * 128) + (j & 3) * 32;
            const uint32_t offv = (j >> 2) * (kDV * 128) + (j & 3) * 32;
            tc::mma_tf32_ss(tb + kColO, tc::smem_desc(vt + offv, 16, 1024), tc::smem_desc(a + offa, 16, 1024),
                            tc::idesc_tf32(kDV, kC, 0, 0), 1);
          }
          tc::mma_commit(&bar_o);
        }
      }

      // ---- P5: outputs of the chunk (WG1: thread = value column)
      if (!SUMMARY && wg == 1) {
        wait_or_abort(&bar_o, n_chunks & 1, abort_flag);
        tc::tmem_fence_after();
        const int dv = tid - 128;
        float* orow = p.o + (((int64_t)b * T + c0) * H + h) * kDV + dv;
        const int64_t ostride = (int64_t)H * kDV;
#pragma unroll 1
        for (int c = 0; c < kC; c += 32) {
          float ov[32];
          tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColO + c), ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c + j < nrows) orow[(int64_t)(c + j) * ostride] = ov[j];
        }
        tc::tmem_fence_before();
      }
      // the chunk's MMAs are done with A (over the raw v) and V^T: fetch the next chunk
      if (issuer && c0 + kC < t1) {
        wait_or_abort(&bar_o, n_chunks & 1, abort_flag);
        ++n_tma;
        tc::mbar_arrive_expect_tx(&bar_tma, 3 * kC * kM * 2);
        tc::tma_load_4d(sm + kOffRaw, &maps.q, &bar_tma, 0, h, c0 + kC, b);
        tc::tma_load_4d(sm + kOffRaw + kC * kM * 2, &maps.k, &bar_tma, 0, h, c0 + kC, b);
        tc::tma_load_4d(sm + kOffRaw + 2 * kC * kM * 2, &maps.v, &bar_tma, 0, h, c0 + kC, b);
      }
      fast_prev = fast;
      ++n_chunks;
      __syncthreads();
      if (s_abort) break;
    }
    if (s_abort) break;

    // ---- end of the item: last carry, then the state goes out
    if (wg == 1) {
      wait_or_abort(&bar_o, (n_chunks - 1) & 1, abort_flag);
      tc::tmem_fence_after();
      const int buf = (n_chunks - 1) & 1;
      const float* Dp = sDc + buf * kM;
      const int* Tp = sTouch + buf * kM;
      float* dst = nullptr;
      if (SUMMARY) dst = p.ws_state + ((int64_t)pair * p.nseg + seg + 1) * kM * kDV;
      else if (last_seg && p.HT) dst = p.HT + (int64_t)pair * kM * kDV;
      const int dv = tid - 128;
#pragma unroll 1
      for (int c = 0; c < kM; c += 32) {
        float hv[32];
        tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColH + c), hv);
        tc::tmem_wait_ld();
        if (fast_prev) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (Tp[c + j]) hv[j] *= Dp[c + j];
        }
        if (dst) {
#pragma unroll
          for (int j = 0; j < 32; ++j) dst[(c + j) * kDV + dv] = hv[j];
        }
      }
      tc::tmem_fence_before();
    }
    if (SUMMARY && wg == 0) {
      const int64_t base = ((int64_t)pair * p.nseg + seg + 1) * kM;
      p.ws_D[base + tid] = sDseg[tid];
      p.ws_touch[base + tid] = sTseg[tid];
    }
    __syncthreads();
  }

  // ---- teardown: let outstanding MMAs finish before the columns are released
  __syncthreads();
  if (issuer && n_chunks > 0) {
    tc::mma_commit(&bar_o);
    tc::mbar_wait(&bar_o, n_chunks & 1);
  }
  // a tile load still in flight (only after an abort) must land before the CTA leaves
  if (issuer && n_tma > n_chunks) tc::mbar_wait(&bar_tma, (n_tma - 1) & 1);
  tc::tmem_fence_before();
  __syncthreads();
  tc::tmem_fence_after();
  if (warp == 4) tc::tmem_dealloc(tb, kTmemCols);
}

// Combines the segment summaries of each (b,h) into start states:
// state[0] = H0 (or 0); state[j] = D_{j-1} * state[j-1] + U_{j-1} on the slots touched in
// segment j-1 (the summary of segment j-1 is stored in slot j and is replaced in place).
__global__ void __launch_bounds__(256) segment_scan_kernel(const Params p) {
  const int pair = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;  // element (slot, column)
  if (e >= kM * kDV) return;
  const int i = e / kDV;
  float* st = p.ws_state + (int64_t)pair * p.nseg * kM * kDV;
  const float* D = p.ws_D + (int64_t)pair * p.nseg * kM;
  const int* touch = p.ws_touch + (int64_t)pair * p.nseg * kM;
  float hcur = p.H0 ? p.H0[(int64_t)pair * kM * kDV + e] : 0.f;
  st[e] = hcur;
  for (int j = 1; j < p.nseg; ++j) {
    if (touch[j * kM + i]) hcur = fmaf(D[j * kM + i], hcur, st[(int64_t)j * kM * kDV + e]);
    st[(int64_t)j * kM * kDV + e] = hcur;
  }
}

// ---------------------------------------------------------------------------------------------
// host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 4-D map over [B, T, H, C] bf16 (C innermost) with a box of one (b, h) and 64 tokens.
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H, int C) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)C * 2, (cuuint64_t)H * C * 2, (cuuint64_t)T * H * C * 2};
  cuuint32_t box[4] = {(cuuint32_t)C, 1, (cuuint32_t)kC, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

struct Plan {
  int nseg, seg_chunks;
};

Plan plan_for(const rsm_forward_args& a, int sms) {
  const int64_t pairs = (int64_t)a.B * a.H;
  const int nchunks = (a.T + kC - 1) / kC;
  int nseg = 1;
  if (pairs > 0 && pairs < sms) nseg = (int)(sms / pairs);
  // segments of at least 4 chunks; never more segments than chunks
  nseg = std::max(1, std::min(nseg, nchunks / 4));
  int seg_chunks = (nchunks + nseg - 1) / nseg;
  if (seg_chunks < 1) seg_chunks = 1;
  nseg = std::max(1, (nchunks + seg_chunks - 1) / seg_chunks);
  return {nseg, seg_chunks};
}

size_t ws_bytes(const rsm_forward_args& a, const Plan& pl) {
  if (pl.nseg <= 1) return 0;
  const size_t per = (size_t)a.B * a.H * pl.nseg;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  return up(per * kM * kDV * 4) + up(per * kM * 4) + up(per * kM * 4);
}

}  // namespace

bool prefill_tc_supported(const rsm_forward_args& a) {
  return a.qkv_dtype == RSM_BF16 && a.M == kM && a.Dv == kDV && a.K <= kKMax;
}

size_t prefill_tc_workspace_bytes(const rsm_forward_args& a) {
  if (!prefill_tc_supported(a)) return 0;
  return ws_bytes(a, plan_for(a, sm_count()));
}

cudaError_t launch_prefill_tc(const rsm_forward_args& a, cudaStream_t stream) {
  const int sms = sm_count();
  const Plan pl = plan_for(a, sms);
  Maps maps;
  if (!make_map(&maps.q, a.q, a.B, a.T, a.H, kM) || !make_map(&maps.k, a.k, a.B, a.T, a.H, kM) ||
      !make_map(&maps.v, a.v, a.B, a.T, a.H, kDV))
    return cudaErrorInvalidValue;
  Params p;
  p.B = a.B; p.T = a.T; p.H = a.H; p.K = a.K;
  p.decay_slot = a.decay == RSM_DECAY_SLOT;
  p.logits = a.logits; p.f = a.f; p.H0 = a.H0;
  p.o = a.o; p.HT = a.HT; p.idx_out = a.idx_out; p.score_out = a.score_out;
  p.validate = (a.flags & RSM_FLAG_VALIDATE) != 0;
  p.nseg = pl.nseg; p.seg_chunks = pl.seg_chunks;
  p.ws_state = nullptr; p.ws_D = nullptr; p.ws_touch = nullptr;
  if (pl.nseg > 1) {
    const size_t per = (size_t)a.B * a.H * pl.nseg;
    auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
    char* w = static_cast<char*>(a.workspace);
    p.ws_state = reinterpret_cast<float*>(w);
    p.ws_D = reinterpret_cast<float*>(w + up(per * kM * kDV * 4));
    p.ws_touch = reinterpret_cast<int*>(w + up(per * kM * kDV * 4) + up(per * kM * 4));
  }
  cudaError_t e0 = cudaFuncSetAttribute(prefill_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e0 == cudaSuccess)
    e0 = cudaFuncSetAttribute(prefill_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e0 != cudaSuccess) return e0;
  const int64_t pairs = (int64_t)a.B * a.H;
  if (pl.nseg > 1) {
    const int items = (int)(pairs * (pl.nseg - 1));
    prefill_tc_kernel<true><<<std::min(items, sms), kThreads, kSmemBytes, stream>>>(maps, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    dim3 g((kM * kDV + 255) / 256, (unsigned)pairs);
    segment_scan_kernel<<<g, 256, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int64_t items = pairs * pl.nseg;
  prefill_tc_kernel<false><<<(unsigned)std::min<int64_t>(items, sms), kThreads, kSmemBytes, stream>>>(maps, p);
  return cudaGetLastError();
}

}  // namespace rsm
