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
// A chunk whose decay is stronger than that bound takes an exact path: A from pairwise sums with
// non-positive exponents, and the carry with weights w * e^{g_end - g} after the state is decayed.
//
// Operands are fp32 tiles rounded to nearest tf32 (kind::tf32), accumulated in fp32. The fp32
// state lives in TMEM as H^T (lane = value column, column = slot); the carry accumulates into it
// and a tf32-rounded copy feeds the next chunk's read as the A operand straight from TMEM.
// TMEM columns: [0,128) H^T, [128,256) rounded H^T, [256,320) O^T, [320,384) S (64-lane layout).
//
// Warp roles (one persistent CTA per SM, 12 warps):
//   warps 0-7  row workers: for each chunk, the routing of 8 rows per warp (TopK, log-decay), a
//              cross-warp prefix of the log-decay, then their rows of the Qh, Wh and Wh^T tiles.
//              They route chunk n+1 while the tensor core and the TMEM workers finish chunk n.
//   warps 8-11 TMEM workers (one per TMEM lane quarter): outputs of chunk n-1, the decay of the
//              state and its rounded copy, the V^T tile of chunk n, the S -> A masking. Thread 256
//              also issues the tile loads and the MMAs.
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

constexpr int kC = 64;         // tokens per chunk
constexpr int kM = 128;        // slots
constexpr int kDV = 128;       // value columns
constexpr int kKMax = 32;      // largest TopK on this path
constexpr int kRWarps = 8;     // row workers
constexpr int kRowsPerWarp = kC / kRWarps;
constexpr int kThreads = 384;
constexpr int kRThreads = kRWarps * 32;
constexpr int kIssuer = kRThreads;  // first thread of the TMEM workers
constexpr float kGMax = 80.f;       // fast-path bound on the in-chunk decay (e^80 fits fp32/tf32)
constexpr float kLog2e = 1.4426950408889634f;

constexpr int kColH = 0, kColHr = 128, kColO = 256, kColS = 320, kTmemCols = 512;

// Dynamic shared memory (offsets from a 1024-byte aligned base). Operand tiles are K-major in the
// swizzled format of tc.cuh; Wh^T and V^T are stored transposed because they are contracted over
// tokens (a tf32 operand cannot be MN-major in this swizzle).
constexpr int kOffQ = 0;                      // Qh   [64 t][128 slot]   (A of S, B of the read)
constexpr int kOffW = kOffQ + 32768;          // Wh   [64 s][128 slot]   (B of S)
constexpr int kOffWt = kOffW + 32768;         // Wh^T [128 slot][64 s]   (B of the carry)
constexpr int kOffVt = kOffWt + 32768;        // V^T  [128 dv][64 s]     (A of carry and A.V)
constexpr int kOffA = kOffVt + 32768;         // A    [64 t][64 s]       (B of A.V)
constexpr int kOffRawV = kOffA + 16384;       // v tiles from TMA, 2 x [64][128] bf16
constexpr int kOffTot = kOffRawV + 2 * 16384; // per-warp log-decay totals, 2 x [8][128] fp32
constexpr int kOffSidx = kOffTot + 2 * kRWarps * kM * 4;   // exact path: written slots [64][32]
constexpr int kOffSw = kOffSidx + kC * kKMax;              // exact path: their write weights
constexpr int kOffSmall = kOffSw + kC * kKMax * 4;
constexpr int kSmallBytes = (2 * kM + 2 * kM + kC) * 4 + 16;  // D[2][M], touched[2][M], cnt[64], fast[2]
constexpr int kSmemBytes = kOffSmall + kSmallBytes + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Maps {
  CUtensorMap v;
};

struct Params {
  int B, T, H, K;
  int decay_slot;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
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

RSM_DEV float4 bf16x4_to_f32(uint2 r) {
  return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u),
                     __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xffff0000u));
}
RSM_DEV float fget(const float4& v, int e) { return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w; }

// Bounded mbarrier wait; on expiry records a timeout and raises the CTA abort flag.
RSM_DEV void wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  if (!tc::mbar_wait(bar, parity)) {
    *abort_flag = 1;
    raise_status(RSM_ERR_TIMEOUT);
  }
}
RSM_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}
// Barrier among the row workers that also ORs a flag over them (every row worker sees the same).
RSM_DEV bool bar_rows_or(bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)flag), "n"(kRThreads)
      : "memory");
  return r != 0;
}

// Position of one chunk in the CTA's work list.
struct Chunk {
  int pair, seg, b, h, c0, nrows;
  bool first, last;
};

// The CTA walks its items (item = blockIdx.x + j*gridDim.x) and each item's chunks in order.
struct Walker {
  int items, pairs, H, T, seg_chunks, item, c0, t0, t1;
  __device__ void start(int items_, int pairs_, int H_, int T_, int seg_chunks_) {
    items = items_; pairs = pairs_; H = H_; T = T_; seg_chunks = seg_chunks_;
    item = blockIdx.x;
    set_item();
  }
  __device__ void set_item() {
    if (item >= items) return;
    const int seg = item / pairs;
    t0 = seg * seg_chunks * kC;
    t1 = min(T, t0 + seg_chunks * kC);
    c0 = t0;
  }
  __device__ bool valid() const { return item < items; }
  __device__ Chunk get() const {
    Chunk c;
    c.pair = item % pairs;
    c.seg = item / pairs;
    c.b = c.pair / H;
    c.h = c.pair % H;
    c.c0 = c0;
    c.nrows = min(kC, t1 - c0);
    c.first = c0 == t0;
    c.last = c0 + kC >= t1;
    return c;
  }
  __device__ void next() {
    c0 += kC;
    if (c0 >= t1) {
      item += gridDim.x;
      set_item();
    }
  }
};

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
  const uint16_t* sRawV = reinterpret_cast<const uint16_t*>(sm + kOffRawV);
  float* sTot = reinterpret_cast<float*>(sm + kOffTot);
  unsigned char* sSidx = sm + kOffSidx;
  float* sSw = reinterpret_cast<float*>(sm + kOffSw);
  float* sDc = reinterpret_cast<float*>(sm + kOffSmall);  // [2][M]
  int* sTouch = reinterpret_cast<int*>(sDc + 2 * kM);      // [2][M]
  int* sCnt = sTouch + 2 * kM;                             // [64]
  int* sFast = sCnt + kC;                                  // [2]

  __shared__ __align__(8) uint64_t bar_tma[2], bar_ready, bar_s, bar_a, bar_o, bar_x;
  __shared__ uint32_t s_tbase;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool row_worker = warp < kRWarps;
  const int T = p.T, H = p.H, K = p.K;
  const int pairs = p.B * H;
  const int segs_here = SUMMARY ? p.nseg - 1 : p.nseg;
  const int items = pairs * segs_here;

  if (warp == kRWarps) tc::tmem_alloc(&s_tbase, kTmemCols);
  if (tid == 0) {
    tc::mbar_init(&bar_tma[0], 1);
    tc::mbar_init(&bar_tma[1], 1);
    tc::mbar_init(&bar_ready, kThreads);
    tc::mbar_init(&bar_s, 1);
    tc::mbar_init(&bar_a, kThreads - kRThreads);
    tc::mbar_init(&bar_o, 1);
    tc::mbar_init(&bar_x, kThreads);
    tc::fence_mbar_init();
    s_abort = 0;
  }
  if (tid == kIssuer) tc::tma_prefetch_desc(&maps.v);
  tc::tmem_fence_before();
  __syncthreads();
  tc::tmem_fence_after();
  const uint32_t tb = s_tbase;
  volatile int* abort_flag = &s_abort;
  uint32_t n_x = 0;  // completed phases of bar_x (exact-path synchronisation), kept by every thread
  auto sync_x = [&]() {
    mbar_arrive(&bar_x);
    wait_or_abort(&bar_x, n_x & 1, abort_flag);
    ++n_x;
  };

  Walker wk;
  wk.start(items, pairs, H, T, p.seg_chunks);

  if (row_worker) {
    // =========================================================================== row workers
    const int w = warp;
    float Dseg[4] = {1.f, 1.f, 1.f, 1.f};  // summary pass, warp 0: product of the chunk decays
    int tseg[4] = {0, 0, 0, 0};
    float tau = 0.f;  // last routing threshold found by this warp (a guess for the next rows)
    for (uint32_t n = 0; wk.valid(); ++n, wk.next()) {
      const Chunk ck = wk.get();
      const int buf = n & 1;
      // ---- stage A: routing and per-slot log-decay of this warp's 8 rows
      float lam[kRowsPerWarp][4];
      uint2 qv[kRowsPerWarp], kv[kRowsPerWarp];
      float4 xv[kRowsPerWarp], fv[kRowsPerWarp];
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) {
        const int t = w * kRowsPerWarp + r;
        const int64_t row = ((int64_t)ck.b * T + ck.c0 + t) * H + ck.h;
        if (t < ck.nrows) {
          xv[r] = reinterpret_cast<const float4*>(p.logits + row * kM)[lane];
          if (p.decay_slot) {
            fv[r] = reinterpret_cast<const float4*>(p.f + row * kM)[lane];
          } else {
            const float fs = p.f[row];
            fv[r] = make_float4(fs, fs, fs, fs);
          }
          kv[r] = reinterpret_cast<const uint2*>(p.k + row * kM)[lane];
          qv[r] = SUMMARY ? make_uint2(0u, 0u) : reinterpret_cast<const uint2*>(p.q + row * kM)[lane];
        } else {
          xv[r] = make_float4(0.f, 0.f, 0.f, 0.f);
          fv[r] = xv[r];
          kv[r] = make_uint2(0u, 0u);
          qv[r] = kv[r];
        }
      }
      float tot[4] = {0.f, 0.f, 0.f, 0.f};
      const bool want_routing = !SUMMARY && (p.idx_out || p.score_out);
#pragma unroll
      for (int r0 = 0; r0 < kRowsPerWarp; r0 += 4) {
        // selection of four rows at a time (their reductions overlap)
        float x[4][4];
        uint32_t sel[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          x[r][0] = xv[r0 + r].x; x[r][1] = xv[r0 + r].y; x[r][2] = xv[r0 + r].z; x[r][3] = xv[r0 + r].w;
        }
        uint32_t ok = 0u;
        if (!want_routing && K >= 2) ok = warp_select_guess_rows<kM, 4>(x, K, tau, sel);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int t = w * kRowsPerWarp + r0 + r;
#pragma unroll
          for (int e = 0; e < 4; ++e) lam[r0 + r][e] = 0.f;
          if (t >= ck.nrows) continue;  // warp-uniform
          const int64_t row = ((int64_t)ck.b * T + ck.c0 + t) * H + ck.h;
          if (p.validate) {
            bool bad = false;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float fe = fget(fv[r0 + r], e);
              bad |= !finite_f32(x[r][e]) || !finite_f32(fe) || fe > 0.f;
            }
            if (__any_sync(kFull, bad) && lane == 0) raise_status(RSM_ERR_NONFINITE);
          }
          if (!(ok & (1u << r))) {
            int32_t* io = want_routing && p.idx_out ? p.idx_out + row * K : nullptr;
            float* so = want_routing && p.score_out ? p.score_out + row * K : nullptr;
            const float(&xr)[4] = x[r];
            sel[r] = warp_topk<kM>(xr, K, lane, [&](int rk, int slot, int e) {
              if (io) io[rk] = slot;
              if (so) so[rk] = sigmoid_f32(xr[e]);
            });
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float s = __frcp_rn(1.f + __expf(-x[r][e]));  // router score (selected slots)
            lam[r0 + r][e] = (sel[r] & (1u << e)) ? s * fget(fv[r0 + r], e) : 0.f;
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
        for (int e = 0; e < 4; ++e) tot[e] += lam[r][e];
      reinterpret_cast<float4*>(sTot + (buf * kRWarps + w) * kM)[lane] = make_float4(tot[0], tot[1], tot[2], tot[3]);
      if (bar_rows_or(*abort_flag != 0)) break;  // every row worker takes the same decision
      float off[4] = {0.f, 0.f, 0.f, 0.f}, gend[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int w2 = 0; w2 < kRWarps; ++w2) {
        const float4 t4 = reinterpret_cast<const float4*>(sTot + (buf * kRWarps + w2) * kM)[lane];
        const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (w2 < w) off[e] += tv[e];
          gend[e] += tv[e];
        }
      }
      bool ok = true;
#pragma unroll
      for (int e = 0; e < 4; ++e) ok &= gend[e] >= -kGMax;
      const bool fast = __all_sync(kFull, ok);
      // ---- the previous chunk's MMAs are done: its operand tiles are free, and the TMEM workers
      // have finished the chunk before it (whose decay buffer this chunk reuses)
      if (n > 0) wait_or_abort(&bar_o, (n - 1) & 1, abort_flag);
      if (w == 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int slot = lane * 4 + e;
          const float D = exp2f(gend[e] * kLog2e);
          const int touched = gend[e] != 0.f;
          sDc[buf * kM + slot] = D;
          sTouch[buf * kM + slot] = touched;
          if (SUMMARY) {
            if (ck.first) {
              Dseg[e] = 1.f;
              tseg[e] = 0;
            }
            Dseg[e] *= D;
            tseg[e] |= touched;
            if (ck.last) {
              const int64_t base = ((int64_t)ck.pair * p.nseg + ck.seg + 1) * kM;
              p.ws_D[base + slot] = Dseg[e];
              p.ws_touch[base + slot] = tseg[e];
            }
          }
        }
        if (lane == 0) sFast[buf] = fast;
      }
      if (fast) {
        // ---- stage B: this warp's rows of Qh, Wh and Wh^T
        float g[4], Eprev[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          g[e] = off[e];
          Eprev[e] = exp2f(-off[e] * kLog2e);
        }
        float stash[4][4];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const int t = w * kRowsPerWarp + r;
          const float4 q4 = bf16x4_to_f32(qv[r]);
          const float4 k4 = bf16x4_to_f32(kv[r]);
          float qh[4], wh[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            g[e] += lam[r][e];
            const float E = exp2f(-g[e] * kLog2e);                 // e^{-g_t}
            wh[e] = tc::to_tf32(fget(k4, e) * (E - Eprev[e]));     // k (1 - a) e^{-g_t}
            Eprev[e] = E;
            qh[e] = SUMMARY ? 0.f : tc::to_tf32(fget(q4, e) * exp2f(g[e] * kLog2e));
            stash[r & 3][e] = wh[e];
          }
          if (!SUMMARY) {
            *reinterpret_cast<float4*>(sQ + tc::swz_offset(kC, t, lane * 4)) = make_float4(qh[0], qh[1], qh[2], qh[3]);
            *reinterpret_cast<float4*>(sW + tc::swz_offset(kC, t, lane * 4)) = make_float4(wh[0], wh[1], wh[2], wh[3]);
          }
          if ((r & 3) == 3) {
            // four consecutive tokens of each of the lane's slots; the slot order is rotated by
            // lane pair so that 8 neighbouring lanes hit 8 different 16-byte bank groups
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int e = (j + (lane >> 1)) & 3;
              float4 v4;
              v4.x = e == 0 ? stash[0][0] : e == 1 ? stash[0][1] : e == 2 ? stash[0][2] : stash[0][3];
              v4.y = e == 0 ? stash[1][0] : e == 1 ? stash[1][1] : e == 2 ? stash[1][2] : stash[1][3];
              v4.z = e == 0 ? stash[2][0] : e == 1 ? stash[2][1] : e == 2 ? stash[2][2] : stash[2][3];
              v4.w = e == 0 ? stash[3][0] : e == 1 ? stash[3][1] : e == 2 ? stash[3][2] : stash[3][3];
              *reinterpret_cast<float4*>(sWt + tc::swz_offset(kM, lane * 4 + e, t - 3)) = v4;
            }
          }
        }
        tc::fence_async_smem();
        mbar_arrive(&bar_ready);
      } else {
        // ---- exact path (rare), with the TMEM workers: the Qh tile as usual, dense q (bf16, in
        // the raw v buffer of this chunk, already converted) and dense g (in the Wh region, unused
        // here), the listed write weights, then A and the end-referenced Wh^T, exponents <= 0
        mbar_arrive(&bar_ready);
        sync_x();  // X0
        uint2* dq = reinterpret_cast<uint2*>(sm + kOffRawV + buf * (kC * kDV * 2));  // plain [64][128] bf16
        float* dg = reinterpret_cast<float*>(sW);                                    // plain [64][128]
        float g[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) g[e] = off[e];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const int t = w * kRowsPerWarp + r;
          const float4 q4 = bf16x4_to_f32(qv[r]);
          const float4 k4 = bf16x4_to_f32(kv[r]);
          float wv[4], qh[4];
          int cnt = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            g[e] += lam[r][e];
            wv[e] = fget(k4, e) * (-expm1f(lam[r][e]));
            cnt += wv[e] != 0.f;
            qh[e] = SUMMARY ? 0.f : tc::to_tf32(fget(q4, e) * expf(g[e]));
          }
          if (!SUMMARY)
            *reinterpret_cast<float4*>(sQ + tc::swz_offset(kC, t, lane * 4)) = make_float4(qh[0], qh[1], qh[2], qh[3]);
          dq[t * (kM / 4) + lane] = qv[r];
          reinterpret_cast<float4*>(dg + t * kM)[lane] = make_float4(g[0], g[1], g[2], g[3]);
          int pre = cnt;  // inclusive scan over lanes
#pragma unroll
          for (int d = 1; d < 32; d <<= 1) {
            const int v = __shfl_up_sync(kFull, pre, d);
            if (lane >= d) pre += v;
          }
          const int total = __shfl_sync(kFull, pre, 31);
          pre -= cnt;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if (wv[e] != 0.f) {
              sSidx[t * kKMax + pre] = (unsigned char)(lane * 4 + e);
              sSw[t * kKMax + pre] = wv[e];
              ++pre;
            }
          }
          if (lane == 0) sCnt[t] = total;  // <= K <= 32: only selected slots have w != 0
        }
        for (int e = tid; e < kC * kM; e += kRThreads)
          *reinterpret_cast<float*>(sWt + tc::swz_offset(kM, e / kC, e % kC)) = 0.f;
        sync_x();  // X1
        const int nrows = ck.nrows;
        for (int e = tid; e < nrows * kKMax; e += kRThreads) {
          const int t = e / kKMax, r = e % kKMax;
          if (r >= sCnt[t]) continue;
          const int i = sSidx[t * kKMax + r];
          const float gend_i = dg[(kC - 1) * kM + i];
          *reinterpret_cast<float*>(sWt + tc::swz_offset(kM, i, t)) =
              tc::to_tf32(sSw[t * kKMax + r] * expf(gend_i - dg[t * kM + i]));
        }
        if (!SUMMARY) {
          for (int e = tid; e < kC * kC; e += kRThreads) {
            const int t = e / kC, s = e % kC;
            float acc = 0.f;
            if (s <= t && t < nrows) {
              const int cs = sCnt[s];
              for (int r = 0; r < cs; ++r) {
                const int i = sSidx[s * kKMax + r];
                const float qti = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(dq)[t * kM + i] << 16);
                acc = fmaf(qti * sSw[s * kKMax + r], expf(dg[t * kM + i] - dg[s * kM + i]), acc);
              }
            }
            *reinterpret_cast<float*>(sA + tc::swz_offset(kC, t, s)) = tc::to_tf32(acc);
          }
        }
        tc::fence_async_smem();
        sync_x();  // X2
      }
    }
  } else {
    // =========================================================================== TMEM workers
    const int dv = tid - kRThreads;                 // TMEM lane = value column
    const uint32_t sub_lane = (uint32_t)((warp & 3) * 32);
    const bool issuer = tid == kIssuer;
    uint32_t n_s = 0, n_tma_issued = 0;
    Chunk prev;
    prev.nrows = 0;
    bool have_prev = false, fast_prev = true;

    // outputs of chunk `prev`, then the decay of the state (or, at the item's end, the state out)
    auto finish_prev = [&](uint32_t n_prev) {
      wait_or_abort(&bar_o, n_prev & 1, abort_flag);
      tc::tmem_fence_after();
      if (!SUMMARY) {
        float* orow = p.o + (((int64_t)prev.b * T + prev.c0) * H + prev.h) * kDV + dv;
        const int64_t ostride = (int64_t)H * kDV;
#pragma unroll 1
        for (int c = 0; c < kC; c += 32) {
          float ov[32];
          tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColO + c), ov);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c + j < prev.nrows) orow[(int64_t)(c + j) * ostride] = ov[j];
        }
      }
      const float* Dp = sDc + (n_prev & 1) * kM;
      const int* Tp = sTouch + (n_prev & 1) * kM;
      float* dst = nullptr;
      if (prev.last) {
        if (SUMMARY) dst = p.ws_state + ((int64_t)prev.pair * p.nseg + prev.seg + 1) * kM * kDV;
        else if (prev.seg == p.nseg - 1 && p.HT) dst = p.HT + (int64_t)prev.pair * kM * kDV;
      }
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
        if (prev.last) {
          if (dst) {
#pragma unroll
            for (int j = 0; j < 32; ++j) dst[(c + j) * kDV + dv] = hv[j];
          }
        } else {
          if (fast_prev) tc::tmem_st32(tc::tmem_addr(tb, sub_lane, kColH + c), hv);
#pragma unroll
          for (int j = 0; j < 32; ++j) hv[j] = tc::to_tf32(hv[j]);
          tc::tmem_st32(tc::tmem_addr(tb, sub_lane, kColHr + c), hv);
        }
      }
      tc::tmem_wait_st();
    };

    if (issuer && wk.valid()) {
      const Chunk c = wk.get();
      ++n_tma_issued;
      tc::mbar_arrive_expect_tx(&bar_tma[0], kC * kDV * 2);
      tc::tma_load_4d(sm + kOffRawV, &maps.v, &bar_tma[0], 0, c.h, c.c0, c.b);
    }
    uint32_t n = 0;
    for (; wk.valid() && !*abort_flag; ++n, wk.next()) {
      const Chunk ck = wk.get();
      const int buf = n & 1;
      if (have_prev) finish_prev(n - 1);
      if (ck.first) {
        // start state of the item into TMEM (fp32 and its tf32-rounded copy)
        const float* Hs = nullptr;
        if (!SUMMARY)
          Hs = p.nseg > 1 ? p.ws_state + ((int64_t)ck.pair * p.nseg + ck.seg) * kM * kDV
                          : (p.H0 ? p.H0 + (int64_t)ck.pair * kM * kDV : nullptr);
#pragma unroll 1
        for (int c = 0; c < kM; c += 32) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = Hs ? Hs[(c + j) * kDV + dv] : 0.f;
          tc::tmem_st32(tc::tmem_addr(tb, sub_lane, kColH + c), v);
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = tc::to_tf32(v[j]);
          tc::tmem_st32(tc::tmem_addr(tb, sub_lane, kColHr + c), v);
        }
        tc::tmem_wait_st();
      }
      // V^T tile of this chunk (thread = value column; conflict-free 16-byte stores)
      wait_or_abort(&bar_tma[buf], (n >> 1) & 1, abort_flag);
      {
        const uint16_t* rv = sRawV + buf * (kC * kDV);
#pragma unroll 4
        for (int s4 = 0; s4 < kC; s4 += 4) {
          const float4 f4 = make_float4(__uint_as_float((uint32_t)rv[(s4 + 0) * kDV + dv] << 16),
                                        __uint_as_float((uint32_t)rv[(s4 + 1) * kDV + dv] << 16),
                                        __uint_as_float((uint32_t)rv[(s4 + 2) * kDV + dv] << 16),
                                        __uint_as_float((uint32_t)rv[(s4 + 3) * kDV + dv] << 16));
          *reinterpret_cast<float4*>(sVt + tc::swz_offset(kDV, dv, s4)) = f4;
        }
      }
      if (issuer) {
        Walker nx = wk;
        nx.next();
        if (nx.valid()) {
          // the other buffer held chunk n-1, whose V^T was built before bar_ready(n-1) completed
          const Chunk c = nx.get();
          ++n_tma_issued;
          tc::mbar_arrive_expect_tx(&bar_tma[buf ^ 1], kC * kDV * 2);
          tc::tma_load_4d(sm + kOffRawV + (buf ^ 1) * (kC * kDV * 2), &maps.v, &bar_tma[buf ^ 1], 0, c.h,
                          c.c0, c.b);
        }
      }
      tc::fence_async_smem();
      tc::tmem_fence_before();
      mbar_arrive(&bar_ready);
      wait_or_abort(&bar_ready, n & 1, abort_flag);
      const bool fast = sFast[buf] != 0;
      const uint32_t q = tc::smem_u32(sQ), w = tc::smem_u32(sW), wt = tc::smem_u32(sWt),
                     vt = tc::smem_u32(sVt), a = tc::smem_u32(sA);
      if (fast) {
        if (!SUMMARY) {
          if (issuer) {
            tc::tmem_fence_after();
#pragma unroll 1
            for (int j = 0; j < kM / 8; ++j) {  // S = Qh Wh^T
              const uint32_t off = (j >> 2) * (kC * 128) + (j & 3) * 32;
              tc::mma_tf32_ss(tb + kColS, tc::smem_desc(q + off, 16, 1024), tc::smem_desc(w + off, 16, 1024),
                              tc::idesc_tf32(64, kC, 0, 0), j > 0);
            }
            tc::mma_commit(&bar_s);
#pragma unroll 1
            for (int j = 0; j < kM / 8; ++j) {  // O^T = Hr^T Qh^T (state read from TMEM)
              const uint32_t off = (j >> 2) * (kC * 128) + (j & 3) * 32;
              tc::mma_tf32_ts(tb + kColO, tb + kColHr + 8 * j, tc::smem_desc(q + off, 16, 1024),
                              tc::idesc_tf32(kDV, kC, 0, 0), j > 0);
            }
#pragma unroll 1
            for (int j = 0; j < kC / 8; ++j) {  // H^T += V^T Wh (carry)
              const uint32_t off = (j >> 2) * (kM * 128) + (j & 3) * 32;
              tc::mma_tf32_ss(tb + kColH, tc::smem_desc(vt + off, 16, 1024), tc::smem_desc(wt + off, 16, 1024),
                              tc::idesc_tf32(kDV, kM, 0, 0), 1);
            }
          }
          // S -> A (rows t = 16*(warp%4) + lane for lane < 16, at TMEM lanes 32*(warp%4) + lane)
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
                const float4 a4 = make_float4(s <= t ? tc::to_tf32(sv[j]) : 0.f,
                                              s + 1 <= t ? tc::to_tf32(sv[j + 1]) : 0.f,
                                              s + 2 <= t ? tc::to_tf32(sv[j + 2]) : 0.f,
                                              s + 3 <= t ? tc::to_tf32(sv[j + 3]) : 0.f);
                *reinterpret_cast<float4*>(sA + tc::swz_offset(kC, t, s)) = a4;
              }
            }
          }
          tc::fence_async_smem();
          tc::tmem_fence_before();
          mbar_arrive(&bar_a);
          if (issuer) {
            wait_or_abort(&bar_a, n_s & 1, abort_flag);
            tc::tmem_fence_after();
#pragma unroll 1
            for (int j = 0; j < kC / 8; ++j) {  // O^T += V^T A^T
              const uint32_t offa = (j >> 2) * (kC * 128) + (j & 3) * 32;
              const uint32_t offv = (j >> 2) * (kDV * 128) + (j & 3) * 32;
              tc::mma_tf32_ss(tb + kColO, tc::smem_desc(vt + offv, 16, 1024), tc::smem_desc(a + offa, 16, 1024),
                              tc::idesc_tf32(kDV, kC, 0, 0), 1);
            }
            tc::mma_commit(&bar_o);
          }
          ++n_s;
        } else if (issuer) {
          tc::tmem_fence_after();
#pragma unroll 1
          for (int j = 0; j < kC / 8; ++j) {  // H^T += V^T Wh (carry)
            const uint32_t off = (j >> 2) * (kM * 128) + (j & 3) * 32;
            tc::mma_tf32_ss(tb + kColH, tc::smem_desc(vt + off, 16, 1024), tc::smem_desc(wt + off, 16, 1024),
                            tc::idesc_tf32(kDV, kM, 0, 0), 1);
          }
          tc::mma_commit(&bar_o);
        }
      } else {
        // ---- exact path: decay the state by this chunk first (end-referenced carry weights)
        sync_x();  // X0
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
        sync_x();  // X1
        sync_x();  // X2: the row workers have written A and Wh^T
        if (issuer) {
          tc::tmem_fence_after();
          if (!SUMMARY) {
#pragma unroll 1
            for (int j = 0; j < kM / 8; ++j) {
              const uint32_t off = (j >> 2) * (kC * 128) + (j & 3) * 32;
              tc::mma_tf32_ts(tb + kColO, tb + kColHr + 8 * j, tc::smem_desc(q + off, 16, 1024),
                              tc::idesc_tf32(kDV, kC, 0, 0), j > 0);
            }
          }
#pragma unroll 1
          for (int j = 0; j < kC / 8; ++j) {
            const uint32_t off = (j >> 2) * (kM * 128) + (j & 3) * 32;
            tc::mma_tf32_ss(tb + kColH, tc::smem_desc(vt + off, 16, 1024), tc::smem_desc(wt + off, 16, 1024),
                            tc::idesc_tf32(kDV, kM, 0, 0), 1);
          }
          if (!SUMMARY) {
#pragma unroll 1
            for (int j = 0; j < kC / 8; ++j) {
              const uint32_t offa = (j >> 2) * (kC * 128) + (j & 3) * 32;
              const uint32_t offv = (j >> 2) * (kDV * 128) + (j & 3) * 32;
              tc::mma_tf32_ss(tb + kColO, tc::smem_desc(vt + offv, 16, 1024), tc::smem_desc(a + offa, 16, 1024),
                              tc::idesc_tf32(kDV, kC, 0, 0), 1);
            }
          }
          tc::mma_commit(&bar_o);
        }
      }
      prev = ck;
      have_prev = true;
      fast_prev = fast;
    }
    if (have_prev && !*abort_flag) finish_prev(n - 1);
    if (issuer) {
      // no MMA or tile load may still be running when the CTA releases its memory
      tc::mma_commit(&bar_o);
      tc::mbar_wait(&bar_o, n & 1);
      if (n_tma_issued > n) tc::mbar_wait(&bar_tma[n & 1], (n >> 1) & 1);
    }
  }

  tc::tmem_fence_before();
  __syncthreads();
  tc::tmem_fence_after();
  if (warp == kRWarps) tc::tmem_dealloc(tb, kTmemCols);
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
  if (!make_map(&maps.v, a.v, a.B, a.T, a.H, kDV)) return cudaErrorInvalidValue;
  Params p;
  p.B = a.B; p.T = a.T; p.H = a.H; p.K = a.K;
  p.decay_slot = a.decay == RSM_DECAY_SLOT;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
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
