// prefill_tc.cu -- chunked prefill on the 5th-generation tensor cores (rsm_forward, tensor path).
//
// Shapes: M = 128 slots, Dv = 128, bf16 q/k/v, K <= 32, per-head or per-slot log-decay.
//
// Chunk algebra (paperlayer.ai summary of the Raven paper, section A.5: T = n*C chunks of C = 64
// tokens), for one (b,h) stream and one chunk, with G_{t,i} = e^{g_{t,i}} the product of the decays
// a = e^lam of slot i from the chunk start through token t, w_{t,i} = k_{t,i} (1 - a_{t,i}) on the
// selected slots and 0 elsewhere, and the reference point at the chunk start:
//   Qh = q * G                (|Qh| <= |q|)
//   Wh = w / G                (finite while every slot decays by less than e^-80 in the chunk)
//   S  = Qh Wh^T,  A = S masked to s <= t           (intra-chunk weights, read after write)
//   O  = Qh H_start + A V                            (chunk outputs)
//   H_end = G_end * (H_start + Wh^T V)               (carry; rows never selected are skipped)
// G and 1/G are running products of a and 1/a down the chunk, so the tiles need no exponential
// per element. A chunk whose decay is stronger than the bound takes an exact path: A from
// pairwise sums with non-positive exponents, and the carry with weights w * e^{g_end - g} after
// the state is decayed.
//
// The routing is not done here: a thread-per-row kernel (route_rec.cu) has already turned the
// logits into one record per row (selection mask, selected slots, lam of each), read here.
//
// Operands are fp32 tiles rounded to nearest tf32 (kind::tf32), accumulated in fp32. The fp32
// state lives in TMEM as H^T (lane = value column, column = slot); the carry accumulates into it
// and a tf32-rounded copy feeds the next chunk's read as the A operand straight from TMEM.
// TMEM columns: [0,128) H^T, [128,256) rounded H^T, [256,320) O^T, [320,384) S (64-lane layout).
//
// Warp roles (one persistent CTA per SM, 12 warps):
//   warps 0-7  row workers, 8 rows of each chunk per warp: the decays of the selected entries of
//              their rows (one lane per entry), the per-slot product over their rows, then, once
//              the previous chunk's MMAs have read the operand tiles, their rows of Qh, Wh, Wh^T.
//              q, k and the records of the next chunk are loaded while this one is processed.
//   warps 8-11 TMEM workers (one per TMEM lane quarter): outputs of chunk n-1, the decay of the
//              state and its rounded copy, the V^T tile of chunk n, the S -> A masking. Thread 256
//              also issues the v tile loads and the MMAs.
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
constexpr int kIssuer = kRThreads;       // first thread of the TMEM workers
constexpr float kDMin = 1.80485139e-35f;  // e^-80: fast-path bound on the in-chunk decay
constexpr int kRecMax = 176;              // routing record bytes for K = 32

constexpr int kColH = 0, kColHr = 128, kColO = 256, kColS = 320, kTmemCols = 512;

// Dynamic shared memory (offsets from a 1024-byte aligned base). Operand tiles are K-major in the
// swizzled format of tc.cuh; Wh^T and V^T are stored transposed because they are contracted over
// tokens (a tf32 operand cannot be MN-major in this swizzle).
constexpr int kOffQ = 0;                      // Qh   [64 t][128 slot]   (A of S, B of the read)
constexpr int kOffW = kOffQ + 32768;          // Wh   [64 s][128 slot]   (B of S); exact path: dense g
constexpr int kOffWt = kOffW + 32768;         // Wh^T [128 slot][64 s]   (B of the carry)
constexpr int kOffVt = kOffWt + 32768;        // V^T  [128 dv][64 s]     (A of carry and A.V)
constexpr int kOffA = kOffVt + 32768;         // A    [64 t][64 s]       (B of A.V)
constexpr int kOffRawV = kOffA + 16384;       // v tile from TMA, [64][128] bf16
constexpr int kOffCmp = kOffRawV + 16384;     // per selected entry (a, 1/a, 1-a, lam), [64][KP] float4
constexpr int kOffRec = kOffCmp + kC * kKMax * 16;                   // records, [8 warps][8 rows][RB]
constexpr int kOffTot = kOffRec + kRWarps * kRowsPerWarp * kRecMax;  // per-warp slot totals, [2][8][128]
constexpr int kOffSmall = kOffTot + 2 * kRWarps * kM * 4;
// D[2][M], touched[2][M], mask OR [2][8][4], fast[2]
constexpr int kSmallBytes = (2 * kM + 2 * kM + 2 * kRWarps * 4 + 2) * 4 + 8;
constexpr int kSmemBytes = kOffSmall + kSmallBytes + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Maps {
  CUtensorMap v;
};

struct Params {
  int B, T, H, K;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const unsigned char* rec;  // routing records, rec_bytes per row, rows in [B, T, H] order
  int rec_bytes;
  const float* H0;
  float* o;
  float* HT;
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
RSM_DEV float bf16_at(const __nv_bfloat16* p) {
  return __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t*>(p)) << 16);
}

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
RSM_DEV void bar_rows() { asm volatile("bar.sync 1, %0;" ::"n"(kRThreads) : "memory"); }

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

// A row worker's inputs for one chunk: q and k of its 8 rows (4 slots per lane) and the pieces of
// its 8 routing records (16 bytes per piece, up to 3 pieces per lane).
struct RowInputs {
  uint2 q[kRowsPerWarp], k[kRowsPerWarp];
  uint4 rec[3];
};

template <bool SUMMARY>
RSM_DEV void load_rows(const Params& p, const Chunk& c, int w, int lane, int n16, RowInputs& in) {
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int t = w * kRowsPerWarp + r;
    in.k[r] = make_uint2(0u, 0u);
    in.q[r] = make_uint2(0u, 0u);
    if (t < c.nrows) {
      const int64_t row = ((int64_t)c.b * p.T + c.c0 + t) * p.H + c.h;
      in.k[r] = reinterpret_cast<const uint2*>(p.k + row * kM)[lane];
      if (!SUMMARY) in.q[r] = reinterpret_cast<const uint2*>(p.q + row * kM)[lane];
    }
  }
#pragma unroll
  for (int u = 0; u < 3; ++u) {
    const int idx = lane + 32 * u;
    const int r = idx / n16, part = idx - r * n16;
    const int t = w * kRowsPerWarp + r;
    in.rec[u] = make_uint4(0u, 0u, 0u, 0u);
    if (r < kRowsPerWarp && t < c.nrows) {
      const int64_t row = ((int64_t)c.b * p.T + c.c0 + t) * p.H + c.h;
      in.rec[u] = *reinterpret_cast<const uint4*>(p.rec + row * p.rec_bytes + part * 16);
    }
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
  const uint16_t* sRawV = reinterpret_cast<const uint16_t*>(sm + kOffRawV);
  float4* sCmp = reinterpret_cast<float4*>(sm + kOffCmp);
  unsigned char* sRec = sm + kOffRec;
  float* sTot = reinterpret_cast<float*>(sm + kOffTot);
  float* sDc = reinterpret_cast<float*>(sm + kOffSmall);         // [2][M]
  int* sTouch = reinterpret_cast<int*>(sDc + 2 * kM);             // [2][M]
  uint32_t* sOr = reinterpret_cast<uint32_t*>(sTouch + 2 * kM);  // [2][8][4]
  int* sFast = reinterpret_cast<int*>(sOr + 2 * kRWarps * 4);    // [2]

  __shared__ __align__(8) uint64_t bar_tma, bar_v, bar_ready, bar_s, bar_a, bar_t, bar_o, bar_x;
  __shared__ uint32_t s_tbase;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool row_worker = warp < kRWarps;
  const int T = p.T, H = p.H, K = p.K;
  const int pairs = p.B * H;
  const int segs_here = SUMMARY ? p.nseg - 1 : p.nseg;
  const int items = pairs * segs_here;
  const int KP = K <= 16 ? 16 : 32;  // entries per row in sCmp

  if (warp == kRWarps) tc::tmem_alloc(&s_tbase, kTmemCols);
  if (tid == 0) {
    tc::mbar_init(&bar_tma, 1);
    tc::mbar_init(&bar_v, kThreads - kRThreads);
    tc::mbar_init(&bar_ready, kThreads);
    tc::mbar_init(&bar_s, 1);
    tc::mbar_init(&bar_a, kThreads - kRThreads);
    tc::mbar_init(&bar_t, 1);
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
    const int RB = p.rec_bytes, n16 = RB / 16;
    const int slot_off = 16, lam_off = 16 + ((K + 15) & ~15);
    unsigned char* myRec = sRec + w * (kRowsPerWarp * kRecMax);  // this warp's 8 records, stride RB
    const int mw = lane >> 3;                  // mask word holding the lane's 4 slots
    const int sh = (lane & 7) * 4;             // bit offset of the lane's slots in that word
    const uint32_t below = (1u << sh) - 1u;    // the word's bits of lower slots
    const int ej = lane % KP, er = lane / KP;  // entry-parallel mapping: entry ej of row r0 + er
    const int rpp = 32 / KP;                   // rows per entry pass
    float Dseg[4] = {1.f, 1.f, 1.f, 1.f};      // summary pass, warp 0: product of the chunk decays
    int tseg[4] = {0, 0, 0, 0};

    RowInputs cur;
    if (wk.valid()) load_rows<SUMMARY>(p, wk.get(), w, lane, n16, cur);
    for (uint32_t n = 0; wk.valid(); ++n, wk.next()) {
      const Chunk ck = wk.get();
      const int buf = n & 1;
      // ---- records into shared memory; the next chunk's inputs start loading
#pragma unroll
      for (int u = 0; u < 3; ++u) {
        const int idx = lane + 32 * u;
        const int r = idx / n16, part = idx - r * n16;
        if (r < kRowsPerWarp) *reinterpret_cast<uint4*>(myRec + r * RB + part * 16) = cur.rec[u];
      }
      RowInputs nxt;
      {
        Walker nx = wk;
        nx.next();
        if (nx.valid()) load_rows<SUMMARY>(p, nx.get(), w, lane, n16, nxt);
      }
      __syncwarp();
      // ---- decay of every selected entry of the warp's rows (one lane per entry)
      for (int r0 = 0; r0 < kRowsPerWarp; r0 += rpp) {
        const int r = r0 + er;
        const int t = w * kRowsPerWarp + r;
        if (ej < K && t < ck.nrows) {
          const float lam = *reinterpret_cast<const float*>(myRec + r * RB + lam_off + 4 * ej);
          sCmp[t * KP + ej] = make_float4(expf(lam), expf(-lam), -expm1f(lam), lam);
        }
      }
      float* tot = sTot + (buf * kRWarps + w) * kM;
      reinterpret_cast<float4*>(tot)[lane] = make_float4(1.f, 1.f, 1.f, 1.f);
      if (lane < 4) {
        uint32_t om = 0u;
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) om |= reinterpret_cast<const uint32_t*>(myRec + r * RB)[lane];
        sOr[(buf * kRWarps + w) * 4 + lane] = om;
      }
      __syncwarp();
      // per-slot product of the decays over the warp's rows, rows in order
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) {
        const int t = w * kRowsPerWarp + r;
        if (lane < K && t < ck.nrows) {
          const int slot = myRec[r * RB + slot_off + lane];
          tot[slot] *= sCmp[t * KP + lane].x;
        }
        __syncwarp();
      }
      if (bar_rows_or(*abort_flag != 0)) break;  // every row worker takes the same decision
      // ---- in-chunk products at the warp's first row (off) and over the chunk (gend)
      float off[4] = {1.f, 1.f, 1.f, 1.f}, gend[4] = {1.f, 1.f, 1.f, 1.f};
      uint32_t orw = 0u;
#pragma unroll
      for (int w2 = 0; w2 < kRWarps; ++w2) {
        const float4 t4 = reinterpret_cast<const float4*>(sTot + (buf * kRWarps + w2) * kM)[lane];
        const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (w2 < w) off[e] *= tv[e];
          gend[e] *= tv[e];
        }
        orw |= sOr[(buf * kRWarps + w2) * 4 + mw];
      }
      bool ok = true;
#pragma unroll
      for (int e = 0; e < 4; ++e) ok &= gend[e] >= kDMin;
      const bool fast = __all_sync(kFull, ok);
      // ---- the previous chunk's MMAs have read the operand tiles (and the TMEM workers have
      // finished the chunk before it, whose decay buffer this chunk reuses)
      if (n > 0) wait_or_abort(&bar_t, (n - 1) & 1, abort_flag);
      if (w == 0) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int slot = lane * 4 + e;
          const int touched = (orw >> (sh + e)) & 1u;
          sDc[buf * kM + slot] = gend[e];
          sTouch[buf * kM + slot] = touched;
          if (SUMMARY) {
            if (ck.first) {
              Dseg[e] = 1.f;
              tseg[e] = 0;
            }
            Dseg[e] *= gend[e];
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
        // ---- this warp's rows of Qh, Wh and Wh^T
        float G[4], Gi[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          G[e] = off[e];
          Gi[e] = 1.f / off[e];
        }
        float stash[4][4];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const int t = w * kRowsPerWarp + r;
          const uint4 mk = *reinterpret_cast<const uint4*>(myRec + r * RB);
          const uint32_t wd = mw == 0 ? mk.x : mw == 1 ? mk.y : mw == 2 ? mk.z : mk.w;
          int base = __popc(wd & below) + (mw > 0 ? __popc(mk.x) : 0) + (mw > 1 ? __popc(mk.y) : 0) +
                     (mw > 2 ? __popc(mk.z) : 0);
          const float4 q4 = bf16x4_to_f32(cur.q[r]);
          const float4 k4 = bf16x4_to_f32(cur.k[r]);
          float qh[4], wh[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float wt = 0.f;
            if ((wd >> (sh + e)) & 1u) {
              const float4 c = sCmp[t * KP + base];
              ++base;
              G[e] *= c.x;
              Gi[e] *= c.y;
              wt = fget(k4, e) * c.z * Gi[e];  // k (1 - a) / G_t
            }
            qh[e] = SUMMARY ? 0.f : tc::to_tf32(fget(q4, e) * G[e]);
            wh[e] = tc::to_tf32(wt);
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
        // ---- exact path (rare), with the TMEM workers: dense g (log domain, in the Wh region),
        // the Qh tile, the end-referenced Wh^T and A from pairwise sums, exponents <= 0
        mbar_arrive(&bar_ready);
        sync_x();  // X0: every row worker is past the product totals; the TMEM workers decay H
        float* totL = sTot + (buf * kRWarps + w) * kM;  // now: per-warp sums of lam
        reinterpret_cast<float4*>(totL)[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
        __syncwarp();
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const int t = w * kRowsPerWarp + r;
          if (lane < K && t < ck.nrows) {
            const int slot = myRec[r * RB + slot_off + lane];
            totL[slot] += sCmp[t * KP + lane].w;
          }
          __syncwarp();
        }
        bar_rows();
        float g[4] = {0.f, 0.f, 0.f, 0.f};
        for (int w2 = 0; w2 < w; ++w2) {
          const float4 t4 = reinterpret_cast<const float4*>(sTot + (buf * kRWarps + w2) * kM)[lane];
          g[0] += t4.x; g[1] += t4.y; g[2] += t4.z; g[3] += t4.w;
        }
        float* dg = reinterpret_cast<float*>(sW);  // plain [64][128]
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const int t = w * kRowsPerWarp + r;
          const uint4 mk = *reinterpret_cast<const uint4*>(myRec + r * RB);
          const uint32_t wd = mw == 0 ? mk.x : mw == 1 ? mk.y : mw == 2 ? mk.z : mk.w;
          int base = __popc(wd & below) + (mw > 0 ? __popc(mk.x) : 0) + (mw > 1 ? __popc(mk.y) : 0) +
                     (mw > 2 ? __popc(mk.z) : 0);
          const float4 q4 = bf16x4_to_f32(cur.q[r]);
          float qh[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            if ((wd >> (sh + e)) & 1u) {
              g[e] += sCmp[t * KP + base].w;
              ++base;
            }
            qh[e] = SUMMARY ? 0.f : tc::to_tf32(fget(q4, e) * expf(g[e]));
          }
          reinterpret_cast<float4*>(dg + t * kM)[lane] = make_float4(g[0], g[1], g[2], g[3]);
          if (!SUMMARY)
            *reinterpret_cast<float4*>(sQ + tc::swz_offset(kC, t, lane * 4)) = make_float4(qh[0], qh[1], qh[2], qh[3]);
        }
        // write weight of every selected entry, w = k (1 - a), into its (unused) 1/a field
        for (int r0 = 0; r0 < kRowsPerWarp; r0 += rpp) {
          const int r = r0 + er;
          const int t = w * kRowsPerWarp + r;
          if (ej < K && t < ck.nrows) {
            const int slot = myRec[r * RB + slot_off + ej];
            const int64_t row = ((int64_t)ck.b * T + ck.c0 + t) * H + ck.h;
            sCmp[t * KP + ej].y = bf16_at(p.k + row * kM + slot) * sCmp[t * KP + ej].z;
          }
        }
        for (int e = tid; e < kC * kM / 4; e += kRThreads)
          reinterpret_cast<float4*>(sWt)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        bar_rows();
        const int nrows = ck.nrows;
        for (int e = tid; e < nrows * KP; e += kRThreads) {
          const int t = e / KP, j = e % KP;
          if (j >= K) continue;
          const unsigned char* rt = sRec + (t / kRowsPerWarp) * (kRowsPerWarp * kRecMax) + (t % kRowsPerWarp) * RB;
          const int i = rt[slot_off + j];
          const float gend_i = dg[(kC - 1) * kM + i];
          *reinterpret_cast<float*>(sWt + tc::swz_offset(kM, i, t)) =
              tc::to_tf32(sCmp[t * KP + j].y * expf(gend_i - dg[t * kM + i]));
        }
        if (!SUMMARY) {
          for (int e = tid; e < kC * kC; e += kRThreads) {
            const int t = e / kC, s = e % kC;
            float acc = 0.f;
            if (s <= t && t < nrows) {
              const unsigned char* rs = sRec + (s / kRowsPerWarp) * (kRowsPerWarp * kRecMax) + (s % kRowsPerWarp) * RB;
              const int64_t rowt = ((int64_t)ck.b * T + ck.c0 + t) * H + ck.h;
              for (int j = 0; j < K; ++j) {
                const int i = rs[slot_off + j];
                const float qti = bf16_at(p.q + rowt * kM + i);
                acc = fmaf(qti * sCmp[s * KP + j].y, expf(dg[t * kM + i] - dg[s * kM + i]), acc);
              }
            }
            *reinterpret_cast<float*>(sA + tc::swz_offset(kC, t, s)) = tc::to_tf32(acc);
          }
        }
        tc::fence_async_smem();
        sync_x();  // X1
      }
      cur = nxt;
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
      tc::mbar_arrive_expect_tx(&bar_tma, kC * kDV * 2);
      tc::tma_load_4d(sm + kOffRawV, &maps.v, &bar_tma, 0, c.h, c.c0, c.b);
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
      wait_or_abort(&bar_tma, n & 1, abort_flag);
#pragma unroll 4
      for (int s4 = 0; s4 < kC; s4 += 4) {
        const float4 f4 = make_float4(__uint_as_float((uint32_t)sRawV[(s4 + 0) * kDV + dv] << 16),
                                      __uint_as_float((uint32_t)sRawV[(s4 + 1) * kDV + dv] << 16),
                                      __uint_as_float((uint32_t)sRawV[(s4 + 2) * kDV + dv] << 16),
                                      __uint_as_float((uint32_t)sRawV[(s4 + 3) * kDV + dv] << 16));
        *reinterpret_cast<float4*>(sVt + tc::swz_offset(kDV, dv, s4)) = f4;
      }
      tc::fence_async_smem();
      mbar_arrive(&bar_v);  // this TMEM worker is done with the raw v tile
      if (issuer) {
        Walker nx = wk;
        nx.next();
        wait_or_abort(&bar_v, n & 1, abort_flag);
        if (nx.valid()) {
          const Chunk c = nx.get();
          ++n_tma_issued;
          tc::mbar_arrive_expect_tx(&bar_tma, kC * kDV * 2);
          tc::tma_load_4d(sm + kOffRawV, &maps.v, &bar_tma, 0, c.h, c.c0, c.b);
        }
      }
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
            tc::mma_commit(&bar_t);  // Qh, Wh, Wh^T are free for the next chunk
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
          tc::mma_commit(&bar_t);
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
        sync_x();  // X1: the row workers have written Qh, A and Wh^T
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
          tc::mma_commit(&bar_t);
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
      if (n_tma_issued > n) tc::mbar_wait(&bar_tma, n & 1);
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

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace: routing records, then (segmented runs) the segment states, decays and touch flags.
struct WsLayout {
  size_t rec, state, D, touch, total;
};
WsLayout ws_layout(const rsm_forward_args& a, const Plan& pl) {
  WsLayout l;
  const size_t rows = (size_t)a.B * a.T * a.H;
  l.rec = 0;
  size_t off = up256(rows * (size_t)route_record_bytes(a.K));
  l.state = l.D = l.touch = off;
  if (pl.nseg > 1) {
    const size_t per = (size_t)a.B * a.H * pl.nseg;
    l.state = off;
    off += up256(per * kM * kDV * 4);
    l.D = off;
    off += up256(per * kM * 4);
    l.touch = off;
    off += up256(per * kM * 4);
  }
  l.total = off;
  return l;
}

}  // namespace

bool prefill_tc_supported(const rsm_forward_args& a) {
  return a.qkv_dtype == RSM_BF16 && a.M == kM && a.Dv == kDV && a.K <= kKMax && route_records_supported(a.M, a.K);
}

size_t prefill_tc_workspace_bytes(const rsm_forward_args& a) {
  if (!prefill_tc_supported(a)) return 0;
  return ws_layout(a, plan_for(a, sm_count())).total;
}

int prefill_tc_launches(const rsm_forward_args& a) {
  if (!prefill_tc_supported(a) || a.T == 0) return 0;
  return plan_for(a, sm_count()).nseg > 1 ? 4 : 2;
}

cudaError_t launch_prefill_tc(const rsm_forward_args& a, cudaStream_t stream) {
  const int sms = sm_count();
  const Plan pl = plan_for(a, sms);
  const WsLayout wl = ws_layout(a, pl);
  char* ws = static_cast<char*>(a.workspace);
  unsigned char* rec = reinterpret_cast<unsigned char*>(ws + wl.rec);
  const int64_t rows = (int64_t)a.B * a.T * a.H;
  cudaError_t e = launch_route_records(a.logits, a.f, rows, a.M, a.K, a.decay == RSM_DECAY_SLOT,
                                       (a.flags & RSM_FLAG_VALIDATE) != 0, rec, a.idx_out, a.score_out, stream);
  if (e != cudaSuccess) return e;
  Maps maps;
  if (!make_map(&maps.v, a.v, a.B, a.T, a.H, kDV)) return cudaErrorInvalidValue;
  Params p;
  p.B = a.B; p.T = a.T; p.H = a.H; p.K = a.K;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.k = static_cast<const __nv_bfloat16*>(a.k);
  p.rec = rec;
  p.rec_bytes = route_record_bytes(a.K);
  p.H0 = a.H0;
  p.o = a.o; p.HT = a.HT;
  p.nseg = pl.nseg; p.seg_chunks = pl.seg_chunks;
  p.ws_state = nullptr; p.ws_D = nullptr; p.ws_touch = nullptr;
  if (pl.nseg > 1) {
    p.ws_state = reinterpret_cast<float*>(ws + wl.state);
    p.ws_D = reinterpret_cast<float*>(ws + wl.D);
    p.ws_touch = reinterpret_cast<int*>(ws + wl.touch);
  }
  e = cudaFuncSetAttribute(prefill_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t pairs = (int64_t)a.B * a.H;
  if (pl.nseg > 1) {
    const int items = (int)(pairs * (pl.nseg - 1));
    prefill_tc_kernel<true><<<std::min(items, sms), kThreads, kSmemBytes, stream>>>(maps, p);
    e = cudaGetLastError();
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
