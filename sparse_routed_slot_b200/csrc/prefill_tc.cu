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
// logits into one record per row (selected slots, lam = log of each decay, w = k (1 - a)), stored
// time-contiguous per (b,h) stream; the chunk's 64 records are read here.
//
// Operands are fp32 tiles rounded to nearest tf32 (kind::tf32), accumulated in fp32. The fp32
// state lives in TMEM as H^T (lane = value column, column = slot); the carry accumulates into it
// and a tf32-rounded copy feeds the next chunk's read as the A operand straight from TMEM (the
// tensor core would truncate fp32, a bias proportional to each output).
// TMEM columns: [0,128) H^T, [128,256) rounded H^T, [256,320) and [320,384) O^T of even and odd
// chunks, [384,448) S (64-lane layout); [384,512) U^T, the carry of an exact-path chunk, shares
// S's columns (an exact chunk has no S, and the next S waits until the epilogue has used U).
//
// Warp roles (one persistent CTA per SM, 13 warps):
//   warps 0-7  row workers; warp w owns tokens 8w..8w+7 of the chunk, lane l slots 4l..4l+3.
//              A warp scatters the decays of its rows' selected entries into its rows of a dense
//              per-chunk table (a = 1 elsewhere, the sign bit marks a selected entry), multiplies
//              along its rows, and exchanges the per-warp products for the in-chunk prefix at its
//              first row. It then walks its rows: the running product G gives Qh = q G and, at
//              the selected entries, G itself, from which each entry's owner forms Wh = w / G in
//              the Wh and Wh^T tiles. Once a chunk's tiles are handed over, the row workers convert
//              its v tile into V^T. q and the records of the next chunk are loaded while this one
//              is processed.
//   warp 8     MMA issuer (one thread): v tile loads (two chunks ahead) and the tcgen05.mma of
//              every chunk, as soon as their operands are ready.
//   warps 9-12 epilogue (one per TMEM lane quarter): S -> A masking, the decay of the state after
//              the carry (and the state in and out at item boundaries), the output of the chunk
//              from TMEM, staged in halves through the A tile's memory and written by bulk tensor
//              stores.
// Per chunk the issuer runs S = Qh Wh^T (as soon as the row tiles are ready), then, once the
// state is decayed, O^T = H^T Qh^T, then (the V^T conversion overlaps the read) the carry
// H^T += V^T Wh, and finally O^T += V^T A^T when the epilogue has masked S into A. An exact-path chunk carries into
// U^T = V^T Wh_end (end-referenced weights) and the epilogue forms H = D H + U.
// Every mbarrier is waited on by a role that the barrier's next phase depends on, so no waiter
// can fall two phases behind (which a parity wait cannot tell from zero).
//
// Long sequences with few (b,h) streams are split into segments processed in parallel: a summary
// kernel (segment_summary_kernel, below) computes for each segment but the last the product of
// its decays and the state it reaches from a zero start, as one accumulation of end-referenced
// weights; a scan combines them into the true start state of every segment; the main pass then
// runs every segment from its start state.
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
constexpr int kRThreads = kRWarps * 32;
constexpr int kIssuerWarp = kRWarps;          // warp 8
constexpr int kEpiThreads = 4 * 32;
constexpr int kEpiThread0 = (kRWarps + 1) * 32;  // issues the output tile stores
constexpr int kThreads = (kRWarps + 1 + 4) * 32;
constexpr float kDMin = 1.80485139e-35f;  // e^-80: fast-path bound on the in-chunk decay

constexpr int kColH = 0, kColHr = 128, kColO = 256, kColS = 384, kColU = 384, kTmemCols = 512;

// Dynamic shared memory (offsets from a 1024-byte aligned base). Operand tiles are K-major in the
// swizzled format of tc.cuh; Wh^T and V^T are stored transposed because they are contracted over
// tokens and every operand tile here is K-major. Qh is double-buffered (chunk n&1), so the row
// workers can build the next chunk's Qh while this chunk's read still uses its own. The Wh tile
// also holds the chunk's decay table before the walk turns it into G (in place) and the post-pass
// into Wh; an exact-path chunk keeps lam and then the dense g there (plain [64][128] layout).
constexpr int kOffQ = 0;                   // Qh   [2][64 t][128 slot] (A of S, B of the read)
constexpr int kOffW = kOffQ + 2 * 32768;   // Wh   [64 s][128 slot]   (B of S); decay table before
constexpr int kOffWt = kOffW + 32768;      // Wh^T [128 slot][64 s]   (B of the carry)
constexpr int kOffVt = kOffWt + 32768;     // V^T  [128 dv][64 s]     (A of carry and A.V)
constexpr int kOffA = kOffVt + 32768;      // A    [64 t][64 s]       (B of A.V)
constexpr int kOffRawV = kOffA + 16384;    // v tiles from TMA, [2][64][128] bf16
constexpr int kOffTot = kOffRawV + 32768;  // per-warp slot products (sums), [2][8][128]
constexpr int kOffSmall = kOffTot + 2 * kRWarps * kM * 4;
// D[2][M], fast[2]
constexpr int kSmallBytes = 2 * kM * 4 + 16;
constexpr int kSmemBytes = kOffSmall + kSmallBytes + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");

struct Maps {
  CUtensorMap v;    // v [B,T,H,Dv] bf16, box: one (b,h), 64 tokens
  CUtensorMap vsw;  // v [B,T,H,Dv] bf16, box: 64 value columns of one (b,h), 64 tokens, 128B swizzle
  CUtensorMap o;    // o [B,T,H,Dv] fp32, box: one (b,h), 32 tokens (output stores)
};

struct Params {
  int B, T, H, K;
  const __nv_bfloat16* q;
  const unsigned char* rec;  // routing records, rec_bytes per row, rows in [B, H, T] order
  int rec_bytes;
  const float* H0;
  float* o;
  float* HT;
  int nseg, seg_chunks;
  int sub, piece_chunks;  // summary pieces per segment and their length in chunks
  int nslot;              // 1 + (nseg - 1) * sub
  float* ws_state;  // [pairs][nslot][M][Dv]: slot 0 = start state, slot 1 + k = summary of piece k
  float* ws_D;      // [pairs][nslot][M]
};

RSM_DEV float4 bf16x4_to_f32(uint2 r) {
  return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xffff0000u),
                     __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xffff0000u));
}
RSM_DEV float fget(const float4& v, int e) { return e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w; }
RSM_DEV float bf16_at(const __nv_bfloat16* p) {
  return __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t*>(p)) << 16);
}
// v[j] *= d[j] for 32 consecutive slots (d in shared memory, 16-byte aligned).
RSM_DEV void scale_by(float (&v)[32], const float* d) {
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    const float4 d4 = *reinterpret_cast<const float4*>(d + j);
    v[j] *= d4.x; v[j + 1] *= d4.y; v[j + 2] *= d4.z; v[j + 3] *= d4.w;
  }
}
RSM_DEV bool sign_set(float x) { return (__float_as_uint(x) >> 31) != 0u; }

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
RSM_DEV void bar_epi() { asm volatile("bar.sync 2, %0;" ::"n"(kEpiThreads) : "memory"); }
// Barrier among the epilogue warps that ORs a flag over them (every epilogue thread sees the same).
RSM_DEV bool bar_epi_or(bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 2, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)flag), "n"(kEpiThreads)
      : "memory");
  return r != 0;
}

// Position of one chunk in the CTA's work list.
struct Chunk {
  int pair, seg, b, h, c0, nrows;
  bool first, last;
};

// The CTA walks its items (item = blockIdx.x + j*gridDim.x) and each item's chunks in order.
// The item's coordinates are computed once per item (integer division is not cheap here); the
// sizes come from the kernel parameters, so a walker is only a few registers.
struct Walker {
  int item, c0, t1, pair, seg, b, h;
  bool first;
  __device__ void start(const Params& p, int items) {
    item = blockIdx.x;
    set_item(p, items);
  }
  __device__ void set_item(const Params& p, int items) {
    if (item >= items) return;
    const int pairs = p.B * p.H;
    seg = item / pairs;
    pair = item - seg * pairs;
    b = pair / p.H;
    h = pair - b * p.H;
    c0 = seg * p.seg_chunks * kC;
    t1 = min(p.T, c0 + p.seg_chunks * kC);
    first = true;
  }
  __device__ bool valid(int items) const { return item < items; }
  __device__ Chunk get(const Params& p) const {
    Chunk c;
    c.pair = pair;
    c.seg = seg;
    c.b = b;
    c.h = h;
    c.c0 = c0;
    c.nrows = min(kC, t1 - c0);
    c.first = first;
    c.last = c0 + kC >= t1;
    return c;
  }
  __device__ void next(const Params& p, int items) {
    c0 += kC;
    first = false;
    if (c0 >= t1) {
      item += gridDim.x;
      set_item(p, items);
    }
  }
};

// A row worker's inputs for one chunk: q of its 8 rows (4 slots per lane) and up to 8 entries of
// its rows' records (groups of 4 consecutive entries: slots, lam, w).
template <int KP>
struct RowInputs {
  static constexpr int kGroups = KP / 16;  // groups of 4 entries per lane
  uint2 q[kRowsPerWarp];
  uint32_t es[kGroups];
  float4 el[kGroups], ew[kGroups];
};

// Entry group g of lane `lane` in a warp's 8 records of KP entries each: row r, first entry j0.
RSM_DEV void entry_pos(int lane, int g, int KP, int& r, int& j0) {
  const int f = (lane + 32 * g) * 4;
  r = f / KP;
  j0 = f - r * KP;
}

template <bool SUMMARY, int KP>
RSM_DEV void load_rows(const Params& p, const Chunk& c, int w, int lane, RowInputs<KP>& in) {
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int t = w * kRowsPerWarp + r;
    in.q[r] = make_uint2(0u, 0u);
    if (!SUMMARY && t < c.nrows) {
      const int64_t row = ((int64_t)c.b * p.T + c.c0 + t) * p.H + c.h;
      in.q[r] = reinterpret_cast<const uint2*>(p.q + row * kM)[lane];
    }
  }
  const unsigned char* rb = p.rec + ((int64_t)c.pair * p.T + c.c0 + w * kRowsPerWarp) * p.rec_bytes;
#pragma unroll
  for (int g = 0; g < RowInputs<KP>::kGroups; ++g) {
    int r, j0;
    entry_pos(lane, g, KP, r, j0);
    in.es[g] = 0u;
    in.el[g] = make_float4(0.f, 0.f, 0.f, 0.f);
    in.ew[g] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < kRowsPerWarp && w * kRowsPerWarp + r < c.nrows) {
      const unsigned char* e = rb + r * p.rec_bytes;
      in.es[g] = *reinterpret_cast<const uint32_t*>(e + j0);
      in.el[g] = *reinterpret_cast<const float4*>(e + KP + 4 * j0);
      in.ew[g] = *reinterpret_cast<const float4*>(e + 5 * KP + 4 * j0);
    }
  }
}

// Calls fn(r, slot, lam, w) for every valid entry of the lane's groups (row r of the warp).
template <int KP, class Fn>
RSM_DEV void for_entries(const RowInputs<KP>& in, int lane, int K, int nrows_w, Fn fn) {
#pragma unroll
  for (int g = 0; g < RowInputs<KP>::kGroups; ++g) {
    int r, j0;
    entry_pos(lane, g, KP, r, j0);
    if (r >= kRowsPerWarp || r >= nrows_w) continue;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (j0 + e < K) fn(r, (int)((in.es[g] >> (8 * e)) & 255u), fget(in.el[g], e), fget(in.ew[g], e));
    }
  }
}

template <int KP>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ Maps maps,
                                                                  const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* sQ = sm + kOffQ;
  unsigned char* sW = sm + kOffW;
  unsigned char* sWt = sm + kOffWt;
  unsigned char* sVt = sm + kOffVt;
  unsigned char* sA = sm + kOffA;
  unsigned char* sRawV = sm + kOffRawV;
  float* sTot = reinterpret_cast<float*>(sm + kOffTot);
  float* sDc = reinterpret_cast<float*>(sm + kOffSmall);    // [2][M]
  int* sFast = reinterpret_cast<int*>(sDc + 2 * kM);         // [2]

  // mbarriers (phase k of a barrier = its k-th completion; every role counts the same way)
  __shared__ __align__(8) uint64_t bar_rdy,  // row tiles of chunk n written         (row threads)
      bar_tma[2],                             // raw v tile of chunk n landed          (TMA, buffer n&1)
      bar_vt,                                 // V^T of chunk n written                (row threads)
      bar_s,                                  // main pass: S of chunk n done          (MMA commit)
      bar_a,                                  // main pass: A of chunk n written       (epilogue)
      bar_t,                                  // read and carry of chunk n done        (MMA commit)
      bar_o,                                  // every MMA of chunk n done             (MMA commit)
      bar_h,                                  // state ready for chunk n               (epilogue)
      bar_of[2],                              // O buffer n&1 stored after chunk n     (epilogue)
      bar_fin;                                // issuer only: every MMA issued is done (MMA commit)
  __shared__ uint32_t s_tbase;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = p.T, H = p.H, K = p.K;
  const int pairs = p.B * H;
  const int items = pairs * p.nseg;

  if (warp == kIssuerWarp) tc::tmem_alloc(&s_tbase, kTmemCols);
  if (tid == 0) {
    tc::mbar_init(&bar_rdy, kRThreads);
    tc::mbar_init(&bar_tma[0], 1);
    tc::mbar_init(&bar_tma[1], 1);
    tc::mbar_init(&bar_vt, kRThreads);
    tc::mbar_init(&bar_s, 1);
    tc::mbar_init(&bar_a, kEpiThreads);
    tc::mbar_init(&bar_t, 1);
    tc::mbar_init(&bar_o, 1);
    tc::mbar_init(&bar_h, kEpiThreads);
    tc::mbar_init(&bar_of[0], kEpiThreads);
    tc::mbar_init(&bar_of[1], kEpiThreads);
    tc::mbar_init(&bar_fin, 1);
    tc::fence_mbar_init();
    s_abort = 0;
  }
  if (warp == kIssuerWarp && lane == 0) tc::tma_prefetch_desc(&maps.v);
  tc::tmem_fence_before();
  __syncthreads();
  tc::tmem_fence_after();
  const uint32_t tb = s_tbase;
  volatile int* abort_flag = &s_abort;

  Walker wk;
  wk.start(p, items);

  if (warp < kRWarps) {
    // =========================================================================== row workers
    const int w = warp;
    const int RB = p.rec_bytes;
    // the decay table lives in the Wh tile: row t = w*8 + r of the warp, 4 slots per lane
    auto tab_row = [&](int r) -> float4* {
      return reinterpret_cast<float4*>(sW + tc::swz_offset(kC, w * kRowsPerWarp + r, lane * 4));
    };

    RowInputs<KP> cur;
    if (wk.valid(items)) load_rows<false, KP>(p, wk.get(p), w, lane, cur);
    for (uint32_t n = 0; wk.valid(items); ++n, wk.next(p, items)) {
      const Chunk ck = wk.get(p);
      const int buf = n & 1;
      const int nrows_w = ck.nrows - w * kRowsPerWarp;  // rows of this warp inside the chunk
      // ---- the previous chunk's S has read the Wh tile (and, issued before it, the read of the
      // chunk before that has read this chunk's Qh buffer)
      if (n > 0) wait_or_abort(&bar_s, (n - 1) & 1, abort_flag);
      // ---- this warp's rows of the decay table: 1 everywhere, -a at the selected entries
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) *tab_row(r) = make_float4(1.f, 1.f, 1.f, 1.f);
      __syncwarp();
      for_entries(cur, lane, K, nrows_w, [&](int r, int slot, float lam, float) {
        *reinterpret_cast<float*>(sW + tc::swz_offset(kC, w * kRowsPerWarp + r, slot)) = -expf(lam);
      });
      __syncwarp();
      // ---- product of the decays over the warp's rows, per slot
      float P[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
      for (int r = 0; r < kRowsPerWarp; ++r) {
        const float4 a4 = *tab_row(r);
        P[0] *= fabsf(a4.x); P[1] *= fabsf(a4.y); P[2] *= fabsf(a4.z); P[3] *= fabsf(a4.w);
      }
      reinterpret_cast<float4*>(sTot + (buf * kRWarps + w) * kM)[lane] = make_float4(P[0], P[1], P[2], P[3]);
      if (bar_rows_or(*abort_flag != 0)) break;  // every row worker takes the same decision
      // ---- in-chunk products before the warp's first row (off) and over the chunk (gend)
      float off[4] = {1.f, 1.f, 1.f, 1.f}, gend[4] = {1.f, 1.f, 1.f, 1.f};
#pragma unroll
      for (int w2 = 0; w2 < kRWarps; ++w2) {
        const float4 t4 = reinterpret_cast<const float4*>(sTot + (buf * kRWarps + w2) * kM)[lane];
        const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (w2 < w) off[e] *= tv[e];
          gend[e] *= tv[e];
        }
      }
      bool ok = true;
#pragma unroll
      for (int e = 0; e < 4; ++e) ok &= gend[e] >= kDMin;
      const bool fast = __all_sync(kFull, ok);
      // the chunk's decays and path, once the epilogue has used those of the chunk before the
      // previous one (its decay of the state precedes the previous chunk's read, and so the carry)
      auto put_decays = [&]() {
        if (w == 0) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int slot = lane * 4 + e;
            sDc[buf * kM + slot] = gend[e];
          }
          if (lane == 0) sFast[buf] = fast;
        }
      };
      unsigned char* sQb = sQ + buf * 32768;  // this chunk's Qh buffer
      if (fast) {
        // ---- walk the warp's rows: Qh = q G, and G at the selected entries (0 elsewhere)
        float G[4] = {off[0], off[1], off[2], off[3]};
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const int t = w * kRowsPerWarp + r;
          const float4 a4 = *tab_row(r);
          const float av[4] = {a4.x, a4.y, a4.z, a4.w};
          const float4 q4 = bf16x4_to_f32(cur.q[r]);
          float qh[4], gw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            G[e] *= fabsf(av[e]);
            qh[e] = tc::to_tf32(fget(q4, e) * G[e]);
            gw[e] = sign_set(av[e]) ? G[e] : 0.f;
          }
          *reinterpret_cast<float4*>(sQb + tc::swz_offset(kC, t, lane * 4)) = make_float4(qh[0], qh[1], qh[2], qh[3]);
          *reinterpret_cast<float4*>(sW + tc::swz_offset(kC, t, lane * 4)) = make_float4(gw[0], gw[1], gw[2], gw[3]);
        }
        // the previous carry has read Wh^T (and the epilogue has used the decays this chunk's
        // buffer held before)
        if (n > 0) wait_or_abort(&bar_t, (n - 1) & 1, abort_flag);
        put_decays();
        // this warp's token columns of Wh^T start at zero
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int slot = lane + 32 * e;  // 8 consecutive rows per 8 lanes: 4-way stores (no conflicts)
          *reinterpret_cast<float4*>(sWt + tc::swz_offset(kM, slot, w * kRowsPerWarp)) = make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(sWt + tc::swz_offset(kM, slot, w * kRowsPerWarp + 4)) =
              make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncwarp();
        // ---- each entry's owner: Wh = w / G_t (finite: G_t >= gend >= e^-80)
        for_entries(cur, lane, K, nrows_w, [&](int r, int slot, float, float wv) {
          const int t = w * kRowsPerWarp + r;
          float* gp = reinterpret_cast<float*>(sW + tc::swz_offset(kC, t, slot));
          const float wh = tc::to_tf32(__fdividef(wv, *gp));
          *gp = wh;
          *reinterpret_cast<float*>(sWt + tc::swz_offset(kM, slot, t)) = wh;
        });
        tc::fence_async_smem();
        mbar_arrive(&bar_rdy);
      } else {
        // ---- exact path (rare): log-domain table and dense g (in the Wh region), the Qh tile,
        // the end-referenced Wh^T and A from pairwise sums, exponents <= 0. The issuer runs the
        // read, the carry into U and A.V; the epilogue then forms H = D H + U.
        // A.V of the chunk before is done with A, and the epilogue has staged that chunk's output
        // through the A tile's memory
        if (n > 0) wait_or_abort(&bar_of[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag);
        put_decays();
        // lam, then the dense g, in the Wh tile's memory in plain [64][128] layout (this warp: rows
        // 8w..8w+7); every row worker is past the swizzled decay table first
        float* tab = reinterpret_cast<float*>(sW) + w * kRowsPerWarp * kM;
        bar_rows();  // every row worker is past the product totals
#pragma unroll
        for (int i = 0; i < kRowsPerWarp; ++i)
          reinterpret_cast<float4*>(tab)[lane + 32 * i] = make_float4(0.f, 0.f, 0.f, 0.f);
        __syncwarp();
        for_entries(cur, lane, K, nrows_w, [&](int r, int slot, float lam, float) { tab[r * kM + slot] = lam; });
        __syncwarp();
        float S[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
          const float4 l4 = reinterpret_cast<const float4*>(tab + r * kM)[lane];
          S[0] += l4.x; S[1] += l4.y; S[2] += l4.z; S[3] += l4.w;
        }
        reinterpret_cast<float4*>(sTot + (buf * kRWarps + w) * kM)[lane] = make_float4(S[0], S[1], S[2], S[3]);
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
          const float4 l4 = reinterpret_cast<const float4*>(tab + r * kM)[lane];
          g[0] += l4.x; g[1] += l4.y; g[2] += l4.z; g[3] += l4.w;
          reinterpret_cast<float4*>(dg + t * kM)[lane] = make_float4(g[0], g[1], g[2], g[3]);
          const float4 q4 = bf16x4_to_f32(cur.q[r]);
          *reinterpret_cast<float4*>(sQb + tc::swz_offset(kC, t, lane * 4)) =
              make_float4(tc::to_tf32(q4.x * expf(g[0])), tc::to_tf32(q4.y * expf(g[1])),
                          tc::to_tf32(q4.z * expf(g[2])), tc::to_tf32(q4.w * expf(g[3])));
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int slot = lane + 32 * e;  // 8 consecutive rows per 8 lanes: 4-way stores (no conflicts)
          *reinterpret_cast<float4*>(sWt + tc::swz_offset(kM, slot, w * kRowsPerWarp)) = make_float4(0.f, 0.f, 0.f, 0.f);
          *reinterpret_cast<float4*>(sWt + tc::swz_offset(kM, slot, w * kRowsPerWarp + 4)) =
              make_float4(0.f, 0.f, 0.f, 0.f);
        }
        bar_rows();  // dense g complete (row 63 holds the chunk totals)
        for_entries(cur, lane, K, nrows_w, [&](int r, int slot, float, float wv) {
          const int t = w * kRowsPerWarp + r;
          *reinterpret_cast<float*>(sWt + tc::swz_offset(kM, slot, t)) =
              tc::to_tf32(wv * expf(dg[(kC - 1) * kM + slot] - dg[t * kM + slot]));
        });
        const int nrows = ck.nrows;
        const unsigned char* rb = p.rec + ((int64_t)ck.pair * T + ck.c0) * RB;
        for (int e = tid; e < kC * kC; e += kRThreads) {
          const int t = e / kC, s = e % kC;
          float acc = 0.f;
          if (s <= t && t < nrows) {
            const int64_t rowt = ((int64_t)ck.b * T + ck.c0 + t) * H + ck.h;
            const unsigned char* rs = rb + s * RB;
            for (int j = 0; j < K; ++j) {
              const int i = rs[j];
              const float wj = reinterpret_cast<const float*>(rs + 5 * KP)[j];
              acc = fmaf(bf16_at(p.q + rowt * kM + i) * wj, expf(dg[t * kM + i] - dg[s * kM + i]), acc);
            }
          }
          *reinterpret_cast<float*>(sA + tc::swz_offset(kC, t, s)) = tc::to_tf32(acc);
        }
        tc::fence_async_smem();
        mbar_arrive(&bar_rdy);
      }
      // ---- the next chunk's q and records start loading (they land during the V^T conversion
      // and the next chunk's table)
      RowInputs<KP> nxt;
      {
        Walker nx = wk;
        nx.next(p, items);
        if (nx.valid(items)) load_rows<false, KP>(p, nx.get(p), w, lane, nxt);
      }
      // ---- V^T of this chunk: its v tile has landed and the chunk before has finished A.V
      if (n > 0) wait_or_abort(&bar_o, (n - 1) & 1, abort_flag);
      wait_or_abort(&bar_tma[n & 1], (n >> 1) & 1, abort_flag);
      {
        const uint16_t* raw = reinterpret_cast<const uint16_t*>(sRawV + (n & 1) * (kC * kDV * 2));
        const int dv = tid & (kDV - 1), s_beg = (tid >> 7) * (kC / 2);
#pragma unroll 4
        for (int s4 = s_beg; s4 < s_beg + kC / 2; s4 += 4) {
          const float4 f4 = make_float4(__uint_as_float((uint32_t)raw[(s4 + 0) * kDV + dv] << 16),
                                        __uint_as_float((uint32_t)raw[(s4 + 1) * kDV + dv] << 16),
                                        __uint_as_float((uint32_t)raw[(s4 + 2) * kDV + dv] << 16),
                                        __uint_as_float((uint32_t)raw[(s4 + 3) * kDV + dv] << 16));
          *reinterpret_cast<float4*>(sVt + tc::swz_offset(kDV, dv, s4)) = f4;
        }
        tc::fence_async_smem();
        mbar_arrive(&bar_vt);
      }
      cur = nxt;
    }
  } else if (warp == kIssuerWarp) {
    // =========================================================================== MMA issuer
    // The whole warp runs the issuer's loop, so that its descriptors and addresses are
    // warp-uniform values; lane 0 alone issues the copies, the MMAs and their commits.
    const bool leader = lane == 0;
    {
      uint32_t n = 0, n_tma = 0;
      auto load_v = [&](const Walker& at, uint32_t j) {  // v tile of the walker's chunk, as chunk j
        if (!at.valid(items)) return;
        const Chunk c = at.get(p);
        if (leader) {
          tc::mbar_arrive_expect_tx(&bar_tma[j & 1], kC * kDV * 2);
          tc::tma_load_4d(sRawV + (j & 1) * (kC * kDV * 2), &maps.v, &bar_tma[j & 1], 0, c.h, c.c0, c.b);
        }
        ++n_tma;
      };
      {
        Walker nx = wk;
        load_v(nx, 0);
        nx.next(p, items);
        load_v(nx, 1);
      }
      // Descriptors are built once per tile; a K step only advances the start-address field (the
      // low 14 bits, in 16-byte units), so each MMA costs the issuing thread about one add. The
      // issuer shares its scheduler with three busy warps: fewer instructions per MMA is what
      // keeps the tensor core fed.
      const uint64_t dQ = tc::smem_desc(tc::smem_u32(sQ), 16, 1024), dW = tc::smem_desc(tc::smem_u32(sW), 16, 1024),
                     dWt = tc::smem_desc(tc::smem_u32(sWt), 16, 1024), dVt = tc::smem_desc(tc::smem_u32(sVt), 16, 1024),
                     dA = tc::smem_desc(tc::smem_u32(sA), 16, 1024);
      // start-address advance of K step j in a tile with R rows: column block j/4 (R*128 bytes),
      // 32 bytes (8 tf32) within the 128-byte row
      auto kstep = [](int R, int j) -> uint64_t { return (uint64_t)(((j >> 2) * (R * 128) + (j & 3) * 32) >> 4); };
      constexpr uint32_t kIdS = tc::idesc_tf32(64, kC, 0, 0), kIdO = tc::idesc_tf32(kDV, kC, 0, 0),
                         kIdC = tc::idesc_tf32(kDV, kM, 0, 0);
      auto mma_s = [&](uint64_t dQn) {  // S = Qh Wh^T
#pragma unroll
        for (int j = 0; j < kM / 8; ++j)
          if (leader) tc::mma_tf32_ss(tb + kColS, dQn + kstep(kC, j), dW + kstep(kC, j), kIdS, j > 0);
      };
      auto mma_read = [&](uint32_t ob, uint64_t dQn) {  // O^T = H^T Qh^T (state read from TMEM)
#pragma unroll
        for (int j = 0; j < kM / 8; ++j)
          if (leader) tc::mma_tf32_ts(tb + kColO + ob, tb + kColHr + 8 * j, dQn + kstep(kC, j), kIdO, j > 0);
      };
      auto mma_carry = [&](uint32_t col, bool acc) {  // H^T += V^T Wh, or U^T = V^T Wh
#pragma unroll
        for (int j = 0; j < kC / 8; ++j)
          if (leader) tc::mma_tf32_ss(tb + col, dVt + kstep(kM, j), dWt + kstep(kM, j), kIdC, (acc || j > 0) ? 1u : 0u);
      };
      auto mma_av = [&](uint32_t ob) {  // O^T += V^T A^T
#pragma unroll
        for (int j = 0; j < kC / 8; ++j)
          if (leader) tc::mma_tf32_ss(tb + kColO + ob, dVt + kstep(kDV, j), dA + kstep(kC, j), kIdO, 1);
      };
      bool prev_exact = false;
      for (; wk.valid(items) && !*abort_flag; ++n, wk.next(p, items)) {
        const uint32_t ob = (n & 1) * kC;  // O buffer of this chunk
        wait_or_abort(&bar_rdy, n & 1, abort_flag);
        const bool fast = sFast[n & 1] != 0;
        tc::tmem_fence_after();
        if (fast && prev_exact) {  // S overwrites the columns of the previous chunk's U
          wait_or_abort(&bar_h, n & 1, abort_flag);
          tc::tmem_fence_after();
        }
        const uint64_t dQn = dQ + (uint64_t)(((n & 1) * 32768) >> 4);  // this chunk's Qh buffer
        if (fast) mma_s(dQn);
        if (leader) tc::mma_commit(&bar_s);  // every main-pass chunk: tells the epilogue the chunk is ready
        wait_or_abort(&bar_h, n & 1, abort_flag);  // state ready
        if (n >= 2) wait_or_abort(&bar_of[n & 1], ((n - 2) >> 1) & 1, abort_flag);  // O buffer free
        tc::tmem_fence_after();
        mma_read(ob, dQn);  // needs no V^T: the conversion overlaps it
        wait_or_abort(&bar_vt, n & 1, abort_flag);  // V^T written
        tc::tmem_fence_after();
        {
          // the raw v buffer of this chunk is free again: load the chunk two ahead into it
          Walker nx = wk;
          nx.next(p, items);
          nx.next(p, items);
          load_v(nx, n + 2);
        }
        mma_carry(fast ? kColH : kColU, fast);
        if (leader) tc::mma_commit(&bar_t);
        wait_or_abort(&bar_a, n & 1, abort_flag);
        tc::tmem_fence_after();
        mma_av(ob);
        if (leader) tc::mma_commit(&bar_o);
        prev_exact = !fast;
      }
      // no MMA or tile load may still be running when the CTA releases its memory (a barrier of
      // its own: another phase of bar_o could overtake the epilogue's last wait on it)
      if (leader) tc::mma_commit(&bar_fin);
      tc::mbar_wait(&bar_fin, 0);
      for (uint32_t j = n; j < n_tma; ++j) tc::mbar_wait(&bar_tma[j & 1], (j >> 1) & 1);
    }
    __syncwarp();  // the whole warp reaches the CTA barrier and the TMEM release together
  } else {
    // =========================================================================== epilogue
    const uint32_t sub_lane = (uint32_t)((warp & 3) * 32);
    const int dv = (int)sub_lane + lane;  // TMEM lane = value column

    // the state of chunk ck's item into TMEM (H0, a segment start state, or zeros)
    auto load_state = [&](const Chunk& ck) {
      const float* Hs = p.nseg > 1 ? p.ws_state + ((int64_t)ck.pair * p.nslot + ck.seg * p.sub) * kM * kDV
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
    };
    if (wk.valid(items)) {
      load_state(wk.get(p));
      tc::tmem_fence_before();
      mbar_arrive(&bar_h);  // phase 0: the first chunk's state
    }
    uint32_t n = 0;
    for (; wk.valid(items); ++n, wk.next(p, items)) {
      if (bar_epi_or(*abort_flag != 0)) break;  // the epilogue warps leave together (named barriers)
      const Chunk ck = wk.get(p);
      const float* Dn = sDc + (n & 1) * kM;
      wait_or_abort(&bar_s, n & 1, abort_flag);
      tc::tmem_fence_after();
      const bool fast = sFast[n & 1] != 0;
      if (fast) {
        // S -> A (rows t = 16*(warp%4) + lane for lane < 16, at TMEM lanes 32*(warp%4) + lane)
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
      }
      tc::tmem_fence_before();
      mbar_arrive(&bar_a);  // every main-pass chunk (an exact chunk's A comes from the row workers)
      // ---- after the carry: the state of the chunk end (fast: H = D H; exact: H = D H + U), the
      // item's state out at its end, the next item's state in at its start
      wait_or_abort(&bar_t, n & 1, abort_flag);
      tc::tmem_fence_after();
      Walker nx = wk;
      nx.next(p, items);
      float* dst = nullptr;
      if (ck.last && ck.seg == p.nseg - 1 && p.HT) dst = p.HT + (int64_t)ck.pair * kM * kDV;
      // the chunk-end state of 32 slots (in hv) is written out at the item's end, else back to
      // TMEM with its tf32-rounded copy
      auto put_state = [&](float (&hv)[32], int cg) {
        if (ck.last) {
          if (dst) {
#pragma unroll
            for (int j = 0; j < 32; ++j) dst[(cg + j) * kDV + dv] = hv[j];
          }
        } else {
          tc::tmem_st32(tc::tmem_addr(tb, sub_lane, kColH + cg), hv);
#pragma unroll
          for (int j = 0; j < 32; ++j) hv[j] = tc::to_tf32(hv[j]);
          tc::tmem_st32(tc::tmem_addr(tb, sub_lane, kColHr + cg), hv);
        }
      };
      if (fast) {
        // H = D H, two groups of 32 slots per TMEM wait
#pragma unroll 1
        for (int c = 0; c < kM; c += 64) {
          float hv[2][32];
          tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColH + c), hv[0]);
          tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColH + c + 32), hv[1]);
          tc::tmem_wait_ld();
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            scale_by(hv[g], Dn + c + 32 * g);  // slots not selected in the chunk: D = 1 exactly
            put_state(hv[g], c + 32 * g);
          }
        }
      } else {
        // exact chunk: H = D H + U
#pragma unroll 1
        for (int c = 0; c < kM; c += 32) {
          float hv[32], uv[32];
          tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColH + c), hv);
          tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColU + c), uv);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            const float4 d4 = *reinterpret_cast<const float4*>(Dn + c + j);
            hv[j] = fmaf(d4.x, hv[j], uv[j]);
            hv[j + 1] = fmaf(d4.y, hv[j + 1], uv[j + 1]);
            hv[j + 2] = fmaf(d4.z, hv[j + 2], uv[j + 2]);
            hv[j + 3] = fmaf(d4.w, hv[j + 3], uv[j + 3]);
          }
          put_state(hv, c);
        }
      }
      tc::tmem_wait_st();
      if (ck.last && nx.valid(items)) load_state(nx.get(p));
      tc::tmem_fence_before();
      mbar_arrive(&bar_h);  // phase n+1: the state of the next chunk
      // ---- every MMA of this chunk is done: its output
      wait_or_abort(&bar_o, n & 1, abort_flag);
      tc::tmem_fence_after();
      float ov[2][32];
      tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColO + (n & 1) * kC), ov[0]);
      tc::tmem_ld32(tc::tmem_addr(tb, sub_lane, kColO + (n & 1) * kC + 32), ov[1]);
      tc::tmem_wait_ld();
      // each half (32 tokens x 128 columns) is staged in the A tile's memory, free after A.V,
      // and written out by one bulk tensor store (tokens past T are clipped by the map)
      float* stg = reinterpret_cast<float*>(sA);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        if (hf == 1) {
          if (tid == kEpiThread0) tc::bulk_wait_read_all();
          bar_epi();
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) stg[j * kDV + dv] = ov[hf][j];
        tc::fence_async_smem();
        bar_epi();
        if (tid == kEpiThread0) {
          tc::tma_store_4d(&maps.o, stg, 0, ck.h, ck.c0 + 32 * hf, ck.b);
          tc::bulk_commit_group();
        }
      }
      if (tid == kEpiThread0) tc::bulk_wait_read_all();
      bar_epi();
      tc::tmem_fence_before();
      mbar_arrive(&bar_of[n & 1]);  // the O buffer and the staging memory are free
    }
    if (tid == kEpiThread0) tc::bulk_wait_all();  // output stores complete before the CTA ends
  }

  tc::tmem_fence_before();
  __syncthreads();
  tc::tmem_fence_after();
  if (warp == kIssuerWarp) tc::tmem_dealloc(tb, kTmemCols);
}

// ---------------------------------------------------------------------------------------------
// Segment summaries (segmented runs). For every segment of a (b,h) stream but the last, the
// state the recurrence reaches at the segment end from a zero start, and the product of the
// segment's decays:
//   D[i] = e^{Lam_i},  Lam_i = sum of lam_{t,i} over the segment's tokens
//   U    = sum_t Wr_t^T v_t,  Wr_{t,i} = w_{t,i} e^{sum of lam_{s,i} over the segment's tokens s > t}
// Referenced to the segment end, every exponent is <= 0: no division, no fast/exact split, and no
// decay of an accumulator between chunks, so U is a single accumulation of V^T Wr over the
// segment (one TMEM accumulator). The chunks are visited from the
// segment's last to its first, so the exponent of a token is the running sum of the lam of the
// tokens after it.
//
// The products run on bf16 operands (kind::f16): v as stored (its TMA tile, used MN-major), and Wr
// split into a bf16 high part and a bf16 low part (about 16 significant bits together). One MMA of
// N = 256 per K step takes both parts as the two halves of its B operand, so v is read once: U^T
// accumulates in fp32 as a high-part sum (TMEM columns 0..127) and a low-part sum (128..255),
// added when U is read out.
//
// Warp roles (two CTAs per SM, each on one segment at a time, 9 warps):
//   warps 0-7  row workers; warp w owns tokens 8w..8w+7 of the chunk, lane l slots 4l..4l+3 of
//              the lam table. Per chunk: scatter the rows' lam into the table, walk the rows from
//              the last to the first (exclusive in-warp suffix sums in place), exchange the warp
//              totals, write Wr (high and low tiles) at the selected entries; at the segment's end
//              read U out of TMEM and write U and D.
//   warp 8     MMA issuer (lane 0 issues): the v tile loads (one chunk ahead) and the 4 MMAs of
//              each chunk, U^T += V^T [Wr_high | Wr_low] (M = value columns, N = 2 x 128 slots,
//              K = 16 tokens per step).
// One Wr tile pair: the row workers build a chunk's table and exponents while the MMAs of the
// chunk before run, and write its Wr once they are done.
constexpr int kSumThreads = (kRWarps + 1) * 32;
constexpr int kSumOffV = 0;                          // v tiles [2][2 halves][64 t][64 dv] bf16, 128B swizzled
constexpr int kSumOffWb = kSumOffV + 2 * 16384;      // Wr high, low [2][64 t][128 slot] bf16, MN-major
constexpr int kSumOffTab = kSumOffWb + 32768;        // lam table [64 t][128 slot], then exponents
constexpr int kSumOffTot = kSumOffTab + 32768;       // per-warp lam sums [2][8][128]
constexpr int kSumOffSuf = kSumOffTot + 2 * kRWarps * kM * 4;  // per-warp exponent offsets [8][128]
constexpr int kSumOffLam = kSumOffSuf + kRWarps * kM * 4;       // Lam of the piece past this chunk [128]
constexpr int kSumSmemBytes = kSumOffLam + kM * 4 + 1024;
constexpr int kSumCtasPerSm = 2;
constexpr int kSumTmemCols = 256;
static_assert(kSumCtasPerSm * (kSumSmemBytes + 1024) <= 233472, "two summary CTAs per SM");

// The bf16 high and low tiles of Wr ([64 t][128 slot] each, MN-major, 16 KB apart): row t, slot i.
RSM_DEV void put_wr_bf16(unsigned char* sWb, int t, int i, float x) {
  uint16_t hi, lo;
  tc::split_bf16(x, hi, lo);
  const uint32_t off = tc::swz16_offset(kC, t, i);
  *reinterpret_cast<uint16_t*>(sWb + off) = hi;
  *reinterpret_cast<uint16_t*>(sWb + 16384 + off) = lo;
}

// The summary kernel visits item (pair, piece) = blockIdx.x + j*gridDim.x, piece < (nseg - 1) * sub
// (piece q of segment j is piece j*sub + q; a segment's pieces split its chunks evenly), and the
// item's chunks from the last to the first; first/last refer to that visiting order. A chunk's
// `seg` field holds the piece.
struct SumWalker {
  int item, pair, piece, b, h, t0, t1, nch, i;
  __device__ void set_item(const Params& p, int items) {
    if (item >= items) return;
    const int pairs = p.B * p.H;
    piece = item / pairs;
    pair = item - piece * pairs;
    b = pair / p.H;
    h = pair - b * p.H;
    const int seg = piece / p.sub, q = piece - seg * p.sub;
    const int c0 = seg * p.seg_chunks + q * p.piece_chunks;
    const int c1 = min((seg + 1) * p.seg_chunks, c0 + p.piece_chunks);
    t0 = c0 * kC;
    t1 = min(p.T, c1 * kC);
    nch = (t1 - t0 + kC - 1) / kC;
    i = 0;
  }
  __device__ void start(const Params& p, int items) {
    item = blockIdx.x;
    set_item(p, items);
  }
  __device__ bool valid(int items) const { return item < items; }
  __device__ Chunk get(const Params& p) const {
    Chunk c;
    c.pair = pair;
    c.seg = piece;
    c.b = b;
    c.h = h;
    c.c0 = t0 + (nch - 1 - i) * kC;
    c.nrows = min(kC, t1 - c.c0);
    c.first = i == 0;
    c.last = i == nch - 1;
    return c;
  }
  __device__ void next(const Params& p, int items) {
    if (++i >= nch) {
      item += gridDim.x;
      set_item(p, items);
    }
  }
};

template <int KP>
__global__ void __launch_bounds__(kSumThreads, kSumCtasPerSm) segment_summary_kernel(const __grid_constant__ Maps maps,
                                                                                     const Params p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* sV = sm + kSumOffV;
  unsigned char* sWb = sm + kSumOffWb;  // [high | low]
  float* sTab = reinterpret_cast<float*>(sm + kSumOffTab);
  float* sTot = reinterpret_cast<float*>(sm + kSumOffTot);
  float* sSuf = reinterpret_cast<float*>(sm + kSumOffSuf);
  float* sLam = reinterpret_cast<float*>(sm + kSumOffLam);

  // mbarriers (phase k of a barrier = its k-th completion)
  __shared__ __align__(8) uint64_t bar_rdy,  // Wr of chunk n written                  (row threads)
      bar_tma[2],                             // v tile of chunk n landed, buffer n&1   (TMA)
      bar_mma,                                // MMAs of chunk n done                   (MMA commit)
      bar_out,                                // U of an item read out of TMEM          (row threads)
      bar_fin;                                // issuer only: every MMA issued is done  (MMA commit)
  __shared__ uint32_t s_tbase;
  __shared__ int s_abort;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int K = p.K;
  const int items = p.B * p.H * (p.nslot - 1);

  if (warp == kIssuerWarp) tc::tmem_alloc(&s_tbase, kSumTmemCols);
  if (tid == 0) {
    tc::mbar_init(&bar_rdy, kRThreads);
    tc::mbar_init(&bar_tma[0], 1);
    tc::mbar_init(&bar_tma[1], 1);
    tc::mbar_init(&bar_mma, 1);
    tc::mbar_init(&bar_out, kRThreads);
    tc::mbar_init(&bar_fin, 1);
    tc::fence_mbar_init();
    s_abort = 0;
  }
  if (warp == kIssuerWarp && lane == 0) tc::tma_prefetch_desc(&maps.vsw);
  tc::tmem_fence_before();
  __syncthreads();
  tc::tmem_fence_after();
  const uint32_t tb = s_tbase;
  volatile int* abort_flag = &s_abort;

  SumWalker wk;
  wk.start(p, items);

  if (warp < kRWarps) {
    // =========================================================================== row workers
    const int w = warp;
    float* tab = sTab + w * kRowsPerWarp * kM;  // this warp's rows of the table
    // The table rows and the warp's token rows of the Wr tiles start at zero; afterwards each
    // entry's owner clears what it wrote (sparse), so no chunk fills them densely.
    uint32_t es1[RowInputs<KP>::kGroups];  // entry slots of the chunk before
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i)
      reinterpret_cast<float4*>(tab)[lane + 32 * i] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const uint32_t off = tc::swz16_offset(kC, w * kRowsPerWarp + r, lane * 4);
      *reinterpret_cast<uint2*>(sWb + off) = make_uint2(0u, 0u);
      *reinterpret_cast<uint2*>(sWb + 16384 + off) = make_uint2(0u, 0u);
    }
#pragma unroll
    for (int g = 0; g < RowInputs<KP>::kGroups; ++g) es1[g] = 0u;
    __syncwarp();
    RowInputs<KP> cur;
    if (wk.valid(items)) load_rows<true, KP>(p, wk.get(p), w, lane, cur);
    for (uint32_t n = 0; wk.valid(items); ++n, wk.next(p, items)) {
      const Chunk ck = wk.get(p);
      const int buf = n & 1;
      const int nrows_w = ck.nrows - w * kRowsPerWarp;
      // the next chunk's records start loading (they have this whole chunk to arrive)
      RowInputs<KP> nxt;
      {
        SumWalker nx = wk;
        nx.next(p, items);
        if (nx.valid(items)) load_rows<true, KP>(p, nx.get(p), w, lane, nxt);
      }
      // ---- the warp's rows of the table (all zero): lam at the selected entries
      for_entries(cur, lane, K, nrows_w, [&](int r, int slot, float lam, float) { tab[r * kM + slot] = lam; });
      __syncwarp();
      // ---- walk the rows from the last: each nonzero entry becomes the sum of lam below it in the
      // warp, zeros stay (an entry with lam = 0 has w = k (1 - e^0) = 0, so its exponent is not used)
      float run[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int r = kRowsPerWarp - 1; r >= 0; --r) {
        float4* row = reinterpret_cast<float4*>(tab + r * kM) + lane;
        const float4 x = *row;
        if (x.x != 0.f || x.y != 0.f || x.z != 0.f || x.w != 0.f)  // all-zero groups stay as they are
          *row = make_float4(x.x != 0.f ? run[0] : 0.f, x.y != 0.f ? run[1] : 0.f, x.z != 0.f ? run[2] : 0.f,
                             x.w != 0.f ? run[3] : 0.f);
        run[0] += x.x; run[1] += x.y; run[2] += x.z; run[3] += x.w;
      }
      reinterpret_cast<float4*>(sTot + (buf * kRWarps + w) * kM)[lane] = make_float4(run[0], run[1], run[2], run[3]);
      if (bar_rows_or(*abort_flag != 0)) break;  // every row worker takes the same decision
      // ---- exponent offsets, one slot per thread (row-worker thread j < M owns slot j): for every
      // warp, the lam of the later warps' rows and of the piece's later chunks; then Lam past this
      // chunk, and at the piece's end D = e^Lam
      {
        const int j = w * 32 + lane;
        if (j < kM) {
          float acc = ck.first ? 0.f : sLam[j];
#pragma unroll
          for (int w2 = kRWarps - 1; w2 >= 0; --w2) {
            sSuf[w2 * kM + j] = acc;
            acc += sTot[(buf * kRWarps + w2) * kM + j];
          }
          sLam[j] = acc;
          if (ck.last) p.ws_D[((int64_t)ck.pair * p.nslot + ck.seg + 1) * kM + j] = expf(acc);
        }
      }
      bar_rows();
      // ---- the Wr tiles are free once the MMAs of the chunk before are done; that chunk's entries
      // leave them (rows past a chunk's end hold slot 0, which clears a zero)
      if (n >= 1) wait_or_abort(&bar_mma, (n - 1) & 1, abort_flag);
#pragma unroll
      for (int g = 0; g < RowInputs<KP>::kGroups; ++g) {
        int r, j0;
        entry_pos(lane, g, KP, r, j0);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (r < kRowsPerWarp && j0 + e < K) {
            const uint32_t off = tc::swz16_offset(kC, w * kRowsPerWarp + r, (int)((es1[g] >> (8 * e)) & 255u));
            *reinterpret_cast<uint16_t*>(sWb + off) = 0;
            *reinterpret_cast<uint16_t*>(sWb + 16384 + off) = 0;
          }
        }
        es1[g] = cur.es[g];
      }
      __syncwarp();
      // ---- each entry's owner: Wr = w e^{exponent} (exponent <= 0); its table entry back to zero
      for_entries(cur, lane, K, nrows_w, [&](int r, int slot, float, float wv) {
        const float x = tab[r * kM + slot] + sSuf[w * kM + slot];
        tab[r * kM + slot] = 0.f;
        put_wr_bf16(sWb, w * kRowsPerWarp + r, slot, wv * expf(x));
      });
      tc::fence_async_smem();
      mbar_arrive(&bar_rdy);
      // ---- the item's last chunk: U out of TMEM (warp w: lanes 32(w%4).., slot columns
      // 64(w/4)..), D = e^Lam
      if (ck.last) {
        wait_or_abort(&bar_mma, n & 1, abort_flag);
        tc::tmem_fence_after();
        const int64_t slot_base = ((int64_t)ck.pair * p.nslot + ck.seg + 1);
        float* dst = p.ws_state + slot_base * kM * kDV;
        const int dv = (w & 3) * 32 + lane;
        const int c0 = (w >> 2) * 64;
#pragma unroll 1
        for (int g = 0; g < 8; ++g) {
          float u[8], ul[8];  // high-part and low-part sums of 8 slots
          tc::tmem_ld8(tc::tmem_addr(tb, (uint32_t)((w & 3) * 32), (uint32_t)(c0 + 8 * g)), u);
          tc::tmem_ld8(tc::tmem_addr(tb, (uint32_t)((w & 3) * 32), (uint32_t)(kM + c0 + 8 * g)), ul);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 8; ++j) dst[(int64_t)(c0 + 8 * g + j) * kDV + dv] = u[j] + ul[j];
        }
        tc::tmem_fence_before();
        mbar_arrive(&bar_out);
      }
      cur = nxt;
    }
  } else {
    // =========================================================================== MMA issuer
    // The whole warp runs the issuer's loop, so that its descriptors and addresses are
    // warp-uniform values; lane 0 alone issues the copies, the MMAs and their commits.
    const bool leader = lane == 0;
    {
      uint32_t n = 0, n_tma = 0, n_items = 0;
      // v tile of the walker's chunk, as chunk j, into buffer j&1: two 64-column halves, each
      // [64 t][64 dv] bf16 with 128-byte swizzle (the MN-major operand layout); rows past the
      // sequence end are zero
      auto load_v = [&](const SumWalker& at, uint32_t j) {
        if (!at.valid(items)) return;
        const Chunk c = at.get(p);
        if (leader) {
          tc::mbar_arrive_expect_tx(&bar_tma[j & 1], kC * kDV * 2);
          tc::tma_load_4d(sV + (j & 1) * 16384, &maps.vsw, &bar_tma[j & 1], 0, c.h, c.c0, c.b);
          tc::tma_load_4d(sV + (j & 1) * 16384 + 8192, &maps.vsw, &bar_tma[j & 1], 64, c.h, c.c0, c.b);
        }
        ++n_tma;
      };
      load_v(wk, 0);
      // v: 64-column halves 8 KB apart, groups of 8 token rows 1 KB apart; [Wr_high | Wr_low]: four
      // 64-slot blocks 8 KB apart (N = 256), the same row groups; a K step of 16 tokens advances both
      // by 2 KB
      const uint64_t dV0 = tc::smem_desc(tc::smem_u32(sV), 8192, 1024), dWb = tc::smem_desc(tc::smem_u32(sWb), 8192, 1024);
      constexpr uint32_t kIdC = tc::idesc_bf16(kDV, 2 * kM, 1, 1);
      for (; wk.valid(items) && !*abort_flag; ++n, wk.next(p, items)) {
        const Chunk ck = wk.get(p);
        {
          // buffer (n+1)&1 is free once the MMAs of chunk n-1 are done: the next chunk's v into it
          if (n >= 1) wait_or_abort(&bar_mma, (n - 1) & 1, abort_flag);
          SumWalker nx = wk;
          nx.next(p, items);
          load_v(nx, n + 1);
        }
        wait_or_abort(&bar_rdy, n & 1, abort_flag);                   // Wr written
        wait_or_abort(&bar_tma[n & 1], (n >> 1) & 1, abort_flag);     // v landed
        // the accumulator of the item before has been read out
        if (ck.first && n_items > 0) wait_or_abort(&bar_out, (n_items - 1) & 1, abort_flag);
        tc::tmem_fence_after();
        const uint64_t dVn = dV0 + (uint64_t)(((n & 1) * 16384) >> 4);
#pragma unroll
        for (int j = 0; j < kC / 16; ++j)
          if (leader)
            tc::mma_bf16_ss(tb, dVn + (uint64_t)((j * 2048) >> 4), dWb + (uint64_t)((j * 2048) >> 4), kIdC,
                            (ck.first && j == 0) ? 0u : 1u);
        if (leader) tc::mma_commit(&bar_mma);
        if (ck.last) ++n_items;
      }
      // nothing may still be running when the CTA releases its memory
      if (leader) tc::mma_commit(&bar_fin);
      tc::mbar_wait(&bar_fin, 0);
      for (uint32_t j = n; j < n_tma; ++j) tc::mbar_wait(&bar_tma[j & 1], (j >> 1) & 1);
    }
    __syncwarp();
  }

  tc::tmem_fence_before();
  __syncthreads();
  tc::tmem_fence_after();
  if (warp == kIssuerWarp) tc::tmem_dealloc(tb, kSumTmemCols);
}

// Combines the piece summaries of each (b,h) into states:
// state[0] = H0 (or 0); state[k] = D_{k-1} * state[k-1] + U_{k-1} (the summary of piece k-1 is
// stored in slot k and is replaced in place), so slot j*sub ends up holding the start state of
// segment j. A slot with D = 1 and U = 0 (not selected in the piece) keeps its bits.
__global__ void __launch_bounds__(256) segment_scan_kernel(const Params p) {
  const int pair = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;  // element (slot, column)
  if (e >= kM * kDV) return;
  const int i = e / kDV;
  float* st = p.ws_state + (int64_t)pair * p.nslot * kM * kDV;
  const float* D = p.ws_D + (int64_t)pair * p.nslot * kM;
  float hcur = p.H0 ? p.H0[(int64_t)pair * kM * kDV + e] : 0.f;
  st[e] = hcur;
  // the summaries are loaded 8 at a time ahead of the dependent chain (one memory round trip per 8)
  constexpr int kBatch = 8;
  for (int j0 = 1; j0 < p.nslot; j0 += kBatch) {
    float d[kBatch], u[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      d[k] = 1.f;
      u[k] = 0.f;
      if (j0 + k < p.nslot) {
        d[k] = D[(j0 + k) * kM + i];
        u[k] = st[(int64_t)(j0 + k) * kM * kDV + e];
      }
    }
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      if (j0 + k < p.nslot) {
        if (d[k] != 1.f || u[k] != 0.f) hcur = fmaf(d[k], hcur, u[k]);
        st[(int64_t)(j0 + k) * kM * kDV + e] = hcur;
      }
    }
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

// 4-D map over [B, T, H, C] (C innermost) with a box of one (b, h) and `box_t` tokens.
bool make_map(CUtensorMap* m, const void* base, int B, int T, int H, int C, bool fp32, int box_t, int box_c = 0,
              bool swizzle128 = false) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t es = fp32 ? 4 : 2;
  cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)C * es, (cuuint64_t)H * C * es, (cuuint64_t)T * H * C * es};
  cuuint32_t box[4] = {(cuuint32_t)(box_c > 0 ? box_c : C), 1, (cuuint32_t)box_t, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, fp32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() { return device_sm_count(); }

struct Plan {
  int nseg, seg_chunks;
  int sub, piece_chunks, nslot;
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
  // the summary pass runs two CTAs per SM: each segment it summarises is split into that many
  // pieces (of at least 4 chunks), combined by the scan
  int sub = seg_chunks >= 4 * kSumCtasPerSm ? kSumCtasPerSm : 1;
  const int piece_chunks = (seg_chunks + sub - 1) / sub;
  sub = (seg_chunks + piece_chunks - 1) / piece_chunks;
  return {nseg, seg_chunks, sub, piece_chunks, 1 + (nseg - 1) * sub};
}

size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace: routing records, then (segmented runs) the segment states and decays.
struct WsLayout {
  size_t rec, state, D, total;
};
WsLayout ws_layout(const rsm_forward_args& a, const Plan& pl) {
  WsLayout l;
  const size_t rows = (size_t)a.B * a.T * a.H;
  l.rec = 0;
  size_t off = up256(rows * (size_t)route_record_bytes(a.K));
  l.state = l.D = off;
  if (pl.nseg > 1) {
    const size_t per = (size_t)a.B * a.H * pl.nslot;
    l.state = off;
    off += up256(per * kM * kDV * 4);
    l.D = off;
    off += up256(per * kM * 4);
  }
  l.total = off;
  return l;
}

// Summary pass + segment scan (segmented runs only), then the main pass.
template <int KP>
cudaError_t launch_passes(const Maps& maps, const Params& p, const Plan& pl, int64_t pairs, int sms,
                          cudaStream_t stream) {
  cudaError_t e =
      set_smem_limit<prefill_tc_kernel<KP>>(kSmemBytes);
  if (e != cudaSuccess) return e;
  if (pl.nseg > 1) {
    e = set_smem_limit<segment_summary_kernel<KP>>(kSumSmemBytes);
    if (e != cudaSuccess) return e;
    const int items = (int)(pairs * (pl.nslot - 1));
    segment_summary_kernel<KP><<<std::min(items, kSumCtasPerSm * sms), kSumThreads, kSumSmemBytes, stream>>>(maps, p);
    e = cudaGetLastError();
    if (e == cudaSuccess) e = profile_mark(stream);
    if (e != cudaSuccess) return e;
    dim3 g((kM * kDV + 255) / 256, (unsigned)pairs);
    segment_scan_kernel<<<g, 256, 0, stream>>>(p);
    e = cudaGetLastError();
    if (e == cudaSuccess) e = profile_mark(stream);
    if (e != cudaSuccess) return e;
  }
  const int64_t items = pairs * pl.nseg;
  prefill_tc_kernel<KP><<<(unsigned)std::min<int64_t>(items, sms), kThreads, kSmemBytes, stream>>>(maps, p);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = profile_mark(stream);
  return e;
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
  return (plan_for(a, sm_count()).nseg > 1 ? 4 : 2) + (a.slot_counts ? 1 : 0);
}

cudaError_t launch_prefill_tc(const rsm_forward_args& a, cudaStream_t stream) {
  const int sms = sm_count();
  const Plan pl = plan_for(a, sms);
  const WsLayout wl = ws_layout(a, pl);
  char* ws = static_cast<char*>(a.workspace);
  unsigned char* rec = reinterpret_cast<unsigned char*>(ws + wl.rec);
  cudaError_t e = launch_route_records(a.logits, a.f, a.k, a.B, a.T, a.H, a.M, a.K, a.decay == RSM_DECAY_SLOT,
                                       (int)a.router, (a.flags & RSM_FLAG_VALIDATE) != 0, rec, a.idx_out,
                                       a.score_out, a.slot_counts, stream);
  if (e == cudaSuccess) e = profile_mark(stream);
  if (e == cudaSuccess && a.slot_counts) {
    e = launch_record_counts(rec, (int64_t)a.B * a.H, a.T, a.K, a.slot_counts, stream);
    if (e == cudaSuccess) e = profile_mark(stream);
  }
  if (e != cudaSuccess) return e;
  Maps maps;
  if (!make_map(&maps.v, a.v, a.B, a.T, a.H, kDV, false, kC)) return cudaErrorInvalidValue;
  if (!make_map(&maps.vsw, a.v, a.B, a.T, a.H, kDV, false, kC, 64, true)) return cudaErrorInvalidValue;
  if (!make_map(&maps.o, a.o, a.B, a.T, a.H, kDV, true, kC / 2)) return cudaErrorInvalidValue;
  Params p;
  p.B = a.B; p.T = a.T; p.H = a.H; p.K = a.K;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.rec = rec;
  p.rec_bytes = route_record_bytes(a.K);
  p.H0 = a.H0;
  p.o = a.o; p.HT = a.HT;
  p.nseg = pl.nseg; p.seg_chunks = pl.seg_chunks;
  p.sub = pl.sub; p.piece_chunks = pl.piece_chunks; p.nslot = pl.nslot;
  p.ws_state = nullptr; p.ws_D = nullptr;
  if (pl.nseg > 1) {
    p.ws_state = reinterpret_cast<float*>(ws + wl.state);
    p.ws_D = reinterpret_cast<float*>(ws + wl.D);
  }
  const int64_t pairs = (int64_t)a.B * a.H;
  return a.K <= 16 ? launch_passes<16>(maps, p, pl, pairs, sms, stream) : launch_passes<32>(maps, p, pl, pairs, sms, stream);
}

}  // namespace rsm
