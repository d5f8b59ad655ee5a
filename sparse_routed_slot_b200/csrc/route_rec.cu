// route_rec.cu -- routing records for the tensor-core prefill (M = 128 slots, K <= 32).
//
// The chunk kernels of the tensor-core prefill read compact routing records instead of the
// logits (Raven README "How Raven Works": route_scores = TopK(sigmoid(r_proj(x))); "Model
// Structure": a = exp(score * f)):
//
//   record (route_record_bytes(K) = 9 * KP bytes, KP = 16 for K <= 16 else 32; rows in
//   [B, H, T] order, so the records of one (b,h) stream are contiguous along time):
//     uint8  slot[KP]   the selected slots (entries >= K: 0)
//     float  lam[KP]    lam = s * f, the log of the slot's decay (<= 0), s the router score
//                       (sigmoid or softmax of the logit, optionally normalised over the K)
//     float  w[KP]      w = k[slot] * (1 - e^lam), the slot's write weight
//   Entries are in rank order (logit descending, slot ascending) except that logits agreeing in
//   their upper 25 key bits may be listed in slot order; when no ranked output is requested and
//   K equals KP, they come in no particular order. The set is always exact.
//
// Two threads per row. A warp takes 16 consecutive rows and copies them into its shared-memory
// buffer with asynchronous 16-byte copies (one 512-byte row per warp instruction). One buffer per
// warp keeps a CTA at 34 KB, so six CTAs (24 warps) share an SM and hide each other's copy
// latency, which measured faster than double-buffering at half the warps. Each thread of the
// pair ranks half of the row's slots; the two sorted halves are merged through shuffles.
// Selection (router scores are monotone in the
// logits, so TopK of the scores = TopK of the logits; -0 ties +0): each logit becomes a packed
// 32-bit key, its order-preserving bit pattern with the low 7 bits replaced by (127 - slot), which
// makes every key distinct and breaks ties to the lower slot. The top N (N = 16 or 32 >= K) keys
// come from sorting networks in registers: each group of N is sorted (odd-even merge sort) and
// merged into the running top N (the larger half of two sorted runs is bitonic; one half-cleaner
// cascade sorts it).
// Dropping the low 7 bits can only misorder logits whose upper 25 key bits agree; if the K-th and
// (K+1)-th keys share them, or ranked outputs are requested and two of the first K share them,
// the whole warp ranks that row exactly with the tournament of common.cuh instead.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rsm {

namespace {

constexpr int kRM = 128;              // slots on this path
constexpr int kRowFloats = kRM + 4;    // staged row stride (16-byte pad: conflict-free float4 reads)
constexpr int kWarps = 4;              // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerTask = 16;       // rows per warp task (two threads per row)
constexpr int kBufBytes = kRowsPerTask * kRowFloats * 4;  // one warp's staged rows
constexpr int kSmem = kWarps * kBufBytes;
constexpr uint32_t kCoarse = ~0x7Fu;   // key bits above the slot field

// The order key of common.cuh with -0 folded into +0 by an add (x + 0 is +0 for x = -0 and x
// otherwise), which runs on the FMA pipe and leaves two logic operations for the ALU.
RSM_DEV uint32_t packed_key(float x, int slot) {
  const uint32_t b = __float_as_uint(x + 0.0f);
  const uint32_t key = b ^ ((uint32_t)((int32_t)b >> 31) | 0x80000000u);
  return (key & kCoarse) | (uint32_t)(127 - slot);
}

// Batcher's odd-even merge sort of N keys, descending (every compare-exchange moves the larger key
// to the lower index): 63 compare-exchanges for 16 keys and 191 for 32, against 80 and 240 for a
// bitonic sorting network. The recursion runs at compile time on the index range LO..HI
// (inclusive), so every index is a constant and the keys stay in registers.
template <int LO, int HI, int R, int N>
RSM_DEV void oe_merge(uint32_t (&a)[N]) {  // merges the sorted halves; elements R apart
  constexpr int step = 2 * R;
  if constexpr (step < HI - LO) {
    oe_merge<LO, HI, step>(a);
    oe_merge<LO + R, HI, step>(a);
#pragma unroll
    for (int i = LO + R; i < HI - R; i += step) cas_desc(a[i], a[i + R]);
  } else {
    cas_desc(a[LO], a[LO + R]);
  }
}
template <int LO, int HI, int N>
RSM_DEV void oe_sort(uint32_t (&a)[N]) {
  if constexpr (HI - LO >= 1) {
    constexpr int mid = LO + (HI - LO) / 2;
    oe_sort<LO, mid>(a);
    oe_sort<mid + 1, HI>(a);
    oe_merge<LO, HI, 1>(a);
  }
}
template <int N>
RSM_DEV void sort_desc(uint32_t (&a)[N]) {
  oe_sort<0, N - 1>(a);
}

// top <- the N largest of top and g (both sorted descending); the largest dropped key is folded
// into `dropped`. Without SORT the N keys are left as a bitonic sequence (the right set, unordered).
template <int N, bool SORT = true>
RSM_DEV void merge_top(uint32_t (&top)[N], const uint32_t (&g)[N], uint32_t& dropped) {
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const uint32_t a = top[i], b = g[N - 1 - i];
    top[i] = max(a, b);
    dropped = max(dropped, min(a, b));
  }
  if constexpr (SORT) {
#pragma unroll
    for (int j = N >> 1; j > 0; j >>= 1) {
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int l = i ^ j;
        if (l > i) cas_desc(top[i], top[l]);
      }
    }
  }
}

RSM_DEV void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(smem)), "l"(gmem) : "memory");
}
RSM_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
RSM_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

struct Rows {
  const float* logits;
  const float* f;
  const uint16_t* k;  // bf16 bits
  int64_t B, T, H;
  int K, decay_slot, router;
  unsigned char* rec;
  int32_t* idx_out;
  float* score_out;
};

// lam and w of one selected slot of input row `ir`, from its router score s.
RSM_DEV void entry_values(const Rows& R, int64_t ir, int slot, float s, float fh, float& lam, float& w) {
  const float fv = R.decay_slot ? __ldg(R.f + ir * kRM + slot) : fh;
  lam = s * fv;
  const float kv = __uint_as_float((uint32_t)__ldg(R.k + ir * kRM + slot) << 16);
  w = kv * (-expm1f(lam));
}

template <int N, bool VALIDATE, bool VARIANT>
__global__ void __launch_bounds__(kThreads) route_rec_kernel(const Rows R) {
  constexpr int KP = N;  // record entries
  // VARIANT: a router other than plain sigmoid scores (the default compiles without that code)
  const int router = VARIANT ? R.router : (int)RSM_ROUTER_SIGMOID;
  extern __shared__ __align__(128) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rl = lane >> 1, half = lane & 1;  // row of the task, half of the row (slots 64*half..)
  const int K = R.K;
  const int64_t rows = R.B * R.H * R.T;
  const int64_t tasks = (rows + kRowsPerTask - 1) / kRowsPerTask;
  const int64_t stride = (int64_t)gridDim.x * kWarps;
  unsigned char* wbuf = smem + warp * kBufBytes;
  // input row index (in the [B, T, H] layout) of row p = 16*task + r of the [B, H, T] order:
  // one division per warp and task (lane 0), then a walk along the stream
  auto input_row = [&](int64_t task, int r) {
    int64_t b = 0, h = 0, t = 0;
    if (lane == 0) {
      const int64_t p0 = task * kRowsPerTask;
      const int64_t bh = p0 / R.T;
      t = p0 - bh * R.T;
      b = bh / R.H;
      h = bh - b * R.H;
    }
    b = __shfl_sync(kFull, b, 0);
    h = __shfl_sync(kFull, h, 0);
    t = __shfl_sync(kFull, t, 0) + r;
    while (t >= R.T) {  // past the end of the stream: the next (b,h)
      t -= R.T;
      if (++h == R.H) {
        h = 0;
        ++b;
      }
    }
    return (b * R.T + t) * R.H + h;
  };
  // the warp copies the 16 rows of task `task` into its buffer (16 bytes per lane per row)
  auto stage = [&](int64_t task) {
    if (task < tasks) {
      const int64_t ir0 = input_row(task, lane & 15);  // lane r (r < 16) knows row r's index
      for (int r = 0; r < kRowsPerTask; ++r) {
        const int64_t irr = __shfl_sync(kFull, ir0, r);
        if (task * kRowsPerTask + r < rows)
          cp_async16(wbuf + (r * kRowFloats + lane * 4) * 4, R.logits + irr * kRM + lane * 4);
      }
      // the k rows (gathered at the selected slots once the rows are ranked) start moving into L2:
      // lane 2r + e fetches the e-th 128-byte half of row r's 256 bytes
      {
        const int64_t irk = __shfl_sync(kFull, ir0, lane >> 1);
        if (task * kRowsPerTask + (lane >> 1) < rows)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(R.k + irk * kRM + (lane & 1) * (kRM / 2)));
      }
    }
    cp_async_commit();
  };
  const int64_t task0 = (int64_t)blockIdx.x * kWarps + warp;
  for (int64_t task = task0; task < tasks; task += stride) {
    stage(task);
    cp_async_wait_all();
    __syncwarp();
    const int64_t p = task * kRowsPerTask + rl;
    const int64_t ir = input_row(task, rl);
    const bool live = p < rows;  // both lanes of a pair agree
    const float* xr = reinterpret_cast<const float*>(wbuf) + rl * kRowFloats;
    const float fh = (R.decay_slot || !live) ? 0.f : __ldg(R.f + ir);

    // ---- top N packed keys of this thread's half of the row, then of the whole row
    uint32_t top[N], g[N], dropped = 0u;
    bool bad = false;
    auto keys = [&](int grp, uint32_t (&dst)[N]) {
#pragma unroll
      for (int i = 0; i < N / 4; ++i) {
        const int s0 = half * (kRM / 2) + grp * N + 4 * i;
        const float4 v = *reinterpret_cast<const float4*>(xr + s0);
        dst[4 * i] = packed_key(v.x, s0);
        dst[4 * i + 1] = packed_key(v.y, s0 + 1);
        dst[4 * i + 2] = packed_key(v.z, s0 + 2);
        dst[4 * i + 3] = packed_key(v.w, s0 + 3);
        if (VALIDATE) bad |= !finite_f32(v.x) || !finite_f32(v.y) || !finite_f32(v.z) || !finite_f32(v.w);
      }
    };
    keys(0, top);
    sort_desc<N>(top);
#pragma unroll 1
    for (int grp = 1; grp < kRM / 2 / N; ++grp) {
      keys(grp, g);
      sort_desc<N>(g);
      merge_top<N>(top, g, dropped);
    }
#pragma unroll
    for (int i = 0; i < N; ++i) g[i] = __shfl_xor_sync(kFull, top[i], 1);  // the partner's half
    // both lanes now hold the row's top N; sorted only where the order is used (ranked outputs, or
    // K < N, where the first K must be the K largest)
    const bool ranked = R.idx_out || R.score_out;
    const bool sorted = ranked || K < N;
    if (sorted) merge_top<N, true>(top, g, dropped);
    else merge_top<N, false>(top, g, dropped);  // lane 2r+1 holds lane 2r's keys in reverse
    dropped = max(dropped, __shfl_xor_sync(kFull, dropped, 1));
    if (VALIDATE && live) {
      if (R.decay_slot) {
        for (int s = half * (kRM / 2); s < (half + 1) * (kRM / 2); ++s) {
          const float fv = __ldg(R.f + ir * kRM + s);
          bad |= !finite_f32(fv) || fv > 0.f;
        }
      } else {
        bad |= !finite_f32(fh) || fh > 0.f;
      }
      if (bad) raise_status(RSM_ERR_NONFINITE);
    }

    // ---- is the coarse order enough? (the K-th and (K+1)-th keys; neighbours among the first K)
    uint32_t kth = 0xffffffffu, next = dropped;
    bool near_tie = false;
#pragma unroll
    for (int r = 0; r < N; ++r) {
      kth = min(kth, r < K ? top[r] : 0xffffffffu);
      next = max(next, r < K ? 0u : top[r]);
      if (r + 1 < N && r + 1 < K) near_tie |= ((top[r] ^ top[r + 1]) & kCoarse) == 0u;
    }
    const bool exact = ((next ^ kth) & kCoarse) == 0u || (ranked && near_tie);
    unsigned char* rp = R.rec + p * (int64_t)(9 * KP);
    int32_t* io = R.idx_out ? R.idx_out + ir * K : nullptr;
    float* so = R.score_out ? R.score_out + ir * K : nullptr;

    // softmax scores need the row's maximum and normalising sum (each lane of a pair: its half)
    float smax = 0.f, rsum = 1.f;
    if (router & RSM_ROUTER_SOFTMAX) {
      float mx = -3.402823466e38f;
#pragma unroll 4
      for (int i = 0; i < kRM / 2; ++i) mx = fmaxf(mx, xr[half * (kRM / 2) + i]);
      smax = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
      float z = 0.f;
#pragma unroll 4
      for (int i = 0; i < kRM / 2; ++i) z += expf(xr[half * (kRM / 2) + i] - smax);
      rsum = 1.0f / (z + __shfl_xor_sync(kFull, z, 1));
    }

    constexpr int KH = KP / 2;
    // the key of this lane's q-th entry: sorted, lane `half` takes rank positions half*KH + q;
    // unsorted, the partner's array is this lane's reversed, so each lane takes its own first half
    auto entry_key = [&](int q) { return (sorted && half) ? top[KH + q] : top[q]; };
    float rnorm = 1.f;
    if (router & 2) {  // normalised scores: 1 / (sum over the row's K selected slots)
      float t = 0.f;
#pragma unroll
      for (int q = 0; q < KH; ++q) {
        const float xq = xr[127 - (int)(entry_key(q) & 0x7Fu)];
        if (half * KH + q < K) t += (router & RSM_ROUTER_SOFTMAX) ? expf(xq - smax) * rsum : sigmoid_f32(xq);
      }
      rnorm = 1.0f / (t + __shfl_xor_sync(kFull, t, 1));
    }
    if (live && !exact) {
      // ---- entries in rank order from the sorted keys; each lane of the pair computes half
      uint32_t sw[KH / 4];
      float lam[KH], wv[KH];
#pragma unroll
      for (int i = 0; i < KH / 4; ++i) sw[i] = 0u;
#pragma unroll
      for (int q = 0; q < KH; ++q) {
        const int r = half * KH + q;
        lam[q] = 0.f;
        wv[q] = 0.f;
        if (r < K) {
          const int slot = 127 - (int)(entry_key(q) & 0x7Fu);
          sw[q / 4] |= (uint32_t)slot << (8 * (q % 4));
          const float xq = xr[slot];
          const float sc = rnorm * ((router & RSM_ROUTER_SOFTMAX) ? expf(xq - smax) * rsum : sigmoid_f32(xq));
          entry_values(R, ir, slot, sc, fh, lam[q], wv[q]);
          if (io) io[r] = slot;
          if (so) so[r] = sc;
        }
      }
#pragma unroll
      for (int i = 0; i < KH / 16; ++i)
        reinterpret_cast<uint4*>(rp + half * KH)[i] = make_uint4(sw[4 * i], sw[4 * i + 1], sw[4 * i + 2], sw[4 * i + 3]);
      if (KH % 16 != 0) {  // KH = 8: two words of slots
        reinterpret_cast<uint2*>(rp + half * KH)[0] = make_uint2(sw[0], sw[1]);
      }
#pragma unroll
      for (int i = 0; i < KH / 4; ++i) {
        reinterpret_cast<float4*>(rp + KP + 4 * half * KH)[i] =
            make_float4(lam[4 * i], lam[4 * i + 1], lam[4 * i + 2], lam[4 * i + 3]);
        reinterpret_cast<float4*>(rp + 5 * KP + 4 * half * KH)[i] =
            make_float4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
      }
    }
    // ---- rare rows (a near-tie at the cut, or ranked output with near-ties among the first K):
    // the whole warp ranks each of them exactly with the tournament (logit desc, slot asc)
    uint32_t pending = __ballot_sync(kFull, live && exact && half == 0);
    while (pending) {
      const int src = __ffs(pending) - 1;
      pending &= pending - 1u;
      const int r = src >> 1;
      const float* xw = reinterpret_cast<const float*>(wbuf) + r * kRowFloats;
      float x4[kRM / 32];
#pragma unroll
      for (int e = 0; e < kRM / 32; ++e) x4[e] = xw[lane * (kRM / 32) + e];
      const int64_t irw = __shfl_sync(kFull, ir, src);
      const int64_t pw = __shfl_sync(kFull, p, src);
      const float fhw = __shfl_sync(kFull, fh, src);
      unsigned char* rpw = R.rec + pw * (int64_t)(9 * KP);
      int32_t* iow = R.idx_out ? R.idx_out + irw * K : nullptr;
      float* sow = R.score_out ? R.score_out + irw * K : nullptr;
      int rank[4] = {0, 0, 0, 0};
      int* rank_p = rank;  // a rare path: local memory is fine here
      const uint32_t sel = warp_topk<kRM>(x4, K, lane, [&](int rk, int slot, int e) {
        rpw[rk] = (unsigned char)slot;
        if (iow) iow[rk] = slot;
        rank_p[e] = rk;
      });
      float scw[4];
      const float(&x4c)[4] = x4;  // (binding first sidesteps a front-end crash of this nvcc)
      warp_router_scores(x4c, sel, router, scw);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if ((sel >> e) & 1u) {
          float lm, wvv;
          entry_values(R, irw, lane * (kRM / 32) + e, scw[e], fhw, lm, wvv);
          reinterpret_cast<float*>(rpw + KP)[rank[e]] = lm;
          reinterpret_cast<float*>(rpw + 5 * KP)[rank[e]] = wvv;
          if (sow) sow[rank[e]] = scw[e];
        }
      }
      if (lane < KP - K) {  // padding entries
        rpw[K + lane] = 0;
        reinterpret_cast<float*>(rpw + KP)[K + lane] = 0.f;
        reinterpret_cast<float*>(rpw + 5 * KP)[K + lane] = 0.f;
      }
    }
    __syncwarp();  // every lane is done with the buffer before it is refilled
  }
  cp_async_wait_all();
}

template <int N, bool V, bool VAR>
cudaError_t launch_n(const Rows& R, cudaStream_t stream) {
  cudaError_t e = set_smem_limit<route_rec_kernel<N, V, VAR>>(kSmem);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  static int per_sm_cached = 0;  // the same on every B200 device
  int per_sm = per_sm_cached;
  if (per_sm <= 0) {
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_rec_kernel<N, V, VAR>, kThreads, kSmem);
    per_sm_cached = per_sm;
  }
  const int64_t rows = R.B * R.H * R.T;
  const int64_t tasks = (rows + kRowsPerTask - 1) / kRowsPerTask;
  const int64_t grid = std::min<int64_t>((tasks + kWarps - 1) / kWarps, (int64_t)sms * std::max(per_sm, 1));
  route_rec_kernel<N, V, VAR><<<(unsigned)grid, kThreads, kSmem, stream>>>(R);
  return cudaGetLastError();
}

// Per-slot selection counts from the records: block (pair, part) counts the selected slots of a
// range of the pair's rows in shared memory and adds them to counts[pair][slot].
__global__ void __launch_bounds__(256) record_counts_kernel(const unsigned char* __restrict__ rec, int64_t T,
                                                            int K, int rec_bytes, int rows_per_block,
                                                            int32_t* __restrict__ counts) {
  __shared__ int hist[kRM];
  const int pair = blockIdx.y;
  for (int i = threadIdx.x; i < kRM; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int64_t t0 = (int64_t)blockIdx.x * rows_per_block;
  const int64_t t1 = min(T, t0 + rows_per_block);
  for (int64_t t = t0 + threadIdx.x; t < t1; t += blockDim.x) {
    const unsigned char* r = rec + ((int64_t)pair * T + t) * rec_bytes;
    for (int j = 0; j < K; ++j) atomicAdd(&hist[r[j]], 1);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kRM; i += blockDim.x)
    if (hist[i]) atomicAdd(counts + (int64_t)pair * kRM + i, hist[i]);
}

}  // namespace

int route_record_bytes(int K) { return 9 * (K <= 16 ? 16 : 32); }

cudaError_t launch_record_counts(const unsigned char* rec, int64_t pairs, int64_t T, int K, int32_t* counts,
                                 cudaStream_t stream) {
  if (pairs == 0 || T == 0) return cudaSuccess;
  const int rows_per_block = 4096;
  dim3 grid((unsigned)((T + rows_per_block - 1) / rows_per_block), (unsigned)pairs);
  record_counts_kernel<<<grid, 256, 0, stream>>>(rec, T, K, route_record_bytes(K), rows_per_block, counts);
  return cudaGetLastError();
}

bool route_records_supported(int M, int K) { return M == kRM && K >= 1 && K <= 32; }

cudaError_t launch_route_records(const float* logits, const float* f, const void* k, int64_t B, int64_t T,
                                 int64_t H, int M, int K, int decay_slot, int router, int validate,
                                 unsigned char* rec, int32_t* idx_out, float* score_out, int32_t* counts,
                                 cudaStream_t stream) {
  if (!route_records_supported(M, K) || !rec || !f || !k) return cudaErrorInvalidValue;
  if (B * T * H == 0) return cudaSuccess;
  Rows R;
  R.logits = logits;
  R.f = f;
  R.k = static_cast<const uint16_t*>(k);
  R.B = B; R.T = T; R.H = H;
  R.K = K;
  R.decay_slot = decay_slot;
  R.router = router;
  R.rec = rec;
  R.idx_out = idx_out;
  R.score_out = score_out;
  cudaError_t e;
  if (router != RSM_ROUTER_SIGMOID) {
    if (K <= 16) e = validate ? launch_n<16, true, true>(R, stream) : launch_n<16, false, true>(R, stream);
    else e = validate ? launch_n<32, true, true>(R, stream) : launch_n<32, false, true>(R, stream);
  } else {
    if (K <= 16) e = validate ? launch_n<16, true, false>(R, stream) : launch_n<16, false, false>(R, stream);
    else e = validate ? launch_n<32, true, false>(R, stream) : launch_n<32, false, false>(R, stream);
  }
  (void)counts;  // counted by launch_record_counts, a launch of its own
  return e;
}

}  // namespace rsm
