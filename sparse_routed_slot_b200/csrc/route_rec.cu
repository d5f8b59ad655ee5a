// route_rec.cu -- routing records for the tensor-core prefill.
//
// The TopK routing of every (token, head) row runs once, ahead of the chunked scan, in a kernel
// with one THREAD per row (all 32 lanes of a warp do useful work on 32 different rows), and its
// result is stored as a compact record that both passes of the scan read instead of the logits:
//
//   record (rec_bytes(K) bytes, 16-byte aligned, row-major like the logits [B, T, H]):
//     uint32 mask[4]                   bit i of the 128-bit mask set <=> slot i selected
//     uint8  slot[roundup(K, 16)]      the selected slots in ascending order (padding 0)
//     float  lam[roundup(K, 4)]        lam_j = sigmoid(logit[slot_j]) * f(slot_j), the log of the
//                                      decay a = e^lam (<= 0) of the j-th selected slot (padding 0)
//
// Selection (router scores are monotone in the logits, so TopK of the scores = TopK of the
// logits; order: logit descending, slot ascending, -0 ties +0): each logit becomes a packed
// 32-bit key, its order-preserving bit pattern with the low 7 bits replaced by (127 - slot), which
// makes every key distinct and breaks ties to the lower slot. The top N (N = 16 or 32 >= K) keys
// of the 128 come from a bitonic network in registers: 128/N sorted runs of N, each merged into
// the running top N (the larger half of two sorted runs is bitonic; one half-cleaner cascade sorts
// it). Dropping the low 7 bits can only misorder logits whose upper 25 key bits agree; if the K-th
// and (K+1)-th keys share them, the row is finished by an exact scan over that bucket.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace rsm {

namespace {

constexpr int kRM = 128;                  // slots on this path
constexpr int kRowFloats = kRM + 4;       // staged row stride (16-byte pad: conflict-free float4 reads)
constexpr int kWarps = 2;                 // warps per CTA
constexpr uint32_t kCoarse = ~0x7Fu;      // key bits above the slot field

RSM_DEV uint32_t packed_key(float x, int slot) { return (order_key(x) & kCoarse) | (uint32_t)(127 - slot); }

// Full bitonic sort of N keys, descending.
template <int N>
RSM_DEV void sort_desc(uint32_t (&a)[N]) {
#pragma unroll
  for (int k = 2; k <= N; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int l = i ^ j;
        if (l > i) {
          if ((i & k) == 0) cas_desc(a[i], a[l]);
          else cas_desc(a[l], a[i]);
        }
      }
    }
  }
}

// top <- the N largest of top and g (both sorted descending); the N smaller ones are dropped and
// the largest dropped key is folded into `dropped`.
template <int N>
RSM_DEV void merge_top(uint32_t (&top)[N], const uint32_t (&g)[N], uint32_t& dropped) {
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const uint32_t a = top[i], b = g[N - 1 - i];
    top[i] = max(a, b);
    dropped = max(dropped, min(a, b));
  }
#pragma unroll
  for (int j = N >> 1; j > 0; j >>= 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const int l = i ^ j;
      if (l > i) cas_desc(top[i], top[l]);
    }
  }
}

RSM_DEV void set_bit(uint32_t (&m)[4], int slot) {
  const uint32_t bit = 1u << (slot & 31);
  const int w = slot >> 5;
  m[0] |= w == 0 ? bit : 0u;
  m[1] |= w == 1 ? bit : 0u;
  m[2] |= w == 2 ? bit : 0u;
  m[3] |= w == 3 ? bit : 0u;
}
RSM_DEV bool has_bit(const uint32_t (&m)[4], int slot) {
  const int w = slot >> 5;
  const uint32_t word = w == 0 ? m[0] : w == 1 ? m[1] : w == 2 ? m[2] : m[3];
  return (word >> (slot & 31)) & 1u;
}

RSM_DEV void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}
RSM_DEV void cp_async_wait_all() { asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory"); }

template <int N, bool VALIDATE>
__global__ void __launch_bounds__(kWarps * 32) route_rec_kernel(const float* __restrict__ logits,
                                                                 const float* __restrict__ f, int64_t rows,
                                                                 int K, int decay_slot, int rec_bytes,
                                                                 unsigned char* __restrict__ rec,
                                                                 int32_t* __restrict__ idx_out,
                                                                 float* __restrict__ score_out) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int stage_bytes = 32 * rec_bytes;
  float* sRows = reinterpret_cast<float*>(smem + warp * (32 * kRowFloats * 4 + stage_bytes));
  unsigned char* sStage = reinterpret_cast<unsigned char*>(sRows + 32 * kRowFloats);
  const int slot_off = 16, lam_off = 16 + ((K + 15) & ~15);
  const int64_t groups = (rows + 31) / 32;

  for (int64_t grp = (int64_t)blockIdx.x * kWarps + warp; grp < groups; grp += (int64_t)gridDim.x * kWarps) {
    const int64_t row0 = grp * 32;
    const int nr = rows - row0 < 32 ? (int)(rows - row0) : 32;
    // ---- stage the warp's rows (one 512-byte row per copy instruction)
    for (int r = 0; r < nr; ++r) cp_async16(sRows + r * kRowFloats + lane * 4, logits + (row0 + r) * kRM + lane * 4);
    float fh = 0.f;
    const int64_t row = row0 + lane;
    const bool live = lane < nr;
    if (live && f && !decay_slot) fh = f[row];
    cp_async_wait_all();
    __syncwarp();

    const float* xr = sRows + lane * kRowFloats;
    uint32_t m[4] = {0u, 0u, 0u, 0u};
    if (live) {
      // ---- top N packed keys
      uint32_t top[N], g[N], dropped = 0u;
      bool bad = false;
#pragma unroll
      for (int i = 0; i < N; i += 4) {
        const float4 v = *reinterpret_cast<const float4*>(xr + i);
        top[i] = packed_key(v.x, i);
        top[i + 1] = packed_key(v.y, i + 1);
        top[i + 2] = packed_key(v.z, i + 2);
        top[i + 3] = packed_key(v.w, i + 3);
        if (VALIDATE) bad |= !finite_f32(v.x) || !finite_f32(v.y) || !finite_f32(v.z) || !finite_f32(v.w);
      }
      sort_desc<N>(top);
#pragma unroll 1
      for (int s0 = N; s0 < kRM; s0 += N) {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
          const float4 v = *reinterpret_cast<const float4*>(xr + s0 + i);
          g[i] = packed_key(v.x, s0 + i);
          g[i + 1] = packed_key(v.y, s0 + i + 1);
          g[i + 2] = packed_key(v.z, s0 + i + 2);
          g[i + 3] = packed_key(v.w, s0 + i + 3);
          if (VALIDATE) bad |= !finite_f32(v.x) || !finite_f32(v.y) || !finite_f32(v.z) || !finite_f32(v.w);
        }
        sort_desc<N>(g);
        merge_top<N>(top, g, dropped);
      }
      if (VALIDATE && f) {
        if (decay_slot) {
          for (int s = 0; s < kRM; ++s) {
            const float fv = f[row * kRM + s];
            bad |= !finite_f32(fv) || fv > 0.f;
          }
        } else {
          bad |= !finite_f32(fh) || fh > 0.f;
        }
      }
      if (VALIDATE && bad) raise_status(RSM_ERR_NONFINITE);
      // ---- the K-th and (K+1)-th keys; the set of the first K
      // (top is sorted: the K-th is the least of the first K, the next the largest of the rest;
      // written as reductions so that no register array is indexed by K)
      uint32_t kth = 0xffffffffu, next = dropped;
#pragma unroll
      for (int r = 0; r < N; ++r) {
        kth = min(kth, r < K ? top[r] : 0xffffffffu);
        next = max(next, r < K ? 0u : top[r]);
      }
      const uint32_t cb = kth & kCoarse;
      const bool exact_needed = (next & kCoarse) == cb;
      int have = 0;
#pragma unroll
      for (int r = 0; r < N; ++r) {
        // with a shared bucket at the cut, keep only the keys strictly above it
        if (r < K && (!exact_needed || (top[r] & kCoarse) > cb)) {
          set_bit(m, 127 - (int)(top[r] & 0x7Fu));
          ++have;
        }
      }
      // ---- rare: fill the cut exactly from the shared bucket (logit desc, slot asc)
      for (; have < K; ++have) {
        int best = -1;
        uint32_t bk = 0u;
        for (int s = 0; s < kRM; ++s) {
          const uint32_t k = order_key(xr[s]);
          if ((k & kCoarse) != cb || has_bit(m, s)) continue;
          if (best < 0 || k > bk) {
            best = s;
            bk = k;
          }
        }
        set_bit(m, best);
      }
    }
    // ---- record of this lane's row into the warp's staging area
    unsigned char* st = sStage + lane * rec_bytes;
    if (live) {
      *reinterpret_cast<uint4*>(st) = make_uint4(m[0], m[1], m[2], m[3]);
      int j = 0;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t mw = m[w];
        while (mw) {
          const int slot = w * 32 + __ffs(mw) - 1;
          mw &= mw - 1u;
          st[slot_off + j] = (unsigned char)slot;
          ++j;
        }
      }
      for (; j < lam_off - slot_off; ++j) st[slot_off + j] = 0;
      uint32_t* keys = reinterpret_cast<uint32_t*>(st + lam_off);  // the lam area, reused first
      float* lam = reinterpret_cast<float*>(st + lam_off);
      if (idx_out || score_out) {
        // rank of each selected slot: the selected slots that beat it (logit desc, slot asc)
        for (int jj = 0; jj < K; ++jj) keys[jj] = order_key(xr[st[slot_off + jj]]);
        for (int jj = 0; jj < K; ++jj) {
          const int sj = st[slot_off + jj];
          const uint32_t kj = keys[jj];
          int rank = 0;
          for (int i = 0; i < K; ++i) {
            const uint32_t ki = keys[i];
            rank += (ki > kj) || (ki == kj && i < jj);  // slots ascending: index order = slot order
          }
          if (idx_out) idx_out[row * K + rank] = sj;
          if (score_out) score_out[row * K + rank] = sigmoid_f32(xr[sj]);
        }
      }
      if (rec) {
        // lam after all slots are known (slot-decay gathers are independent loads)
#pragma unroll 4
        for (int jj = 0; jj < K; ++jj) {
          const int slot = st[slot_off + jj];
          const float fv = decay_slot ? f[row * kRM + slot] : fh;
          lam[jj] = sigmoid_f32(xr[slot]) * fv;
        }
        for (int jj = K; jj < (rec_bytes - lam_off) / 4; ++jj) lam[jj] = 0.f;
      }
    }
    __syncwarp();
    if (rec) {
      // coalesced copy-out of the warp's records (consecutive rows are consecutive records)
      const int n16 = nr * rec_bytes / 16;
      uint4* dst = reinterpret_cast<uint4*>(rec + row0 * rec_bytes);
      const uint4* src = reinterpret_cast<const uint4*>(sStage);
      for (int i = lane; i < n16; i += 32) dst[i] = src[i];
    }
    __syncwarp();
  }
}

template <int N, bool V>
cudaError_t launch_n(const float* logits, const float* f, int64_t rows, int K, int decay_slot,
                     unsigned char* rec, int32_t* idx_out, float* score_out, cudaStream_t stream) {
  const int rb = route_record_bytes(K);
  const int smem = kWarps * (32 * kRowFloats * 4 + 32 * rb);
  cudaError_t e = cudaFuncSetAttribute(route_rec_kernel<N, V>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_rec_kernel<N, V>, kWarps * 32, smem);
  const int64_t ctas_needed = ((rows + 31) / 32 + kWarps - 1) / kWarps;
  const int64_t grid = std::min<int64_t>(ctas_needed, (int64_t)sms * std::max(per_sm, 1));
  route_rec_kernel<N, V><<<(unsigned)grid, kWarps * 32, smem, stream>>>(logits, f, rows, K, decay_slot, rb, rec,
                                                                        idx_out, score_out);
  return cudaGetLastError();
}

}  // namespace

int route_record_bytes(int K) { return 16 + ((K + 15) & ~15) + 4 * ((K + 3) & ~3); }

bool route_records_supported(int M, int K) { return M == kRM && K >= 1 && K <= 32; }

cudaError_t launch_route_records(const float* logits, const float* f, int64_t rows, int M, int K, int decay_slot,
                                 int validate, unsigned char* rec, int32_t* idx_out, float* score_out,
                                 cudaStream_t stream) {
  if (!route_records_supported(M, K)) return cudaErrorInvalidValue;
  if (rows == 0) return cudaSuccess;
  if (K <= 16) {
    return validate ? launch_n<16, true>(logits, f, rows, K, decay_slot, rec, idx_out, score_out, stream)
                    : launch_n<16, false>(logits, f, rows, K, decay_slot, rec, idx_out, score_out, stream);
  }
  return validate ? launch_n<32, true>(logits, f, rows, K, decay_slot, rec, idx_out, score_out, stream)
                  : launch_n<32, false>(logits, f, rows, K, decay_slot, rec, idx_out, score_out, stream);
}

}  // namespace rsm
