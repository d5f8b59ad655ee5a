// route_rec.cu -- TopK routing, one THREAD per row (M = 128 slots, K <= 32).
//
// Used by rsm_route (indices and scores in rank order) and by the tensor-core prefill, which
// reads compact routing records instead of the logits (Raven README "How Raven Works":
// route_scores = TopK(sigmoid(r_proj(x))); "Model Structure": a = exp(score * f)):
//
//   record (route_record_bytes(K) = 9 * KP bytes, KP = 16 for K <= 16 else 32; rows in
//   [B, H, T] order, so the records of one (b,h) stream are contiguous along time):
//     uint8  slot[KP]   the selected slots (entries >= K: 0)
//     float  lam[KP]    lam = sigmoid(logit[slot]) * f, the log of the slot's decay (<= 0)
//     float  w[KP]      w = k[slot] * (1 - e^lam), the slot's write weight
//   Entries are in rank order (logit descending, slot ascending) except that logits agreeing in
//   their upper 25 key bits may be listed in slot order; the set is always exact.
//
// Selection (router scores are monotone in the logits, so TopK of the scores = TopK of the
// logits; -0 ties +0): each logit becomes a packed 32-bit key, its order-preserving bit pattern
// with the low 7 bits replaced by (127 - slot), which makes every key distinct and breaks ties to
// the lower slot. The top N (N = 16 or 32 >= K) keys come from a bitonic network in registers: the
// row is read in groups of N logits straight from global memory (the next group is in flight while
// the current one is sorted), each group is sorted and merged into the running top N (the larger
// half of two sorted runs is bitonic; one half-cleaner cascade sorts it). Dropping the low 7 bits
// can only misorder logits whose upper 25 key bits agree; if the K-th and (K+1)-th keys share them,
// or ranked outputs are requested and two of the first K share them, the row is finished by an
// exact selection over the full keys instead.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace rsm {

namespace {

constexpr int kRM = 128;              // slots on this path
constexpr int kThreads = 128;
constexpr uint32_t kCoarse = ~0x7Fu;  // key bits above the slot field

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

// top <- the N largest of top and g (both sorted descending); the largest dropped key is folded
// into `dropped`.
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

RSM_DEV bool has_bit(const uint32_t (&m)[4], int slot) {
  const int w = slot >> 5;
  const uint32_t word = w == 0 ? m[0] : w == 1 ? m[1] : w == 2 ? m[2] : m[3];
  return (word >> (slot & 31)) & 1u;
}
RSM_DEV void set_bit(uint32_t (&m)[4], int slot) {
  const uint32_t bit = 1u << (slot & 31);
  const int w = slot >> 5;
  m[0] |= w == 0 ? bit : 0u;
  m[1] |= w == 1 ? bit : 0u;
  m[2] |= w == 2 ? bit : 0u;
  m[3] |= w == 3 ? bit : 0u;
}

template <int N>
RSM_DEV void load_group(const float* row, int g, float4 (&v)[N / 4]) {
#pragma unroll
  for (int i = 0; i < N / 4; ++i) v[i] = __ldg(reinterpret_cast<const float4*>(row + g * N) + i);
}

struct Rows {
  const float* logits;
  const float* f;
  const uint16_t* k;  // bf16 bits
  int64_t B, T, H;
  int K, decay_slot;
  unsigned char* rec;
  int32_t* idx_out;
  float* score_out;
};

// The lam and w of one selected slot of input row `ir`.
RSM_DEV void entry_values(const Rows& R, int64_t ir, int slot, float fh, float& s, float& lam, float& w) {
  const float x = __ldg(R.logits + ir * kRM + slot);
  s = sigmoid_f32(x);
  const float fv = R.decay_slot ? __ldg(R.f + ir * kRM + slot) : fh;
  lam = s * fv;
  const float kv = __uint_as_float((uint32_t)__ldg(R.k + ir * kRM + slot) << 16);
  w = kv * (-expm1f(lam));
}

template <int N, bool VALIDATE>
__global__ void __launch_bounds__(kThreads) route_rec_kernel(const Rows R) {
  constexpr int KP = N;  // record entries
  const int K = R.K;
  const int64_t rows = R.B * R.H * R.T;
  for (int64_t p = (int64_t)blockIdx.x * kThreads + threadIdx.x; p < rows; p += (int64_t)gridDim.x * kThreads) {
    // p enumerates rows in [B, H, T] order; ir is the row's index in the [B, T, H] input layout
    const int64_t bh = p / R.T, t = p - bh * R.T;
    const int64_t b = bh / R.H, h = bh - b * R.H;
    const int64_t ir = (b * R.T + t) * R.H + h;
    const float* xr = R.logits + ir * kRM;
    const float fh = (R.f && !R.decay_slot) ? __ldg(R.f + ir) : 0.f;

    // ---- top N packed keys
    uint32_t top[N], g[N], dropped = 0u;
    bool bad = false;
    float4 cur[N / 4], nxt[N / 4];
    auto keys = [&](int grp, uint32_t (&dst)[N]) {
#pragma unroll
      for (int i = 0; i < N / 4; ++i) {
        const int s0 = grp * N + 4 * i;
        dst[4 * i] = packed_key(cur[i].x, s0);
        dst[4 * i + 1] = packed_key(cur[i].y, s0 + 1);
        dst[4 * i + 2] = packed_key(cur[i].z, s0 + 2);
        dst[4 * i + 3] = packed_key(cur[i].w, s0 + 3);
        if (VALIDATE)
          bad |= !finite_f32(cur[i].x) || !finite_f32(cur[i].y) || !finite_f32(cur[i].z) || !finite_f32(cur[i].w);
      }
    };
    load_group<N>(xr, 0, cur);
    load_group<N>(xr, 1, nxt);
    keys(0, top);
    sort_desc<N>(top);
#pragma unroll 1
    for (int grp = 1; grp < kRM / N; ++grp) {
#pragma unroll
      for (int i = 0; i < N / 4; ++i) cur[i] = nxt[i];
      if (grp + 1 < kRM / N) load_group<N>(xr, grp + 1, nxt);
      keys(grp, g);
      sort_desc<N>(g);
      merge_top<N>(top, g, dropped);
    }
    if (VALIDATE && R.f) {
      if (R.decay_slot) {
        for (int s = 0; s < kRM; ++s) {
          const float fv = __ldg(R.f + ir * kRM + s);
          bad |= !finite_f32(fv) || fv > 0.f;
        }
      } else {
        bad |= !finite_f32(fh) || fh > 0.f;
      }
    }
    if (VALIDATE && bad) raise_status(RSM_ERR_NONFINITE);

    // ---- is the coarse order enough? (the K-th and (K+1)-th keys; neighbours among the first K)
    uint32_t kth = 0xffffffffu, next = dropped;
    bool near_tie = false;
#pragma unroll
    for (int r = 0; r < N; ++r) {
      kth = min(kth, r < K ? top[r] : 0xffffffffu);
      next = max(next, r < K ? 0u : top[r]);
      if (r + 1 < N && r + 1 < K) near_tie |= ((top[r] ^ top[r + 1]) & kCoarse) == 0u;
    }
    const bool ranked = R.idx_out || R.score_out;
    const bool exact = ((next ^ kth) & kCoarse) == 0u || (ranked && near_tie);
    const bool rec = R.rec != nullptr;
    unsigned char* rp = rec ? R.rec + p * (int64_t)(9 * KP) : nullptr;
    int32_t* io = R.idx_out ? R.idx_out + ir * K : nullptr;
    float* so = R.score_out ? R.score_out + ir * K : nullptr;

    if (!exact) {
      // ---- entries in rank order from the sorted keys
      uint32_t sw[KP / 4];
      float lam[KP], wv[KP];
#pragma unroll
      for (int i = 0; i < KP / 4; ++i) sw[i] = 0u;
#pragma unroll
      for (int r = 0; r < KP; ++r) {
        lam[r] = 0.f;
        wv[r] = 0.f;
        if (r < K) {
          const int slot = 127 - (int)(top[r] & 0x7Fu);
          sw[r / 4] |= (uint32_t)slot << (8 * (r % 4));
          float s;
          if (rec) {
            entry_values(R, ir, slot, fh, s, lam[r], wv[r]);
          } else {
            s = sigmoid_f32(__ldg(xr + slot));
          }
          if (io) io[r] = slot;
          if (so) so[r] = s;
        }
      }
      if (rec) {
#pragma unroll
        for (int i = 0; i < KP / 16; ++i)
          reinterpret_cast<uint4*>(rp)[i] = make_uint4(sw[4 * i], sw[4 * i + 1], sw[4 * i + 2], sw[4 * i + 3]);
#pragma unroll
        for (int i = 0; i < KP / 4; ++i) {
          reinterpret_cast<float4*>(rp + KP)[i] = make_float4(lam[4 * i], lam[4 * i + 1], lam[4 * i + 2], lam[4 * i + 3]);
          reinterpret_cast<float4*>(rp + 5 * KP)[i] = make_float4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
        }
      }
    } else {
      // ---- rare: exact selection on the full keys, one rank at a time (logit desc, slot asc)
      uint32_t chosen[4] = {0u, 0u, 0u, 0u};
      for (int j = 0; j < KP; ++j) {
        if (j >= K) {
          if (rec) {
            rp[j] = 0;
            reinterpret_cast<float*>(rp + KP)[j] = 0.f;
            reinterpret_cast<float*>(rp + 5 * KP)[j] = 0.f;
          }
          continue;
        }
        int best = -1;
        uint32_t bk = 0u;
        for (int s = 0; s < kRM; ++s) {
          if (has_bit(chosen, s)) continue;
          const uint32_t kx = order_key(__ldg(xr + s));
          if (best < 0 || kx > bk) {
            best = s;
            bk = kx;
          }
        }
        set_bit(chosen, best);
        float s, lam = 0.f, wv = 0.f;
        if (rec) entry_values(R, ir, best, fh, s, lam, wv);
        else s = sigmoid_f32(__ldg(xr + best));
        if (rec) {
          rp[j] = (unsigned char)best;
          reinterpret_cast<float*>(rp + KP)[j] = lam;
          reinterpret_cast<float*>(rp + 5 * KP)[j] = wv;
        }
        if (io) io[j] = best;
        if (so) so[j] = s;
      }
    }
  }
}

template <int N, bool V>
cudaError_t launch_n(const Rows& R, cudaStream_t stream) {
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, route_rec_kernel<N, V>, kThreads, 0);
  const int64_t rows = R.B * R.H * R.T;
  const int64_t need = (rows + kThreads - 1) / kThreads;
  const int64_t grid = std::min<int64_t>(need, (int64_t)sms * std::max(per_sm, 1) * 4);
  route_rec_kernel<N, V><<<(unsigned)grid, kThreads, 0, stream>>>(R);
  return cudaGetLastError();
}

}  // namespace

int route_record_bytes(int K) { return 9 * (K <= 16 ? 16 : 32); }

bool route_records_supported(int M, int K) { return M == kRM && K >= 1 && K <= 32; }

cudaError_t launch_route_records(const float* logits, const float* f, const void* k, int64_t B, int64_t T,
                                 int64_t H, int M, int K, int decay_slot, int validate, unsigned char* rec,
                                 int32_t* idx_out, float* score_out, cudaStream_t stream) {
  if (!route_records_supported(M, K)) return cudaErrorInvalidValue;
  if (B * T * H == 0) return cudaSuccess;
  if (rec && (!f || !k)) return cudaErrorInvalidValue;
  Rows R;
  R.logits = logits;
  R.f = f;
  R.k = static_cast<const uint16_t*>(k);
  R.B = B; R.T = T; R.H = H;
  R.K = K;
  R.decay_slot = decay_slot;
  R.rec = rec;
  R.idx_out = idx_out;
  R.score_out = score_out;
  if (K <= 16) return validate ? launch_n<16, true>(R, stream) : launch_n<16, false>(R, stream);
  return validate ? launch_n<32, true>(R, stream) : launch_n<32, false>(R, stream);
}

}  // namespace rsm
