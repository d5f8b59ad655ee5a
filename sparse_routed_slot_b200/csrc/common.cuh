// common.cuh -- device helpers shared by the librsm kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "rsm.h"

#define RSM_DEV __device__ __forceinline__

namespace rsm {

constexpr unsigned kFull = 0xffffffffu;

// Device status word (one per device): bits are rsm_status values OR-ed as (1u << status).
extern __device__ unsigned int g_device_status;

RSM_DEV void raise_status(rsm_status s) { atomicOr(&g_device_status, 1u << (unsigned)s); }

// ---------------------------------------------------------------------------------------------
// Input element loads (q, k, v may be fp32 or bf16; everything is computed in fp32).
template <typename T> struct In;
template <> struct In<float> {
  static RSM_DEV float ld(const float* p) { return *p; }
  static RSM_DEV void ld4(const float* p, float (&x)[4]) {
    float4 t = *reinterpret_cast<const float4*>(p);
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  }
};
template <> struct In<__nv_bfloat16> {
  static RSM_DEV float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
  static RSM_DEV void ld4(const __nv_bfloat16* p, float (&x)[4]) {
    uint2 t = *reinterpret_cast<const uint2*>(p);
    x[0] = __uint_as_float(t.x << 16); x[1] = __uint_as_float(t.x & 0xffff0000u);
    x[2] = __uint_as_float(t.y << 16); x[3] = __uint_as_float(t.y & 0xffff0000u);
  }
};

// ---------------------------------------------------------------------------------------------
// Router pieces.
//
// Ranking key: an order-preserving map of an fp32 logit to uint32 (larger float -> larger key),
// with -0.0 mapped onto +0.0 so that the two tie. Inputs are finite (precondition).
RSM_DEV uint32_t order_key(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// sigmoid in fp32 (the router score of a selected slot).
RSM_DEV float sigmoid_f32(float x) { return 1.0f / (1.0f + expf(-x)); }

// Compare-and-swap so that a >= b afterwards.
RSM_DEV void cas_desc(uint32_t& a, uint32_t& b) {
  uint32_t hi = max(a, b), lo = min(a, b);
  a = hi; b = lo;
}

// Warp-wide TopK over one row of M logits (M = 32 * E). Lane l holds slots [l*E, l*E + E) in x.
//
// Order: logit descending, then slot index ascending. Result: a bit mask over the lane's E
// elements (bit e set <=> slot l*E + e is selected). After the selection is final,
// `emit(rank, slot, e)` is called by the lane that owns each selected slot, once per selected
// slot, with its rank in [0, K).
//
// Fast path: a K-round tournament on packed 32-bit keys (ranking key with its low log2(M) bits
// replaced by the inverted slot index, which makes every key unique and breaks ties to the lower
// index). Dropping those low bits can only misorder slots whose logits share the truncated key;
// if any two consecutive entries among the top K+1 share it, the row is re-ranked exactly by
// counting, for each slot, the slots that beat it on the full (key, index) order.
template <int M, class Emit>
RSM_DEV uint32_t warp_topk(const float (&x)[M / 32], int K, int lane, Emit emit) {
  constexpr int E = M / 32;
  constexpr uint32_t kIdxMask = (uint32_t)M - 1u;
  uint32_t key[E], p[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    key[e] = order_key(x[e]);
    p[e] = (key[e] & ~kIdxMask) | (kIdxMask - (uint32_t)(lane * E + e));
  }
  // odd-even transposition sort, descending
#pragma unroll
  for (int r = 0; r < E; ++r) {
#pragma unroll
    for (int i = r & 1; i + 1 < E; i += 2) cas_desc(p[i], p[i + 1]);
  }
  uint32_t sel = 0u;
  uint32_t prev = 0u;
  bool collide = false;
  int rank[E];
#pragma unroll
  for (int e = 0; e < E; ++e) rank[e] = 0;
  const int rounds = K < M ? K + 1 : K;  // one extra peek at the (K+1)-th for the check
  for (int r = 0; r < rounds; ++r) {
    const uint32_t m = __reduce_max_sync(kFull, p[0]);
    if (r > 0) collide |= ((m & ~kIdxMask) == (prev & ~kIdxMask));
    prev = m;
    if (r == K) break;
    if (p[0] == m) {
#pragma unroll
      for (int e = 0; e + 1 < E; ++e) p[e] = p[e + 1];
      p[E - 1] = 0u;
      const int e = (int)(kIdxMask - (m & kIdxMask)) - lane * E;
#pragma unroll
      for (int e2 = 0; e2 < E; ++e2) rank[e2] = (e2 == e) ? r : rank[e2];
      sel |= 1u << e;
    }
  }
  if (__any_sync(kFull, collide)) {
    // Exact re-ranking (rare: a near-tie or an exact tie at or around the cut).
#pragma unroll
    for (int e = 0; e < E; ++e) rank[e] = 0;
    for (int src = 0; src < 32; ++src) {
#pragma unroll
      for (int e2 = 0; e2 < E; ++e2) {
        const uint32_t kj = __shfl_sync(kFull, key[e2], src);
        const int j = src * E + e2;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int i = lane * E + e;
          rank[e] += (kj > key[e]) || (kj == key[e] && j < i);
        }
      }
    }
    sel = 0u;
#pragma unroll
    for (int e = 0; e < E; ++e) sel |= (rank[e] < K ? 1u : 0u) << e;
  }
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (sel & (1u << e)) emit(rank[e], lane * E + e, e);
  return sel;
}

// Loads the lane's E contiguous logits of a row.
template <int M>
RSM_DEV void load_row_logits(const float* row, int lane, float (&x)[M / 32]) {
  constexpr int E = M / 32;
  const float* p = row + lane * E;
  if constexpr (E == 1) {
    x[0] = p[0];
  } else if constexpr (E == 2) {
    float2 t = *reinterpret_cast<const float2*>(p);
    x[0] = t.x; x[1] = t.y;
  } else {
#pragma unroll
    for (int c = 0; c < E / 4; ++c) {
      float4 t = *reinterpret_cast<const float4*>(p + 4 * c);
      x[4 * c] = t.x; x[4 * c + 1] = t.y; x[4 * c + 2] = t.z; x[4 * c + 3] = t.w;
    }
  }
}

// Validation helpers (used only under RSM_FLAG_VALIDATE).
RSM_DEV bool finite_f32(float x) { return (__float_as_uint(x) & 0x7f800000u) != 0x7f800000u; }

}  // namespace rsm
