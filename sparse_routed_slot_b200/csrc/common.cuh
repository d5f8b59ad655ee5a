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

// Warp-wide sum / max / min by xor-shuffle butterflies (every lane gets the result).
RSM_DEV float warp_sum_f(float v) {
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) v += __shfl_xor_sync(kFull, v, d);
  return v;
}
RSM_DEV float warp_max_f(float v) {
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, d));
  return v;
}
RSM_DEV int warp_sum(int v) {
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) v += __shfl_xor_sync(kFull, v, d);
  return v;
}
RSM_DEV uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) v = max(v, (uint32_t)__shfl_xor_sync(kFull, v, d));
  return v;
}
RSM_DEV uint32_t warp_min_u32(uint32_t v) {
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) v = min(v, (uint32_t)__shfl_xor_sync(kFull, v, d));
  return v;
}

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

// Selection of the TopK set only (no ranks): finds a threshold t with exactly K values >= t. Every
// member of {x >= t} is then strictly larger than every non-member, so it is the TopK set under any
// tie-breaking. The search runs in the value domain from a guess (for example the previous row's
// threshold): rows of one stream share a logit distribution, so the first counts usually bracket
// the cut tightly and a few interpolation steps on the empirical distribution land between the
// K-th and (K+1)-th values. The bracket always stays valid: lo with more than K values >= lo, hi
// with fewer than K values >= hi (the row max and min start it). `guess` is replaced by the
// threshold found. Returns false, without a result, when no such threshold exists (a tie at the
// cut) or the bracket closes without one (near-ties); the caller then uses warp_topk. Needs
// 2 <= K < M.
template <int M>
RSM_DEV bool warp_select_guess(const float (&x)[M / 32], int K, float& guess, uint32_t& sel) {
  constexpr int E = M / 32;
  auto count_ge = [&](float t) {
    int c = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) c += x[e] >= t ? 1 : 0;
    return (int)__reduce_add_sync(kFull, (unsigned)c);
  };
  float lmax = x[0], lmin = x[0];
#pragma unroll
  for (int e = 1; e < E; ++e) {
    lmax = fmaxf(lmax, x[e]);
    lmin = fminf(lmin, x[e]);
  }
  // row max / min through order-preserving keys (exact, -0 and +0 alike)
  const uint32_t kmax = __reduce_max_sync(kFull, order_key(lmax));
  const uint32_t kmin = __reduce_min_sync(kFull, order_key(lmin));
  auto key_to_float = [](uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
  };
  float hi = key_to_float(kmax), lo = key_to_float(kmin);
  int chi = count_ge(hi);  // multiplicity of the max
  if (chi >= K) return false;  // K-way tie (or more) at the max
  int clo = M;             // every value is >= the min
  float t = guess;
  if (!(t > lo && t < hi)) t = lo + (hi - lo) * ((float)(M - K) / (float)M);
  bool found = false;
  for (int it = 0; it < 24; ++it) {
    const int c = count_ge(t);
    if (c == K) {
      found = true;
      break;
    }
    if (c > K) {
      lo = t;
      clo = c;
    } else {
      hi = t;
      chi = c;
    }
    // next probe: linear interpolation of the count between the bracket ends, aimed half a
    // value past the K-th; every third step bisects to guarantee progress
    float nt = (it % 3 == 2) ? 0.5f * (lo + hi)
                             : lo + (hi - lo) * __fdividef((float)clo - (float)K - 0.5f, (float)(clo - chi));
    if (!(nt > lo && nt < hi)) nt = 0.5f * (lo + hi);
    if (!(nt > lo && nt < hi)) return false;  // adjacent floats: a tie or near-tie at the cut
    t = nt;
  }
  if (!found) return false;
  guess = t;
  sel = 0u;
#pragma unroll
  for (int e = 0; e < E; ++e) sel |= (x[e] >= t ? 1u : 0u) << e;
  return true;
}

// Router variant scores of a row held by a warp (lane: E logits x[e]; sel: the lane's selected
// elements, bit e). s[e] is the score of each selected element, 0 elsewhere:
//   RSM_ROUTER_SIGMOID       sigmoid(x)
//   RSM_ROUTER_SOFTMAX       e^{x - max} / sum over the whole row of e^{x_j - max}
//   *_NORM                   the above divided by its sum over the selected elements
// Every lane of the warp must call it (warp reductions).
template <int E>
RSM_DEV void warp_router_scores(const float (&x)[E], uint32_t sel, int router, float (&s)[E]) {
  if (router & RSM_ROUTER_SOFTMAX) {
    float mx = x[0];
#pragma unroll
    for (int e = 1; e < E; ++e) mx = fmaxf(mx, x[e]);
    mx = warp_max_f(mx);
    float z = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      s[e] = expf(x[e] - mx);
      z += s[e];
    }
    const float rz = 1.0f / warp_sum_f(z);
#pragma unroll
    for (int e = 0; e < E; ++e) s[e] = (sel >> e) & 1u ? s[e] * rz : 0.f;
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) s[e] = (sel >> e) & 1u ? sigmoid_f32(x[e]) : 0.f;
  }
  if (router & 2) {  // normalised over the selected slots
    float t = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) t += s[e];
    const float rt = 1.0f / warp_sum_f(t);
#pragma unroll
    for (int e = 0; e < E; ++e) s[e] *= rt;
  }
}

// rank[e] = r for element e (unrolled select, so that a runtime e keeps the array in registers).
template <int E>
RSM_DEV void set_rank(int (&rank)[E], int e, int r) {
#pragma unroll
  for (int e2 = 0; e2 < E; ++e2) rank[e2] = (e2 == e) ? r : rank[e2];
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

// ---------------------------------------------------------------------------------------------
// Host-side launch set-up, cached per device: the multiprocessor count, and each kernel's
// dynamic shared-memory limit (an attribute of the function in the device's context; setting it
// on every call costs host time that small launches would wait on).
inline int device_sm_count() {
  static int cached[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 148;
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

template <auto Kernel>
inline cudaError_t set_smem_limit(int bytes) {
  static int done[64] = {};  // bytes already allowed, per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && done[dev] >= bytes) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = bytes;
  return e;
}

// Validation helpers (used only under RSM_FLAG_VALIDATE).
RSM_DEV bool finite_f32(float x) { return (__float_as_uint(x) & 0x7f800000u) != 0x7f800000u; }

}  // namespace rsm
