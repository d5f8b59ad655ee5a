// decode.cu -- one generation step per (b,h) (rsm_decode_step).
//
// The step streams the whole fp32 state once: for every (b,h) it reads the M x Dv state, writes
// back only the K selected rows and produces o = sum_i q_i H'[i,:] (Raven README "Model Structure":
// the fused recurrent form used for generation). Bytes per (b,h): M*Dv*4 read + K*Dv*4 written +
// the token's inputs, so the kernel is bound by HBM bandwidth and is organised to keep the copy
// engine busy without pause:
//
//   one persistent CTA per SM owns a contiguous range of (b,h) items (ranges differ by at most one
//   item) and splits the work among three warp roles that meet at mbarriers in shared memory:
//     producer  (1 thread)   streams the state of its items, block by block (32 KB of rows per
//                            block), through a ring of kStages buffers with cp.async.bulk;
//     routers   (kRouters warps) run ahead of the consumers: TopK of the item's logits, the
//                            router scores s (sigmoid or softmax, optionally normalised), then the
//                            decay a = e^{s f} and write weight w = k (1 - a) of every slot (a = 1,
//                            w = 0 off the selection), q and v, into a ring of routing slots;
//     consumers (8 warps)    apply the update to the selected rows of each block, store those rows,
//                            accumulate the read over all rows, and reduce o at the item's end.
//   Selected slots carry their decay with the sign bit set (-a), so one load tells a consumer both
//   whether to write the row and by how much to decay it.
//
// Every wait is bounded; on expiry the CTA records RSM_ERR_TIMEOUT, stops, and the producer waits
// (bounded) for its copies still in flight before the CTA exits. RSM_FLAG_TEST_STALL_ROUTING
// exercises that path on purpose: the routers hand over nothing and the consumers' wait for the
// first routing slot uses a short limit, so every CTA takes the timeout exit.
#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace rsm {

namespace {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kRouters = 4;                       // routing warps
constexpr int kProducerWarp = kConsumerWarps;     // warp 8
constexpr int kRouterWarp0 = kConsumerWarps + 1;  // warps 9..12
constexpr int kThreads = (kConsumerWarps + 1 + kRouters) * 32;
constexpr int kStages = 6;
constexpr int kStageBytes = 32 * 1024;  // 16 KB blocks measured slower: per-block consumer overhead
constexpr int kRouteSlotsMax = 8;
constexpr int kSmemMax = 232448;       // dynamic shared memory per CTA on sm_100
constexpr int kRedBytes = 2 * 8 * 32 * 16;

// Bytes of one routing slot: a[M], w[M], q[M] (fp32) and v[Dv] (fp32).
__host__ __device__ constexpr int route_slot_bytes(int M, int Dv) { return (3 * M + Dv) * 4; }

// Routing slots that fit beside the state ring (2 to kRouteSlotsMax).
__host__ __device__ constexpr int route_slots(int M, int Dv) {
  return (kSmemMax - kStages * kStageBytes - kRedBytes) / route_slot_bytes(M, Dv) < kRouteSlotsMax
             ? (kSmemMax - kStages * kStageBytes - kRedBytes) / route_slot_bytes(M, Dv)
             : kRouteSlotsMax;
}

struct Smem {
  unsigned char* stage;  // [kStages][kStageBytes]
  unsigned char* route;  // [nslots][route_slot_bytes]
  float4* red;           // [2][kConsumers]
};

RSM_DEV void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          tc::smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
      : "memory");
}
RSM_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}
// Barrier among the consumer warps that also ORs a flag over them (all of them get the result).
RSM_DEV bool bar_consumers_or(bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)flag), "n"(kConsumers)
      : "memory");
  return r != 0;
}

static_assert(kRedBytes == 2 * kConsumers * 16, "reduction buffer");
static_assert(route_slots(256, 256) >= kRouters, "routing ring too small for the largest shape");

template <int M, typename TIn>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(rsm_decode_args a) {
  constexpr int E = M / 32;
  const int Dv = a.Dv, K = a.K;
  const int rows_blk = min(M, kStageBytes / (Dv * 4));  // state rows per block
  const int nblk = (M + rows_blk - 1) / rows_blk;        // blocks per item
  const int slot_bytes = route_slot_bytes(M, Dv);
  const int nslots = route_slots(M, Dv);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // this CTA's items: a contiguous range, sizes differing by at most one across CTAs
  const int64_t items = (int64_t)a.B * a.H;
  const int64_t it0 = items * blockIdx.x / gridDim.x;
  const int64_t it1 = items * (blockIdx.x + 1) / gridDim.x;
  const int nitems = (int)(it1 - it0);

  extern __shared__ __align__(128) unsigned char dsm[];
  Smem s;
  s.stage = dsm;
  s.route = dsm + kStages * kStageBytes;
  s.red = reinterpret_cast<float4*>(s.route + nslots * slot_bytes);
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages], rfull[kRouteSlotsMax], rempty[kRouteSlotsMax];
  __shared__ int s_abort;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      tc::mbar_init(&full[i], 1);
      tc::mbar_init(&empty[i], kConsumerWarps);
    }
    for (int i = 0; i < kRouteSlotsMax; ++i) {
      tc::mbar_init(&rfull[i], 1);
      tc::mbar_init(&rempty[i], 1);
    }
    tc::fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();
  volatile int* abort_flag = &s_abort;
  auto fail = [&]() {
    *abort_flag = 1;
    raise_status(RSM_ERR_TIMEOUT);
  };

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------------------ producer
    if (lane == 0) {
      const int total = nitems * nblk;
      int n = 0;
      for (; n < total && !*abort_flag; ++n) {
        const int st = n % kStages;
        if (n >= kStages && !tc::mbar_wait(&empty[st], ((n / kStages) - 1) & 1)) {
          fail();
          break;
        }
        const int64_t item = it0 + n / nblk;
        const int r0 = (n % nblk) * rows_blk;
        const uint32_t bytes = (uint32_t)(min(rows_blk, M - r0) * Dv * 4);
        tc::mbar_arrive_expect_tx(&full[st], bytes);
        bulk_load(s.stage + st * kStageBytes, a.state + (item * M + r0) * (int64_t)Dv, bytes, &full[st]);
      }
      // copies still in flight must land before the CTA's shared memory is released
      for (int m = max(0, n - kStages); m < n; ++m) tc::mbar_wait(&full[m % kStages], (m / kStages) & 1);
    }
  } else if (warp >= kRouterWarp0) {
    // ------------------------------------------------------------------------------ routers
    const int r = warp - kRouterWarp0;
    // testing aid: no routing slot is ever handed over, so the consumers' bounded wait expires
    const int route_items = (a.flags & RSM_FLAG_TEST_STALL_ROUTING) ? 0 : nitems;
    for (int m = r; m < route_items && !*abort_flag; m += kRouters) {
      const int slot = m % nslots;
      if (m >= nslots && !tc::mbar_wait(&rempty[slot], ((m / nslots) - 1) & 1)) {
        fail();
        break;
      }
      const int64_t pair = it0 + m;
      float* sa = reinterpret_cast<float*>(s.route + slot * slot_bytes);
      float* sw = sa + M;
      float* sq = sw + M;
      float* sv = sq + M;
      const TIn* q = reinterpret_cast<const TIn*>(a.q) + pair * M;
      const TIn* k = reinterpret_cast<const TIn*>(a.k) + pair * M;
      const TIn* v = reinterpret_cast<const TIn*>(a.v) + pair * Dv;
      float x[E], fv[E], kv[E];
      load_row_logits<M>(a.logits + pair * M, lane, x);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int i = lane * E + e;
        fv[e] = (a.decay == RSM_DECAY_SLOT) ? a.f[pair * M + i] : a.f[pair];
        kv[e] = In<TIn>::ld(k + i);
        sq[i] = In<TIn>::ld(q + i);
      }
      for (int d = lane; d < Dv; d += 32) sv[d] = In<TIn>::ld(v + d);
      if (a.flags & RSM_FLAG_VALIDATE) {
        bool bad = false;
#pragma unroll
        for (int e = 0; e < E; ++e) bad |= !finite_f32(x[e]) || !finite_f32(fv[e]) || fv[e] > 0.f;
        if (__any_sync(kFull, bad) && lane == 0) raise_status(RSM_ERR_NONFINITE);
      }
      int32_t* io = a.idx_out ? a.idx_out + pair * K : nullptr;
      float* so = a.score_out ? a.score_out + pair * K : nullptr;
      int32_t* cnt = a.slot_counts ? a.slot_counts + pair * M : nullptr;
      int rank[E];
      const uint32_t sel = warp_topk<M>(x, K, lane, [&](int rk, int slot_i, int e) {
        if (io) io[rk] = slot_i;
        if (cnt) cnt[slot_i] += 1;  // one router warp per (b,h): no other writer
        set_rank<E>(rank, e, rk);
      });
      float sc[E];
      warp_router_scores<E>(x, sel, a.router, sc);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int i = lane * E + e;
        if (sel & (1u << e)) {
          if (so) so[rank[e]] = sc[e];
          const float lam = sc[e] * fv[e];   // log of the decay, <= 0
          sa[i] = -expf(lam);                // sign bit: selected
          sw[i] = kv[e] * (-expm1f(lam));    // k_i (1 - a_i)
        } else {
          sa[i] = 1.f;
          sw[i] = 0.f;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&rfull[slot]);
    }
  } else {
    // ------------------------------------------------------------------------------ consumers
    const int CG = Dv >> 2;          // float4 column groups
    const int RG = kConsumers / CG;  // row groups
    const int cg = tid % CG, rg = tid / CG;
    const bool active = rg < RG;
    // the hand-off wait's poll limit: the default bound, or a short one under the testing aid
    const uint32_t rfull_limit = (a.flags & RSM_FLAG_TEST_STALL_ROUTING) ? (1u << 10) : (1u << 22);
    int n = 0;
    for (int m = 0; m < nitems; ++m) {
      // A thread that sees a failure stops waiting and computing but still reaches the item's
      // barrier, which ORs the failure over all consumers, so that they leave together.
      bool ab = false;
      const int slot = m % nslots;
      if (!tc::mbar_wait(&rfull[slot], (m / nslots) & 1, rfull_limit)) {
        fail();
        ab = true;
      }
      const float* sa = reinterpret_cast<const float*>(s.route + slot * slot_bytes);
      const float* sw = sa + M;
      const float* sq = sw + M;
      const float4 vv = active ? reinterpret_cast<const float4*>(sq + M)[cg] : make_float4(0.f, 0.f, 0.f, 0.f);
      float* state = a.state + (it0 + m) * (int64_t)M * Dv;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int blk = 0; blk < nblk; ++blk, ++n) {
        const int st = n % kStages;
        ab = ab || *abort_flag;
        if (!ab && !tc::mbar_wait(&full[st], (n / kStages) & 1)) {
          fail();
          ab = true;
        }
        const float* sb = reinterpret_cast<const float*>(s.stage + st * kStageBytes);
        const int r0 = blk * rows_blk;
        const int rows = min(rows_blk, M - r0);
        if (active && !ab) {
#pragma unroll 4
          for (int rr = rg; rr < rows; rr += RG) {
            const int row = r0 + rr;
            float4 hv = reinterpret_cast<const float4*>(sb + rr * Dv)[cg];
            const float as = sa[row];
            if (__float_as_uint(as) & 0x80000000u) {
              const float ar = -as, wr = sw[row];
              hv.x = fmaf(ar, hv.x, wr * vv.x);
              hv.y = fmaf(ar, hv.y, wr * vv.y);
              hv.z = fmaf(ar, hv.z, wr * vv.z);
              hv.w = fmaf(ar, hv.w, wr * vv.w);
              reinterpret_cast<float4*>(state + (int64_t)row * Dv)[cg] = hv;
            }
            const float qr = sq[row];
            acc.x = fmaf(qr, hv.x, acc.x);
            acc.y = fmaf(qr, hv.y, acc.y);
            acc.z = fmaf(qr, hv.z, acc.z);
            acc.w = fmaf(qr, hv.w, acc.w);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);  // this warp is done with the buffer
      }
      // o = sum over the row groups (double-buffered partials: one barrier per item)
      float4* red = s.red + (m & 1) * kConsumers;
      if (active) red[rg * CG + cg] = acc;
      if (bar_consumers_or(ab || *abort_flag)) break;
      for (int c = tid; c < CG; c += kConsumers) {
        float4 o4 = red[c];
        for (int g = 1; g < RG; ++g) {
          const float4 p = red[g * CG + c];
          o4.x += p.x; o4.y += p.y; o4.z += p.z; o4.w += p.w;
        }
        reinterpret_cast<float4*>(a.o + (it0 + m) * (int64_t)Dv)[c] = o4;
      }
      if (tid == 0) mbar_arrive(&rempty[slot]);  // every consumer is past the routing slot
    }
  }
}


template <int M, typename TIn>
cudaError_t launch_t(const rsm_decode_args& a, cudaStream_t stream) {
  const int smem = kStages * kStageBytes + route_slots(M, a.Dv) * route_slot_bytes(M, a.Dv) + kRedBytes;
  cudaError_t e = set_smem_limit<decode_kernel<M, TIn>>(smem);
  if (e != cudaSuccess) return e;
  const int64_t items = (int64_t)a.B * a.H;
  const unsigned grid = (unsigned)std::min<int64_t>(items, (int64_t)device_sm_count());
  decode_kernel<M, TIn><<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int M>
cudaError_t launch_m(const rsm_decode_args& a, cudaStream_t stream) {
  return a.qkv_dtype == RSM_BF16 ? launch_t<M, __nv_bfloat16>(a, stream) : launch_t<M, float>(a, stream);
}

}  // namespace

cudaError_t launch_decode(const rsm_decode_args& a, cudaStream_t stream) {
  if ((int64_t)a.B * a.H == 0) return cudaSuccess;
  switch (a.M) {
    case 32: return launch_m<32>(a, stream);
    case 64: return launch_m<64>(a, stream);
    case 128: return launch_m<128>(a, stream);
    case 256: return launch_m<256>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace rsm
