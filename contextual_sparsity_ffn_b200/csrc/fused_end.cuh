// End phase shared by the decode-step kernels: the output (the sum of the CTAs' partial outputs in
// L2) and the compaction of the active list.
//
// Before it every CTA of the step has added its partial output into one of kFusedAccCopies fp32
// accumulators in the workspace (red_add_v4) and written the keep flag and the kept activations of
// every row position it decided.
#pragma once

#include "common.cuh"
#include "kernels.h"

namespace csffn {

// Fused control words (FusedArgs::ctl).
constexpr int kCtlDone = 0;  // CTAs whose partial sums and flags are written (wraps to 0 on the last)
constexpr int kCtlY = 2;     // CTAs whose share of the predictor's y is written (predictor mode)

constexpr int kTicketCounters = 1;  // ticket counters in use (FusedArgs::tickets)
constexpr int kCounterStride = 32;  // 32-bit words between counters (128 bytes)

constexpr int kFinishHalf = 128;       // threads of each end-phase group (out | compaction)
constexpr int kCountLoads = 16;        // 16-byte flag loads in flight per thread (compaction)

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// out[0..3] += (a, b, c, e) as one vector reduction in L2 (no return value); 16-byte aligned.
__device__ __forceinline__ void red_add_v4(float* out, float a, float b, float c, float e) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(out), "f"(a), "f"(b), "f"(c), "f"(e)
               : "memory");
}

// Bounded wait until *p == 0 (acquire).  Gives up after a second and records the timeout.
__device__ __forceinline__ void wait_zero(const uint32_t* p, uint32_t* err) {
  if (ld_acquire_u32(p) == 0u) return;
  const uint64_t t0 = globaltimer_now();
  while (ld_acquire_u32(p) != 0u) {
    if (globaltimer_now() - t0 > 1000000000ull) {
      atomicOr(err, kDevErrTimeout);
      return;
    }
    __nanosleep(64);
  }
}

// Bounded wait until *p >= target (acquire).  Gives up after a second and records the timeout.
__device__ __forceinline__ void wait_at_least(const uint32_t* p, uint32_t target, uint32_t* err) {
  if (ld_acquire_u32(p) >= target) return;
  const uint64_t t0 = globaltimer_now();
  while (ld_acquire_u32(p) < target) {
    if (globaltimer_now() - t0 > 1000000000ull) {
      atomicOr(err, kDevErrTimeout);
      return;
    }
    __nanosleep(64);
  }
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Row position j of the step -> neuron (the candidate list's entry, or j itself).  A candidate
// outside 0 .. h - 1 (a malformed list) maps to neuron 0, so every access stays in bounds.
__device__ __forceinline__ int step_neuron(const int32_t* cand, int h, int j) {
  if (!cand) return j;
  const int r = __ldg(cand + j);
  return (unsigned)r < (unsigned)h ? r : 0;
}

// Compaction of a step's keep flags into idx / a_val / count, by 128 threads of every CTA of the
// grid (ct = 0 .. 127 their index, named barrier `bar` among them): CTA k owns a fixed range of
// 32-position words, counts the kept positions before it from the flag bytes (each 0 or 1, so a
// 32-bit word's popcount counts its kept rows) and writes its positions' neurons and kept
// activations in ascending order; the last CTA writes the count.
template <int NB>
__device__ __forceinline__ void compact_flags(const FusedArgs& p, int n_rows, uint32_t* s_cnt, int ct, int bar) {
  const int lane = ct & 31, cw = ct >> 5;
  const int B = p.B, h = p.h;
  const int n_words = (n_rows + kWarp - 1) / kWarp;
  const int wa = (int)((long long)n_words * blockIdx.x / gridDim.x);
  const int wb = (int)((long long)n_words * (blockIdx.x + 1) / gridDim.x);
  if (!(wa < wb || blockIdx.x == gridDim.x - 1)) return;
  bool f;
  int nr;
  float av[NB];
  auto load_pass = [&](int w0) {  // flag, neuron and activations of position (w0 + cw) * 32 + lane
    const int jp = (w0 + cw) * kWarp + lane;
    const bool in = w0 + cw < wb && jp < n_rows;
    f = in && __ldcg(p.flags + jp) != 0;
    nr = in ? step_neuron(p.cand_idx, h, jp) : 0;
#pragma unroll
    for (int b = 0; b < NB; ++b) av[b] = (in && b < B) ? __ldcg(p.afull + (size_t)b * h + jp) : 0.f;
  };
  load_pass(wa);
  uint32_t before = 0;
  const uint4* f4 = reinterpret_cast<const uint4*>(p.flags);
  for (int i0 = ct; i0 < wa * 2; i0 += kFinishHalf * kCountLoads) {  // each batch's loads issued together
    uint4 fw[kCountLoads];
#pragma unroll
    for (int u = 0; u < kCountLoads; ++u)
      fw[u] = i0 + u * kFinishHalf < wa * 2 ? __ldcg(f4 + i0 + u * kFinishHalf) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int u = 0; u < kCountLoads; ++u)
      before += __popc(fw[u].x) + __popc(fw[u].y) + __popc(fw[u].z) + __popc(fw[u].w);
  }
  before = warp_sum_u32(before);
  if (lane == 0) s_cnt[cw] = before;
  named_sync(bar, kFinishHalf);
  uint32_t base = 0;
#pragma unroll
  for (int w = 0; w < kFinishHalf / kWarp; ++w) base += s_cnt[w];
  named_sync(bar, kFinishHalf);
  for (int w0 = wa; w0 < wb; w0 += kFinishHalf / kWarp) {
    const uint32_t m = __ballot_sync(0xffffffffu, f);
    if (lane == 0) s_cnt[cw] = __popc(m);
    named_sync(bar, kFinishHalf);
    uint32_t off = base, total = base;
#pragma unroll
    for (int ww = 0; ww < kFinishHalf / kWarp; ++ww) {
      off += ww < cw ? s_cnt[ww] : 0u;
      total += s_cnt[ww];
    }
    if (f) {
      const uint32_t pos = off + __popc(m & ((1u << lane) - 1u));
      p.idx[pos] = nr;
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (b < B) p.a_val[(size_t)b * h + pos] = av[b];
    }
    base = total;
    named_sync(bar, kFinishHalf);
    load_pass(w0 + kFinishHalf / kWarp);
  }
  if (blockIdx.x == gridDim.x - 1 && ct == 0) *p.count = (int32_t)base;
}

// The end phase, called by every thread of the CTA (blockDim.x >= 2 * kFinishHalf) once every CTA's
// partial output is in the accumulators and every keep flag is written (after the meeting below, or
// in a kernel that follows the one that wrote them).  Threads [0, kFinishHalf) write out (the sum of
// the accumulators, plus the old out when accumulating) over an equal share of the columns and
// clear the accumulators for the next launch; threads [kFinishHalf, 2 kFinishHalf) compact idx /
// a_val / count from the keep flags (compact_flags, named barrier 2).
template <int NB>
__device__ void fused_finish_work(const FusedArgs& p, int n_rows, uint32_t* s_cnt) {
  const int tid = threadIdx.x;
  const int B = p.B, d = p.d;
  if (tid < kFinishHalf) {
    const int n4 = B * d / 4;
    const int i0 = (int)((long long)n4 * blockIdx.x / gridDim.x);
    const int i1 = (int)((long long)n4 * (blockIdx.x + 1) / gridDim.x);
    for (int i = i0 + tid; i < i1; i += kFinishHalf) {
      float4 s4[kFusedAccCopies];
#pragma unroll
      for (int c = 0; c < kFusedAccCopies; ++c)
        s4[c] = __ldcg(reinterpret_cast<const float4*>(p.facc + (size_t)c * B * d) + i);
      float4 t4 = s4[0];
#pragma unroll
      for (int c = 1; c < kFusedAccCopies; ++c) {
        t4.x += s4[c].x;
        t4.y += s4[c].y;
        t4.z += s4[c].z;
        t4.w += s4[c].w;
      }
      if (p.out_mode == CSFFN_OUT_BF16) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(t4.x, t4.y), hi = __floats2bfloat162_rn(t4.z, t4.w);
        uint2 pk;
        pk.x = *reinterpret_cast<uint32_t*>(&lo);
        pk.y = *reinterpret_cast<uint32_t*>(&hi);
        reinterpret_cast<uint2*>(p.out)[i] = pk;
      } else {
        float4* of = reinterpret_cast<float4*>(p.out) + i;
        if (p.out_mode == CSFFN_OUT_F32_ACCUMULATE) {
          const float4 prev = *of;
          t4.x += prev.x;
          t4.y += prev.y;
          t4.z += prev.z;
          t4.w += prev.w;
        }
        *of = t4;
      }
#pragma unroll
      for (int c = 0; c < kFusedAccCopies; ++c)
        __stcg(reinterpret_cast<float4*>(p.facc + (size_t)c * B * d) + i, make_float4(0.f, 0.f, 0.f, 0.f));
    }
  } else if (tid < 2 * kFinishHalf) {
    compact_flags<NB>(p, n_rows, s_cnt, tid - kFinishHalf, 2);
  }
}

// One grid-wide meeting, then the end phase.  The arrival counter wraps to zero on the last arrival
// (atomicInc) and the others wait for that zero, so it is ready for the next launch without a
// reset; the last CTA also clears the ticket counter and the predictor's count (every CTA has drawn
// its last ticket and passed that count before it arrives).  Only for cooperative launches: all
// CTAs are co-resident, so the meeting cannot wait on a CTA that has not started.
template <int NB>
__device__ void fused_finish(const FusedArgs& p, int n_rows, uint32_t* s_cnt) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (atomicInc(&p.ctl[kCtlDone], gridDim.x - 1u) == gridDim.x - 1u) {
      for (int i = 0; i < kTicketCounters; ++i) {
        p.tickets[i * kCounterStride] = 0u;
        p.tickets[i * kCounterStride + 1] = 0u;
      }
      p.ctl[kCtlY] = 0u;
      __threadfence();  // with the counter read above: the other CTAs' sums are visible here
    } else {
      wait_zero(&p.ctl[kCtlDone], p.err);
    }
  }
  __syncthreads();
  fused_finish_work<NB>(p, n_rows, s_cnt);
}

}  // namespace csffn
