// One-launch CATS decode step: gate + threshold + up (phase A), grid barrier, gathered down
// projection and active-list compaction (phase B).
//
// "CATS: Contextually-Aware Thresholding for Sparsity in Large Language Models", abstract: the
// gate GEMV, the compare and the flag-gated GEMV of its custom kernel; here all of one decode step
// of an FFN layer runs in a single persistent grid.  A decode step reads a few hundred MB, and a
// separate launch per stage pays its ramp-up and tail every time (measured on B200: a bare
// 45 MB row stream reaches 3.6 TB/s, a 720 MB one 6.8 TB/s), so the stages share one launch.
//
// Phase A: warp per neuron row; rows come one at a time from ticket counters (an up row follows
//   only a kept gate row, so static shares would be uneven).  The warp reduces W_gate[r] against
//   the tokens staged in shared memory, applies bias, activation and the threshold per token,
//   writes the keep flag and the kept activations, and if any token keeps the row streams W_up[r]
//   at once and writes v[b, r] = a[b, r] * u[b, r].  It then counts the row (and whether it was
//   kept) for its neuron range with a release increment.
// Phase B (dataflow, no grid barrier): a CTA whose warps find no more rows takes phase-B tiles in
//   range order from a tile counter.  Tile (range q, slice s) waits (bounded) until every row of
//   range q has been counted, then its warps ballot the range's flags word by word and stream the
//   slice (16 bytes per lane) of each kept row of W_down^T, accumulating v[b, r] * W_down^T[r, s]
//   in registers; warps reduce in shared memory, the tile writes one partial per (range, token,
//   column), and the last tile of a slice sums the partials in range order (deterministic).  The
//   slice-0 tile of a range also writes the range's part of idx / a_val at the offset given by the
//   kept counts of the earlier ranges (once those are complete), and the last range writes count.
//   Ranges complete roughly in order (tickets hand out rows in increasing order), so phase B of
//   the early ranges runs while phase A finishes the late rows.
// Every row is owned by a running warp before any CTA waits on a range, so nothing here depends on
// CTAs that have not started; all waits are bounded.  The last CTA to finish resets the counters.
#include "common.cuh"
#include "gemv.cuh"
#include "kernels.h"

namespace csffn {

constexpr int kFusedThreads = 256;
constexpr int kFusedWarps = kFusedThreads / kWarp;
constexpr int kFusedWordBlock = 256;  // 32-neuron words compacted per pass in phase B
// Row tickets: counter i hands out rows i, i + kTicketCounters, ... to the warps with
// gw % kTicketCounters == i; the counters sit kTicketStride words (128 bytes) apart so that the
// warps' atomics spread over L2 instead of serialising on one address.
constexpr int kTicketCounters = 64;
constexpr int kTicketStride = 32;

__device__ __forceinline__ uint8_t ld_cg_u8(const uint8_t* p) { return __ldcg(p); }


__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ uint32_t atom_add_release_u32(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.add.release.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Bounded wait until *p >= target (acquire).  Returns false after a second (error recorded).
__device__ __forceinline__ bool wait_at_least(const uint32_t* p, uint32_t target, uint32_t* err) {
  if (ld_acquire_u32(p) >= target) return true;
  const uint64_t t0 = globaltimer_now();
  while (ld_acquire_u32(p) < target) {
    if (globaltimer_now() - t0 > 1000000000ull) {
      atomicOr(err, kDevErrTimeout);
      return false;
    }
    __nanosleep(64);
  }
  return true;
}

// Dot products of one row with the staged tokens: acc[b] += W[row] . x_b (this lane's share).
template <typename WT, int NB, int U>
__device__ __forceinline__ void row_dot(const WT* __restrict__ row, const WT* __restrict__ xs, int K, int lane,
                                        float (&acc)[NB]) {
  constexpr int EPV = Vec<WT>::N;
  const int NV = K / EPV;
  for (int v0 = lane; v0 < NV; v0 += kWarp * U) {
    uint4 w[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * kWarp;
      w[u] = v < NV ? ld_stream(row + (size_t)v * EPV) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * kWarp;
      if (v < NV) {
        float wf[EPV];
        unpack(w[u], wf);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float xf[EPV];
          load_x<EPV>(xs + (size_t)b * K + (size_t)v * EPV, xf);
#pragma unroll
          for (int e = 0; e < EPV; ++e) acc[b] = fmaf(wf[e], xf[e], acc[b]);
        }
      }
    }
  }
}

// Rows of one 32-neuron word consumed per phase-B batch (two batches in flight per warp).
template <int NB> struct FusedDownU { static constexpr int value = NB <= 2 ? 4 : 2; };

// Range (of p.ranges) holding 32-neuron word w when n_words words are split evenly.
__device__ __forceinline__ int range_of_word(int w, int n_words, int ranges) {
  return (int)(((long long)(w + 1) * ranges - 1) / n_words);
}

// Fused control words (FusedArgs::ctl, 32-bit each): row-ticket counters sit elsewhere.
constexpr int kCtlTile = 0;     // phase-B tile counter
constexpr int kCtlExit = 1;     // CTAs finished
constexpr int kCtlWords = 2;

template <typename WT, int NB>
__global__ void __launch_bounds__(kFusedThreads, 4) cats_fused_kernel(const FusedArgs p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  constexpr int EPV = Vec<WT>::N;
  constexpr int SW = kWarp * EPV;  // columns per phase-B slice
  constexpr int U = GemvUnroll<NB>::value;
  constexpr int UD = FusedDownU<NB>::value;
  __shared__ float red[kFusedWarps][SW];
  __shared__ uint32_t s_wcnt[kFusedWordBlock];
  __shared__ uint32_t s_offset;
  __shared__ int s_tile;
  __shared__ bool s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = p.d, h = p.h;
  const int n_words = (h + kWarp - 1) / kWarp;
  WT* xs = reinterpret_cast<WT*>(smem_raw);
  const WT* Wg = reinterpret_cast<const WT*>(p.W_gate);
  const WT* Wu = reinterpret_cast<const WT*>(p.W_up);
  const WT* Wd = reinterpret_cast<const WT*>(p.W_down_t);
  uint32_t* range_done = p.range_cnt;                  // rows counted per range
  uint32_t* range_kept = p.range_cnt + kMaxRowRanges;  // kept rows per range

  // ---------------------------------------------------------------- phase A: gate + up
  stage_tokens<WT, NB>(xs, reinterpret_cast<const WT*>(p.x), p.B, d);
  __syncthreads();
  // Rows come one at a time from ticket counters, so the data-dependent up rows balance out; the
  // next ticket is fetched while the current row streams.
  // A warp whose counter runs dry marks it exhausted (word 1 of the counter's line) and moves to a
  // counter that still has rows; it leaves phase A only when all counters are dry, so by then every
  // row belongs to a running warp.
  const int gw = blockIdx.x * kFusedWarps + warp;
  int tc = gw % kTicketCounters;
  auto take = [&](int c) -> int {  // lane 0: next row of counter c (>= h when it is dry)
    return c + kTicketCounters * (int)atomicAdd(p.tickets + c * kTicketStride, 1u);
  };
  int r_next = 0;
  if (lane == 0) r_next = take(tc);
  r_next = __shfl_sync(0xffffffffu, r_next, 0);
  for (;;) {
    if (r_next >= h) {
      if (lane == 0) p.tickets[tc * kTicketStride + 1] = 1u;
      const bool dry_lo = __ldcg(p.tickets + lane * kTicketStride + 1) != 0u;
      const bool dry_hi = __ldcg(p.tickets + (lane + kWarp) * kTicketStride + 1) != 0u;
      const uint32_t live_lo = __ballot_sync(0xffffffffu, !dry_lo), live_hi = __ballot_sync(0xffffffffu, !dry_hi);
      if (!live_lo && !live_hi) break;
      tc = live_lo ? __ffs(live_lo) - 1 : kWarp + __ffs(live_hi) - 1;
      if (lane == 0) r_next = take(tc);
      r_next = __shfl_sync(0xffffffffu, r_next, 0);
      continue;
    }
    const int r = r_next;
    if (lane == 0) r_next = take(tc);
    float acc[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b] = 0.f;
    row_dot<WT, NB, U>(Wg + (size_t)r * d, xs, d, lane, acc);
    const float beta = p.bias ? p.bias[r] : 0.f;
    float a[NB];
    bool any = false;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float z = warp_sum(acc[b]) + beta;
      const float ab = gate_act(z, p.act);
      const bool kb = b < p.B && fabsf(ab) > p.t;
      a[b] = kb ? ab : 0.f;
      any |= kb;
    }
    if (lane == 0) {
      p.flags[r] = any ? 1 : 0;
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (b < p.B) p.afull[(size_t)b * h + r] = a[b];
    }
    if (any) {
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[b] = 0.f;
      row_dot<WT, NB, U>(Wu + (size_t)r * d, xs, d, lane, acc);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float u = warp_sum(acc[b]);
        if (lane == 0 && b < p.B) p.v[(size_t)b * h + r] = a[b] * u;
      }
    }
    if (lane == 0) {
      const int q = range_of_word(r / kWarp, n_words, p.ranges);
      if (any) atomicAdd(&range_kept[q], 1u);
      atom_add_release_u32(&range_done[q], 1u);  // the row's outputs are visible before it counts
    }
    r_next = __shfl_sync(0xffffffffu, r_next, 0);
  }
  __syncthreads();

  // ---------------------------------------------------------------- phase B: down + compaction
  const int n_tiles = p.slices * p.ranges;
  for (;;) {
    if (tid == 0) s_tile = (int)atomicAdd(&p.ctl[kCtlTile], 1u);
    __syncthreads();
    const int tile = s_tile;
    __syncthreads();
    if (tile >= n_tiles) break;
    const int q = tile / p.slices, slice = tile % p.slices;  // range-major: early ranges first
    const int w0 = (int)((long long)n_words * q / p.ranges), w1 = (int)((long long)n_words * (q + 1) / p.ranges);
    const int rows_q = min(h, w1 * kWarp) - w0 * kWarp;
    if (tid == 0) wait_at_least(&range_done[q], (uint32_t)rows_q, p.err);
    __syncthreads();
    const int c0 = slice * SW + lane * EPV;
    const bool col_ok = c0 < d;
    float acc[NB][EPV];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[b][e] = 0.f;

    // Words w0 + warp, w0 + warp + 8, ...: ballot the word's flags, then stream its kept rows in
    // batches of UD, two batches in flight; the next word's flags and v are fetched ahead.
    auto fetch_word = [&](int w, uint32_t& m, float (&vv)[NB]) {
      const int r = w * kWarp + lane;
      const bool f = w < w1 && r < h && ld_cg_u8(p.flags + r) != 0;
      m = __ballot_sync(0xffffffffu, f);
#pragma unroll
      for (int b = 0; b < NB; ++b) vv[b] = (f && b < p.B) ? __ldcg(p.v + (size_t)b * h + r) : 0.f;
    };
    auto fill = [&](int w, uint32_t& mm, uint4 (&wv)[UD], int (&src)[UD]) {
#pragma unroll
      for (int u = 0; u < UD; ++u) {
        src[u] = mm ? __ffs(mm) - 1 : -1;
        mm &= mm - 1u;
        const int row = w * kWarp + (src[u] < 0 ? 0 : src[u]);
        wv[u] = (src[u] >= 0 && col_ok) ? ld_stream(Wd + (size_t)row * d + c0) : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    auto consume = [&](const uint4 (&wv)[UD], const int (&src)[UD], const float (&vv)[NB]) {
#pragma unroll
      for (int u = 0; u < UD; ++u) {
        float wf[EPV];
        unpack(wv[u], wf);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float vb = __shfl_sync(0xffffffffu, vv[b], src[u] < 0 ? 0 : src[u]);
          if (src[u] >= 0) {
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc[b][e] = fmaf(vb, wf[e], acc[b][e]);
          }
        }
      }
    };
    {
      uint32_t m_cur, m_nxt;
      float v_cur[NB], v_nxt[NB];
      int w = w0 + warp;
      fetch_word(w, m_cur, v_cur);
      for (; w < w1; w += kFusedWarps) {
        fetch_word(w + kFusedWarps, m_nxt, v_nxt);
        uint32_t mm = m_cur;
        uint4 wa[UD], wb[UD];
        int sa[UD], sb[UD];
        fill(w, mm, wa, sa);
        while (sa[0] >= 0) {
          fill(w, mm, wb, sb);
          consume(wa, sa, v_cur);
          if (sb[0] < 0) break;
          fill(w, mm, wa, sa);
          consume(wb, sb, v_cur);
        }
        m_cur = m_nxt;
#pragma unroll
        for (int b = 0; b < NB; ++b) v_cur[b] = v_nxt[b];
      }
    }

    // cross-warp reduction, one partial row per token
    const int col = slice * SW + tid;
    for (int b = 0; b < p.B && b < NB; ++b) {
#pragma unroll
      for (int bb = 0; bb < NB; ++bb)
        if (bb == b)
#pragma unroll
          for (int e = 0; e < EPV; ++e) red[warp][lane * EPV + e] = acc[bb][e];
      __syncthreads();
      if (tid < SW && col < d) {
        float sum = 0.f;
#pragma unroll
        for (int ww = 0; ww < kFusedWarps; ++ww) sum += red[ww][tid];
        p.partial[((size_t)q * p.B + b) * d + col] = sum;
      }
      __syncthreads();
    }

    // compacted outputs for this range (slice-0 tile), at the offset of the earlier ranges' kept rows
    if (slice == 0) {
      if (tid == 0) {
        uint32_t before = 0;
        for (int qq = 0; qq < q; ++qq) {
          const int a0 = (int)((long long)n_words * qq / p.ranges), a1 = (int)((long long)n_words * (qq + 1) / p.ranges);
          wait_at_least(&range_done[qq], (uint32_t)(min(h, a1 * kWarp) - a0 * kWarp), p.err);
          before += ld_acquire_u32(&range_kept[qq]);
        }
        s_offset = before;
      }
      __syncthreads();
      uint32_t off = s_offset;
      for (int wb = w0; wb < w1; wb += kFusedWordBlock) {
        const int we = min(w1, wb + kFusedWordBlock);
        for (int w = wb + warp; w < we; w += kFusedWarps) {
          const int r = w * kWarp + lane;
          const bool f = r < h && ld_cg_u8(p.flags + r) != 0;
          const uint32_t m = __ballot_sync(0xffffffffu, f);
          if (lane == 0) s_wcnt[w - wb] = __popc(m);
        }
        __syncthreads();
        if (tid == 0) {
          uint32_t run = off;
          for (int w = wb; w < we; ++w) {
            const uint32_t c = s_wcnt[w - wb];
            s_wcnt[w - wb] = run;
            run += c;
          }
          s_offset = run;
        }
        __syncthreads();
        for (int w = wb + warp; w < we; w += kFusedWarps) {
          const int r = w * kWarp + lane;
          const bool f = r < h && ld_cg_u8(p.flags + r) != 0;
          const uint32_t m = __ballot_sync(0xffffffffu, f);
          if (f) {
            const uint32_t pos = s_wcnt[w - wb] + __popc(m & ((1u << lane) - 1u));
            if (pos < (uint32_t)h) {
              p.idx[pos] = r;
#pragma unroll
              for (int b = 0; b < NB; ++b)
                if (b < p.B) p.a_val[(size_t)b * h + pos] = __ldcg(p.afull + (size_t)b * h + r);
            }
          }
        }
        off = s_offset;
        __syncthreads();
      }
      if (q == p.ranges - 1 && tid == 0) *p.count = (int32_t)off;
    }

    // the last tile of this slice sums the partials in range order
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&p.slice_ctr[slice], 1u) == (uint32_t)(p.ranges - 1);
    __syncthreads();
    if (s_last) {
      __threadfence();
      if (tid < SW && col < d) {
        for (int b = 0; b < p.B; ++b) {
          float sum = 0.f;
          for (int rr = 0; rr < p.ranges; ++rr) sum += __ldcg(p.partial + ((size_t)rr * p.B + b) * d + col);
          const size_t o = (size_t)b * d + col;
          if (p.out_mode == CSFFN_OUT_BF16)
            reinterpret_cast<bf16*>(p.out)[o] = __float2bfloat16_rn(sum);
          else if (p.out_mode == CSFFN_OUT_F32)
            reinterpret_cast<float*>(p.out)[o] = sum;
          else
            reinterpret_cast<float*>(p.out)[o] += sum;
        }
      }
      if (tid == 0) p.slice_ctr[slice] = 0u;
    }
  }

  // the last CTA out resets every counter for the next launch
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(&p.ctl[kCtlExit], 1u) == gridDim.x - 1) {
      for (int i = 0; i < kTicketCounters; ++i) {
        p.tickets[i * kTicketStride] = 0u;
        p.tickets[i * kTicketStride + 1] = 0u;
      }
      for (int i = 0; i < 2 * kMaxRowRanges; ++i) p.range_cnt[i] = 0u;
      p.ctl[kCtlTile] = 0u;
      p.ctl[kCtlExit] = 0u;
      __threadfence();
    }
  }
}

template <typename WT, int NB>
static cudaError_t fused_t(FusedArgs a, cudaStream_t s) {
  auto kern = cats_fused_kernel<WT, NB>;
  const size_t smem = (size_t)NB * a.d * sizeof(WT);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  int occ = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kFusedThreads, smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  const int grid = sm_count() * occ;
  constexpr int SW = kWarp * Vec<WT>::N;
  a.slices = (a.d + SW - 1) / SW;
  if (a.slices > grid || a.slices > kMaxSlices) return cudaErrorInvalidConfiguration;
  const int n_words = (a.h + kWarp - 1) / kWarp;
  a.ranges = grid / a.slices;
  if (a.ranges > kMaxRowRanges) a.ranges = kMaxRowRanges;
  if (a.ranges > n_words) a.ranges = n_words;
  if (a.ranges < 1) a.ranges = 1;
  kern<<<grid, kFusedThreads, smem, s>>>(a);
  return cudaGetLastError();
}

bool cats_fused_supported(int d, int B, int wdtype) {
  const size_t es = wdtype == CSFFN_F32 ? 4 : 2;
  return B >= 1 && B <= 4 && (size_t)batch_tier(B) * d * es <= 48 * 1024;
}

cudaError_t launch_cats_fused(const FusedArgs& a, int wdtype, cudaStream_t s) {
  const int t = batch_tier(a.B);
  if (wdtype == CSFFN_F32) {
    switch (t) {
      case 1: return fused_t<float, 1>(a, s);
      case 2: return fused_t<float, 2>(a, s);
      default: return fused_t<float, 4>(a, s);
    }
  }
  switch (t) {
    case 1: return fused_t<bf16, 1>(a, s);
    case 2: return fused_t<bf16, 2>(a, s);
    default: return fused_t<bf16, 4>(a, s);
  }
}

}  // namespace csffn
