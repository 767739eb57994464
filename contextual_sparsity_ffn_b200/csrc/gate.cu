// Fused gate GEMV + activation + threshold + union over tokens + active-index compaction.
//
// "CATS: Contextually-Aware Thresholding for Sparsity in Large Language Models", abstract: the
// gate activations below a threshold are zeroed, and the custom kernel fuses the gate GEMV with
// the compare and a flag.  "SVD Contextual Sparsity Predictors for Fast LLM Inference", Fig. 1
// (predictor output against per-neuron thresholds) and Fig. 3 (the gate runs only on the
// predicted set) reuse the same kernel with a candidate list or in predictor mode.
//
// Work is split into chunks of kChunkRows consecutive rows (of 0..h-1, or of the candidate
// list).  CTAs take chunks in order from a ticket counter, so every chunk's predecessors are
// already running; after its GEMV a CTA ballots its chunk's keep flags, publishes the chunk
// count and finds its output offset by a decoupled look-back over the predecessors' status
// words (each tagged with the launch epoch, so stale words from earlier launches never match).
// Output indices therefore come out ascending without a second pass or a host round trip.
#include "common.cuh"
#include "gemv.cuh"
#include "kernels.h"

namespace csffn {

constexpr int kGateThreads = 256;
constexpr int kGateWarps = kGateThreads / kWarp;
constexpr int kGateRowsPerWarp = kChunkRows / kGateWarps;
static_assert(kChunkRows <= kWarp, "one ballot per chunk");
static_assert(kGateRowsPerWarp * kGateWarps == kChunkRows, "chunk tiles the warps");

template <typename WT, typename XT, int NB, int MODE>
__global__ void __launch_bounds__(kGateThreads) gate_compact_kernel(const GateArgs p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  XT* xs = reinterpret_cast<XT*>(smem_raw);
  __shared__ float s_val[NB][kChunkRows];
  __shared__ uint32_t s_keep[kChunkRows];
  __shared__ int s_ticket;
  __shared__ uint32_t s_epoch;

  constexpr int R = kGateRowsPerWarp;
  constexpr int U = GemvUnroll<NB>::value;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.K;

  stage_tokens<XT, NB>(xs, reinterpret_cast<const XT*>(p.x), p.B, K);
  // Rows considered; a candidate count is clamped to [0, h] so no write can leave the buffers.
  const int n_rows = p.cand_count ? min(max(*p.cand_count, 0), p.h) : p.h;
  const int n_chunks = (n_rows + kChunkRows - 1) / kChunkRows;
  if (tid == 0) s_epoch = *reinterpret_cast<volatile uint32_t*>(&p.ctl->epoch);
  __syncthreads();
  const uint32_t epoch = s_epoch;
  const WT* W = reinterpret_cast<const WT*>(p.W);

  for (;;) {
    if (tid == 0) s_ticket = (int)atomicAdd(&p.ctl->ticket, 1u);
    __syncthreads();
    const int c = s_ticket;
    if (c >= n_chunks) {
      if (c == 0 && tid == 0) *p.count = 0;  // empty row set
      break;
    }

    // ---- GEMV over this warp's rows of the chunk
    const int j0 = c * kChunkRows + warp * R;
    int rowid[R];
    bool valid[R];
    const WT* rp[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = j0 + r;
      valid[r] = j < n_rows;
      rowid[r] = valid[r] ? (p.cand_idx ? p.cand_idx[j] : j) : 0;
      if ((unsigned)rowid[r] >= (unsigned)p.h) rowid[r] = 0;  // malformed candidate: stay in bounds
      rp[r] = W + (size_t)rowid[r] * K;
    }
    float acc[R][NB];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
    rows_dot<WT, XT, NB, R, U>(rp, valid, xs, K, lane, acc);
    warp_reduce_all<R, NB>(acc);

    // ---- activation, threshold, union over tokens (lane r finalises row r)
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (lane == r) {
        bool keep_any = false;
        if (valid[r]) {
          const int i = rowid[r];
          const float beta = p.bias ? p.bias[i] : 0.f;
          const float thr = MODE == kModePred ? p.tau[i] : p.t;
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            if (b < p.B) {
              const float z = acc[r][b] + beta;
              bool k;
              if (MODE == kModeCats) {
                const float a = gate_act(z, p.act);
                k = fabsf(a) > thr;
                s_val[b][warp * R + r] = k ? a : 0.f;
              } else {
                k = z > thr;
              }
              keep_any |= k;
            }
          }
        }
        s_keep[warp * R + r] = keep_any ? 1u : 0u;
      }
    }
    __syncthreads();

    // ---- ballot, decoupled look-back, scatter (warp 0)
    if (warp == 0) {
      const bool keep = lane < kChunkRows && s_keep[lane] != 0u;
      const uint32_t mask = __ballot_sync(0xffffffffu, keep);
      const uint32_t agg = __popc(mask);
      const uint32_t prefix = warp_lookback(p.status, c, epoch, agg, p.err, lane);
      if (keep) {
        const uint32_t pos = prefix + __popc(mask & ((1u << lane) - 1u));
        if (pos < (uint32_t)p.h) {
          const int j = c * kChunkRows + lane;
          p.idx[pos] = p.cand_idx ? p.cand_idx[j] : j;
          if (MODE == kModeCats) {
#pragma unroll
            for (int b = 0; b < NB; ++b)
              if (b < p.B) p.a_val[(size_t)b * p.h + pos] = s_val[b][lane];
          }
        }
      }
      if (c == n_chunks - 1 && lane == 0) *p.count = (int32_t)(prefix + agg);
    }
    __syncthreads();
  }

  // ---- the last CTA out resets the tickets and opens the next epoch
  if (tid == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(&p.ctl->done, 1u);
    if (prev == gridDim.x - 1) {
      p.ctl->ticket = 0u;
      p.ctl->done = 0u;
      p.ctl->epoch = epoch + 1u;
      __threadfence();
    }
  }
}

template <typename WT, typename XT, int NB, int MODE>
static cudaError_t launch_gate_t(const GateArgs& a, cudaStream_t s) {
  auto kern = gate_compact_kernel<WT, XT, NB, MODE>;
  const size_t smem = (size_t)NB * a.K * sizeof(XT);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  int occ = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kGateThreads, smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  const int max_chunks = (a.h + kChunkRows - 1) / kChunkRows;
  int grid = sm_count() * occ;
  if (grid > max_chunks) grid = max_chunks;
  if (grid < 1) grid = 1;
  kern<<<grid, kGateThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename WT, typename XT, int MODE>
static cudaError_t launch_gate_nb(const GateArgs& a, cudaStream_t s) {
  switch (batch_tier(a.B)) {
    case 1: return launch_gate_t<WT, XT, 1, MODE>(a, s);
    case 2: return launch_gate_t<WT, XT, 2, MODE>(a, s);
    case 4: return launch_gate_t<WT, XT, 4, MODE>(a, s);
    case 8: return launch_gate_t<WT, XT, 8, MODE>(a, s);
    default: return launch_gate_t<WT, XT, 16, MODE>(a, s);
  }
}

cudaError_t launch_gate_compact(const GateArgs& a, int wdtype, bool x_f32, int mode, cudaStream_t s) {
  if (wdtype == CSFFN_F32) {
    return mode == kModeCats ? launch_gate_nb<float, float, kModeCats>(a, s)
                             : launch_gate_nb<float, float, kModePred>(a, s);
  }
  if (x_f32) {
    return mode == kModeCats ? launch_gate_nb<bf16, float, kModeCats>(a, s)
                             : launch_gate_nb<bf16, float, kModePred>(a, s);
  }
  return mode == kModeCats ? launch_gate_nb<bf16, bf16, kModeCats>(a, s)
                           : launch_gate_nb<bf16, bf16, kModePred>(a, s);
}

}  // namespace csffn
