// Streaming version of the fused gate GEMV + threshold + compaction kernel.
//
// Same result as gate_compact_kernel (gate.cu): "CATS: Contextually-Aware Thresholding for
// Sparsity in Large Language Models", abstract (gate GEMV fused with the compare and a flag), and
// "SVD Contextual Sparsity Predictors for Fast LLM Inference", Fig. 1 and Fig. 3 (predictor
// compare; gate on the predicted set).  Organisation, one CTA per SM:
//
//   warps 0-15 (streaming): CTA b owns chunks b, b + G, b + 2G, ... (16 rows each, G = grid size;
//          every chunk is the same amount of work, so a static assignment balances as well as
//          tickets would, without their round trips).  Warp w reduces row w of each of its CTA's
//          chunks against the tokens staged in shared memory.  A row is read as two halves of
//          16-byte vectors held in registers, double-buffered across rows: the loads of the next
//          row's half are issued before the current half is consumed, so each warp keeps a whole
//          row (8 KB at d = 4096) in flight without pause.  After a row the warp applies bias,
//          activation and threshold, writes the result into the chunk's result buffer, and the
//          last warp to finish a chunk publishes its count (the look-back aggregate) at once.
//   warp 16 (compaction): per chunk, ballots the keep flags, finds the output offset by the
//          warp-parallel decoupled look-back (common.cuh) over epoch-tagged status words,
//          publishes the inclusive prefix and scatters idx and a_val, while the streaming warps
//          are already on later chunks.
//
// The look-back only waits on chunks owned by CTAs of this grid, all resident at once (one CTA
// per SM, grid <= SM count, launched after the previous kernel on the stream has finished), and
// every wait is bounded.
#include "common.cuh"
#include "gemv.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace csffn {

constexpr int kStreamWarps = 16;
constexpr int kStreamThreads = (kStreamWarps + 1) * kWarp;
constexpr int kStreamBufs = 8;  // chunk result buffers
static_assert(kStreamWarps == kChunkRows, "one row of every chunk per streaming warp");

template <int NB>
struct StreamShared {
  uint64_t chunk_full[kStreamBufs];
  uint64_t chunk_empty[kStreamBufs];
  float val[kStreamBufs][kChunkRows][NB];
  uint32_t keep[kStreamBufs][kChunkRows];
  uint32_t cnt[kStreamBufs];
  uint32_t arrived[kStreamBufs];
  int abort;
  uint32_t epoch;
};

// 16-byte vectors per lane per pipeline unit, and units in flight per warp (the ring holds one
// more: the unit being consumed).
template <int NB> struct StreamU { static constexpr int value = NB <= 4 ? 4 : 2; };
template <int NB> struct StreamInFlight { static constexpr int value = NB <= 2 ? 5 : (NB <= 8 ? 3 : 2); };

template <typename WT, typename XT, int NB, int MODE>
__global__ void __launch_bounds__(kStreamThreads, 1) gate_stream_kernel(const GateArgs p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ StreamShared<NB> sh;
  constexpr int EPV = Vec<WT>::N;
  constexpr int U = StreamU<NB>::value;
  constexpr int kInFlight = StreamInFlight<NB>::value;
  constexpr int nstage = kInFlight + 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.K;
  const size_t x_bytes = align_up((size_t)NB * K * sizeof(XT), 16);
  XT* xs = reinterpret_cast<XT*>(smem_raw);

  if (tid == 0) {
    for (int i = 0; i < kStreamBufs; ++i) {
      mbar_init(&sh.chunk_full[i], kStreamWarps);
      mbar_init(&sh.chunk_empty[i], 1);
      sh.cnt[i] = 0u;
      sh.arrived[i] = 0u;
    }
    sh.abort = 0;
    sh.epoch = *reinterpret_cast<volatile uint32_t*>(&p.ctl->epoch);
    fence_mbar_init();
  }
  stage_tokens<XT, NB>(xs, reinterpret_cast<const XT*>(p.x), p.B, K);
  __syncthreads();

  const int n_rows = p.cand_count ? min(max(*p.cand_count, 0), p.h) : p.h;
  const int n_chunks = (n_rows + kChunkRows - 1) / kChunkRows;
  const int G = gridDim.x;
  const int my_chunks = n_chunks > (int)blockIdx.x ? (n_chunks - 1 - (int)blockIdx.x) / G + 1 : 0;
  const uint32_t epoch = sh.epoch;
  volatile int* abort = &sh.abort;
  auto row_of = [&](int j) -> int {
    int r = p.cand_idx ? p.cand_idx[j] : j;
    return ((unsigned)r < (unsigned)p.h) ? r : 0;
  };
  if (blockIdx.x == 0 && n_chunks == 0 && tid == 0) *p.count = 0;  // empty row set

  if (warp < kStreamWarps) {
    // ------------------------------------------------------------------ streaming warps
    // A row is streamed as units of U 16-byte vectors per lane (U * 512 bytes per warp).  Units
    // go through a per-warp ring of S slots in shared memory by cp.async; each lane consumes only
    // the vectors it copied itself, so cp.async.wait_group is the only synchronisation and S
    // units (S * U * 512 bytes) stay in flight per warp while one is consumed.
    const WT* W = reinterpret_cast<const WT*>(p.W);
    const int NV = K / EPV;                             // 16-byte vectors per row
    const int upr = (NV + kWarp * U - 1) / (kWarp * U);  // units per row
    const int total = my_chunks * upr;
    uint4* ring = reinterpret_cast<uint4*>(smem_raw + x_bytes) + (size_t)warp * nstage * U * kWarp;
    auto row_ptr = [&](int k, bool& ok) -> const WT* {
      const int j = ((int)blockIdx.x + k * G) * kChunkRows + warp;
      ok = k < my_chunks && j < n_rows;
      return W + (size_t)(ok ? row_of(j) : 0) * K;
    };
    // issue unit t (row t / upr, vectors of group t % upr) into slot t % nstage
    int issue_k = -1;
    const WT* issue_row = W;
    bool issue_ok = false;
    auto issue = [&](int t, uint32_t after) {
      if (t < total) {
        const int k = t / upr;
        if (k != issue_k) {
          issue_k = k;
          issue_row = row_ptr(k, issue_ok);
        }
        uint4* slot = ring + (size_t)(t % nstage) * U * kWarp;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = ((t % upr) * U + u) * kWarp + lane;
          if (issue_ok && v < NV) cp_async16(slot + u * kWarp + lane, issue_row + (size_t)v * EPV, after);
        }
      }
      cp_async_commit();  // one group per unit, possibly empty, keeps the group count uniform
    };
    for (int t = 0; t < nstage - 1; ++t) issue(t, 0u);
    float acc[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b] = 0.f;
    for (int t = 0; t < total; ++t) {
      issue(t + nstage - 1, __float_as_uint(acc[0]));
      cp_async_wait<kInFlight>();  // unit t has landed (only later units may be pending)
      const int k = t / upr;
      const int ut = t % upr;
      const uint4* slot = ring + (size_t)(t % nstage) * U * kWarp;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = (ut * U + u) * kWarp + lane;
        if (v < NV) {
          float wf[EPV];
          unpack(slot[u * kWarp + lane], wf);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            float xf[EPV];
            load_x<EPV>(xs + (size_t)b * K + (size_t)v * EPV, xf);
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc[b] = fmaf(wf[e], xf[e], acc[b]);
          }
        }
      }
      if (ut == upr - 1) {
        // ---- row k finished: reduce, threshold, hand to the chunk buffer
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = warp_sum(acc[b]);
        const int cb = k % kStreamBufs;
        if (!mbar_wait(&sh.chunk_empty[cb], ((k / kStreamBufs) & 1) ^ 1, p.err, abort)) break;
        const int c = (int)blockIdx.x + k * G;
        const int j = c * kChunkRows + warp;
        if (lane == 0) {
          bool keep_any = false;
          if (j < n_rows) {
            const int i = row_of(j);
            const float beta = p.bias ? p.bias[i] : 0.f;
            const float thr = MODE == kModePred ? p.tau[i] : p.t;
#pragma unroll
            for (int b = 0; b < NB; ++b) {
              if (b < p.B) {
                const float z = acc[b] + beta;
                bool kb;
                if (MODE == kModeCats) {
                  const float a = gate_act(z, p.act);
                  kb = fabsf(a) > thr;
                  sh.val[cb][warp][b] = kb ? a : 0.f;
                } else {
                  kb = z > thr;
                }
                keep_any |= kb;
              }
            }
          }
          sh.keep[cb][warp] = keep_any ? 1u : 0u;
          if (keep_any) atomicAdd(&sh.cnt[cb], 1u);
          __threadfence_block();
          if (atomicAdd(&sh.arrived[cb], 1u) == (uint32_t)(kStreamWarps - 1)) {
            // last row of the chunk: publish its aggregate now (chunk 0: its inclusive prefix)
            const uint32_t agg = atomicAdd(&sh.cnt[cb], 0u);
            st_status(&p.status[c], status_word(epoch, c == 0 ? kFlagInclusive : kFlagAggregate, agg));
          }
          mbar_arrive(&sh.chunk_full[cb]);
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = 0.f;
      }
    }
    cp_async_wait<0>();  // nothing of ours may still be landing when the CTA exits
  } else {
    // ------------------------------------------------------------------ compaction warp
    for (int k = 0; k < my_chunks; ++k) {
      const int cb = k % kStreamBufs;
      if (!mbar_wait(&sh.chunk_full[cb], (k / kStreamBufs) & 1, p.err, abort)) break;
      const int c = (int)blockIdx.x + k * G;
      const bool keep = lane < kChunkRows && sh.keep[cb][lane] != 0u;
      const uint32_t mask = __ballot_sync(0xffffffffu, keep);
      const uint32_t agg = __popc(mask);
      const uint32_t prefix = warp_lookback(p.status, c, epoch, agg, p.err, lane, /*agg_published=*/true);
      if (keep) {
        const uint32_t pos = prefix + __popc(mask & ((1u << lane) - 1u));
        if (pos < (uint32_t)p.h) {
          p.idx[pos] = row_of(c * kChunkRows + lane);
          if (MODE == kModeCats) {
#pragma unroll
            for (int b = 0; b < NB; ++b)
              if (b < p.B) p.a_val[(size_t)b * p.h + pos] = sh.val[cb][lane][b];
          }
        }
      }
      if (c == n_chunks - 1 && lane == 0) *p.count = (int32_t)(prefix + agg);
      __syncwarp();
      if (lane == 0) {
        sh.cnt[cb] = 0u;
        sh.arrived[cb] = 0u;
        mbar_arrive(&sh.chunk_empty[cb]);
      }
    }
  }

  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t prev = atomicAdd(&p.ctl->done, 1u);
    if (prev == gridDim.x - 1) {
      p.ctl->done = 0u;
      p.ctl->epoch = epoch + 1u;
      __threadfence();
    }
  }
}

template <int NB>
static size_t stream_ring_bytes() {
  return (size_t)kStreamWarps * (StreamInFlight<NB>::value + 1) * StreamU<NB>::value * kWarp * 16;
}

template <typename WT, typename XT, int NB, int MODE>
static cudaError_t launch_stream_t(const GateArgs& a, cudaStream_t s) {
  auto kern = gate_stream_kernel<WT, XT, NB, MODE>;
  const size_t smem = align_up((size_t)NB * a.K * sizeof(XT), 16) + stream_ring_bytes<NB>();
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int max_chunks = (a.h + kChunkRows - 1) / kChunkRows;
  int grid = sm_count();
  if (grid > max_chunks) grid = max_chunks;
  if (grid < 1) grid = 1;
  kern<<<grid, kStreamThreads, smem, s>>>(a);
  return cudaGetLastError();
}

bool gate_stream_supported(int K, int B, int wdtype, bool x_f32) {
  const size_t xs = x_f32 || wdtype == CSFFN_F32 ? 4 : 2;
  const int t = batch_tier(B);
  const size_t ring = t == 1 ? stream_ring_bytes<1>() : t == 2 ? stream_ring_bytes<2>() : t == 4 ? stream_ring_bytes<4>()
                    : t == 8 ? stream_ring_bytes<8>() : stream_ring_bytes<16>();
  return align_up((size_t)t * K * xs, 16) + ring <= 220 * 1024;
}

template <typename WT, typename XT, int MODE>
static cudaError_t launch_stream_nb(const GateArgs& a, cudaStream_t s) {
  switch (batch_tier(a.B)) {
    case 1: return launch_stream_t<WT, XT, 1, MODE>(a, s);
    case 2: return launch_stream_t<WT, XT, 2, MODE>(a, s);
    case 4: return launch_stream_t<WT, XT, 4, MODE>(a, s);
    case 8: return launch_stream_t<WT, XT, 8, MODE>(a, s);
    default: return launch_stream_t<WT, XT, 16, MODE>(a, s);
  }
}

cudaError_t launch_gate_stream(const GateArgs& a, int wdtype, bool x_f32, int mode, cudaStream_t s) {
  if (wdtype == CSFFN_F32) {
    return mode == kModeCats ? launch_stream_nb<float, float, kModeCats>(a, s)
                             : launch_stream_nb<float, float, kModePred>(a, s);
  }
  if (x_f32) {
    return mode == kModeCats ? launch_stream_nb<bf16, float, kModeCats>(a, s)
                             : launch_stream_nb<bf16, float, kModePred>(a, s);
  }
  return mode == kModeCats ? launch_stream_nb<bf16, bf16, kModeCats>(a, s)
                           : launch_stream_nb<bf16, bf16, kModePred>(a, s);
}

}  // namespace csffn
