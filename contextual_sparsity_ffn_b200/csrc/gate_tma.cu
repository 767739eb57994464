// Warp-specialised, bulk-copy-fed version of the fused gate GEMV + threshold + compaction kernel.
//
// Same result as gate_compact_kernel (gate.cu): "CATS: Contextually-Aware Thresholding for
// Sparsity in Large Language Models", abstract (gate GEMV fused with the compare and a flag), and
// "SVD Contextual Sparsity Predictors for Fast LLM Inference", Fig. 1 and Fig. 3 (predictor
// compare; gate on the predicted set).  What changes is how HBM is kept busy:
//
//   warp 8 (producer, one thread): takes 16-row chunks from the ticket counter and streams their
//          weight rows into a ring of shared-memory slots (RPS rows per slot) with 1-D bulk copies
//          that complete on the slot's "full" mbarrier.  It runs up to the ring's depth ahead of
//          the consumers, independent of everything below.  A bulk copy costs a roughly fixed
//          time per copy on B200, so without a candidate list a slot's RPS = 2 consecutive rows
//          (contiguous in the neuron-major layout) move as one 16 KB copy at d = 4096; gathered
//          candidate rows move one copy per row.
//   warps 0-7 (consumers): warp w takes every slot q with q = w (mod 8), reduces the slot's rows
//          against the tokens staged in shared memory, applies bias, activation and threshold,
//          writes the results into the chunk's result buffer and releases the slot.  The ring
//          depth is a multiple of 8, so slot q % depth always belongs to the same warp, which has
//          finished item q - depth before it waits for item q: a parity wait can never match a
//          phase from two fills earlier.
//          The last consumer warp to finish a chunk publishes the chunk's count (its look-back
//          aggregate) at once, so other CTAs' look-backs never wait on this CTA's compaction warp.
//   warp 9 (compaction): per chunk, ballots the 16 keep flags, finds the output offset by a
//          warp-parallel decoupled look-back over epoch-tagged status words, publishes the
//          inclusive prefix and scatters idx and a_val, while the consumers work on later chunks.
//
// CTA b's first chunk is chunk b; later chunks come from a ticket counter, in increasing order,
// to running CTAs only, and each CTA compacts its chunks in order, so the smallest unfinished
// chunk can always finish: the look-back never waits on work that cannot progress.  The producer
// starts streaming while the consumers stage the tokens.  Every wait is bounded (tma.cuh,
// common.cuh).
#include "common.cuh"
#include "gemv.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace csffn {

constexpr int kTmaConsumers = 8;
constexpr int kTmaThreads = (kTmaConsumers + 2) * kWarp;  // + producer warp + compaction warp
constexpr int kMaxRingSlots = 32;
constexpr int kChunkBufs = 8;
constexpr size_t kTmaSmemBudget = 220 * 1024;

struct GateTmaShared {
  uint64_t full[kMaxRingSlots];
  uint64_t empty[kMaxRingSlots];
  uint64_t chunk_full[kChunkBufs];
  uint64_t chunk_empty[kChunkBufs];
  int slot_chunk[kMaxRingSlots];
  int res_chunk[kChunkBufs];
  uint32_t res_keep[kChunkBufs][kChunkRows];
  uint32_t res_cnt[kChunkBufs];     // kept rows of the chunk so far
  uint32_t res_arrived[kChunkBufs]; // consumer slots of the chunk finished so far
  int abort;
  uint32_t epoch;
};

template <typename WT, typename XT, int NB, int MODE, int RPS>
__global__ void __launch_bounds__(kTmaThreads, 1) gate_tma_kernel(const GateArgs p, int nslots) {
  constexpr int kRowsPerSlot = RPS;
  constexpr int kSlotsPerChunk = kChunkRows / RPS;
  static_assert(kSlotsPerChunk % kTmaConsumers == 0, "each chunk gives every consumer whole slots");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ GateTmaShared sh;
  __shared__ float res_val[kChunkBufs][kChunkRows][NB];

  constexpr int EPV = Vec<WT>::N;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.K;
  const size_t x_bytes = align_up((size_t)NB * K * sizeof(XT), 128);
  const uint32_t row_bytes = (uint32_t)(K * sizeof(WT));
  const uint32_t slot_bytes = row_bytes * kRowsPerSlot;
  XT* xs = reinterpret_cast<XT*>(smem_raw);
  unsigned char* ring = smem_raw + x_bytes;

  if (tid == 0) {
    for (int i = 0; i < nslots; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int i = 0; i < kChunkBufs; ++i) {
      mbar_init(&sh.chunk_full[i], kSlotsPerChunk);
      mbar_init(&sh.chunk_empty[i], 1);
      sh.res_cnt[i] = 0u;
      sh.res_arrived[i] = 0u;
    }
    sh.abort = 0;
    sh.epoch = *reinterpret_cast<volatile uint32_t*>(&p.ctl->epoch);
    fence_mbar_init();
  }
  __syncthreads();

  const int n_rows = p.cand_count ? min(max(*p.cand_count, 0), p.h) : p.h;
  const int n_chunks = (n_rows + kChunkRows - 1) / kChunkRows;
  const uint32_t epoch = sh.epoch;
  volatile int* abort = &sh.abort;
  auto row_of = [&](int j) -> int {
    int r = p.cand_idx ? p.cand_idx[j] : j;
    return ((unsigned)r < (unsigned)p.h) ? r : 0;
  };

  if (warp == kTmaConsumers) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      const WT* W = reinterpret_cast<const WT*>(p.W);
      int q = 0;
      int c_next = (int)blockIdx.x;  // first chunk: no ticket needed
      bool ok = true;
      for (bool done = false; !done && ok;) {
        const int c = c_next;
        done = c >= n_chunks;
        if (c == 0 && n_chunks == 0) *p.count = 0;  // empty row set
        if (!done) c_next = (int)gridDim.x + (int)atomicAdd(&p.ctl->ticket, 1u);
        for (int g = 0; g < kSlotsPerChunk; ++g, ++q) {
          const int slot = q % nslots;
          if (!(ok = mbar_wait(&sh.empty[slot], ((q / nslots) & 1) ^ 1, p.err, abort))) break;
          sh.slot_chunk[slot] = done ? -1 : c;
          const int j0 = c * kChunkRows + g * kRowsPerSlot;
          const int nvalid = done ? 0 : max(0, min(kRowsPerSlot, n_rows - j0));
          if (nvalid == 0) {
            mbar_arrive(&sh.full[slot]);
          } else {
            mbar_arrive_expect_tx(&sh.full[slot], row_bytes * nvalid);
            if (p.cand_idx == nullptr) {  // consecutive rows: one copy for the whole slot
              bulk_load(ring + (size_t)slot * slot_bytes, W + (size_t)j0 * K, row_bytes * nvalid, &sh.full[slot]);
            } else {
              for (int r = 0; r < nvalid; ++r)
                bulk_load(ring + (size_t)slot * slot_bytes + (size_t)r * row_bytes,
                          W + (size_t)row_of(j0 + r) * K, row_bytes, &sh.full[slot]);
            }
          }
        }
      }
      if (!ok) {
        // Aborted: wait (bounded) for every copy this thread may still have in flight.
        for (int k = 1; k <= nslots && k <= q; ++k) {
          const int qq = q - k;
          const int slot = qq % nslots;
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&sh.full[slot], (qq / nslots) & 1) && globaltimer_ns() - t0 < kWaitNs) {
          }
        }
      }
    }
  } else if (warp < kTmaConsumers) {
    // ------------------------------------------------------------------ consumers
    constexpr int R = kRowsPerSlot;
    const int NV = K / EPV;
    {  // stage the tokens (consumer warps only; the producer is already streaming)
      const int per_tok = (int)((size_t)K * sizeof(XT) / 16);
      uint4* dst = reinterpret_cast<uint4*>(xs);
      const uint4* src = reinterpret_cast<const uint4*>(p.x);
      for (int e = tid; e < NB * per_tok; e += kTmaConsumers * kWarp)
        dst[e] = (e / per_tok) < p.B ? src[e] : make_uint4(0u, 0u, 0u, 0u);
      asm volatile("bar.sync 1, %0;" ::"n"(kTmaConsumers * kWarp) : "memory");
    }
    for (int q = warp;; q += kTmaConsumers) {
      const int slot = q % nslots;
      if (!mbar_wait(&sh.full[slot], (q / nslots) & 1, p.err, abort)) break;
      const int c = sh.slot_chunk[slot];
      const int s = q / kSlotsPerChunk;  // this CTA's chunk sequence number
      const int cb = s % kChunkBufs;
      if (c < 0) {  // sentinel chunk: tell the compaction warp to stop
        if (!mbar_wait(&sh.chunk_empty[cb], ((s / kChunkBufs) & 1) ^ 1, p.err, abort)) break;
        if (q % kSlotsPerChunk == 0 && lane == 0) sh.res_chunk[cb] = -1;
        __syncwarp();
        if (lane == 0) {
          // arrive for every slot of the sentinel chunk this warp owns; the later ones are never read
          for (int k = 0; k < kSlotsPerChunk / kTmaConsumers; ++k) mbar_arrive(&sh.chunk_full[cb]);
          mbar_arrive(&sh.empty[slot]);
        }
        break;
      }
      const int pos = (q % kSlotsPerChunk) * R;  // first row of this slot within the chunk
      const int j0 = c * kChunkRows + pos;
      const WT* rows = reinterpret_cast<const WT*>(ring + (size_t)slot * slot_bytes);
      // Two partial sums per (row, token) halve the dependent FMA chain.
      float acc2[R][NB][2];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < NB; ++b) acc2[r][b][0] = acc2[r][b][1] = 0.f;
#pragma unroll 4
      for (int v = lane; v < NV; v += kWarp) {
        float wf[R][EPV];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint4 w = *reinterpret_cast<const uint4*>(rows + (size_t)r * K + (size_t)v * EPV);
          unpack(w, wf[r]);
        }
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float xf[EPV];
          load_x<EPV>(xs + (size_t)b * K + (size_t)v * EPV, xf);
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc2[r][b][e & 1] = fmaf(wf[r][e], xf[e], acc2[r][b][e & 1]);
        }
      }
      // The slot's data is in registers: hand the slot back to the producer before anything else.
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh.empty[slot]);
      float acc[R][NB];
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[r][b] = acc2[r][b][0] + acc2[r][b][1];
      if (!mbar_wait(&sh.chunk_empty[cb], ((s / kChunkBufs) & 1) ^ 1, p.err, abort)) break;
      warp_reduce_all<R, NB>(acc);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (lane == r) {
          const int j = j0 + r;
          bool keep_any = false;
          if (j < n_rows) {
            const int i = row_of(j);
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
                  res_val[cb][pos + r][b] = k ? a : 0.f;
                } else {
                  k = z > thr;
                }
                keep_any |= k;
              }
            }
          }
          sh.res_keep[cb][pos + r] = keep_any ? 1u : 0u;
        }
      }
      if (pos == 0 && lane == 0) sh.res_chunk[cb] = c;
      __syncwarp();
      if (lane == 0) {
        uint32_t kept = 0;
#pragma unroll
        for (int r = 0; r < R; ++r) kept += sh.res_keep[cb][pos + r];
        atomicAdd(&sh.res_cnt[cb], kept);
        __threadfence_block();  // the count is in before this slot is counted as finished
        if (atomicAdd(&sh.res_arrived[cb], 1u) == (uint32_t)(kSlotsPerChunk - 1)) {
          // last slot of the chunk: publish the aggregate now (chunk 0: its inclusive prefix)
          const uint32_t agg = atomicAdd(&sh.res_cnt[cb], 0u);
          st_status(&p.status[c], status_word(epoch, c == 0 ? kFlagInclusive : kFlagAggregate, agg));
        }
        mbar_arrive(&sh.chunk_full[cb]);
      }
    }
  } else {
    // ------------------------------------------------------------------ compaction
    for (int s = 0;; ++s) {
      const int cb = s % kChunkBufs;
      if (!mbar_wait(&sh.chunk_full[cb], (s / kChunkBufs) & 1, p.err, abort)) break;
      const int c = sh.res_chunk[cb];
      if (c < 0) break;
      const bool keep = lane < kChunkRows && sh.res_keep[cb][lane] != 0u;
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
              if (b < p.B) p.a_val[(size_t)b * p.h + pos] = res_val[cb][lane][b];
          }
        }
      }
      if (c == n_chunks - 1 && lane == 0) *p.count = (int32_t)(prefix + agg);
      __syncwarp();
      if (lane == 0) {
        sh.res_cnt[cb] = 0u;
        sh.res_arrived[cb] = 0u;
        mbar_arrive(&sh.chunk_empty[cb]);
      }
    }
  }

  __syncthreads();
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

// Ring depth for a slot size: a multiple of the consumer count, or 0 if not even one slot per
// consumer fits beside the staged tokens.
static int ring_slots(size_t x_bytes, size_t slot) {
  const size_t avail = kTmaSmemBudget > x_bytes ? kTmaSmemBudget - x_bytes : 0;
  size_t n = avail / slot;
  if (n > (size_t)kMaxRingSlots) n = kMaxRingSlots;
  n -= n % kTmaConsumers;
  return (int)n;
}

template <typename WT, typename XT, int NB, int MODE, int RPS>
static cudaError_t launch_gate_tma_r(const GateArgs& a, cudaStream_t s) {
  auto kern = gate_tma_kernel<WT, XT, NB, MODE, RPS>;
  const size_t x_bytes = align_up((size_t)NB * a.K * sizeof(XT), 128);
  const size_t slot_bytes = (size_t)a.K * sizeof(WT) * RPS;
  const int nslots = ring_slots(x_bytes, slot_bytes);
  if (nslots == 0) return cudaErrorInvalidConfiguration;
  const size_t smem = x_bytes + (size_t)nslots * slot_bytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int max_chunks = (a.h + kChunkRows - 1) / kChunkRows;
  int grid = sm_count();
  if (grid > max_chunks) grid = max_chunks;
  if (grid < 1) grid = 1;
  kern<<<grid, kTmaThreads, smem, s>>>(a, nslots);
  return cudaGetLastError();
}

// Two rows per slot when the rows are consecutive and the ring still holds 8 such slots.
static bool two_rows_per_slot(const GateArgs& a, size_t x_bytes, size_t row_bytes) {
  return a.cand_idx == nullptr && ring_slots(x_bytes, 2 * row_bytes) >= kTmaConsumers;
}

template <typename WT, typename XT, int NB, int MODE>
static cudaError_t launch_gate_tma_t(const GateArgs& a, cudaStream_t s) {
  const size_t x_bytes = align_up((size_t)NB * a.K * sizeof(XT), 128);
  const size_t row_bytes = (size_t)a.K * sizeof(WT);
  return two_rows_per_slot(a, x_bytes, row_bytes) ? launch_gate_tma_r<WT, XT, NB, MODE, 2>(a, s)
                                                  : launch_gate_tma_r<WT, XT, NB, MODE, 1>(a, s);
}

bool gate_tma_supported(int K, int B, int wdtype, bool x_f32) {
  const size_t xs = x_f32 || wdtype == CSFFN_F32 ? 4 : 2;
  const size_t ws = wdtype == CSFFN_F32 ? 4 : 2;
  return ring_slots(align_up((size_t)batch_tier(B) * K * xs, 128), (size_t)K * ws) >= kTmaConsumers;
}

template <typename WT, typename XT, int MODE>
static cudaError_t launch_gate_tma_nb(const GateArgs& a, cudaStream_t s) {
  switch (batch_tier(a.B)) {
    case 1: return launch_gate_tma_t<WT, XT, 1, MODE>(a, s);
    case 2: return launch_gate_tma_t<WT, XT, 2, MODE>(a, s);
    case 4: return launch_gate_tma_t<WT, XT, 4, MODE>(a, s);
    case 8: return launch_gate_tma_t<WT, XT, 8, MODE>(a, s);
    default: return launch_gate_tma_t<WT, XT, 16, MODE>(a, s);
  }
}

cudaError_t launch_gate_tma(const GateArgs& a, int wdtype, bool x_f32, int mode, cudaStream_t s) {
  if (wdtype == CSFFN_F32) {
    return mode == kModeCats ? launch_gate_tma_nb<float, float, kModeCats>(a, s)
                             : launch_gate_tma_nb<float, float, kModePred>(a, s);
  }
  if (x_f32) {
    return mode == kModeCats ? launch_gate_tma_nb<bf16, float, kModeCats>(a, s)
                             : launch_gate_tma_nb<bf16, float, kModePred>(a, s);
  }
  return mode == kModeCats ? launch_gate_tma_nb<bf16, bf16, kModeCats>(a, s)
                           : launch_gate_tma_nb<bf16, bf16, kModePred>(a, s);
}

}  // namespace csffn
