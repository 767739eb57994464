// One-launch CATS decode step: gate, threshold, up and down projection in a single pass over the
// neuron rows, then one cross-CTA sum and the compaction of the active list.
//
// "CATS: Contextually-Aware Thresholding for Sparsity in Large Language Models", abstract and the
// section on the custom kernel: the gate GEMV, the compare against t and the flag-gated up and
// down GEMVs.  Here every stage of one decode step of an FFN layer runs in one persistent grid.
// A decode step reads a few hundred MB, and a separate launch per stage pays its ramp-up and tail
// each time (measured on B200: a bare 45 MB row stream reaches 3.6 TB/s, a 720 MB one 6.8 TB/s),
// and a statically partitioned stream ends in a long tail (CTAs with equal shares finished up to
// 2.5x apart), so the rows are handed out dynamically in small chunks.
//
// Chunks of kChunk neuron rows (kTailChunk at the end of the range) go to CTA b first (chunk b,
// no draw), then come from a ticket counter in row order; the next ticket is drawn one chunk
// ahead, so its round trip is hidden and 1.4 K draws per step do not contend.
// The chunk's W_gate rows (contiguous) arrive in shared memory by one bulk copy issued while the
// previous chunk is still being worked on.  For its chunk a CTA
//   1. has warp w reduce gate row w against the tokens (both in shared memory), add the bias,
//      apply the activation and the threshold per token, and record the keep flag and the kept
//      activations; after one block barrier thread 0 issues the next chunk's bulk copy;
//   2. appends the chunk's kept rows to a ring queue in shared memory.  Whenever 8 rows are
//      queued (and for the rest after the CTA's last chunk) it flushes them: warp w streams W_up of
//      queued row w from HBM and forms v[b] = a[b] * u[b]; after a barrier each warp streams its
//      fixed 1/8 of the columns of the 8 W_down^T rows and accumulates v[b] * W_down^T[r, cols] in
//      registers over all its batches (no atomics, no cross-warp traffic until the end).
// So the up and down round trips are paid once per 8 kept rows, not once per chunk: at high
// sparsity the chunk loop is a gate stream.
// When the tickets run out each CTA adds its register partial of out (fp32 [B, d]) into one of a
// few accumulators in L2 by vector reductions, so the CTAs that finish early do so while the rest
// are still streaming.  After one grid-wide meeting (all CTAs are co-resident: cooperative launch)
// half of each CTA's warps turn an equal share of the accumulators into out and clear it, while
// the other half compact the active list from the keep flags: CTA k takes a fixed range of 32-row
// words, counts the flags before it, and writes idx / a_val in ascending neuron order.  Every wait
// is bounded; the counters return to zero by themselves (the ticket counter is cleared by the
// last CTA to arrive at the meeting).
#include "common.cuh"
#include "fused_end.cuh"
#include "gemv.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace csffn {

constexpr int kFusedThreads = 256;
constexpr int kFusedWarps = kFusedThreads / kWarp;
constexpr int kChunk = kFusedWarps;  // neuron rows per chunk, one per warp
constexpr int kQueueBatch = kFusedWarps;      // kept rows per up/down batch, one W_up row per warp
constexpr int kQueueSlots = 2 * kQueueBatch;  // ring of queued kept rows (a chunk adds at most kChunk)
constexpr int kCounters = kTicketCounters;
constexpr int kTailChunk = 4;        // rows per chunk at the end of the row range
constexpr int kTailGrids = 2;        // the last kTailGrids * grid chunks are of kTailChunk rows

// acc[b] += W[row] . x_b over this lane's share (U 16-byte vectors in flight per lane).
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

template <int NB> struct FusedGateU { static constexpr int value = NB <= 2 ? 16 : 8; };
// Kept rows whose W_down^T slices are loaded together.
template <int NB, int KD> struct FusedDownRows {
  static constexpr int value = NB * KD <= 2 ? 8 : (NB * KD <= 4 ? 4 : 2);  // a whole chunk at batch 1
};

// Chunks in row order: `big` rows each, then `small` rows each for the last `tail` rows (at
// least), so that the work a CTA still holds when the tickets run out is small and the CTAs
// finish close together.
struct ChunkMap {
  int n_rows, big, small, n_big, n_chunks;
  __device__ void init(int rows, int big_rows, int small_rows, int tail) {
    n_rows = rows;
    big = big_rows;
    small = small_rows;
    n_big = rows > tail ? (rows - tail) / big : 0;
    n_chunks = n_big + (rows - n_big * big + small - 1) / small;
  }
  __device__ void rows(int c, int& j0, int& n) const {
    if (c < n_big) {
      j0 = c * big;
      n = big;
    } else {
      j0 = n_big * big + (c - n_big) * small;
      n = min(small, n_rows - j0);
    }
  }
};

// Predictor mode: at most this many groups of kChunk V_r rows per chunk (and 64 KB of rows).
constexpr int kPredSubMax = 16;
__host__ __device__ inline int pred_sub_max(int rank, int es) {
  const int r = 65536 / (kChunk * rank * es);
  return r < 1 ? 1 : (r > kPredSubMax ? kPredSubMax : r);
}

// Tickets, drawn by thread 0, for the chunks after the first grid width (CTA b starts on chunk b
// without a draw).  Counter g hands out chunks base + [lo(g), lo(g + 1)); a counter found dry is
// flagged (word 1 of its line) and the thread moves on to the next counter not flagged.
// resolve() returns -1 once every counter is dry.
struct Tickets {
  uint32_t* ctr;
  int base, n_chunks, G;
  __device__ int lo(int g) const { return (int)((long long)n_chunks * g / G); }
  __device__ uint32_t draw(int g) const { return atomicAdd(ctr + g * kCounterStride, 1u); }
  __device__ int resolve(int& g, uint32_t t) const {
    for (;;) {
      const int c = lo(g) + (int)t;
      if (c < lo(g + 1)) return base + c;
      ctr[g * kCounterStride + 1] = 1u;
      uint32_t live = 0;  // bit i: counter i not flagged dry
#pragma unroll
      for (int i = 0; i < kCounters; ++i)
        live |= (i < G && i != g && __ldcg(ctr + i * kCounterStride + 1) == 0u) ? 1u << i : 0u;
      if (!live) return -1;
      // first live counter after g, cyclically
      const uint32_t above = g + 1 < kCounters ? live & (~0u << (g + 1)) : 0u;
      g = __ffs(above ? above : live) - 1;
      t = draw(g);
    }
  }
};

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// PRED: predictor mode ("SVD Contextual Sparsity Predictors for Fast LLM Inference", Fig. 1 and
// Fig. 3).  Before the chunk loop the grid computes y = x U_r (a warp per row of U_r^T) and meets
// at a grid-wide count; the chunks then prefetch rows of V_r instead of W_gate, each warp forms
// p = y . V_r[i] + beta_i, and only a neuron predicted by some token (p > tau_i) has its W_gate
// row streamed and its activation thresholded; up and down follow as in the CATS mode.
template <typename WT, int NB, int KD, bool PRED>
__global__ void __launch_bounds__(kFusedThreads, 2) cats_fused_kernel(const FusedArgs p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  constexpr int EPV = Vec<WT>::N;
  constexpr int U = FusedGateU<NB>::value;
  constexpr int DR = FusedDownRows<NB, KD>::value;
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ int s_abort;
  __shared__ float s_v[kQueueBatch][NB];        // v of the batch being flushed
  __shared__ int s_drow[kQueueBatch];            // its neurons
  __shared__ uint8_t s_keep[2][kChunk];          // keep flags of the chunk or round (by parity)
  __shared__ int s_plist[PRED ? 2 : 1][kFusedWarps][kPredSubMax];  // predictor: predicted rows per warp
  __shared__ int s_pcnt[PRED ? 2 : 1][kFusedWarps];
  __shared__ int s_qrow[kQueueSlots];            // queued kept rows: neuron
  __shared__ float s_qa[kQueueSlots][NB];        // and kept activations per token
  __shared__ int s_next[2];
  __shared__ uint32_t s_cnt[kFusedWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = p.d, h = p.h, B = p.B;
  const int cpw = d / EPV / kFusedWarps;  // 16-byte columns of W_down^T owned by each warp
  WT* xs = reinterpret_cast<WT*>(smem_raw);
  const int rowlen = PRED ? p.rank : d;  // elements of a prefetched row (V_r or W_gate)
  WT* gbuf = xs + (size_t)NB * d;         // prefetched rows of the current chunk [chunk rows][rowlen]
  // predictor mode: y [NB][rank] after the largest chunk of V_r rows
  float* ys = reinterpret_cast<float*>(gbuf + (size_t)kChunk * (PRED ? pred_sub_max(p.rank, (int)sizeof(WT)) : 1) * rowlen);
  const WT* Wg = reinterpret_cast<const WT*>(p.W_gate);
  const WT* Wu = reinterpret_cast<const WT*>(p.W_up);
  const WT* Wd = reinterpret_cast<const WT*>(p.W_down_t);
  const uint32_t row_bytes = (uint32_t)(rowlen * sizeof(WT));
  const WT* Wpre = PRED ? reinterpret_cast<const WT*>(p.v_r) : Wg;  // the rows the chunks prefetch

  // Rows are positions 0 .. n_rows - 1 of the candidate list (neuron cand_idx[j]) or, without one,
  // the neurons themselves.  Keep flags and kept activations are stored by position.  A candidate
  // outside 0 .. h - 1 (a malformed list) reads row 0, so every access stays in bounds.
  const int32_t* cand = p.cand_idx;
  const int n_rows = cand ? min(max(__ldg(p.cand_count), 0), h) : h;
  auto neuron = [&](int j) {
    if (!cand) return j;
    const int r = __ldg(cand + j);
    return (unsigned)r < (unsigned)h ? r : 0;
  };

  ChunkMap cm;
  if constexpr (PRED) {
    // one chunk per CTA where the rows allow: the work per row is a few hundred bytes of V_r, so a
    // chunk's round trips, not its bytes, set its time
    const int per = (n_rows + (int)gridDim.x - 1) / (int)gridDim.x;
    const int cs = max(kChunk, min((per + kChunk - 1) / kChunk * kChunk, kChunk * pred_sub_max(p.rank, (int)sizeof(WT))));
    cm.init(n_rows, cs, cs, 0);
  } else {
    cm.init(n_rows, kChunk, kTailChunk, kTailGrids * (int)gridDim.x * kTailChunk);
  }
  Tickets tk;
  tk.ctr = p.tickets;
  tk.base = min((int)gridDim.x, cm.n_chunks);
  tk.n_chunks = cm.n_chunks - tk.base;
  tk.G = tk.n_chunks < kCounters ? (tk.n_chunks > 0 ? tk.n_chunks : 1) : kCounters;
  int g = blockIdx.x % tk.G;
  uint32_t t_pending = 0;  // thread 0: ticket drawn for the chunk after the one in flight
  auto issue_gate = [&](int c) {  // thread 0: the chunk's W_gate rows -> gbuf (one copy, or one per row)
    int j0, n;
    cm.rows(c, j0, n);
    mbar_arrive_expect_tx(&s_bar, (uint32_t)n * row_bytes);
    if (!cand) {
      bulk_load(gbuf, Wpre + (size_t)j0 * rowlen, (uint32_t)n * row_bytes, &s_bar);
    } else {
      int rows[kChunk];  // all indices fetched before the first copy, so their loads overlap
#pragma unroll
      for (int jj = 0; jj < kChunk; ++jj) rows[jj] = jj < n ? neuron(j0 + jj) : 0;
#pragma unroll
      for (int jj = 0; jj < kChunk; ++jj)
        if (jj < n) bulk_load(gbuf + (size_t)jj * d, Wg + (size_t)rows[jj] * d, row_bytes, &s_bar);
    }
  };

  if (tid == 0) {
    s_abort = 0;
    mbar_init(&s_bar, 1);
    fence_mbar_init();
    const int c0 = (int)blockIdx.x < cm.n_chunks ? (int)blockIdx.x : -1;
    s_next[0] = c0;
    if (c0 >= 0) issue_gate(c0);
    t_pending = tk.draw(g);
  }
  stage_tokens<WT, NB>(xs, reinterpret_cast<const WT*>(p.x), B, d);
  __syncthreads();

  if constexpr (PRED) {
    // y[b][k] = x_b . U_r^T[k]: a warp per row, over the whole grid; then every CTA takes all of y
    const WT* Urt = reinterpret_cast<const WT*>(p.u_rt);
    const int rank = p.rank;
    for (int k = blockIdx.x * kFusedWarps + warp; k < rank; k += gridDim.x * kFusedWarps) {
      float yk[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) yk[b] = 0.f;
      row_dot<WT, NB, FusedGateU<NB>::value>(Urt + (size_t)k * d, xs, d, lane, yk);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        yk[b] = warp_sum(yk[b]);
        if (lane == 0 && b < B) __stcg(p.ybuf + (size_t)b * rank + k, yk[b]);
      }
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      atomicAdd(&p.ctl[kCtlY], 1u);
      wait_at_least(&p.ctl[kCtlY], gridDim.x, p.err);
    }
    __syncthreads();
    for (int e = tid; e < NB * rank; e += kFusedThreads) ys[e] = e / rank < B ? __ldcg(p.ybuf + e) : 0.f;
    __syncthreads();
  }

  float acc[NB][KD][EPV];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int k = 0; k < KD; ++k)
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[b][k][e] = 0.f;

  // Kept rows wait in a ring of kQueueSlots entries (neuron, kept activations); q_head / q_tail are
  // the same in every thread.  flush(n) runs up and down for the n oldest entries: warp w streams
  // W_up of entry w and forms v, then every warp streams its columns of the n W_down^T rows.
  int q_head = 0, q_tail = 0;
  auto flush = [&](int n) {
    __syncthreads();  // queued entries are visible; the last batch's v and rows are no longer read
    float v[NB];
    int r = 0;
#pragma unroll
    for (int b = 0; b < NB; ++b) v[b] = 0.f;
    if (warp < n) {
      const int slot = (q_head + warp) & (kQueueSlots - 1);
      r = s_qrow[slot];
      float u[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) u[b] = 0.f;
      row_dot<WT, NB, U>(Wu + (size_t)r * d, xs, d, lane, u);
#pragma unroll
      for (int b = 0; b < NB; ++b) v[b] = s_qa[slot][b] * warp_sum(u[b]);
    }
    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < NB; ++b) s_v[warp][b] = v[b];
      s_drow[warp] = r;
    }
    __syncthreads();
    uint32_t m = (1u << n) - 1u;
    while (m) {
      int js[DR];
      uint4 w[DR][KD];
#pragma unroll
      for (int q = 0; q < DR; ++q) {
        js[q] = m ? __ffs(m) - 1 : -1;
        m &= m - 1u;
        const WT* row = Wd + (size_t)s_drow[js[q] < 0 ? 0 : js[q]] * d;
#pragma unroll
        for (int k = 0; k < KD; ++k) {
          const int c = lane + k * kWarp;
          w[q][k] = (js[q] >= 0 && c < cpw) ? ld_stream(row + (size_t)(warp * cpw + c) * EPV)
                                            : make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int q = 0; q < DR; ++q) {
        if (js[q] < 0) continue;
#pragma unroll
        for (int k = 0; k < KD; ++k) {
          float wf[EPV];
          unpack(w[q][k], wf);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const float vb = s_v[js[q]][b];
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc[b][k][e] = fmaf(vb, wf[e], acc[b][k][e]);
          }
        }
      }
    }
    q_head += n;
  };

  // Threshold one gate row: per token the activation of z + beta against t; records the keep flag
  // and the kept activations of position j and returns whether any token keeps the row.
  auto decide = [&](int j, float (&z)[NB], float beta, float (&a)[NB]) {
    bool any = false;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const float ab = gate_act(warp_sum(z[b]) + beta, p.act);
      const bool kb = b < B && fabsf(ab) > p.t;
      a[b] = kb ? ab : 0.f;
      any |= kb;
    }
    if (lane == 0) {
      p.flags[j] = any ? 1 : 0;
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (b < B) p.afull[(size_t)b * h + j] = a[b];
    }
    return any;
  };
  // Thread 0 resolves the ticket drawn a chunk ago and publishes it; after the block barrier (the
  // step's shared writes are visible, gbuf is free) it issues that chunk's copy and draws again.
  auto advance = [&](int buf) {
    int cn = -1;
    if (tid == 0) {
      cn = tk.resolve(g, t_pending);
      s_next[buf ^ 1] = cn;
    }
    __syncthreads();
    if (tid == 0 && cn >= 0) {
      fence_proxy_async_smem();
      issue_gate(cn);
      t_pending = tk.draw(g);
    }
    return s_next[buf ^ 1];
  };
  // Append the kept rows of one step (warp w's row r when keep[w]) to the queue, in warp order, and
  // flush a batch once kQueueBatch are waiting.
  auto enqueue = [&](bool any, int r, const float (&a)[NB], const uint8_t* keep) {
    uint32_t mask = 0;
#pragma unroll
    for (int jj = 0; jj < kChunk; ++jj) mask |= keep[jj] ? 1u << jj : 0u;
    if (any && lane == 0) {
      const int slot = (q_tail + __popc(mask & ((1u << warp) - 1u))) & (kQueueSlots - 1);
      s_qrow[slot] = r;
#pragma unroll
      for (int b = 0; b < NB; ++b) s_qa[slot][b] = a[b];
    }
    q_tail += __popc(mask);
    if (q_tail - q_head >= kQueueBatch) flush(kQueueBatch);
  };

  int chunk = s_next[0];
  int kr = 0;  // predictor mode: rounds so far (parity of their keep flags)
  for (int it = 0; chunk >= 0; ++it) {
    const int buf = it & 1;
    // A copy that never lands (a wait that ran out: the error word is set) ends the chunk loop in
    // every thread together, so no math runs on a buffer that did not arrive.
    if (__syncthreads_or(!mbar_wait(&s_bar, (uint32_t)(it & 1), p.err, &s_abort))) break;
    int j0, n_in;
    cm.rows(chunk, j0, n_in);
    int next;
    if constexpr (!PRED) {
      // 1. gate and threshold for position j (neuron r; one per warp) from the prefetched rows
      const int j = j0 + warp;
      const int r = warp < n_in ? neuron(j) : 0;
      float a[NB];
      bool any = false;
#pragma unroll
      for (int b = 0; b < NB; ++b) a[b] = 0.f;
      if (warp < n_in) {
        float z[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) z[b] = 0.f;
        const float beta = p.bias ? __ldg(p.bias + r) : 0.f;
        smem_row_dot<WT, NB>(gbuf + (size_t)warp * d, xs, d, lane, z);
        any = decide(j, z, beta, a);
      }
      if (lane == 0) s_keep[buf][warp] = any ? 1 : 0;
      next = advance(buf);
      // 2. queue the chunk's kept rows; up and down run on batches of kQueueBatch queued rows
      enqueue(any, r, a, s_keep[buf]);
    } else {
      // a. the prediction p = y . V_r[j] + beta_j against tau_j (union over tokens) for every row of
      //    the chunk, warp w taking rows w, w + 8, ...; a row not predicted is final here.  Lane i
      //    fetches tau and beta of the warp's row i, so those loads overlap.
      float tau_l = 0.f, beta_l = 0.f;
      {
        const int qi = warp + lane * kFusedWarps;
        if (lane < kPredSubMax && qi < n_in) {
          tau_l = __ldg(p.tau + neuron(j0 + qi));
          beta_l = p.bias ? __ldg(p.bias + neuron(j0 + qi)) : 0.f;
        }
      }
      int pc = 0;
      for (int i = 0; warp + i * kFusedWarps < n_in; ++i) {
        const int q = warp + i * kFusedWarps;
        float z[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) z[b] = 0.f;
        smem_dot_f32<WT, NB>(gbuf + (size_t)q * rowlen, ys, rowlen, lane, z);
        const float tau = __shfl_sync(0xffffffffu, tau_l, i), beta = __shfl_sync(0xffffffffu, beta_l, i);
        bool pred = false;
#pragma unroll
        for (int b = 0; b < NB; ++b) pred |= b < B && warp_sum(z[b]) + beta > tau;
        if (pred) {
          if (lane == 0) s_plist[buf][warp][pc] = q;
          ++pc;
        } else if (lane == 0) {
          p.flags[j0 + q] = 0;
#pragma unroll
          for (int b = 0; b < NB; ++b)
            if (b < B) p.afull[(size_t)b * h + j0 + q] = 0.f;
        }
      }
      if (lane == 0) s_pcnt[buf][warp] = pc;
      next = advance(buf);
      // b. rounds of up to kFusedWarps predicted rows: warp w streams the W_gate row of one from HBM
      //    and thresholds it; each round's kept rows go to the queue
      int pre[kFusedWarps + 1];
      pre[0] = 0;
#pragma unroll
      for (int w = 0; w < kFusedWarps; ++w) pre[w + 1] = pre[w] + s_pcnt[buf][w];
      const int P = pre[kFusedWarps];
      for (int base = 0; base < P; base += kFusedWarps) {
        const int k = base + warp;
        int r = 0;
        float a[NB];
        bool any = false;
#pragma unroll
        for (int b = 0; b < NB; ++b) a[b] = 0.f;
        if (k < P) {
          int w = 0;
#pragma unroll
          for (int ww = 1; ww < kFusedWarps; ++ww) w += k >= pre[ww] ? 1 : 0;
          const int jq = j0 + s_plist[buf][w][k - pre[w]];
          r = neuron(jq);
          const float beta = p.bias ? __ldg(p.bias + r) : 0.f;
          float z[NB];
#pragma unroll
          for (int b = 0; b < NB; ++b) z[b] = 0.f;
          row_dot<WT, NB, FusedGateU<NB>::value>(Wg + (size_t)r * d, xs, d, lane, z);
          any = decide(jq, z, beta, a);
        }
        if (lane == 0) s_keep[kr & 1][warp] = any ? 1 : 0;
        __syncthreads();  // the round's keep flags are visible
        enqueue(any, r, a, s_keep[kr & 1]);
        ++kr;
      }
    }
    if (next < 0 && q_tail > q_head) flush(q_tail - q_head);  // this CTA's last chunk: drain
    chunk = next;
  }

  // ---------------------------------------------------------------- partial sums, then one grid meeting
  // The CTA adds its register partial of out into accumulator blockIdx % kFusedAccCopies with
  // vector reductions in L2, issued the moment its chunks are done, so they overlap the other
  // CTAs' last chunks; spreading the CTAs over several accumulators shortens the queue of
  // reductions on each address.
  {
    float* accp = p.facc + (size_t)(blockIdx.x % kFusedAccCopies) * B * d;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b < B) {
#pragma unroll
        for (int k = 0; k < KD; ++k) {
          const int c = lane + k * kWarp;
          if (c < cpw) {
            float* dst = accp + (size_t)b * d + (size_t)(warp * cpw + c) * EPV;
#pragma unroll
            for (int e = 0; e < EPV; e += 4)
              red_add_v4(dst + e, acc[b][k][e], acc[b][k][e + 1], acc[b][k][e + 2], acc[b][k][e + 3]);
          }
        }
      }
    }
  }
  fused_finish<NB>(p, n_rows, s_cnt);
}

// Dynamic shared memory: the staged tokens and one chunk of prefetched rows (W_gate, or V_r in
// predictor mode, with the predictor's y beside them).
static size_t fused_smem_bytes(int d, int nb, size_t es, int rank = 0) {
  if (rank > 0)
    return (size_t)nb * d * es + (size_t)kChunk * pred_sub_max(rank, (int)es) * rank * es +
           (size_t)nb * rank * sizeof(float);
  return (size_t)(nb + kChunk) * d * es;
}

// Down-slice width per lane (16-byte columns) for a shape, 0 when the fused kernel does not take it.
static int fused_kd(int d, int B, int wdtype) {
  const int epv = wdtype == CSFFN_F32 ? 4 : 8;
  if (d % (epv * kFusedWarps) != 0) return 0;
  const int cpw = d / epv / kFusedWarps;
  const int kd = cpw <= 32 ? 1 : cpw <= 64 ? 2 : cpw <= 128 ? 4 : 0;
  // register budget: the down accumulators (tokens x kd x epv floats) beside a streamed row
  if (kd == 0 || batch_tier(B) * kd * epv > 64 || (epv == 8 && kd == 4 && B > 1)) return 0;
  return kd;
}

template <typename WT, int NB, int KD, bool PRED>
static cudaError_t fused_t(FusedArgs a, cudaStream_t s) {
  auto kern = cats_fused_kernel<WT, NB, KD, PRED>;
  const size_t smem = fused_smem_bytes(a.d, NB, sizeof(WT), PRED ? a.rank : 0);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  int occ = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kFusedThreads, smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorInvalidConfiguration;
  if (occ > 2) occ = 2;
  const int grid = sm_count() * occ;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a);
}

bool cats_fused_supported(int d, int B, int wdtype, int rank) {
  const size_t es = wdtype == CSFFN_F32 ? 4 : 2;
  return B >= 1 && B <= kFusedMaxBatch && fused_smem_bytes(d, batch_tier(B), es) <= 200 * 1024 &&
         fused_smem_bytes(d, batch_tier(B), es, rank) <= 200 * 1024 && fused_kd(d, B, wdtype) > 0;
}

template <typename WT, int NB, bool PRED>
static cudaError_t fused_kd_t(const FusedArgs& a, int kd, cudaStream_t s) {
  switch (kd) {
    case 1: return fused_t<WT, NB, 1, PRED>(a, s);
    case 2: return fused_t<WT, NB, 2, PRED>(a, s);
    default:
      if constexpr (Vec<WT>::N == 8 && NB > 1) return cudaErrorInvalidValue;  // rejected by fused_kd
      else return fused_t<WT, NB, 4, PRED>(a, s);
  }
}

template <bool PRED>
static cudaError_t launch_fused_mode(const FusedArgs& a, int wdtype, int kd, cudaStream_t s) {
  const int t = batch_tier(a.B);
  if (wdtype == CSFFN_F32) {
    switch (t) {
      case 1: return fused_kd_t<float, 1, PRED>(a, kd, s);
      case 2: return fused_kd_t<float, 2, PRED>(a, kd, s);
      default: return fused_kd_t<float, 4, PRED>(a, kd, s);
    }
  }
  switch (t) {
    case 1: return fused_kd_t<bf16, 1, PRED>(a, kd, s);
    case 2: return fused_kd_t<bf16, 2, PRED>(a, kd, s);
    default: return fused_kd_t<bf16, 4, PRED>(a, kd, s);
  }
}

cudaError_t launch_cats_fused(const FusedArgs& a, int wdtype, cudaStream_t s) {
  const int kd = fused_kd(a.d, a.B, wdtype);
  if (kd == 0) return cudaErrorInvalidValue;
  return a.u_rt ? launch_fused_mode<true>(a, wdtype, kd, s) : launch_fused_mode<false>(a, wdtype, kd, s);
}

}  // namespace csffn
