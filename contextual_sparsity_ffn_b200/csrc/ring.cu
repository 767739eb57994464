// CATS decode step on shared-memory rings fed by bulk copies: gate, threshold, up and down
// projection of one FFN layer in one streaming kernel, then the output and the compaction of the
// active list in a short second kernel.
//
// "CATS: Contextually-Aware Thresholding for Sparsity in Large Language Models", abstract and the
// section on the custom kernel: the gate GEMV, the compare against t, and the flag-gated up and down
// GEMVs.  The step is a stream of weight rows: all of W_gate, then the W_up and W_down^T rows of the
// neurons that survive the threshold.  A decode step moves 100-300 MB, so it is bound by how many
// bytes each SM keeps in flight, and by the dependent round trip gate -> up -> down at the end.
//
// One CTA per SM.  Every weight row reaches shared memory by one 1-D bulk copy (cp.async.bulk, no
// tensor map, no multicast), completing on its slot's mbarrier.  Warps:
//   1 .. 8   gate warps.  Each is its own stream: it draws tickets of kRingChunk gate rows from one
//            counter (its first chunk is fixed), keeps R rows in flight in its own R slots, dots each
//            row with the tokens (staged in shared memory as fp32), and decides it at once: bias,
//            activation and threshold per token, the keep flag and the kept activations.  The slot a
//            kept row frees takes that neuron's W_up row next; after its dot the warp hands
//            v_b = a_b u_b (with the neuron) to the producer through a queue in shared memory.
//   0        producer: turns the queue into bulk copies of W_down^T rows into the down ring.
//   9 .. 16  down warps: down warp c owns 1/8 of the output columns and accumulates v_b W_down^T[n]
//            for them in registers; a slot of the down ring is released when all eight are done.
// No warp handles a row it does no work on, and the gate path has no central issuer: the bytes in
// flight are the gate warps' slots (16 rows per SM at d = 4096) plus the down ring.
// No CTA waits for another: each adds its partial output into the workspace accumulators, writes
// the keep flags of its rows and exits; a small second kernel (ring_finish_kernel) writes out and
// compacts idx / a_val / count.  Both are launched as programmatic dependents of the kernel before
// them on the stream: a streaming CTA may start on an SM the previous step's streaming CTA has left
// while the previous step still finishes, and it fetches its first W_gate rows (weights, which no
// kernel writes) before griddepcontrol.wait; everything else -- the tokens, the candidate list, the
// workspace, the outputs -- is touched only after it.
// Every wait is bounded (a second); a wait that runs out records the timeout in the error word and
// ends the CTA's loops, after waiting (again bounded) for the CTA's own copies still in flight.
#include "common.cuh"
#include "fused_end.cuh"
#include "kernels.h"
#include "tma.cuh"

namespace csffn {

constexpr int kGateWarps = 8;
constexpr int kDownWarps = 8;
constexpr int kRingThreads = (1 + kGateWarps + kDownWarps) * kWarp;
constexpr int kRingChunk = 2;      // gate rows per ticket
constexpr int kDownQueue = 64;     // kept neurons between the gate warps and the producer
constexpr bool kPrefetchBeforeWait = true;
constexpr size_t kRingSmemBudget = 220 * 1024;
constexpr uint32_t kFullMask = 0xffffffffu;

enum : int { kItemGate = 0, kItemUp = 1, kItemDown = 2, kItemEnd = 3 };

// A slot's item.  GATE: row position j, neuron n, gate bias beta.  UP: neuron n, kept activations a.
// DOWN: neuron n, v = a * u per token in a.
struct __align__(16) RingDesc {
  int kind;
  int j;
  int n;
  float beta;
  float a[kFusedMaxBatch];
};

// Non-blocking test of an mbarrier phase.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Warp-wide bounded wait for a phase.  Every lane tests the barrier (one try_wait per lane, without
// divergence: cheaper than a lane-0 test and a warp barrier); a phase still open sends the whole
// warp to the slow path, which looks at the abort flag and the clock between tests.  Returns the
// same value in every lane; false when the CTA aborted or the wait ran out (then the error word and
// the abort flag are set).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t* err, volatile int* abort) {
  if (__all_sync(kFullMask, mbar_try_wait(bar, parity))) return true;
  bool ok = true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort) {
      ok = false;
      break;
    }
    if (globaltimer_ns() - t0 > kWaitNs) {
      atomicOr(err, kDevErrTimeout);
      *abort = 1;
      ok = false;
      break;
    }
  }
  return __all_sync(kFullMask, ok);
}

// One arrive from lane 0 of the warp, as a predicated instruction (no branch around it).
__device__ __forceinline__ void lane0_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.eq.u32 p, %1, 0;\n\t"
      "@p mbarrier.arrive.shared::cta.b64 _, [%0];\n\t}" ::"r"(smem_u32(bar)),
      "r"(threadIdx.x & 31u)
      : "memory");
}

// Ring geometry: R = 2^lr slots per gate warp, R_d = 2^lrd slots in the down ring.
struct RingGeom {
  int lr, lrd;
};

// Dynamic shared memory of the ring kernel.
struct RingSmem {
  size_t gring, dring, xs, gdesc, ddesc, gfull, dfull, dempty, dq, dq_flag, total;
};
__host__ __device__ inline RingSmem ring_smem(int d, int es, int nb, RingGeom g) {
  const size_t gs = (size_t)kGateWarps << g.lr, ds = (size_t)1 << g.lrd;
  RingSmem L;
  size_t o = 0;
  L.gring = o;   o += gs * d * es;
  L.dring = o;   o += ds * d * es;
  o = align_up(o, 16);
  L.xs = o;      o += sizeof(float) * (size_t)nb * d;  // tokens as fp32
  o = align_up(o, 16);
  L.gdesc = o;   o += sizeof(RingDesc) * gs;
  L.ddesc = o;   o += sizeof(RingDesc) * ds;
  L.dq = o;      o += sizeof(RingDesc) * kDownQueue;
  o = align_up(o, 8);
  L.gfull = o;   o += sizeof(uint64_t) * gs;
  L.dfull = o;   o += sizeof(uint64_t) * ds;
  L.dempty = o;  o += sizeof(uint64_t) * ds;
  L.dq_flag = o; o += sizeof(int) * kDownQueue;
  L.total = o;
  return L;
}

// The largest rings that fit the budget beside the tokens; {-1, -1} when not even the smallest fits.
__host__ __device__ inline RingGeom ring_geom(int d, int es, int nb) {
  const RingGeom options[] = {{1, 3}, {1, 2}, {1, 1}, {0, 2}, {0, 1}};
  for (const RingGeom& g : options)
    if (ring_smem(d, es, nb, g).total <= kRingSmemBudget) return g;
  return RingGeom{-1, -1};
}

// Shared counters of the down queue.
struct RingShared {
  int dq_tail;    // entries claimed by the gate warps (atomicAdd)
  int dq_head;    // entries the producer has taken (the gate warps' flow control)
  int gate_done;  // gate warps that have pushed their last entry
  int abort;
};

__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename WT, int NB, int KV>
__global__ void __launch_bounds__(kRingThreads, 1) cats_ring_kernel(const FusedArgs p, const RingGeom geo) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  __shared__ RingShared sh;
  constexpr int EPV = Vec<WT>::N;
  constexpr int XH = EPV / 4;  // float4 halves of a 16-byte weight vector
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = p.d, h = p.h, B = p.B;
  const int NV = d / EPV;  // 16-byte vectors per row
  const uint32_t rowbytes = (uint32_t)(d * sizeof(WT));
  const int LR = geo.lr, LRD = geo.lrd;
  const int R = 1 << LR, DS = 1 << LRD;
  const RingSmem L = ring_smem(d, (int)sizeof(WT), NB, geo);
  WT* gring = reinterpret_cast<WT*>(smem_raw + L.gring);
  WT* dring = reinterpret_cast<WT*>(smem_raw + L.dring);
  // tokens as fp32, [NB][XH][NV] float4: the two float4 halves of vector v apart, so that a warp's
  // loads of one half are contiguous
  float4* xs4 = reinterpret_cast<float4*>(smem_raw + L.xs);
  RingDesc* gdesc = reinterpret_cast<RingDesc*>(smem_raw + L.gdesc);
  RingDesc* ddesc = reinterpret_cast<RingDesc*>(smem_raw + L.ddesc);
  RingDesc* dq = reinterpret_cast<RingDesc*>(smem_raw + L.dq);
  uint64_t* gfull = reinterpret_cast<uint64_t*>(smem_raw + L.gfull);
  uint64_t* dfull = reinterpret_cast<uint64_t*>(smem_raw + L.dfull);
  uint64_t* dempty = reinterpret_cast<uint64_t*>(smem_raw + L.dempty);
  volatile int* dq_flag = reinterpret_cast<volatile int*>(smem_raw + L.dq_flag);
  volatile int* abort = &sh.abort;

  pdl_launch_dependents();  // the next step may start on the SMs this one leaves

  // A candidate list (and its count) may come from the kernel before: read after the wait.
  const int32_t* cand = p.cand_idx;
  const int n_streams = (int)gridDim.x * kGateWarps;  // gate warps in the grid; chunk g goes to stream g first

  if (tid == 0) {
    sh.dq_tail = 0;
    sh.dq_head = 0;
    sh.gate_done = 0;
    sh.abort = 0;
    for (int s = 0; s < (kGateWarps << LR); ++s) mbar_init(&gfull[s], 1);
    for (int s = 0; s < DS; ++s) {
      mbar_init(&dfull[s], 1);
      mbar_init(&dempty[s], kDownWarps);
    }
    fence_mbar_init();
  }
  for (int i = tid; i < kDownQueue; i += kRingThreads) dq_flag[i] = 0;
  __syncthreads();

  if (warp == 0) {
    // ------------------------------------------------------------------------------ producer
    pdl_wait();
    const WT* Wd = reinterpret_cast<const WT*>(p.W_down_t);
    int head = 0, dseq = 0, ddone = 0;
    bool ok = true;
    uint64_t t_idle = 0;
    auto dslot = [&](int q) { return q & (DS - 1); };
    auto dpar = [&](int q) { return (uint32_t)((q >> LRD) & 1); };
    for (;;) {
      // down slots that came back (lane 0 tests them in order)
      int rd = 0;
      if (lane == 0)
        while (ddone + rd < dseq && mbar_test(&dempty[dslot(ddone + rd)], dpar(ddone + rd))) ++rd;
      ddone += __shfl_sync(kFullMask, rd, 0);
      const int free_d = ddone + DS - dseq;
      // queue entries published in order from head (lane i looks at entry head + i)
      const bool pub = lane < free_d && dq_flag[(head + lane) % kDownQueue] == head + lane + 1;
      const uint32_t m_pub = __ballot_sync(kFullMask, pub);
      const int m = m_pub == kFullMask ? kWarp : __ffs(~m_pub) - 1;
      if (m > 0) {
        __threadfence_block();  // the entries' contents after their flags
        if (lane < m) {
          const RingDesc& e = dq[(head + lane) % kDownQueue];
          const int sd = dslot(dseq + lane);
          RingDesc& ds = ddesc[sd];
          ds.kind = kItemDown;
          ds.j = 0;
          ds.n = e.n;
#pragma unroll
          for (int b = 0; b < kFusedMaxBatch; ++b) ds.a[b] = e.a[b];
          // the down warps released this slot (arrive, release) after their reads of its previous
          // row, and this lane acquired that: the copy may overwrite it
          mbar_arrive_expect_tx(&dfull[sd], rowbytes);
          bulk_load_hint(dring + (size_t)sd * d, Wd + (size_t)e.n * d, rowbytes, &dfull[sd], l2_evict_first_policy());
        }
        __syncwarp();
        head += m;
        dseq += m;
        if (lane == 0) *reinterpret_cast<volatile int*>(&sh.dq_head) = head;
        t_idle = 0;
        continue;
      }
      // nothing to issue: done once every gate warp has pushed its last entry and all are taken
      const bool gates_done = *reinterpret_cast<volatile int*>(&sh.gate_done) == kGateWarps;
      __threadfence_block();
      const bool drained = gates_done && *reinterpret_cast<volatile int*>(&sh.dq_tail) == head;
      if (__shfl_sync(kFullMask, drained, 0) && free_d > 0) {
        if (lane == 0) {
          const int sd = dslot(dseq);
          ddesc[sd].kind = kItemEnd;
          mbar_arrive(&dfull[sd]);
        }
        __syncwarp();
        ++dseq;
        break;
      }
      if (*abort) {
        ok = false;
        break;
      }
      const uint64_t now = globaltimer_ns();
      if (t_idle == 0) {
        t_idle = now;
      } else if (now - t_idle > kWaitNs) {
        if (lane == 0) {
          atomicOr(p.err, kDevErrTimeout);
          *abort = 1;
        }
        ok = false;
        break;
      }
      __nanosleep(64);
    }
    if (!ok && lane == 0) {
      // every down copy this CTA issued lands before the CTA may exit
      const uint64_t t0 = globaltimer_ns();
      for (int q = ddone; q < dseq; ++q) {
        const int s = dslot(q);
        if (ddesc[s].kind == kItemEnd) continue;
        while (!mbar_test(&dfull[s], dpar(q)) && globaltimer_ns() - t0 < kWaitNs) {
        }
      }
    }
    __syncwarp();
  } else if (warp <= kGateWarps) {
    // ------------------------------------------------------------------------------ gate warps
    const int gw = warp - 1;
    const WT* Wg = reinterpret_cast<const WT*>(p.W_gate);
    const WT* Wu = reinterpret_cast<const WT*>(p.W_up);
    uint64_t* full = gfull + (gw << LR);
    RingDesc* desc = gdesc + (gw << LR);
    WT* ring = gring + ((size_t)gw << LR) * d;
    const int stream = (int)blockIdx.x * kGateWarps + gw;
    const float zero[NB] = {};

    // lane 0 fills the slot's descriptor and issues its row (the slot's previous row was read by
    // this warp, whose lanes finished with it before the warp barrier that precedes every issue)
    auto issue = [&](int q, int kind, int j, int n, float beta, const float (&a)[NB], const WT* src) {
      const int s = q & (R - 1);
      if (lane == 0) {
        RingDesc& ds = desc[s];
        ds.kind = kind;
        ds.j = j;
        ds.n = n;
        ds.beta = beta;
#pragma unroll
        for (int b = 0; b < kFusedMaxBatch; ++b) ds.a[b] = b < NB ? a[b] : 0.f;
        mbar_arrive_expect_tx(&full[s], rowbytes);
        bulk_load_hint(ring + (size_t)s * d, src, rowbytes, &full[s], l2_evict_first_policy());
      }
    };
    // Without a candidate list the stream's first chunk is rows 2 stream and 2 stream + 1 of W_gate:
    // its copies go out before the wait (and before the tokens are staged).
    int iss = 0;  // items issued; item q sits in slot q mod R
    int pre = 0;  // rows of the first chunk issued before the wait
    if (kPrefetchBeforeWait && !cand && stream * kRingChunk < h) {
      const int rows = min(kRingChunk, min(R, h - stream * kRingChunk));
      for (int i = 0; i < rows; ++i) {
        const int n = stream * kRingChunk + i;
        issue(iss++, kItemGate, n, n, p.bias ? __ldg(p.bias + n) : 0.f, zero, Wg + (size_t)n * d);
      }
      pre = rows;
    }
    pdl_wait();
    const int n_rows = cand ? min(max(__ldg(p.cand_count), 0), h) : h;
    const int n_chunks = (n_rows + kRingChunk - 1) / kRingChunk;
    // The first ticket draw goes out now, so that its round trip overlaps the staging of the tokens.
    uint32_t ticket = 0;  // lane 0: a draw in flight
    if (lane == 0 && n_streams < n_chunks) ticket = atomicAdd(p.tickets, 1u);
    bool drawn = n_streams < n_chunks;
    // tokens -> shared memory as fp32 (zero past B), then a barrier among the gate warps; the loads
    // of a batch all go out before the first conversion
    constexpr int kXLoads = 4;  // 16-byte token loads per thread and batch
    for (int e0 = tid - kWarp; e0 < NB * NV; e0 += kXLoads * kGateWarps * kWarp) {
      uint4 raw[kXLoads];
#pragma unroll
      for (int u = 0; u < kXLoads; ++u) {
        const int e = e0 + u * kGateWarps * kWarp;
        const int b = e / NV, v = e - b * NV;
        raw[u] = make_uint4(0u, 0u, 0u, 0u);
        if (e < NB * NV && b < B)
          raw[u] = *reinterpret_cast<const uint4*>(reinterpret_cast<const WT*>(p.x) + (size_t)b * d + (size_t)v * EPV);
      }
#pragma unroll
      for (int u = 0; u < kXLoads; ++u) {
        const int e = e0 + u * kGateWarps * kWarp;
        if (e < NB * NV) {
          const int b = e / NV, v = e - b * NV;
          float f[EPV];
          unpack(raw[u], f);
#pragma unroll
          for (int hh = 0; hh < XH; ++hh)
            xs4[((size_t)b * XH + hh) * NV + v] = make_float4(f[4 * hh], f[4 * hh + 1], f[4 * hh + 2], f[4 * hh + 3]);
        }
      }
    }
    named_sync(1, kGateWarps * kWarp);

    // Chunks of gate rows: this stream's first chunk is its own number; later ones come from the
    // ticket counter.  A ticket is drawn when the current chunk's last row goes out (the first one
    // right after the wait), so its round trip hides behind the row in flight, and when the counter
    // runs dry a warp holds no more than the rows of its current chunk and one drawn chunk.  Lane
    // i < kRingChunk holds the neuron and the gate bias of row i of the current chunk.
    auto chunk_rows = [&](int c) { return min(kRingChunk, n_rows - c * kRingChunk); };
    auto chunk_row = [&](int c, int& n, float& beta) {
      const int j = c * kRingChunk + lane;
      const bool in = c >= 0 && lane < kRingChunk && j < n_rows;
      n = in ? step_neuron(cand, h, j) : 0;
      beta = (in && p.bias) ? __ldg(p.bias + n) : 0.f;
    };
    bool more = n_streams < n_chunks;  // the counter may still hand out chunks
    int cur_c = stream < n_chunks ? stream : -1, cur_i = pre, cur_n;
    float cur_b;
    chunk_row(cur_c, cur_n, cur_b);
    auto draw = [&]() {
      if (lane == 0) ticket = atomicAdd(p.tickets, 1u);
      drawn = true;
    };
    auto gate_row_left = [&]() -> bool {  // moves to the next chunk when the current one is issued
      if (cur_c < 0) return false;
      const int rows = chunk_rows(cur_c);
      if (cur_i < rows) {
        if (cur_i == rows - 1 && more && !drawn) draw();
        return true;
      }
      if (!more) {
        cur_c = -1;
        return false;
      }
      if (!drawn) draw();
      const int c = n_streams + (int)__shfl_sync(kFullMask, ticket, 0);
      drawn = false;
      if (c >= n_chunks) {
        more = false;
        cur_c = -1;
        return false;
      }
      cur_c = c;
      cur_i = 0;
      chunk_row(cur_c, cur_n, cur_b);
      return true;
    };

    auto issue_gate_row = [&](int q) {
      const int n = __shfl_sync(kFullMask, cur_n, cur_i);
      const float beta = __shfl_sync(kFullMask, cur_b, cur_i);
      issue(q, kItemGate, cur_c * kRingChunk + cur_i, n, beta, zero, Wg + (size_t)n * d);
      ++cur_i;
    };

    while (iss < R && gate_row_left()) issue_gate_row(iss++);
    bool ok = true;
    for (int k = 0; k < iss; ++k) {
      const int s = k & (R - 1);
      if (!warp_wait(&full[s], (uint32_t)((k >> LR) & 1), p.err, abort)) {
        ok = false;
        break;
      }
      const RingDesc ds = desc[s];
      const WT* row = ring + (size_t)s * d;
      // the whole row against the tokens, four independent partial sums per token
      float z[NB][4];
#pragma unroll
      for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int i = 0; i < 4; ++i) z[b][i] = 0.f;
      int v = lane;
      for (; v + 3 * kWarp < NV; v += 4 * kWarp) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float wf[EPV];
          unpack(*reinterpret_cast<const uint4*>(row + (size_t)(v + i * kWarp) * EPV), wf);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
#pragma unroll
            for (int hh = 0; hh < XH; ++hh) {
              const float4 xv = xs4[((size_t)b * XH + hh) * NV + v + i * kWarp];
              z[b][i] = fmaf(wf[4 * hh], xv.x, z[b][i]);
              z[b][i] = fmaf(wf[4 * hh + 1], xv.y, z[b][i]);
              z[b][i] = fmaf(wf[4 * hh + 2], xv.z, z[b][i]);
              z[b][i] = fmaf(wf[4 * hh + 3], xv.w, z[b][i]);
            }
          }
        }
      }
      for (; v < NV; v += kWarp) {  // ragged end of the row
        float wf[EPV];
        unpack(*reinterpret_cast<const uint4*>(row + (size_t)v * EPV), wf);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
#pragma unroll
          for (int hh = 0; hh < XH; ++hh) {
            const float4 xv = xs4[((size_t)b * XH + hh) * NV + v];
            z[b][0] = fmaf(wf[4 * hh], xv.x, z[b][0]);
            z[b][0] = fmaf(wf[4 * hh + 1], xv.y, z[b][0]);
            z[b][0] = fmaf(wf[4 * hh + 2], xv.z, z[b][0]);
            z[b][0] = fmaf(wf[4 * hh + 3], xv.w, z[b][0]);
          }
        }
      }
      float zb[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b)  // lane 0's sum in every lane, so every lane takes the same decision
        zb[b] = __shfl_sync(kFullMask, warp_sum((z[b][0] + z[b][1]) + (z[b][2] + z[b][3])), 0);
      __syncwarp();  // every lane is done with the slot's row: it may be refilled
      if (ds.kind == kItemGate) {
        float a[NB];
        bool kept = false;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float ab = gate_act(zb[b] + ds.beta, p.act);
          const bool kb = b < B && fabsf(ab) > p.t;
          a[b] = kb ? ab : 0.f;
          kept |= kb;
        }
        if (lane == 0) {
          p.flags[ds.j] = kept ? 1 : 0;
#pragma unroll
          for (int b = 0; b < NB; ++b)
            if (b < B) p.afull[(size_t)b * h + ds.j] = a[b];
        }
        if (kept) {
          // The freed slot takes the neuron's W_up row; its W_down^T row, which the producer copies
          // once the up dot is done, is fetched into L2 now, so that copy does not wait on HBM.
          if (lane == 0) bulk_prefetch_l2(reinterpret_cast<const WT*>(p.W_down_t) + (size_t)ds.n * d, rowbytes);
          issue(iss++, kItemUp, 0, ds.n, 0.f, a, Wu + (size_t)ds.n * d);
        }
        else if (gate_row_left())
          issue_gate_row(iss++);
      } else {
        // UP: v = a * u goes to the producer, which issues the neuron's W_down^T row
        if (lane == 0) {
          const int e = atomicAdd(&sh.dq_tail, 1);
          const uint64_t t0 = globaltimer_ns();
          while (e - *reinterpret_cast<volatile int*>(&sh.dq_head) >= kDownQueue) {  // queue full
            if (*abort || globaltimer_ns() - t0 > kWaitNs) {
              atomicOr(p.err, kDevErrTimeout);
              *abort = 1;
              break;
            }
            __nanosleep(32);
          }
          RingDesc& en = dq[e % kDownQueue];
          en.kind = kItemDown;
          en.n = ds.n;
#pragma unroll
          for (int b = 0; b < kFusedMaxBatch; ++b) en.a[b] = b < NB ? ds.a[b] * zb[b] : 0.f;
          __threadfence_block();
          dq_flag[e % kDownQueue] = e + 1;
        }
        if (gate_row_left()) issue_gate_row(iss++);
      }
      __syncwarp();
    }
    if (!ok && lane == 0) {
      // every copy this warp issued lands before the CTA may exit
      const uint64_t t0 = globaltimer_ns();
      for (int q = 0; q < iss; ++q)
        while (!mbar_test(&full[q & (R - 1)], (uint32_t)((q >> LR) & 1)) && globaltimer_ns() - t0 < kWaitNs) {
        }
    }
    // this warp's last entry is in the queue
    __threadfence_block();
    if (lane == 0) atomicAdd(&sh.gate_done, 1);
  } else {
    // ------------------------------------------------------------------------------ down warps
    // Down warp cw owns the 16-byte column vectors cw*32 + lane + k*256 (k < KV) of out.
    pdl_wait();
    const int cw = warp - 1 - kGateWarps;
    float acc[NB][KV][EPV];
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
      for (int k = 0; k < KV; ++k)
#pragma unroll
        for (int e = 0; e < EPV; ++e) acc[b][k][e] = 0.f;
    for (int q = 0;; ++q) {
      const int s = q & (DS - 1);
      if (!warp_wait(&dfull[s], (uint32_t)((q >> LRD) & 1), p.err, abort)) break;
      if (ddesc[s].kind == kItemEnd) break;
      float vb[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) vb[b] = ddesc[s].a[b];
      const WT* row = dring + (size_t)s * d;
#pragma unroll
      for (int k = 0; k < KV; ++k) {
        const int v = cw * kWarp + lane + k * kWarp * kDownWarps;
        if (v < NV) {
          float wf[EPV];
          unpack(*reinterpret_cast<const uint4*>(row + (size_t)v * EPV), wf);
#pragma unroll
          for (int b = 0; b < NB; ++b)
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc[b][k][e] = fmaf(vb[b], wf[e], acc[b][k][e]);
        }
      }
      lane0_arrive(&dempty[s]);
    }
    // the partial output of this CTA into accumulator blockIdx % kFusedAccCopies (vector
    // reductions in L2, issued while other CTAs still stream)
    float* accp = p.facc + (size_t)(blockIdx.x % kFusedAccCopies) * B * d;
#pragma unroll
    for (int k = 0; k < KV; ++k) {
      const int v = cw * kWarp + lane + k * kWarp * kDownWarps;
      if (v < NV) {
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b < B) {
            float* dst = accp + (size_t)b * d + (size_t)v * EPV;
#pragma unroll
            for (int e = 0; e < EPV; e += 4)
              red_add_v4(dst + e, acc[b][k][e], acc[b][k][e + 1], acc[b][k][e + 2], acc[b][k][e + 3]);
          }
        }
      }
    }
  }
}

// The end of the step, in a kernel of its own after the streaming kernel (the kernel boundary is the
// grid-wide barrier): the output and the compaction of idx / a_val / count, spread over the grid;
// CTA 0 clears the ticket counter for the next step.  Launched as a programmatic dependent too: its
// CTAs may start beside the streaming kernel's and wait there, and the next step's streaming kernel
// may start beside them.
template <int NB>
__global__ void __launch_bounds__(2 * kFinishHalf) ring_finish_kernel(const FusedArgs p) {
  __shared__ uint32_t s_cnt[kFinishHalf / kWarp];
  pdl_launch_dependents();
  pdl_wait();
  const int n_rows = p.cand_idx ? min(max(__ldg(p.cand_count), 0), p.h) : p.h;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    p.tickets[0] = 0u;
    p.tickets[1] = 0u;
  }
  fused_finish_work<NB>(p, n_rows, s_cnt);
}

// 16-byte vectors per lane of the down projection's columns for a shape (0 when the ring kernel does
// not take it): the output accumulators of a lane's columns stay in registers.
static int ring_kv(int d, int B, int wdtype) {
  const int epv = wdtype == CSFFN_F32 ? 4 : 8;
  if (d % epv != 0 || B < 1 || B > kFusedMaxBatch) return 0;
  const int nv = d / epv;
  const int kv = (nv + kWarp * kDownWarps - 1) / (kWarp * kDownWarps);
  const int k = kv <= 1 ? 1 : kv <= 2 ? 2 : kv <= 3 ? 3 : kv <= 4 ? 4 : kv <= 8 ? 8 : 0;
  if (k == 0 || batch_tier(B) * k * epv > 64) return 0;
  return k;
}

bool cats_ring_supported(int d, int B, int wdtype) {
  const int es = wdtype == CSFFN_F32 ? 4 : 2;
  return ring_kv(d, B, wdtype) > 0 && ring_geom(d, es, batch_tier(B)).lr >= 0;
}

template <typename WT, int NB, int KV>
static cudaError_t ring_t(const FusedArgs& a, cudaStream_t st) {
  auto kern = cats_ring_kernel<WT, NB, KV>;
  const RingGeom geo = ring_geom(a.d, (int)sizeof(WT), NB);
  if (geo.lr < 0) return cudaErrorInvalidValue;
  const size_t smem = ring_smem(a.d, (int)sizeof(WT), NB, geo).total;
  // The shared-memory attribute on every call: it belongs to the CUDA context, which a device reset
  // replaces.  The one-CTA-per-SM check once per device and instance (again when a larger shape
  // needs more shared memory).
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  static int ready[64] = {0};
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (ready[dev] < (int)smem) {
    int occ = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kRingThreads, smem);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    ready[dev] = (int)smem;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sm_count());
  cfg.blockDim = dim3(kRingThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a, geo);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t fin = cfg;
  fin.blockDim = dim3(2 * kFinishHalf);
  fin.dynamicSmemBytes = 0;
  return cudaLaunchKernelEx(&fin, ring_finish_kernel<NB>, a);
}

template <typename WT, int NB>
static cudaError_t ring_kv_t(const FusedArgs& a, int kv, cudaStream_t s) {
  constexpr int EPV = Vec<WT>::N;
  switch (kv) {
    case 1: return ring_t<WT, NB, 1>(a, s);
    case 2:
      if constexpr (NB * 2 * EPV <= 64) return ring_t<WT, NB, 2>(a, s);
      break;
    case 3:
      if constexpr (NB * 3 * EPV <= 64) return ring_t<WT, NB, 3>(a, s);
      break;
    case 4:
      if constexpr (NB * 4 * EPV <= 64) return ring_t<WT, NB, 4>(a, s);
      break;
    case 8:
      if constexpr (NB * 8 * EPV <= 64) return ring_t<WT, NB, 8>(a, s);
      break;
    default: break;
  }
  return cudaErrorInvalidValue;
}

// Tokens from mapped page-locked host memory into the workspace, once per step, so that the step's
// CTAs read them from device memory and not each over the host link.  A programmatic dependent of the
// kernel before it: it copies only after griddepcontrol.wait (the previous step may still read dst,
// and the source may be an earlier step's output), and the step's kernel after it may start early.
__global__ void __launch_bounds__(512) stage_tokens_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                          int n16) {
  pdl_launch_dependents();
  pdl_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n16) dst[i] = src[i];
}

cudaError_t launch_stage_tokens(const void* src, void* dst, size_t bytes, cudaStream_t s) {
  if (bytes % 16 != 0 || ((uintptr_t)src & 15u) || ((uintptr_t)dst & 15u)) return cudaErrorInvalidValue;
  const int n16 = (int)(bytes / 16);
  if (n16 == 0) return cudaSuccess;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((n16 + 511) / 512));
  cfg.blockDim = dim3(512);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, stage_tokens_kernel, reinterpret_cast<const uint4*>(src),
                            reinterpret_cast<uint4*>(dst), n16);
}

cudaError_t launch_cats_ring(const FusedArgs& a, int wdtype, cudaStream_t s) {
  const int kv = ring_kv(a.d, a.B, wdtype);
  if (kv == 0 || a.u_rt) return cudaErrorInvalidValue;
  const int t = batch_tier(a.B);
  if (wdtype == CSFFN_F32) {
    switch (t) {
      case 1: return ring_kv_t<float, 1>(a, kv, s);
      case 2: return ring_kv_t<float, 2>(a, kv, s);
      default: return ring_kv_t<float, 4>(a, kv, s);
    }
  }
  switch (t) {
    case 1: return ring_kv_t<bf16, 1>(a, kv, s);
    case 2: return ring_kv_t<bf16, 2>(a, kv, s);
    default: return ring_kv_t<bf16, 4>(a, kv, s);
  }
}

}  // namespace csffn
