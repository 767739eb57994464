// SVD-predicted sparse FFN decode step (batches of up to 4 tokens) in one cooperative launch.
//
// "SVD Contextual Sparsity Predictors for Fast LLM Inference": Fig. 1 (the predictor p = x U_r
// V_r^T + beta against per-neuron thresholds tau), Fig. 3 (the gate runs on the predicted set, up
// and down on the active set) and Table 3 (the parallel pipeline: gate and up both on the predicted
// set).  A neuron is processed when some token predicts it (p > tau); each token then keeps it when
// |act(z + beta)| > t, as in the CATS step.
//
// The step reads a few tens of MB in a chain of dependent round trips (U_r, then V_r, then the
// predicted W_gate rows, then the kept W_up / W_down^T rows), so it is laid out to keep that chain
// short rather than to stream.  One CTA per SM, each owning a fixed range of neurons:
//  * y = x U_r: CTA c bulk-copies rows c, c + G, ... of U_r^T into shared memory and writes those
//    entries of y; the CTAs then meet at one grid-wide count (all are resident: cooperative launch).
//    The CTA's V_r rows are copied in at the same time, so they are there when y is.
//  * Each CTA forms p for its rows, fetches the predicted rows' W_gate (and W_up, parallel pipeline)
//    in one wave of bulk copies, thresholds them, and fetches the kept rows' W_up and W_down^T
//    together (their copies do not depend on each other); v = a * u times the W_down^T rows
//    accumulates in registers, and the CTA adds its partial output into one of a few fp32
//    accumulators in L2.
//  * After a second grid-wide count (every partial output and every CTA's kept count is written),
//    each CTA writes its kept rows into idx / a_val at the offset the counts before it give, and sums
//    an equal slice of the accumulators into out (clearing them).
// Every wait is bounded; the counters and the accumulators return to zero by themselves.
#include "common.cuh"
#include "fused_end.cuh"
#include "gemv.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace csffn {

constexpr int kSvdThreads = 512;
constexpr int kSvdWarps = kSvdThreads / kWarp;
// FusedArgs::ctl words of the two grid-wide counts (each a count and a generation)
constexpr int kCtlSvdDone = 4, kCtlSvdDoneGen = 6;  // CTAs whose partial output and kept count are written
constexpr int kCtlSvdY = 5, kCtlSvdYGen = 7;        // CTAs whose entries of y are written
constexpr size_t kSvdSmemBudget = 200 * 1024;  // dynamic shared memory of the step kernel
constexpr size_t kSvdVBudget = 96 * 1024;      // V_r rows staged at a time
constexpr int kSvdMinSlots = 4;                // weight-row slots at least (else the fused kernel runs)

__device__ __forceinline__ void proxy_fence_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void svd_pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// One grid-wide count, by one thread of each CTA (all CTAs resident): the last to arrive resets the
// count to zero and advances the generation, which the others wait for (bounded).  Self-resetting:
// the next launch finds the count at zero.
__device__ __forceinline__ void grid_count(uint32_t* count, uint32_t* gen, uint32_t n, uint32_t* err) {
  const uint32_t g0 = ld_acquire_u32(gen);  // read before arriving: the last arrival changes it
  if (atomicAdd(count, 1u) == n - 1u) {
    *reinterpret_cast<volatile uint32_t*>(count) = 0u;
    __threadfence();
    atomicAdd(gen, 1u);
    return;
  }
  if (ld_acquire_u32(gen) != g0) return;
  const uint64_t t0 = globaltimer_now();
  while (ld_acquire_u32(gen) == g0) {
    if (globaltimer_now() - t0 > 1000000000ull) {
      atomicOr(err, kDevErrTimeout);
      return;
    }
    __nanosleep(32);
  }
}

// Shared-memory plan of the step kernel (host and device compute the same).
struct SvdPlan {
  int rows_max;    // neurons per CTA at most
  int vrows;       // V_r rows per staged chunk
  int slots;       // weight-row slots of d elements
  size_t v_off, x_off, y_off, slot_off, total;
};

__host__ __device__ inline SvdPlan svd_plan(int d, int h, int rank, int nb, int es, int grid) {
  SvdPlan s;
  s.rows_max = (h + grid - 1) / grid;
  const size_t vrow = (size_t)rank * es;
  const size_t vmax = kSvdVBudget / vrow;
  s.vrows = (int)((size_t)s.rows_max < vmax ? (size_t)s.rows_max : vmax);
  s.v_off = 0;
  s.x_off = align_up((size_t)s.vrows * vrow, 128);
  s.y_off = s.x_off + align_up((size_t)nb * d * es, 128);
  s.slot_off = s.y_off + align_up((size_t)nb * rank * sizeof(float), 128);
  const size_t left = kSvdSmemBudget > s.slot_off ? kSvdSmemBudget - s.slot_off : 0;
  s.slots = (int)(left / ((size_t)d * es));
  if (s.slots > 32) s.slots = 32;
  s.total = s.slot_off + (size_t)s.slots * d * es;
  return s;
}

// ---------------------------------------------------------------------------------------------
// The step: predictor, gate, up and down for neurons [h * c / G, h * (c + 1) / G) of CTA c.
// ---------------------------------------------------------------------------------------------
constexpr int kSvdMaxRows = 256;  // neurons per CTA at most
constexpr int kSvdMaxSlots = 32;

template <typename WT, int NB, int KD, bool PAR>
__global__ void __launch_bounds__(kSvdThreads, 1) svd_step_kernel(const FusedArgs p, const SvdPlan pl) {
  extern __shared__ __align__(128) unsigned char svd_smem[];
  constexpr int EPV = Vec<WT>::N;
  __shared__ __align__(8) uint64_t s_vbar, s_gbar, s_ubar, s_ybar;
  __shared__ int s_abort;
  __shared__ uint8_t s_pred[kSvdMaxRows];     // predicted (some token), by local row
  __shared__ int s_plist[kSvdMaxRows];         // predicted local rows, ascending
  __shared__ int s_klist[kSvdMaxRows];         // kept neurons, ascending
  __shared__ float s_ka[kSvdMaxRows][NB];      // their activations (0 for a token that rejects)
  __shared__ float s_ku[PAR ? kSvdMaxRows : 1][NB];  // parallel pipeline: their up projections
  __shared__ uint8_t s_keep[kSvdMaxSlots];     // keep flag of each row of a gate wave
  __shared__ float s_wa[kSvdMaxSlots][NB];     // a (and u) of each row of a gate wave
  __shared__ float s_wu[PAR ? kSvdMaxSlots : 1][NB];
  __shared__ float s_v[kSvdMaxSlots][NB];      // v = a * u of each row of an up/down wave
  __shared__ int s_npred, s_nkept;
  __shared__ float s_tau[kSvdMaxRows], s_beta[kSvdMaxRows];  // thresholds and gate biases of the rows
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int d = p.d, h = p.h, B = p.B, rank = p.rank;
  const int r0 = (int)((long long)h * blockIdx.x / gridDim.x);
  const int nrows = (int)((long long)h * (blockIdx.x + 1) / gridDim.x) - r0;
  WT* vs = reinterpret_cast<WT*>(svd_smem + pl.v_off);
  WT* xs = reinterpret_cast<WT*>(svd_smem + pl.x_off);
  float* ys = reinterpret_cast<float*>(svd_smem + pl.y_off);
  WT* slots = reinterpret_cast<WT*>(svd_smem + pl.slot_off);
  const WT* Vr = reinterpret_cast<const WT*>(p.v_r);
  const WT* Wg = reinterpret_cast<const WT*>(p.W_gate);
  const WT* Wu = reinterpret_cast<const WT*>(p.W_up);
  const WT* Wd = reinterpret_cast<const WT*>(p.W_down_t);
  const uint32_t vrow_bytes = (uint32_t)(rank * sizeof(WT)), row_bytes = (uint32_t)(d * sizeof(WT));
  uint32_t issued[3] = {0u, 0u, 0u};  // thread 0: copies issued on s_vbar, s_gbar, s_ubar (phases)
  uint32_t waited[3] = {0u, 0u, 0u};  // phases every thread has waited for

  // rows of U_r^T whose y this CTA computes: k = c, c + G, ... (at most pl.slots of them)
  const int G = gridDim.x;
  const int ymine = (int)blockIdx.x < rank ? (rank - (int)blockIdx.x + G - 1) / G : 0;
  svd_pdl_wait();  // the inputs may come from the previous kernel
  if (tid == 0) {
    s_abort = 0;
    s_nkept = 0;
    mbar_init(&s_vbar, 1);
    mbar_init(&s_gbar, 1);
    mbar_init(&s_ubar, 1);
    mbar_init(&s_ybar, 1);
    fence_mbar_init();
    // the tokens and this CTA's rows of U_r^T for y, then the first chunk of its V_r rows (in
    // flight during the y phase): all at once
    mbar_arrive_expect_tx(&s_ybar, (uint32_t)(ymine + B) * row_bytes);
    bulk_load(xs, p.x, (uint32_t)B * row_bytes, &s_ybar);
    for (int i = 0; i < ymine; ++i)
      bulk_load(slots + (size_t)i * d, reinterpret_cast<const WT*>(p.u_rt) + (size_t)((int)blockIdx.x + i * G) * d,
                row_bytes, &s_ybar);
    if (nrows > 0) {
      const int n0 = min(nrows, pl.vrows);
      mbar_arrive_expect_tx(&s_vbar, (uint32_t)n0 * vrow_bytes);
      bulk_load(vs, Vr + (size_t)r0 * rank, (uint32_t)n0 * vrow_bytes, &s_vbar);
      issued[0] = 1;
    }
  }
  {  // tokens B..NB-1 of the staged block read as zeros
    uint4* xz = reinterpret_cast<uint4*>(xs + (size_t)B * d);
    for (int e = tid; e < (NB - B) * (int)(row_bytes / 16); e += kSvdThreads) xz[e] = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();

  bool ok = true;
  // ---- 0. y = x U_r: this CTA's rows (one warp each), then one grid-wide count
  if (__syncthreads_or(!mbar_wait(&s_ybar, 0u, p.err, &s_abort))) ok = false;
  for (int i = warp; ok && i < ymine; i += kSvdWarps) {
    float yk[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) yk[b] = 0.f;
    smem_row_dot<WT, NB>(slots + (size_t)i * d, xs, d, lane, yk);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      yk[b] = warp_sum(yk[b]);
      if (lane == 0 && b < B) __stcg(p.ybuf + (size_t)b * rank + (int)blockIdx.x + i * G, yk[b]);
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) grid_count(p.ctl + kCtlSvdY, p.ctl + kCtlSvdYGen, (uint32_t)G, p.err);
  // thresholds and gate biases of this CTA's rows, loaded while the count completes
  for (int q = tid; q < nrows; q += kSvdThreads) {
    s_tau[q] = __ldg(p.tau + r0 + q);
    s_beta[q] = p.bias ? __ldg(p.bias + r0 + q) : 0.f;
  }
  __syncthreads();
  __threadfence();
  for (int e = tid; e < NB * rank; e += kSvdThreads) ys[e] = e / rank < B ? __ldcg(p.ybuf + e) : 0.f;
  __syncthreads();

  // ---- 1. the prediction p = y . V_r[i] + beta_i against tau_i, union over tokens
  for (int c0 = 0; ok && c0 < nrows; c0 += pl.vrows) {
    const int n = min(pl.vrows, nrows - c0);
    if (__syncthreads_or(!mbar_wait(&s_vbar, waited[0] & 1u, p.err, &s_abort))) {
      ok = false;
      break;
    }
    ++waited[0];
    for (int q = warp; q < n; q += kSvdWarps) {
      float z[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) z[b] = 0.f;
      smem_dot_f32<WT, NB>(vs + (size_t)q * rank, ys, rank, lane, z);
      const float tau = s_tau[c0 + q], beta = s_beta[c0 + q];
      bool pred = false;
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float pb = warp_sum(z[b]) + beta;
        pred |= b < B && pb > tau;
      }
      if (lane == 0) s_pred[c0 + q] = pred ? 1 : 0;
    }
    __syncthreads();  // the chunk is read
    if (tid == 0 && c0 + pl.vrows < nrows) {
      const int n1 = min(pl.vrows, nrows - c0 - pl.vrows);
      proxy_fence_smem();
      mbar_arrive_expect_tx(&s_vbar, (uint32_t)n1 * vrow_bytes);
      bulk_load(vs, Vr + (size_t)(r0 + c0 + pl.vrows) * rank, (uint32_t)n1 * vrow_bytes, &s_vbar);
      ++issued[0];
    }
  }
  if (warp == 0) {  // the predicted rows in ascending order
    int cnt = 0;
    for (int base = 0; base < nrows; base += kWarp) {
      const bool f = ok && base + lane < nrows && s_pred[base + lane];
      const uint32_t m = __ballot_sync(0xffffffffu, f);
      if (f) s_plist[cnt + __popc(m & ((1u << lane) - 1u))] = base + lane;
      cnt += __popc(m);
    }
    if (lane == 0) s_npred = cnt;
  }
  __syncthreads();

  // ---- 2. gate (and up, parallel pipeline) of the predicted rows, in waves of slot-fulls
  const int npred = s_npred;
  const int grow = PAR ? pl.slots / 2 : pl.slots;
  for (int w0 = 0; ok && w0 < npred; w0 += grow) {
    const int n = min(grow, npred - w0);
    if (tid == 0) {
      proxy_fence_smem();  // the slots' previous contents were read through the generic proxy
      mbar_arrive_expect_tx(&s_gbar, (uint32_t)n * (PAR ? 2u : 1u) * row_bytes);
      for (int k = 0; k < n; ++k) {
        const int i = r0 + s_plist[w0 + k];
        bulk_load(slots + (size_t)k * d, Wg + (size_t)i * d, row_bytes, &s_gbar);
        if (PAR) bulk_load(slots + (size_t)(n + k) * d, Wu + (size_t)i * d, row_bytes, &s_gbar);
      }
      ++issued[1];
    }
    if (__syncthreads_or(!mbar_wait(&s_gbar, waited[1] & 1u, p.err, &s_abort))) {
      ok = false;
      break;
    }
    ++waited[1];
    for (int k = warp; k < n; k += kSvdWarps) {
      const int q = s_plist[w0 + k], i = r0 + q;
      float z[NB], u[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) z[b] = u[b] = 0.f;
      smem_row_dot<WT, NB>(slots + (size_t)k * d, xs, d, lane, z);
      if (PAR) smem_row_dot<WT, NB>(slots + (size_t)(n + k) * d, xs, d, lane, u);
      const float beta = s_beta[q];
      bool any = false;
      float a[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float ab = gate_act(warp_sum(z[b]) + beta, p.act);
        const bool kb = b < B && fabsf(ab) > p.t;
        a[b] = kb ? ab : 0.f;
        any |= kb;
        if (PAR) u[b] = warp_sum(u[b]);
      }
      if (lane == 0) {
        s_keep[k] = any ? 1 : 0;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          s_wa[k][b] = a[b];
          if (PAR) s_wu[PAR ? k : 0][b] = u[b];
        }
      }
    }
    __syncthreads();
    if (warp == 0) {  // append the wave's kept rows, in order
      int nk = s_nkept;
      for (int base = 0; base < n; base += kWarp) {
        const bool f = base + lane < n && s_keep[base + lane];
        const uint32_t m = __ballot_sync(0xffffffffu, f);
        if (f) {
          const int pos = nk + __popc(m & ((1u << lane) - 1u));
          s_klist[pos] = r0 + s_plist[w0 + base + lane];
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            s_ka[pos][b] = s_wa[base + lane][b];
            if (PAR) s_ku[PAR ? pos : 0][b] = s_wu[PAR ? base + lane : 0][b];
          }
        }
        nk += __popc(m);
      }
      if (lane == 0) s_nkept = nk;
    }
    __syncthreads();
  }

  // ---- 3. up and down of the kept rows: both rows of a kept neuron are copied together
  float acc[NB][KD][EPV];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int k = 0; k < KD; ++k)
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[b][k][e] = 0.f;
  const int nkept = ok ? s_nkept : 0;
  const int urow = PAR ? pl.slots : pl.slots / 2;
  for (int w0 = 0; ok && w0 < nkept; w0 += urow) {
    const int n = min(urow, nkept - w0);
    if (tid == 0) {
      proxy_fence_smem();
      mbar_arrive_expect_tx(&s_ubar, (uint32_t)n * (PAR ? 1u : 2u) * row_bytes);
      for (int k = 0; k < n; ++k) {
        const int i = s_klist[w0 + k];
        bulk_load(slots + (size_t)k * d, Wd + (size_t)i * d, row_bytes, &s_ubar);
        if (!PAR) bulk_load(slots + (size_t)(n + k) * d, Wu + (size_t)i * d, row_bytes, &s_ubar);
      }
      ++issued[2];
    }
    if (__syncthreads_or(!mbar_wait(&s_ubar, waited[2] & 1u, p.err, &s_abort))) {
      ok = false;
      break;
    }
    ++waited[2];
    if (!PAR) {
      for (int k = warp; k < n; k += kSvdWarps) {
        float u[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) u[b] = 0.f;
        smem_row_dot<WT, NB>(slots + (size_t)(n + k) * d, xs, d, lane, u);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          u[b] = warp_sum(u[b]);
          if (lane == 0) s_v[k][b] = s_ka[w0 + k][b] * u[b];
        }
      }
    } else {
      for (int e = tid; e < n * NB; e += kSvdThreads)
        s_v[e / NB][e % NB] = s_ka[w0 + e / NB][e % NB] * s_ku[PAR ? w0 + e / NB : 0][e % NB];
    }
    __syncthreads();
    for (int k = 0; k < n; ++k) {
      const WT* row = slots + (size_t)k * d;
#pragma unroll
      for (int kd = 0; kd < KD; ++kd) {
        const int c = (kd * kSvdThreads + tid) * EPV;
        if (c < d) {
          float wf[EPV];
          unpack(*reinterpret_cast<const uint4*>(row + c), wf);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            const float vb = s_v[k][b];
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc[b][kd][e] = fmaf(vb, wf[e], acc[b][kd][e]);
          }
        }
      }
    }
    __syncthreads();  // the slots are refilled by the next wave
  }
  if (nkept > 0) {
    float* accp = p.facc + (size_t)(blockIdx.x % kFusedAccCopies) * B * d;
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      if (b < B) {
#pragma unroll
        for (int kd = 0; kd < KD; ++kd) {
          const int c = (kd * kSvdThreads + tid) * EPV;
          if (c < d) {
#pragma unroll
            for (int e = 0; e < EPV; e += 4)
              red_add_v4(accp + (size_t)b * d + c + e, acc[b][kd][e], acc[b][kd][e + 1], acc[b][kd][e + 2],
                         acc[b][kd][e + 3]);
          }
        }
      }
    }
  }
  if (tid == 0) {  // copies issued but never waited for (a wait that ran out) land before the CTA ends
    uint64_t* bars[3] = {&s_vbar, &s_gbar, &s_ubar};
    for (int k = 0; k < 3; ++k)
      if (issued[k] > waited[k]) mbar_wait_drain(bars[k], (issued[k] - 1u) & 1u, p.err);
  }

  // ---- 4. one more grid-wide count, then every CTA writes its kept rows and a slice of out
  if (tid == 0) p.svd_counts[blockIdx.x] = ok ? (uint32_t)nkept : 0u;
  __threadfence();
  __syncthreads();
  if (tid == 0) grid_count(p.ctl + kCtlSvdDone, p.ctl + kCtlSvdDoneGen, (uint32_t)G, p.err);
  __syncthreads();
  __threadfence();
  // the kept rows of the CTAs before this one set where this CTA's kept rows go in idx / a_val
  if (warp == 0) {
    uint32_t before = 0u, total = 0u;
    for (int c = lane; c < G; c += kWarp) {
      const uint32_t v = __ldcg(p.svd_counts + c);
      before += c < (int)blockIdx.x ? v : 0u;
      total += v;
    }
    before = warp_sum_u32(before);
    total = warp_sum_u32(total);
    for (int k = lane; k < nkept; k += kWarp) {
      p.idx[before + k] = s_klist[k];
#pragma unroll
      for (int b = 0; b < NB; ++b)
        if (b < B) p.a_val[(size_t)b * h + before + k] = s_ka[k][b];
    }
    if (blockIdx.x == 0 && lane == 0) *p.count = (int32_t)total;
  } else {
    // out over this CTA's slice of the columns: the sum of the accumulators, which are cleared
    const int n4 = B * d / 4;
    const int i0 = (int)((long long)n4 * blockIdx.x / G), i1 = (int)((long long)n4 * (blockIdx.x + 1) / G);
    for (int i = i0 + tid - kWarp; i < i1; i += kSvdThreads - kWarp) {
      float4 s4[kFusedAccCopies];
#pragma unroll
      for (int c = 0; c < kFusedAccCopies; ++c) s4[c] = __ldcg(reinterpret_cast<const float4*>(p.facc + (size_t)c * B * d) + i);
      float4 t4 = s4[0];
#pragma unroll
      for (int c = 1; c < kFusedAccCopies; ++c) {
        t4.x += s4[c].x;
        t4.y += s4[c].y;
        t4.z += s4[c].z;
        t4.w += s4[c].w;
      }
#pragma unroll
      for (int c = 0; c < kFusedAccCopies; ++c)
        __stcg(reinterpret_cast<float4*>(p.facc + (size_t)c * B * d) + i, make_float4(0.f, 0.f, 0.f, 0.f));
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
    }
  }
}

// ---------------------------------------------------------------------------------------------
// Launcher
// ---------------------------------------------------------------------------------------------
namespace {

int svd_kd(int d, int epv) { return (d + kSvdThreads * epv - 1) / (kSvdThreads * epv); }

template <typename WT, int NB, int KD, bool PAR>
cudaError_t launch_step_t(const FusedArgs& a, const SvdPlan& pl, int grid, cudaStream_t s) {
  auto kern = svd_step_kernel<WT, NB, KD, PAR>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pl.total);
  if (e != cudaSuccess) return e;
  // one CTA per SM, all resident at once (the y count waits for every CTA)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kSvdThreads);
  cfg.gridDim = dim3(grid);
  cfg.dynamicSmemBytes = pl.total;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, pl);
}

template <typename WT, int NB, bool PAR>
cudaError_t launch_kd(const FusedArgs& a, const SvdPlan& pl, int grid, int kd, cudaStream_t s) {
  constexpr int EPV = Vec<WT>::N;
  switch (kd) {
    case 1: return launch_step_t<WT, NB, 1, PAR>(a, pl, grid, s);
    case 2:
      if constexpr (NB * 2 * EPV <= 32) return launch_step_t<WT, NB, 2, PAR>(a, pl, grid, s);
      break;
    case 4:
      if constexpr (NB * 4 * EPV <= 32) return launch_step_t<WT, NB, 4, PAR>(a, pl, grid, s);
      break;
    default: break;
  }
  return cudaErrorInvalidValue;
}

template <typename WT, bool PAR>
cudaError_t launch_nb(const FusedArgs& a, const SvdPlan& pl, int grid, int kd, cudaStream_t s) {
  switch (batch_tier(a.B)) {
    case 1: return launch_kd<WT, 1, PAR>(a, pl, grid, kd, s);
    case 2: return launch_kd<WT, 2, PAR>(a, pl, grid, kd, s);
    case 4: return launch_kd<WT, 4, PAR>(a, pl, grid, kd, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool svd_step_supported(int d, int h, int B, int wdtype, int rank) {
  const int es = wdtype == CSFFN_F32 ? 4 : 2, epv = 16 / es;
  if (B < 1 || B > 4 || rank < 1 || rank % epv != 0 || d % epv != 0) return false;
  int kd = svd_kd(d, epv);
  kd = kd <= 1 ? 1 : kd <= 2 ? 2 : kd <= 4 ? 4 : 0;
  if (kd == 0 || batch_tier(B) * kd * epv > 32) return false;
  const int grid = sm_count();
  if (grid < 1 || grid > kTcMaxCtas || (h + grid - 1) / grid > kSvdMaxRows) return false;
  const SvdPlan pl = svd_plan(d, h, rank, batch_tier(B), es, grid);
  return pl.vrows >= 1 && pl.slots >= kSvdMinSlots && pl.slots >= (rank + grid - 1) / grid &&
         pl.total <= kSvdSmemBudget;
}

cudaError_t launch_svd_step(const FusedArgs& a, int wdtype, bool parallel, cudaStream_t s) {
  if (!svd_step_supported(a.d, a.h, a.B, wdtype, a.rank)) return cudaErrorInvalidValue;
  const int es = wdtype == CSFFN_F32 ? 4 : 2, epv = 16 / es;
  int kd = svd_kd(a.d, epv);
  kd = kd <= 1 ? 1 : kd <= 2 ? 2 : 4;
  const int grid = sm_count();
  const SvdPlan pl = svd_plan(a.d, a.h, a.rank, batch_tier(a.B), es, grid);
  if (wdtype == CSFFN_F32)
    return parallel ? launch_nb<float, true>(a, pl, grid, kd, s) : launch_nb<float, false>(a, pl, grid, kd, s);
  return parallel ? launch_nb<bf16, true>(a, pl, grid, kd, s) : launch_nb<bf16, false>(a, pl, grid, kd, s);
}

}  // namespace csffn
