// Gathered up- and down-projection over the active neurons, the dense gate/up pass, and a
// plain row GEMV (predictor y = x U_r, calibration activations).
//
// "CATS: Contextually-Aware Thresholding for Sparsity in Large Language Models", abstract: a
// flag-gated GEMV reads only the weights of neurons whose gate survived the threshold.  With
// neuron-major W_up and W_down^T, that is a gather of whole contiguous rows.
//
// Down projection layout: the grid is (column slices) x (row ranges).  A slice is 512 bytes of a
// row (one 16-byte vector per lane); a CTA's 8 warps stream interleaved rows of its range and
// accumulate in registers, reduce across warps in shared memory, write one partial per
// (row range, token, column), and the last CTA to finish a slice sums that slice's partials in
// row-range order.  The result is deterministic and needs no atomics on the data.
#include "common.cuh"
#include "gemv.cuh"
#include "kernels.h"

#include <mutex>

namespace csffn {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / kWarp;

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

template <typename K>
static int occupancy(K kern, int threads, size_t smem) {
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, smem) != cudaSuccess) return 1;
  return occ < 1 ? 1 : occ;
}

template <typename K>
static cudaError_t allow_smem(K kern, size_t smem) {
  if (smem <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

// ------------------------------------------------------------------------------------------
// Up projection over the compacted active list: v[b, j] = a_val[b, j] * (x_b . W_up[idx[j]])
// ------------------------------------------------------------------------------------------
// One row per warp at a time with GemvUnroll vectors in flight per lane, four CTAs per SM: many
// independent row streams keep HBM busy (a gathered row cannot be fetched as one large block).
// A warp's row indices and a_val values are fetched once, up front, one per lane.  The tokens are
// staged in shared memory (measured faster than reading them through the read-only cache).
template <typename WT, int NB>
__global__ void __launch_bounds__(kThreads, 4) up_gather_kernel(const UpArgs p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  constexpr bool kStage = true;
  constexpr int EPV = Vec<WT>::N;
  constexpr int U = GemvUnroll<NB>::value;
  const int lane = threadIdx.x & 31;
  const WT* xs = reinterpret_cast<const WT*>(p.x);
  if (kStage) {
    stage_tokens<WT, NB>(reinterpret_cast<WT*>(smem_raw), reinterpret_cast<const WT*>(p.x), p.B, p.d);
    __syncthreads();
    xs = reinterpret_cast<const WT*>(smem_raw);
  }
  const int n = min(max(*p.count, 0), p.h);
  const int gw = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int GW = gridDim.x * kWarps;
  const WT* W = reinterpret_cast<const WT*>(p.W_up);
  const int NV = p.d / EPV;
  for (int j0 = gw; j0 < n; j0 += GW * kWarp) {
    // rows j0 + k*GW for k = 0..31, one per lane: index and per-token a_val
    const int my_j = j0 + lane * GW;
    int my_row = my_j < n ? p.idx[my_j] : 0;
    if ((unsigned)my_row >= (unsigned)p.h) my_row = 0;  // malformed index: stay in bounds
    float my_a[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) my_a[b] = (my_j < n && b < p.B) ? p.a_val[(size_t)b * p.h + my_j] : 0.f;
    const int cnt = __popc(__ballot_sync(0xffffffffu, my_j < n));
    for (int k = 0; k < cnt; ++k) {
      const WT* row = W + (size_t)__shfl_sync(0xffffffffu, my_row, k) * p.d;
      float acc[NB];
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[b] = 0.f;
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
              if (kStage) {
                load_x<EPV>(xs + (size_t)b * p.d + (size_t)v * EPV, xf);
              } else {
                const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xs + (size_t)b * p.d + (size_t)v * EPV));
                unpack_x<WT>(xv, xf);
              }
#pragma unroll
              for (int e = 0; e < EPV; ++e) acc[b] = fmaf(wf[e], xf[e], acc[b]);
            }
          }
        }
      }
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[b] = warp_sum(acc[b]);
      if (lane == k) {
#pragma unroll
        for (int b = 0; b < NB; ++b)
          if (b < p.B) p.v[(size_t)b * p.h + my_j] = my_a[b] * acc[b];
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// Dense gate and up: v[b, i] = act(x_b . W_gate[i] + beta_i) * (x_b . W_up[i]) for all i
// ------------------------------------------------------------------------------------------
template <typename WT, int NB>
__global__ void __launch_bounds__(kThreads) dense_gate_up_kernel(const DenseGateUpArgs p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  WT* xs = reinterpret_cast<WT*>(smem_raw);
  constexpr int N = 2;  // neurons per warp pass (2 gate rows + 2 up rows)
  constexpr int R = 2 * N;
  constexpr int U = GemvUnroll<NB>::value > 1 ? GemvUnroll<NB>::value / 2 : 1;
  const int lane = threadIdx.x & 31;
  stage_tokens<WT, NB>(xs, reinterpret_cast<const WT*>(p.x), p.B, p.d);
  __syncthreads();
  const int groups = (p.h + N - 1) / N;
  const int gw = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int GW = gridDim.x * kWarps;
  const WT* Wg = reinterpret_cast<const WT*>(p.W_gate);
  const WT* Wu = reinterpret_cast<const WT*>(p.W_up);
  for (int g = gw; g < groups; g += GW) {
    const WT* rp[R];
    bool valid[R];
#pragma unroll
    for (int q = 0; q < N; ++q) {
      const int i = g * N + q;
      const bool ok = i < p.h;
      valid[q] = ok;
      valid[N + q] = ok;
      rp[q] = Wg + (size_t)(ok ? i : 0) * p.d;
      rp[N + q] = Wu + (size_t)(ok ? i : 0) * p.d;
    }
    float acc[R][NB];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
    rows_dot<WT, WT, NB, R, U>(rp, valid, xs, p.d, lane, acc);
    warp_reduce_all<R, NB>(acc);
#pragma unroll
    for (int q = 0; q < N; ++q) {
      if (lane == q && valid[q]) {
        const int i = g * N + q;
        const float beta = p.bias ? p.bias[i] : 0.f;
#pragma unroll
        for (int b = 0; b < NB; ++b)
          if (b < p.B) p.v[(size_t)b * p.h + i] = gate_act(acc[q][b] + beta, p.act) * acc[N + q][b];
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// Down projection over rows idx[0..n): out[b, :] = sum_j v[b, j] * W_down^T[idx[j], :]
// ------------------------------------------------------------------------------------------
// Rows per pipeline unit (one 16-byte vector per lane per row) and resident CTAs per SM the
// register budget is capped for.
template <int NB> struct DownUnroll { static constexpr int value = NB <= 2 ? 4 : 2; };
template <int NB> struct DownMinBlocks { static constexpr int value = NB <= 2 ? 4 : (NB <= 4 ? 3 : 1); };

template <typename WT, int NB>
__global__ void __launch_bounds__(kThreads, DownMinBlocks<NB>::value) down_gather_kernel(const DownArgs p) {
  constexpr int EPV = Vec<WT>::N;
  constexpr int SW = kWarp * EPV;  // columns per slice
  constexpr int U = DownUnroll<NB>::value;
  static_assert(kWarp % U == 0, "units never straddle a 32-row batch");
  __shared__ float red[kWarps][SW];
  __shared__ bool s_last;

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int slice = blockIdx.x, ry = blockIdx.y, RY = gridDim.y;
  const int n = p.count ? min(max(*p.count, 0), p.h) : p.n_host;
  const int jb = (int)((long long)n * ry / RY), je = (int)((long long)n * (ry + 1) / RY);
  const int c0 = slice * SW + lane * EPV;
  const bool col_ok = c0 < p.d;
  const WT* Wd = reinterpret_cast<const WT*>(p.W_down_t);

  float acc[NB][EPV];
#pragma unroll
  for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[b][e] = 0.f;

  // This warp's rows: m-th row is jb + warp + 8m, m < M.  Row indices and v values come in
  // batches of 32 (one per lane), the next batch fetched while the current one streams; the
  // weight loads run as a double-buffered pipeline of U-row units.
  const int M = je - jb - warp > 0 ? (je - jb - warp + kWarps - 1) / kWarps : 0;
  auto fetch = [&](int batch, int& row, float (&v)[NB]) {
    const int m = batch * kWarp + lane;
    const int j = jb + warp + m * kWarps;
    const bool ok = m < M;
    row = ok ? (p.idx ? p.idx[j] : j) : 0;
    if ((unsigned)row >= (unsigned)p.h) row = 0;  // malformed index: stay in bounds
#pragma unroll
    for (int b = 0; b < NB; ++b) v[b] = (ok && b < p.B) ? p.v[(size_t)b * p.h + j] : 0.f;
  };
  int cur_row = 0, nxt_row = 0;
  float cur_v[NB], nxt_v[NB];
  fetch(0, cur_row, cur_v);
  fetch(1, nxt_row, nxt_v);
  const int units = (M + U - 1) / U;
  constexpr int UPB = kWarp / U;  // units per batch
  uint4 bufA[U], bufB[U];
  auto load_unit = [&](int t, int cb, uint4 (&buf)[U]) {
    const int from_next = (t / UPB) != cb;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int m = t * U + u;
      const int src = m % kWarp;
      const int r = __shfl_sync(0xffffffffu, from_next ? nxt_row : cur_row, src);
      buf[u] = (m < M && col_ok) ? ld_stream(Wd + (size_t)r * p.d + c0) : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  auto consume = [&](int t, const uint4 (&buf)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int m = t * U + u;
      float wf[EPV];
      unpack(buf[u], wf);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const float vb = __shfl_sync(0xffffffffu, cur_v[b], m % kWarp);
        if (m < M) {
#pragma unroll
          for (int e = 0; e < EPV; ++e) acc[b][e] = fmaf(vb, wf[e], acc[b][e]);
        }
      }
    }
  };
  int cb = 0;  // batch held in cur_*
  if (units > 0) load_unit(0, cb, bufA);
  for (int t = 0; t < units; t += 2) {
    if (t + 1 < units) load_unit(t + 1, cb, bufB);
    consume(t, bufA);
    if ((t + 1) % UPB == 0 && t + 1 < units) {  // unit t closed batch cb
      ++cb;
      cur_row = nxt_row;
#pragma unroll
      for (int b = 0; b < NB; ++b) cur_v[b] = nxt_v[b];
      fetch(cb + 1, nxt_row, nxt_v);
    }
    if (t + 1 >= units) break;
    if (t + 2 < units) load_unit(t + 2, cb, bufA);
    consume(t + 1, bufB);
    if ((t + 2) % UPB == 0 && t + 2 < units) {  // unit t + 1 closed batch cb
      ++cb;
      cur_row = nxt_row;
#pragma unroll
      for (int b = 0; b < NB; ++b) cur_v[b] = nxt_v[b];
      fetch(cb + 1, nxt_row, nxt_v);
    }
  }

  // Cross-warp reduction, one partial row per token.
  const int col = slice * SW + threadIdx.x;
  for (int b = 0; b < p.B && b < NB; ++b) {
#pragma unroll
    for (int bb = 0; bb < NB; ++bb) {
      if (bb == b) {
#pragma unroll
        for (int e = 0; e < EPV; ++e) red[warp][lane * EPV + e] = acc[bb][e];
      }
    }
    __syncthreads();
    if (threadIdx.x < SW && col < p.d) {
      float s = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += red[w][threadIdx.x];
      p.partial[((size_t)ry * p.B + b) * p.d + col] = s;
    }
    __syncthreads();
  }

  // The last CTA of this slice sums the partials in row-range order.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t prev = atomicAdd(&p.slice_ctr[slice], 1u);
    s_last = prev == (uint32_t)(RY - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (threadIdx.x < SW && col < p.d) {
    for (int b = 0; b < p.B; ++b) {
      float s = 0.f;
      for (int r = 0; r < RY; ++r) s += __ldcg(p.partial + ((size_t)r * p.B + b) * p.d + col);
      const size_t o = (size_t)b * p.d + col;
      if (p.out_mode == CSFFN_OUT_BF16)
        reinterpret_cast<bf16*>(p.out)[o] = __float2bfloat16_rn(s);
      else if (p.out_mode == CSFFN_OUT_F32)
        reinterpret_cast<float*>(p.out)[o] = s;
      else
        reinterpret_cast<float*>(p.out)[o] += s;
    }
  }
  if (threadIdx.x == 0) p.slice_ctr[slice] = 0u;
}

// ------------------------------------------------------------------------------------------
// Plain row GEMV: y[b, row] = f(x_b . W[row] + bias[row]) (predictor, calibration)
// ------------------------------------------------------------------------------------------
template <typename WT, typename XT, int NB>
__global__ void __launch_bounds__(kThreads) row_gemv_kernel(const RowGemvArgs p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  XT* xs = reinterpret_cast<XT*>(smem_raw);
  constexpr int R = 2;
  constexpr int U = GemvUnroll<NB>::value;
  const int lane = threadIdx.x & 31;
  stage_tokens<XT, NB>(xs, reinterpret_cast<const XT*>(p.x), p.B, p.K);
  __syncthreads();
  const int groups = (p.rows + R - 1) / R;
  const int gw = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int GW = gridDim.x * kWarps;
  const WT* W = reinterpret_cast<const WT*>(p.W);
  for (int g = gw; g < groups; g += GW) {
    const WT* rp[R];
    bool valid[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int i = g * R + r;
      valid[r] = i < p.rows;
      rp[r] = W + (size_t)(valid[r] ? i : 0) * p.K;
    }
    float acc[R][NB];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
    rows_dot<WT, XT, NB, R, U>(rp, valid, xs, p.K, lane, acc);
    warp_reduce_all<R, NB>(acc);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (lane == r && valid[r]) {
        const int i = g * R + r;
        const float beta = p.bias ? p.bias[i] : 0.f;
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          if (b < p.B) {
            float y = acc[r][b] + beta;
            if (p.act >= 0) y = gate_act(y, p.act);
            if (p.abs_out) y = fabsf(y);
            const size_t o = p.transpose_out ? (size_t)i * p.y_stride + b : (size_t)b * p.y_stride + i;
            p.y[o] = y;
          }
        }
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// Launchers
// ------------------------------------------------------------------------------------------
template <typename KernT>
static int grid_for(KernT kern, size_t smem, int work_warps) {
  const int occ = occupancy(kern, kThreads, smem);
  int grid = sm_count() * occ;
  const int need = (work_warps + kWarps - 1) / kWarps;
  if (need < grid) grid = need;
  return grid < 1 ? 1 : grid;
}

template <typename WT, int NB>
static cudaError_t up_t(const UpArgs& a, cudaStream_t s) {
  auto kern = up_gather_kernel<WT, NB>;
  const size_t smem = (size_t)NB * a.d * sizeof(WT);
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  const int grid = grid_for(kern, smem, a.h);
  kern<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename WT, int NB>
static cudaError_t dense_t(const DenseGateUpArgs& a, cudaStream_t s) {
  auto kern = dense_gate_up_kernel<WT, NB>;
  const size_t smem = (size_t)NB * a.d * sizeof(WT);
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  const int grid = grid_for(kern, smem, (a.h + 1) / 2);
  kern<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <typename WT, int NB>
static cudaError_t down_t(const DownArgs& a, cudaStream_t s) {
  auto kern = down_gather_kernel<WT, NB>;
  constexpr int SW = kWarp * Vec<WT>::N;
  const int slices = (a.d + SW - 1) / SW;
  const int occ = occupancy(kern, kThreads, 0);
  int ry = (sm_count() * occ) / slices;  // one wave: every CTA resident at once
  if (ry < 1) ry = 1;
  if (ry > kMaxRowRanges) ry = kMaxRowRanges;
  const int max_rows = a.count ? a.h : a.n_host;
  if (ry > max_rows) ry = max_rows > 0 ? max_rows : 1;
  dim3 grid(slices, ry);
  kern<<<grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

template <typename WT, typename XT, int NB>
static cudaError_t gemv_t(const RowGemvArgs& a, cudaStream_t s) {
  auto kern = row_gemv_kernel<WT, XT, NB>;
  const size_t smem = (size_t)NB * a.K * sizeof(XT);
  cudaError_t e = allow_smem(kern, smem);
  if (e != cudaSuccess) return e;
  const int grid = grid_for(kern, smem, (a.rows + 1) / 2);
  kern<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

#define CSFFN_NB_SWITCH(B, CALL)               \
  switch (batch_tier(B)) {                     \
    case 1: return CALL(1);                    \
    case 2: return CALL(2);                    \
    case 4: return CALL(4);                    \
    case 8: return CALL(8);                    \
    default: return CALL(16);                  \
  }

cudaError_t launch_up_gather(const UpArgs& a, int wdtype, cudaStream_t s) {
  if (wdtype == CSFFN_F32) {
#define CALL(nb) up_t<float, nb>(a, s)
    CSFFN_NB_SWITCH(a.B, CALL)
#undef CALL
  }
#define CALL(nb) up_t<bf16, nb>(a, s)
  CSFFN_NB_SWITCH(a.B, CALL)
#undef CALL
}

cudaError_t launch_dense_gate_up(const DenseGateUpArgs& a, int wdtype, cudaStream_t s) {
  if (wdtype == CSFFN_F32) {
#define CALL(nb) dense_t<float, nb>(a, s)
    CSFFN_NB_SWITCH(a.B, CALL)
#undef CALL
  }
#define CALL(nb) dense_t<bf16, nb>(a, s)
  CSFFN_NB_SWITCH(a.B, CALL)
#undef CALL
}

cudaError_t launch_down_gather(const DownArgs& a, int wdtype, cudaStream_t s) {
  if (wdtype == CSFFN_F32) {
#define CALL(nb) down_t<float, nb>(a, s)
    CSFFN_NB_SWITCH(a.B, CALL)
#undef CALL
  }
#define CALL(nb) down_t<bf16, nb>(a, s)
  CSFFN_NB_SWITCH(a.B, CALL)
#undef CALL
}

cudaError_t launch_row_gemv(const RowGemvArgs& a, int wdtype, bool x_f32, cudaStream_t s) {
  if (wdtype == CSFFN_F32) {
#define CALL(nb) gemv_t<float, float, nb>(a, s)
    CSFFN_NB_SWITCH(a.B, CALL)
#undef CALL
  }
  if (x_f32) {
#define CALL(nb) gemv_t<bf16, float, nb>(a, s)
    CSFFN_NB_SWITCH(a.B, CALL)
#undef CALL
  }
#define CALL(nb) gemv_t<bf16, bf16, nb>(a, s)
  CSFFN_NB_SWITCH(a.B, CALL)
#undef CALL
}

}  // namespace csffn
