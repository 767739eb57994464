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
template <typename WT, int NB>
__global__ void __launch_bounds__(kThreads, 4) up_gather_kernel(const UpArgs p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  WT* xs = reinterpret_cast<WT*>(smem_raw);
  constexpr int R = 1;
  constexpr int U = GemvUnroll<NB>::value;
  const int lane = threadIdx.x & 31;
  stage_tokens<WT, NB>(xs, reinterpret_cast<const WT*>(p.x), p.B, p.d);
  __syncthreads();
  const int n = min(max(*p.count, 0), p.h);
  const int groups = (n + R - 1) / R;
  const int gw = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int GW = gridDim.x * kWarps;
  const WT* W = reinterpret_cast<const WT*>(p.W_up);
  for (int g = gw; g < groups; g += GW) {
    const WT* rp[R];
    bool valid[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int j = g * R + r;
      valid[r] = j < n;
      int row = valid[r] ? p.idx[j] : 0;
      if ((unsigned)row >= (unsigned)p.h) row = 0;  // malformed index: stay in bounds
      rp[r] = W + (size_t)row * p.d;
    }
    float acc[R][NB];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
    rows_dot<WT, WT, NB, R, U>(rp, valid, xs, p.d, lane, acc);
    warp_reduce_all<R, NB>(acc);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (lane == r && valid[r]) {
        const size_t j = (size_t)g * R + r;
#pragma unroll
        for (int b = 0; b < NB; ++b)
          if (b < p.B) p.v[(size_t)b * p.h + j] = p.a_val[(size_t)b * p.h + j] * acc[r][b];
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
template <int NB> struct DownUnroll { static constexpr int value = NB <= 2 ? 8 : (NB <= 4 ? 4 : 2); };

template <typename WT, int NB>
__global__ void __launch_bounds__(kThreads) down_gather_kernel(const DownArgs p) {
  constexpr int EPV = Vec<WT>::N;
  constexpr int SW = kWarp * EPV;  // columns per slice
  constexpr int U = DownUnroll<NB>::value;
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

  // This warp's rows: jb + warp, jb + warp + 8, ...; fetched 32 at a time (one per lane).
  for (int m0 = jb + warp; m0 < je; m0 += kWarps * kWarp) {
    const int my_j = m0 + lane * kWarps;
    const bool my_ok = my_j < je;
    int my_row = my_ok ? (p.idx ? p.idx[my_j] : my_j) : 0;
    if ((unsigned)my_row >= (unsigned)p.h) my_row = 0;  // malformed index: stay in bounds
    float my_v[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) my_v[b] = (my_ok && b < p.B) ? p.v[(size_t)b * p.h + my_j] : 0.f;
    const int cnt = __popc(__ballot_sync(0xffffffffu, my_ok));
    for (int q = 0; q < cnt; q += U) {
      uint4 w[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int row = __shfl_sync(0xffffffffu, my_row, (q + u) & 31);
        w[u] = (q + u < cnt && col_ok) ? ld_stream(Wd + (size_t)row * p.d + c0) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        float wf[EPV];
        unpack(w[u], wf);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          const float vb = __shfl_sync(0xffffffffu, my_v[b], (q + u) & 31);
          if (q + u < cnt) {
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc[b][e] = fmaf(vb, wf[e], acc[b][e]);
          }
        }
      }
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
