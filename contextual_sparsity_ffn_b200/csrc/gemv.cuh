// Warp-level multi-row GEMV core shared by the gate, up, dense and predictor kernels.
//
// A warp reduces R weight rows (contiguous, 16-byte vectors, streamed once from HBM with
// non-allocating loads) against NB token vectors held in shared memory.  Each lane walks the
// row in 16-byte vectors strided by the warp width; U vectors per row are loaded before any is
// used, so a warp keeps R*U*512 bytes of loads in flight.
#pragma once

#include "common.cuh"

namespace csffn {

// Unroll depth (16-byte vectors per row in flight per lane) by token capacity.
template <int NB>
struct GemvUnroll {
  static constexpr int value = NB <= 2 ? 8 : (NB <= 4 ? 4 : (NB <= 8 ? 2 : 1));
};

// acc[r][b] += sum_k W_r[k] * x_b[k] over this lane's share of k; caller reduces over the warp.
//   rows[r]: start of row r (global), valid[r]: row exists (warp-uniform).
//   xs: shared memory [NB][K] (tokens >= B zero-filled), K % Vec<WT>::N == 0.
template <typename WT, typename XT, int NB, int R, int U>
__device__ __forceinline__ void rows_dot(const WT* const (&rows)[R], const bool (&valid)[R],
                                         const XT* __restrict__ xs, int K, int lane,
                                         float (&acc)[R][NB]) {
  constexpr int EPV = Vec<WT>::N;
  const int NV = K / EPV;
  for (int v0 = lane; v0 < NV; v0 += kWarp * U) {
    uint4 w[U][R];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * kWarp;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (valid[r] && v < NV)
          w[u][r] = ld_stream(rows[r] + (size_t)v * EPV);
        else
          w[u][r] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * kWarp;
      if (v < NV) {
        float wf[R][EPV];
#pragma unroll
        for (int r = 0; r < R; ++r) unpack(w[u][r], wf[r]);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          float xf[EPV];
          load_x<EPV>(xs + (size_t)b * K + (size_t)v * EPV, xf);
#pragma unroll
          for (int r = 0; r < R; ++r) {
#pragma unroll
            for (int e = 0; e < EPV; ++e) acc[r][b] = fmaf(wf[r][e], xf[e], acc[r][b]);
          }
        }
      }
    }
  }
}

template <int R, int NB>
__device__ __forceinline__ void warp_reduce_all(float (&acc)[R][NB]) {
#pragma unroll
  for (int r = 0; r < R; ++r) {
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = warp_sum(acc[r][b]);
  }
}

// Copy B token vectors [B][K] (global, type XT) into shared memory [NB][K], zero-filling tokens
// B..NB-1.  K * sizeof(XT) is a multiple of 16 bytes; the whole block participates.
template <typename XT, int NB>
__device__ __forceinline__ void stage_tokens(XT* xs, const XT* __restrict__ xg, int B, int K) {
  const int per_tok = (int)((size_t)K * sizeof(XT) / 16);
  uint4* dst = reinterpret_cast<uint4*>(xs);
  const uint4* src = reinterpret_cast<const uint4*>(xg);
  for (int e = threadIdx.x; e < NB * per_tok; e += blockDim.x) {
    const int b = e / per_tok;
    dst[e] = b < B ? src[e] : make_uint4(0u, 0u, 0u, 0u);
  }
}

// acc[b] += W[row] . x_b over this lane's share, row and tokens both in shared memory.
template <typename WT, int NB>
__device__ __forceinline__ void smem_row_dot(const WT* row, const WT* xs, int K, int lane, float (&acc)[NB]) {
  constexpr int EPV = Vec<WT>::N;
  const int NV = K / EPV;
#pragma unroll 4
  for (int v = lane; v < NV; v += kWarp) {
    const uint4 w = *reinterpret_cast<const uint4*>(row + (size_t)v * EPV);
    float wf[EPV];
    unpack(w, wf);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float xf[EPV];
      load_x<EPV>(xs + (size_t)b * K + (size_t)v * EPV, xf);
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[b] = fmaf(wf[e], xf[e], acc[b]);
    }
  }
}

// acc[b] += row[0 .. n) . y_b[0 .. n): a row in shared memory against fp32 vectors y_b = ys + b * n.
template <typename WT, int NB>
__device__ __forceinline__ void smem_dot_f32(const WT* row, const float* ys, int n, int lane, float (&acc)[NB]) {
  constexpr int EPV = Vec<WT>::N;
  const int nv = n / EPV;
#pragma unroll 4
  for (int v = lane; v < nv; v += kWarp) {
    float wf[EPV];
    unpack(*reinterpret_cast<const uint4*>(row + (size_t)v * EPV), wf);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float yf[EPV];
      load_x<EPV>(ys + (size_t)b * n + (size_t)v * EPV, yf);
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[b] = fmaf(wf[e], yf[e], acc[b]);
    }
  }
}

}  // namespace csffn
