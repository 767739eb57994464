// Dense FFN of a block of up to 16 tokens on the tensor cores (bf16 in, fp32 accumulate).
//
// "Sirius: Contextual Sparsity with Correction for Efficient LLMs", section on the correction
// step: the full model re-reads a chunk of recent tokens in parallel, so the dense FFN runs on a
// block of tokens (16 here) instead of one.  At B = 16 the FFN does 16 multiply-adds per weight
// element: fp32 FMA on the CUDA cores would take longer than streaming the weights, the tensor
// cores keep it bound by HBM.
//
// Gate and up (dense_gate_up_mma_kernel): warp tile = 16 neurons x 16 tokens, mma.sync
// m16n8k16 with the neurons as M and the tokens as N.  The weight rows stream from HBM straight
// into A fragments: a dot product may take its k terms in any order, so lane (g, q) loads 16-byte
// vectors of rows g and g + 8 and the B fragments (tokens, staged in shared memory in 512-column
// chunks) are read with the same permutation of k.  Epilogue: v[b, i] = act(z + beta) * u.
//
// Down (down_mma_kernel): out[b, :] = sum_i v[b, i] W_down^T[i, :] with M = tokens, N = output
// columns and K = neurons.  Tiles of W_down^T (64 neurons x 64 columns) and the matching tiles of v
// arrive by TMA tensor copies (cp.async.bulk.tensor with the 128-byte swizzle, no multicast) in a
// four-stage ring on mbarriers; W_down^T is read as B fragments by ldmatrix .trans.
// The gate/up epilogue stores v as bf16 high and low parts (two MMAs), so
// the product carries about 16 mantissa bits of v.  Column tiles x neuron ranges, partials
// summed by the last CTA of each column tile (in range order).
#include <cuda.h>  // CUtensorMap and its encoder's types (the encoder itself comes from the runtime)

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tma.cuh"

namespace csffn {

constexpr int kMmaThreads = 128;
constexpr int kMmaWarps = kMmaThreads / kWarp;
constexpr int kXChunk = 512;                 // token columns staged per step
constexpr int kXRow = kXChunk + 32;          // shared row stride in elements (1088 B: conflict-free)

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t word(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// ------------------------------------------------------------------------------------------
// Gate and up.  NT token tiles of 8 (B <= 8: 1, else 2).
// ------------------------------------------------------------------------------------------
template <int NT>
__global__ void __launch_bounds__(kMmaThreads, 4) dense_gate_up_mma_kernel(const DenseGateUpArgs p) {
  __shared__ __align__(128) bf16 xs[2][16 * kXRow];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, q = lane & 3;
  const int d = p.d, h = p.h, B = p.B;
  const bf16* Wg = reinterpret_cast<const bf16*>(p.W_gate);
  const bf16* Wu = reinterpret_cast<const bf16*>(p.W_up);
  const bf16* xg = reinterpret_cast<const bf16*>(p.x);
  bf16* vhi = reinterpret_cast<bf16*>(p.v);  // [B, h] high parts, then [B, h] low parts
  bf16* vlo = vhi + (size_t)B * h;
  const int n_ctiles = ((h + 15) / 16 + kMmaWarps - 1) / kMmaWarps;
  const int n_chunks = (d + kXChunk - 1) / kXChunk;

  // tokens B..15 stay zero in both buffers
  for (int e = tid; e < 2 * 16 * kXRow / 8; e += kMmaThreads)
    reinterpret_cast<uint4*>(&xs[0][0])[e] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  auto stage = [&](int c, int buf) {
    const int c0 = c * kXChunk, vecs = min(kXChunk, d - c0) / 8;
    for (int e = tid; e < B * vecs; e += kMmaThreads) {
      const int b = e / vecs, v = e - b * vecs;
      cp_async16(&xs[buf][b * kXRow + v * 8], xg + (size_t)b * d + c0 + v * 8, 0u);
    }
    cp_async_commit();
  };

  for (int ct = blockIdx.x; ct < n_ctiles; ct += gridDim.x) {
    const int i0 = (ct * kMmaWarps + warp) * 16;
    const int r_lo = i0 + g, r_hi = i0 + g + 8;
    const bool ok_lo = r_lo < h, ok_hi = r_hi < h;
    const bf16* g_lo = Wg + (size_t)(ok_lo ? r_lo : 0) * d;
    const bf16* g_hi = Wg + (size_t)(ok_hi ? r_hi : 0) * d;
    const bf16* u_lo = Wu + (size_t)(ok_lo ? r_lo : 0) * d;
    const bf16* u_hi = Wu + (size_t)(ok_hi ? r_hi : 0) * d;
    float zg[NT][4], zu[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) zg[t][e] = zu[t][e] = 0.f;

    stage(0, 0);
    for (int c = 0; c < n_chunks; ++c) {
      const int buf = c & 1;
      if (c + 1 < n_chunks) {
        stage(c + 1, buf ^ 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const int c0 = c * kXChunk, w = min(kXChunk, d - c0);
      const bf16* xb = xs[buf];
#pragma unroll 1
      for (int ks = 0; ks < w; ks += 128) {
        // lane (g, q) holds k = k0 + (4 j + q) * 8 + 0..7 of its rows, j = 0..3 (256 B per row per quad)
        const size_t k0 = (size_t)c0 + ks;
        uint4 a_glo[4], a_ghi[4], a_ulo[4], a_uhi[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const size_t off = k0 + (size_t)(4 * j + q) * 8;
          const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
          a_glo[j] = ok_lo ? ld_stream(g_lo + off) : z4;
          a_ghi[j] = ok_hi ? ld_stream(g_hi + off) : z4;
          a_ulo[j] = ok_lo ? ld_stream(u_lo + off) : z4;
          a_uhi[j] = ok_hi ? ld_stream(u_hi + off) : z4;
        }
        uint4 xb4[NT][4];
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            xb4[t][j] = *reinterpret_cast<const uint4*>(xb + (g + 8 * t) * kXRow + ks + (4 * j + q) * 8);
        // sub-step s: words (u, u + 1) of vector j = s / 2, u = 2 (s % 2); the same words of the
        // token vectors give the matching B fragment
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          const int j = s >> 1, u = (s & 1) * 2;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const uint32_t b0 = word(xb4[t][j], u), b1 = word(xb4[t][j], u + 1);
            mma_16816(zg[t], word(a_glo[j], u), word(a_ghi[j], u), word(a_glo[j], u + 1), word(a_ghi[j], u + 1),
                      b0, b1);
            mma_16816(zu[t], word(a_ulo[j], u), word(a_uhi[j], u), word(a_ulo[j], u + 1), word(a_uhi[j], u + 1),
                      b0, b1);
          }
        }
      }
      __syncthreads();  // this buffer is restaged two chunks later
    }

    // C fragment: c[0], c[1] = (row g, tokens 2q, 2q + 1); c[2], c[3] = (row g + 8, same tokens)
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int i = half ? r_hi : r_lo;
      if (i >= h) continue;
      const float beta = p.bias ? p.bias[i] : 0.f;
#pragma unroll
      for (int t = 0; t < NT; ++t)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int b = 8 * t + 2 * q + e;
          if (b < B) {
            // v in two bf16 parts, hi = bf16(v) and lo = bf16(v - hi): the down MMAs take both
            const float v = gate_act(zg[t][2 * half + e] + beta, p.act) * zu[t][2 * half + e];
            const bf16 hi = __float2bfloat16_rn(v);
            vhi[(size_t)b * h + i] = hi;
            vlo[(size_t)b * h + i] = __float2bfloat16_rn(v - __bfloat162float(hi));
          }
        }
    }
  }
}

// ------------------------------------------------------------------------------------------
// Down: out[b, :] = sum_i v[b, i] * W_down^T[i, :] for i < h.
// CTA tile: 64 output columns x a range of neurons; warp w owns columns 16 w .. 16 w + 15 (two
// n tiles) for all 16 tokens.  Per 64-neuron block, two TMA tensor copies fill a stage of a
// four-stage ring: the 64 x 64 W_down^T tile (2-D map over [h, d]) and the tokens' v for the same
// neurons, both bf16 parts (3-D map over [2][B][h]; token rows past B arrive as zeros).  Both land
// with the 128-byte swizzle (16-byte chunk c of a 128-byte row r sits at chunk c ^ (r mod 8)), which
// the ldmatrix and A-fragment addresses undo, so the reads are free of bank conflicts.
// ------------------------------------------------------------------------------------------
constexpr int kDnCols = 64;
constexpr int kDnK = 64;                             // neurons per staged block
constexpr int kDnStages = 4;                         // staged blocks (three in flight while one is used)
constexpr uint32_t kDnWBytes = kDnK * kDnCols * 2;   // W_down^T tile: 64 rows of 128 B
constexpr uint32_t kDnVBytes = 2 * 16 * kDnK * 2;    // v tile: [part][token] rows of 128 B
constexpr uint32_t kDnStageBytes = kDnWBytes + kDnVBytes;  // 12 KB, a multiple of 1 KB

// Byte offset of byte `col_byte` of row `row` in a tile of 128-byte rows written with the 128-byte swizzle.
__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t col_byte) {
  return row * 128u + ((((col_byte >> 4) ^ (row & 7u)) << 4) | (col_byte & 15u));
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, int x, int y, int z, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t& r0, uint32_t& r1, const void* smem_row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1)
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_row))));
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __launch_bounds__(kMmaThreads, 4) down_mma_kernel(const DownArgs p, int ranges,
                                                                  const __grid_constant__ CUtensorMap tm_w,
                                                                  const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ __align__(1024) unsigned char dn_smem_raw[];
  __shared__ __align__(8) uint64_t s_bar[kDnStages];
  __shared__ int s_abort;
  __shared__ bool s_last;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, q = lane & 3;
  const int d = p.d, B = p.B;
  // the swizzle pattern repeats every 1 KB: stage buffers start on a 1 KB boundary
  unsigned char* dn_smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(dn_smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int col0 = blockIdx.x * kDnCols;
  const int ry = blockIdx.y;
  // neuron range of this CTA, in whole 64-neuron blocks; rows past h arrive as zeros
  const int n_blk = (p.n_host + kDnK - 1) / kDnK;
  const int blk_lo = (int)((long long)n_blk * ry / ranges), blk_hi = (int)((long long)n_blk * (ry + 1) / ranges);
  const int k_lo = blk_lo * kDnK;
  const int n_blocks = blk_hi - blk_lo;

  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < kDnStages; ++i) mbar_init(&s_bar[i], 1);
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int blk) {  // thread 0: block blk into its stage
    const int buf = blk % kDnStages, r0 = k_lo + blk * kDnK;
    unsigned char* st = dn_smem + (size_t)buf * kDnStageBytes;
    mbar_arrive_expect_tx(&s_bar[buf], kDnStageBytes);
    tma_load_2d(st, &tm_w, col0, r0, &s_bar[buf]);
    tma_load_3d(st + kDnWBytes, &tm_v, r0, 0, 0, &s_bar[buf]);
  };
  if (tid == 0)
    for (int b0 = 0; b0 < kDnStages - 1 && b0 < n_blocks; ++b0) issue(b0);

  float acc[2][4];
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;

  for (int blk = 0; blk < n_blocks; ++blk) {
    // the stage of block blk - 1 is free (barrier at the end of the last iteration): refill it
    if (tid == 0 && blk + kDnStages - 1 < n_blocks) {
      fence_proxy_async_smem();
      issue(blk + kDnStages - 1);
    }
    const int buf = blk % kDnStages;
    mbar_wait(&s_bar[buf], (uint32_t)((blk / kDnStages) & 1), p.err, &s_abort);
    const unsigned char* wt = dn_smem + (size_t)buf * kDnStageBytes;
    const unsigned char* vt = wt + kDnWBytes;
#pragma unroll
    for (int kk = 0; kk < kDnK; kk += 16) {
      // A fragments (tokens x neurons) of both parts of v: rows g and g + 8, neurons kk + 2q (+1, +8, +9)
      uint32_t ah[4], al[4];
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        uint32_t* a = part ? al : ah;
        const uint32_t r_lo = part * 16 + g, r_hi = part * 16 + g + 8;
        const uint32_t c0 = (kk + 2 * q) * 2, c8 = (kk + 2 * q + 8) * 2;
        a[0] = *reinterpret_cast<const uint32_t*>(vt + swz(r_lo, c0));
        a[1] = *reinterpret_cast<const uint32_t*>(vt + swz(r_hi, c0));
        a[2] = *reinterpret_cast<const uint32_t*>(vt + swz(r_lo, c8));
        a[3] = *reinterpret_cast<const uint32_t*>(vt + swz(r_hi, c8));
      }
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        // B fragment: neurons kk .. kk + 15 (rows of the staged tile), columns 16 warp + 8 t ..
        uint32_t b0, b1;
        const uint32_t lrow = kk + (lane & 15);
        ldmatrix_x2_trans(b0, b1, wt + swz(lrow, (warp * 16 + t * 8) * 2));
        mma_16816(acc[t], ah[0], ah[1], ah[2], ah[3], b0, b1);
        mma_16816(acc[t], al[0], al[1], al[2], al[3], b0, b1);
      }
    }
    __syncthreads();
  }

  // partial of this neuron range: C rows = tokens g, g + 8; columns 16 warp + 8 t + 2q (+1)
  float* part = p.partial + (size_t)ry * B * d;
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int b = g + 8 * (e >> 1);
      const int col = col0 + warp * 16 + t * 8 + 2 * q + (e & 1);
      if (b < B && col < d) __stcg(part + (size_t)b * d + col, acc[t][e]);
    }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&p.slice_ctr[blockIdx.x], 1u) == (uint32_t)(ranges - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int e = tid; e < B * kDnCols; e += kMmaThreads) {
    const int b = e / kDnCols, col = col0 + e % kDnCols;
    if (col >= d) continue;
    float sum = 0.f;
    for (int r = 0; r < ranges; ++r) sum += __ldcg(p.partial + ((size_t)r * B + b) * d + col);
    const size_t o = (size_t)b * d + col;
    if (p.out_mode == CSFFN_OUT_BF16)
      reinterpret_cast<bf16*>(p.out)[o] = __float2bfloat16_rn(sum);
    else if (p.out_mode == CSFFN_OUT_F32)
      reinterpret_cast<float*>(p.out)[o] = sum;
    else
      reinterpret_cast<float*>(p.out)[o] += sum;
  }
  if (tid == 0) p.slice_ctr[blockIdx.x] = 0u;
}

// ------------------------------------------------------------------------------------------
// Launchers
// ------------------------------------------------------------------------------------------
bool dense_mma_supported(int d, int h, int B, int wdtype) {
  return wdtype == CSFFN_BF16 && B >= kDenseMmaMinBatch && B <= 16 && d % 128 == 0 && d % kDnCols == 0 &&
         d / kDnCols <= kMaxSlices && h >= 16 && h % 8 == 0;
}

cudaError_t launch_dense_gate_up_mma(const DenseGateUpArgs& a, cudaStream_t s) {
  const int n_ctiles = ((a.h + 15) / 16 + kMmaWarps - 1) / kMmaWarps;
  int occ = 0;
  cudaError_t e = a.B <= 8 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, dense_gate_up_mma_kernel<1>, kMmaThreads, 0)
                           : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, dense_gate_up_mma_kernel<2>, kMmaThreads, 0);
  if (e != cudaSuccess) return e;
  int grid = sm_count() * (occ > 0 ? occ : 1);
  if (grid > n_ctiles) grid = n_ctiles;
  if (a.B <= 8)
    dense_gate_up_mma_kernel<1><<<grid, kMmaThreads, 0, s>>>(a);
  else
    dense_gate_up_mma_kernel<2><<<grid, kMmaThreads, 0, s>>>(a);
  return cudaGetLastError();
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no link against libcuda).
TensorMapEncodeFn tensor_map_encoder() {
  static TensorMapEncodeFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<TensorMapEncodeFn>(nullptr);
    return reinterpret_cast<TensorMapEncodeFn>(ptr);
  }();
  return fn;
}

cudaError_t launch_down_mma(const DownArgs& a, int max_ranges, cudaStream_t s) {
  TensorMapEncodeFn encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  // W_down^T [h][d] bf16: boxes of 64 columns x 64 rows
  CUtensorMap tm_w, tm_v;
  const cuuint64_t wdim[2] = {(cuuint64_t)a.d, (cuuint64_t)a.h};
  const cuuint64_t wstride[1] = {(cuuint64_t)a.d * 2};
  const cuuint32_t wbox[2] = {kDnCols, kDnK};
  const cuuint32_t ones[3] = {1, 1, 1};
  if (encode(&tm_w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.W_down_t), wdim, wstride, wbox, ones,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // v as [2 parts][B][h] bf16: boxes of 64 neurons x 16 tokens x 2 parts
  const cuuint64_t vdim[3] = {(cuuint64_t)a.h, (cuuint64_t)a.B, 2};
  const cuuint64_t vstride[2] = {(cuuint64_t)a.h * 2, (cuuint64_t)a.B * a.h * 2};
  const cuuint32_t vbox[3] = {kDnK, 16, 2};
  if (encode(&tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<float*>(a.v), vdim, vstride, vbox, ones,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  const int slices = a.d / kDnCols;
  const size_t smem = kDnStages * kDnStageBytes + 1024;  // + room to align the ring to 1 KB
  cudaError_t e = cudaFuncSetAttribute(down_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, down_mma_kernel, kMmaThreads, smem);
  if (e != cudaSuccess) return e;
  int ranges = sm_count() * (occ > 0 ? occ : 1) / slices;  // one wave
  if (ranges < 1) ranges = 1;
  if (ranges > max_ranges) ranges = max_ranges;
  if (ranges > (a.n_host + kDnK - 1) / kDnK) ranges = (a.n_host + kDnK - 1) / kDnK;
  dim3 grid(slices, ranges);
  down_mma_kernel<<<grid, kMmaThreads, smem, s>>>(a, ranges, tm_w, tm_v);
  return cudaGetLastError();
}

}  // namespace csffn
