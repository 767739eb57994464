// Order-statistic selection for threshold calibration, RMSNorm for FFN stacks, and the
// failure-detection self-test.
//
// Calibration ("CATS: Contextually-Aware Thresholding for Sparsity in Large Language Models",
// abstract; "SVD Contextual Sparsity Predictors for Fast LLM Inference", Fig. 1 and Table 3,
// calibrated per-neuron thresholds) needs the exact k-th smallest of many activations.  Global
// selection is an MSD radix select on order-preserving 32-bit keys: four 8-bit passes, each a
// grid-wide histogram of the keys that still match the chosen prefix plus a one-block pick of
// the digit.  Per-neuron selection sorts each neuron's calibration values in shared memory.
#include "common.cuh"
#include "kernels.h"

namespace csffn {

struct KthState {
  uint32_t prefix;
  uint32_t mask;
  unsigned long long krem;  // rank still to find inside the current prefix (1-indexed)
  uint32_t hist[256];
};

size_t kth_state_bytes() { return align_up(sizeof(KthState), 256); }

// Float bits -> unsigned key with the same order as the float values (finite inputs).
__device__ __forceinline__ uint32_t f2key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key2f(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

__global__ void kth_init_kernel(KthState* st, unsigned long long k) {
  const int t = threadIdx.x;
  st->hist[t] = 0u;
  if (t == 0) {
    st->prefix = 0u;
    st->mask = 0u;
    st->krem = k;
  }
}

__global__ void __launch_bounds__(256) kth_hist_kernel(const float* __restrict__ v, long long n,
                                                       KthState* st, int shift) {
  __shared__ uint32_t sh[256];
  sh[threadIdx.x] = 0u;
  __syncthreads();
  const uint32_t prefix = st->prefix, mask = st->mask;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const uint32_t key = f2key(v[i]);
    if ((key & mask) == prefix) atomicAdd(&sh[(key >> shift) & 0xFFu], 1u);
  }
  __syncthreads();
  const uint32_t c = sh[threadIdx.x];
  if (c) atomicAdd(&st->hist[threadIdx.x], c);
}

// One block of 256 threads: choose the digit whose bucket holds the krem-th key.
__global__ void kth_pick_kernel(KthState* st, int shift, float* out) {
  __shared__ unsigned long long cum[256];
  const int t = threadIdx.x;
  cum[t] = st->hist[t];
  __syncthreads();
  // inclusive scan (Hillis-Steele)
  for (int o = 1; o < 256; o <<= 1) {
    const unsigned long long add = t >= o ? cum[t - o] : 0ull;
    __syncthreads();
    cum[t] += add;
    __syncthreads();
  }
  const unsigned long long before = t == 0 ? 0ull : cum[t - 1];
  const unsigned long long k = st->krem;
  __syncthreads();
  if (before < k && k <= cum[t]) {  // exactly one digit satisfies this
    st->prefix |= (uint32_t)t << shift;
    st->mask |= 0xFFu << shift;
    st->krem = k - before;
    if (shift == 0) *out = key2f(st->prefix);
  }
  __syncthreads();
  st->hist[t] = 0u;
}

cudaError_t launch_kth_smallest(const float* values, int64_t n, int64_t k, float* out, void* state,
                                cudaStream_t s) {
  KthState* st = reinterpret_cast<KthState*>(state);
  kth_init_kernel<<<1, 256, 0, s>>>(st, (unsigned long long)k);
  long long blocks = (n + 255) / 256;
  const long long cap = (long long)sm_count() * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  for (int shift = 24; shift >= 0; shift -= 8) {
    kth_hist_kernel<<<(unsigned)blocks, 256, 0, s>>>(values, n, st, shift);
    kth_pick_kernel<<<1, 256, 0, s>>>(st, shift, out);
  }
  return cudaGetLastError();
}

// Ascending bitonic sort of sv[0, n2) in shared memory by the whole block (n2 a power of two); the
// block's threads are synchronised on return.
__device__ void block_bitonic_sort(float* sv, int n2) {
  for (int kk = 2; kk <= n2; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const bool up = (i & kk) == 0;
          const float a = sv[i], b = sv[ixj];
          if ((a > b) == up) {
            sv[i] = b;
            sv[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }
}

// out[r] = k-th smallest (1-indexed) of values[r*n .. r*n + n), by a bitonic sort in shared
// memory (n padded with +inf up to a power of two).
__global__ void __launch_bounds__(256) rows_kth_kernel(const float* __restrict__ values, int n, int n2,
                                                       int k, float* __restrict__ out) {
  extern __shared__ float sv[];
  const float* row = values + (size_t)blockIdx.x * n;
  for (int i = threadIdx.x; i < n2; i += blockDim.x) sv[i] = i < n ? row[i] : __int_as_float(0x7f800000);
  __syncthreads();
  block_bitonic_sort(sv, n2);
  if (threadIdx.x == 0) out[blockIdx.x] = sv[k - 1];
}

cudaError_t launch_rows_kth(const float* values, int rows, int n, int k, float* out, cudaStream_t s) {
  int n2 = 1;
  while (n2 < n) n2 <<= 1;
  const size_t smem = (size_t)n2 * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(rows_kth_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  rows_kth_kernel<<<rows, 256, smem, s>>>(values, n, n2, k, out);
  return cudaGetLastError();
}

// ceil(R * m) for a float R in [0, 1] and 0 <= m < 2^31, exactly: R = mant * 2^-sh with a 24-bit
// integer mant, so R * m = mant * m / 2^sh with the numerator below 2^55.
__device__ __forceinline__ int exact_ceil_mul(float R, int m) {
  if (!(R > 0.f) || m <= 0) return 0;
  const uint32_t b = __float_as_uint(R);
  const int e = (int)((b >> 23) & 0xffu);
  const unsigned long long mant = e ? ((b & 0x7fffffu) | 0x800000u) : (b & 0x7fffffu);
  const int sh = e ? 150 - e : 149;
  const unsigned long long num = mant * (unsigned long long)m;
  unsigned long long q = sh >= 64 ? (num ? 1ull : 0ull) : ((num >> sh) + (((num >> sh) << sh) != num ? 1ull : 0ull));
  return q > (unsigned long long)m ? m : (int)q;
}

// Per-neuron thresholds for a target recall R of the active set: row r of pt and zt holds the
// predictor outputs p_r and the gate pre-activations z_r of the n calibration vectors.  The outputs
// of the active vectors (z > 0) are sorted, the others set to +inf; with m active and c = ceil(R m),
// out[r] is the largest float below the c-th largest active output (so p > out[r] holds for exactly
// the outputs at or above it), or +inf when c = 0.
__global__ void __launch_bounds__(256) rows_recall_kernel(const float* __restrict__ pt, const float* __restrict__ zt,
                                                          int n, int n2, float R, float* __restrict__ out) {
  extern __shared__ float sv[];
  __shared__ int s_m;
  const float* prow = pt + (size_t)blockIdx.x * n;
  const float* zrow = zt + (size_t)blockIdx.x * n;
  if (threadIdx.x == 0) s_m = 0;
  __syncthreads();
  int m = 0;
  for (int i = threadIdx.x; i < n2; i += blockDim.x) {
    const bool active = i < n && zrow[i] > 0.f;
    sv[i] = active ? prow[i] : __int_as_float(0x7f800000);
    m += active ? 1 : 0;
  }
  atomicAdd(&s_m, m);
  __syncthreads();
  block_bitonic_sort(sv, n2);
  if (threadIdx.x == 0) {
    const int ma = s_m;
    const int c = exact_ceil_mul(R, ma);
    out[blockIdx.x] = c == 0 ? __int_as_float(0x7f800000) : nextafterf(sv[ma - c], -INFINITY);
  }
}

cudaError_t launch_rows_recall(const float* pt, const float* zt, int rows, int n, float recall, float* out,
                               cudaStream_t s) {
  int n2 = 1;
  while (n2 < n) n2 <<= 1;
  const size_t smem = (size_t)n2 * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(rows_recall_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  rows_recall_kernel<<<rows, 256, smem, s>>>(pt, zt, n, n2, recall, out);
  return cudaGetLastError();
}

__global__ void fill_kernel(float* p, float v, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) p[i] = v;
}

cudaError_t launch_fill(float* p, float v, int n, cudaStream_t s) {
  fill_kernel<<<(n + 255) / 256, 256, 0, s>>>(p, v, n);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// RMSNorm (unit gain) rounded to bf16: one block per token.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) rmsnorm_bf16_kernel(const float* __restrict__ h, int d, float eps,
                                                           bf16* __restrict__ xn) {
  __shared__ float part[8];
  const float* row = h + (size_t)blockIdx.x * d;
  float ss = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) ss = fmaf(row[c], row[c], ss);
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 8; ++w) tot += part[w];
  const float scale = 1.0f / sqrtf(tot / (float)d + eps);
  bf16* o = xn + (size_t)blockIdx.x * d;
  for (int c = threadIdx.x; c < d; c += blockDim.x) o[c] = __float2bfloat16_rn(row[c] * scale);
}

cudaError_t launch_rmsnorm_bf16(const float* h, int B, int d, float eps, void* xn, cudaStream_t s) {
  rmsnorm_bf16_kernel<<<B, 256, 0, s>>>(h, d, eps, reinterpret_cast<bf16*>(xn));
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Failure-detection self-test: wait on a word nothing sets, with the library's bounded wait.
// ------------------------------------------------------------------------------------------
__global__ void timeout_selftest_kernel(const uint64_t* flag, uint32_t* err, uint32_t limit) {
  uint64_t v = 0;
  bounded_wait(flag, limit, err, [](uint64_t w) { return w != 0ull; }, &v);
}

cudaError_t launch_timeout_selftest(uint64_t* flag, uint32_t* err, int spin_limit, cudaStream_t s) {
  timeout_selftest_kernel<<<1, 1, 0, s>>>(flag, err, (uint32_t)spin_limit);
  return cudaGetLastError();
}

}  // namespace csffn
