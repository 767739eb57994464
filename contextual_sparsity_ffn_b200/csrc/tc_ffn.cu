// Gated FFN of a block of up to 16 tokens on the fifth-generation tensor cores.
//
// "Sirius: Contextual Sparsity with Correction for Efficient LLMs", the correction step: the full
// model re-reads a chunk of recent tokens in parallel, so the dense FFN runs on a block of tokens.
// "CATS: Contextually-Aware Thresholding for Sparsity in Large Language Models", abstract: the
// same FFN with the activations at or below the threshold zeroed (the masked mode here).  At up to
// 16 tokens the work is 16 multiply-adds per weight element, far below the tensor cores' rate, so
// both kernels are bound by streaming the weights from HBM once.
//
// Gate/up (tc_gate_up_kernel), swap-AB: D[neuron, token] = W[neuron, :] . x[token, :] with the
// neurons as M = 128, the tokens as N = 16 (padded with zero rows), K = d in 64-element k-blocks.
// Each k-block stage holds the W_gate tile, the W_up tile (128 rows x 128 bytes each, K-major) and
// the tokens' tile (16 x 128 bytes), all by TMA tensor copies with the 128-byte swizzle; one thread
// issues tcgen05.mma into fp32 accumulators in TMEM (16 columns each, double-buffered; the k-steps
// alternate between two accumulators per matrix, summed in the epilogue).
// Epilogue (4 warps, one TMEM lane = one neuron each): v = act(z + beta) * u, stored as bf16 high
// part and bf16 low part (v - high), so the down MMAs carry about 16 mantissa bits of v.
//
// Down (tc_down_kernel): D[column, token] = sum_i W_down^T[i, column] v[token, i], the output
// columns as M = 128, the tokens as N = 16, the neurons as K.  W_down^T rows are contiguous along
// the columns, so the A operand is MN-major: two 64-column boxes per k-block.  The v tile (high
// parts over low parts, 32 rows) is the K-major B operand of one N = 32 MMA per k-step; the k-steps
// alternate between two accumulators.
//
// Work split (both kernels): the tiles' k-blocks, tile-major, are cut into G equal contiguous runs,
// one per CTA (G = number of SMs), so every SM streams the same number of bytes.  A run covers
// whole tiles and at most a partial tile at each end; a CTA that finishes a partial tile stores its
// accumulators in its own slot, adds its k-block count to the tile's counter, and the CTA whose
// addition completes the count adds the other slots and writes the tile (then clears the counter
// for the next launch).  No CTA waits for another.
//
// Warp roles (192 threads): warp 0 issues the TMA copies, warp 1 owns the TMEM allocation and
// issues the MMAs, warps 2-5 run the epilogue.  Every wait is bounded (one second); a wait that
// runs out records the timeout and ends the kernel after the copies and MMAs in flight complete.
// The two kernels are chained by programmatic dependent launch: each prefetches its first weight
// tiles before waiting for the previous kernel, and reads nothing the previous kernel writes before.
#include "common.cuh"
#include "fused_end.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace csffn {

constexpr int kTcThreads = 192;
constexpr int kTcN = 16;   // tokens per MMA (N)
constexpr int kTcKB = 64;  // contraction elements per staged k-block (one 128-byte row)

// gate/up stage: W_gate tile, W_up tile, tokens tile
constexpr uint32_t kGuWBytes = kTcTile * kTcKB * 2;  // 16 KB
constexpr uint32_t kGuXBytes = kTcN * kTcKB * 2;     // 2 KB
constexpr uint32_t kGuStage = 2 * kGuWBytes + kGuXBytes;
constexpr int kGuStages = 6;
// Accumulators: the k-steps of a stage alternate between two accumulators per matrix, so that
// consecutive MMAs do not wait on one another's sums.  Per buffer: gate even / odd k-steps, up
// even / odd, 16 fp32 columns each; two buffers (one drained while the next tile accumulates).
constexpr uint32_t kGuAccCols = 64;
constexpr uint32_t kGuTmemCols = 2 * kGuAccCols;

// down stage: two 64-column boxes of W_down^T (64 neurons each), v tile (2 parts x 16 tokens)
constexpr uint32_t kDnBox = 64 * kTcKB * 2;          // 8 KB
constexpr uint32_t kDnWBytesTc = 2 * kDnBox;         // 16 KB
constexpr uint32_t kDnVBytesTc = 2 * kTcN * kTcKB * 2;  // 4 KB
constexpr uint32_t kDnStage = kDnWBytesTc + kDnVBytesTc;
constexpr int kDnStagesTc = 10;
// The v tile's high and low parts are stacked as one N = 32 operand (columns 0..15 of D take the
// high parts, 16..31 the low parts).  Per buffer: two accumulators (even / odd k-steps) of 32 fp32
// columns; two buffers.
constexpr int kDnN = 2 * kTcN;
constexpr uint32_t kDnAccCols = 2 * kDnN;
constexpr uint32_t kDnTmemCols = 2 * kDnAccCols;

constexpr size_t kGuSmem = (size_t)kGuStages * kGuStage + 1024;
constexpr size_t kDnSmem = (size_t)kDnStagesTc * kDnStage + 1024;

// ---------------------------------------------------------------------------------------------
// The even split of n_it k-block iterations over G CTAs.
// ---------------------------------------------------------------------------------------------
__host__ __device__ inline long long run_start(int c, long long n_it, int G) { return (long long)c * n_it / G; }
// The CTA whose run holds iteration j.
__device__ inline int run_owner(long long j, long long n_it, int G) { return (int)(((j + 1) * G - 1) / n_it); }

// Slot of CTA c's partial accumulators for its segment in the tile that starts at iteration
// tile_it0: slot 0 for the segment its run starts with, slot 1 for the one it ends with.
__device__ inline int run_slot(int c, long long tile_it0, long long n_it, int G) {
  return run_start(c, n_it, G) >= tile_it0 ? 0 : 1;
}

// Stage ring position: slot and the number of times the ring has wrapped (its phase parity).
struct RingPos {
  int slot = 0;
  uint32_t round = 0;
  __device__ void next(int n) {
    if (++slot == n) {
      slot = 0;
      ++round;
    }
  }
};

// The split-tile protocol of the epilogue (128 threads, et = 0..127, named barrier 1): store this
// CTA's `n` partial values per lane, add `seg_len` to the tile's counter, and report whether this
// CTA completed the tile; if so, `acc` becomes the sum of all the tile's partials, added in CTA order
// (the same bits whichever CTA completes it), and the counter is cleared.
template <int N>
__device__ bool finish_split_tile(float (&acc)[N], const TcArgs& p, uint32_t* ctr, int et, long long tile_it0,
                                  long long tile_it1, long long seg_start, int seg_len, int n_kb, long long n_it,
                                  uint32_t* s_flag) {
  const int c = blockIdx.x, G = gridDim.x;
  const int slot = seg_start == run_start(c, n_it, G) ? 0 : 1;
  float* mine = p.part + (size_t)(c * 2 + slot) * 32 * kTcTile;
#pragma unroll
  for (int v = 0; v < N; ++v) __stcg(mine + v * kTcTile + et, acc[v]);
  __threadfence();
  named_sync(1, 4 * kWarp);
  if (et == 0) {
    const uint32_t old = atomicAdd(ctr, (uint32_t)seg_len);
    *s_flag = old + (uint32_t)seg_len == (uint32_t)n_kb ? 1u : 0u;
  }
  named_sync(1, 4 * kWarp);
  const bool last = *s_flag != 0u;
  named_sync(1, 4 * kWarp);  // s_flag is rewritten by the next split tile
  if (!last) return false;
  __threadfence();
  // the partials in CTA order, whichever CTA came last: the sum does not depend on the timing
  const int c_lo = run_owner(tile_it0, n_it, G), c_hi = run_owner(tile_it1 - 1, n_it, G);
  float own[N];
#pragma unroll
  for (int v = 0; v < N; ++v) {
    own[v] = acc[v];
    acc[v] = 0.f;
  }
  for (int cc = c_lo; cc <= c_hi; ++cc) {
    if (cc == c) {
#pragma unroll
      for (int v = 0; v < N; ++v) acc[v] += own[v];
      continue;
    }
    if (run_start(cc + 1, n_it, G) <= run_start(cc, n_it, G)) continue;
    const float* other = p.part + (size_t)(cc * 2 + run_slot(cc, tile_it0, n_it, G)) * 32 * kTcTile;
#pragma unroll
    for (int v = 0; v < N; ++v) acc[v] += __ldcg(other + v * kTcTile + et);
  }
  if (et == 0) *ctr = 0u;
  return true;
}

// Bounded wait used by every role (aborts with the CTA's flag).
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, const TcArgs& p, volatile int* abort) {
  return mbar_wait(bar, parity, p.err, abort);
}

// ---------------------------------------------------------------------------------------------
// Gate / up
// ---------------------------------------------------------------------------------------------
template <bool kMasked>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_gate_up_kernel(const TcArgs p, const __grid_constant__ CUtensorMap tm_g, const __grid_constant__ CUtensorMap tm_u,
                      const __grid_constant__ CUtensorMap tm_x) {
  extern __shared__ __align__(1024) unsigned char tc_raw[];
  __shared__ __align__(8) uint64_t full[kGuStages], empty[kGuStages], accf[2], acce[2], drain;
  __shared__ uint32_t s_tmem, s_flag;
  __shared__ int s_abort;
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(tc_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = p.h, B = p.B;
  const int n_tiles = (h + kTcTile - 1) / kTcTile, n_kb = (p.d + kTcKB - 1) / kTcKB;
  const long long n_it = (long long)n_tiles * n_kb;
  const long long it0 = run_start(blockIdx.x, n_it, gridDim.x), it1 = run_start(blockIdx.x + 1, n_it, gridDim.x);

  pdl_trigger();
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < kGuStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 4);
    }
    mbar_init(&drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, kGuTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    if (lane == 0 && it1 > it0) {
      // ---- producer: weight tiles of the first stages before the dependency wait, tokens after
      const uint64_t pol = l2_evict_first_policy();
      const int pre = (int)min((long long)kGuStages, it1 - it0);
      int t = (int)(it0 / n_kb), kb = (int)(it0 % n_kb);
      for (int q = 0; q < pre; ++q) {
        unsigned char* st = smem + (size_t)q * kGuStage;
        mbar_arrive_expect_tx(&full[q], kGuStage);
        tma_load_2d_hint(st, &tm_g, kb * kTcKB, t * kTcTile, &full[q], pol);
        tma_load_2d_hint(st + kGuWBytes, &tm_u, kb * kTcKB, t * kTcTile, &full[q], pol);
        if (++kb == n_kb) kb = 0, ++t;
      }
      pdl_wait_prior();
      t = (int)(it0 / n_kb), kb = (int)(it0 % n_kb);
      for (int q = 0; q < pre; ++q) {
        tma_load_2d_plain(smem + (size_t)q * kGuStage + 2 * kGuWBytes, &tm_x, kb * kTcKB, 0, &full[q]);
        if (++kb == n_kb) kb = 0, ++t;
      }
      RingPos r;
      for (int q = 0; q < pre; ++q) r.next(kGuStages);
      long long issued = pre;
      for (long long j = it0 + pre; j < it1; ++j, ++issued) {
        if (!tc_wait(&empty[r.slot], (r.round - 1) & 1, p, &s_abort)) break;
        unsigned char* st = smem + (size_t)r.slot * kGuStage;
        mbar_arrive_expect_tx(&full[r.slot], kGuStage);
        tma_load_2d_hint(st, &tm_g, kb * kTcKB, t * kTcTile, &full[r.slot], pol);
        tma_load_2d_hint(st + kGuWBytes, &tm_u, kb * kTcKB, t * kTcTile, &full[r.slot], pol);
        tma_load_2d_plain(st + 2 * kGuWBytes, &tm_x, kb * kTcKB, 0, &full[r.slot]);
        if (++kb == n_kb) kb = 0, ++t;
        r.next(kGuStages);
      }
      // the copies in flight land before the CTA's shared memory is released
      RingPos w;
      for (long long q = 0; q < issued; ++q) {
        if (q + kGuStages >= issued) mbar_wait_drain(&full[w.slot], w.round & 1, p.err);
        w.next(kGuStages);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && it1 > it0) {
      // ---- MMA issuer
      const uint32_t idesc = umma_idesc_bf16(kTcTile, kTcN, false);
      RingPos r;
      int m = 0;
      long long j = it0;
      bool ok = true;
      while (ok && j < it1) {
        const long long tile = j / n_kb;
        const long long seg_end = min(it1, (tile + 1) * n_kb);
        const int a = m & 1;
        if (m >= 2 && !tc_wait(&acce[a], ((m >> 1) - 1) & 1, p, &s_abort)) break;
        tc_fence_after();
        const uint32_t dbase = tmem + (uint32_t)a * kGuAccCols;
        for (long long jj = j; jj < seg_end; ++jj) {
          if (!tc_wait(&full[r.slot], r.round & 1, p, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + (size_t)r.slot * kGuStage);
#pragma unroll
          for (int k = 0; k < kTcKB / 16; ++k) {
            const uint32_t acc = (jj == j && k < 2) ? 0u : 1u;  // each accumulator's first k-step overwrites
            const uint32_t dg = dbase + 16u * (k & 1), du = dg + 32u;
            const uint64_t bx = umma_desc_k(sb + 2 * kGuWBytes + 32u * k);
            umma_bf16(dg, umma_desc_k(sb + 32u * k), bx, idesc, acc);
            umma_bf16(du, umma_desc_k(sb + kGuWBytes + 32u * k), bx, idesc, acc);
          }
          umma_commit(&empty[r.slot]);
          r.next(kGuStages);
        }
        if (!ok) break;
        umma_commit(&accf[a]);
        ++m;
        j = seg_end;
      }
      // every MMA issued has completed before TMEM is released
      umma_commit(&drain);
      mbar_wait_drain(&drain, 0, p.err);
    }
  } else {
    // ---- epilogue: warps 2..5, TMEM lane quarter warp % 4, one neuron per thread
    const int et = threadIdx.x - 2 * kWarp;
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    pdl_wait_prior();
    int m = 0;
    long long j = it0;
    while (j < it1) {
      const long long tile = j / n_kb;
      const long long tile_it0 = tile * n_kb, tile_it1 = tile_it0 + n_kb;
      const long long seg_end = min(it1, tile_it1);
      const int a = m & 1;
      // every epilogue warp leaves together (the split-tile protocol meets at a named barrier)
      if (!named_all(3, 4 * kWarp, tc_wait(&accf[a], (m >> 1) & 1, p, &s_abort))) break;
      tc_fence_after();
      float acc[32], odd[32];  // gate sums of tokens 0..15, then up sums (even and odd k-steps)
      tmem_ld16(lane_base + (uint32_t)a * kGuAccCols, acc);
      tmem_ld16(lane_base + (uint32_t)a * kGuAccCols + 16u, odd);
      tmem_ld16(lane_base + (uint32_t)a * kGuAccCols + 32u, acc + 16);
      tmem_ld16(lane_base + (uint32_t)a * kGuAccCols + 48u, odd + 16);
      tmem_ld_wait();
#pragma unroll
      for (int v = 0; v < 32; ++v) acc[v] += odd[v];
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[a]);
      bool fin = j == tile_it0 && seg_end == tile_it1;
      if (!fin)
        fin = finish_split_tile<32>(acc, p, p.ctr + tile, et, tile_it0, tile_it1, j, (int)(seg_end - j), n_kb, n_it,
                                    &s_flag);
      if (fin) {
        const int i = (int)tile * kTcTile + row;
        if (i < h) {
          const float beta = p.bias ? p.bias[i] : 0.f;
          bool any = false;
#pragma unroll
          for (int b = 0; b < kTcN; ++b) {
            if (b < B) {
              const float av = gate_act(acc[b] + beta, p.act);
              float v;
              if (kMasked) {
                const bool keep = fabsf(av) > p.t;
                v = keep ? av * acc[16 + b] : 0.f;
                p.afull[(size_t)b * h + i] = keep ? av : 0.f;
                any |= keep;
              } else {
                v = av * acc[16 + b];
              }
              const bf16 hi = __float2bfloat16_rn(v);
              const bf16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
              p.v[(size_t)b * h + i] = __bfloat16_as_ushort(hi);
              p.v[(size_t)(B + b) * h + i] = __bfloat16_as_ushort(lo);
            }
          }
          if (kMasked) p.flags[i] = any ? 1 : 0;
        }
      }
      ++m;
      j = seg_end;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kGuTmemCols);
  }
}

// ---------------------------------------------------------------------------------------------
// Down (and, in masked mode, the compaction of the keep flags)
// ---------------------------------------------------------------------------------------------
template <int NB>  // token tier of the compaction (masked mode); 0: no compaction
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_down_kernel(const TcArgs p, const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ __align__(1024) unsigned char tc_raw[];
  __shared__ __align__(8) uint64_t full[kDnStagesTc], empty[kDnStagesTc], accf[2], acce[2], drain;
  __shared__ uint32_t s_tmem, s_flag;
  __shared__ uint32_t s_cnt[4];
  __shared__ int s_abort;
  unsigned char* smem =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(tc_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = p.d, h = p.h, B = p.B;
  const int n_ct = (d + kTcTile - 1) / kTcTile, n_kb = (h + kTcKB - 1) / kTcKB;
  const long long n_it = (long long)n_ct * n_kb;
  const long long it0 = run_start(blockIdx.x, n_it, gridDim.x), it1 = run_start(blockIdx.x + 1, n_it, gridDim.x);
  uint32_t* ctr = p.ctr + (h + kTcTile - 1) / kTcTile;  // column-tile counters follow the gate/up ones

  pdl_trigger();
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int i = 0; i < kDnStagesTc; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 4);
    }
    mbar_init(&drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, kDnTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    if (lane == 0 && it1 > it0) {
      // ---- producer: W_down^T boxes of the first stages before the dependency wait, v after
      const uint64_t pol = l2_evict_first_policy();
      const int pre = (int)min((long long)kDnStagesTc, it1 - it0);
      int ct = (int)(it0 / n_kb), kb = (int)(it0 % n_kb);
      for (int q = 0; q < pre; ++q) {
        unsigned char* st = smem + (size_t)q * kDnStage;
        mbar_arrive_expect_tx(&full[q], kDnStage);
        tma_load_2d_hint(st, &tm_w, ct * kTcTile, kb * kTcKB, &full[q], pol);
        tma_load_2d_hint(st + kDnBox, &tm_w, ct * kTcTile + 64, kb * kTcKB, &full[q], pol);
        if (++kb == n_kb) kb = 0, ++ct;
      }
      pdl_wait_prior();
      ct = (int)(it0 / n_kb), kb = (int)(it0 % n_kb);
      for (int q = 0; q < pre; ++q) {
        tma_load_3d_plain(smem + (size_t)q * kDnStage + kDnWBytesTc, &tm_v, kb * kTcKB, 0, 0, &full[q]);
        if (++kb == n_kb) kb = 0, ++ct;
      }
      RingPos r;
      for (int q = 0; q < pre; ++q) r.next(kDnStagesTc);
      long long issued = pre;
      for (long long j = it0 + pre; j < it1; ++j, ++issued) {
        if (!tc_wait(&empty[r.slot], (r.round - 1) & 1, p, &s_abort)) break;
        unsigned char* st = smem + (size_t)r.slot * kDnStage;
        mbar_arrive_expect_tx(&full[r.slot], kDnStage);
        tma_load_2d_hint(st, &tm_w, ct * kTcTile, kb * kTcKB, &full[r.slot], pol);
        tma_load_2d_hint(st + kDnBox, &tm_w, ct * kTcTile + 64, kb * kTcKB, &full[r.slot], pol);
        tma_load_3d_plain(st + kDnWBytesTc, &tm_v, kb * kTcKB, 0, 0, &full[r.slot]);
        if (++kb == n_kb) kb = 0, ++ct;
        r.next(kDnStagesTc);
      }
      RingPos w;
      for (long long q = 0; q < issued; ++q) {
        if (q + kDnStagesTc >= issued) mbar_wait_drain(&full[w.slot], w.round & 1, p.err);
        w.next(kDnStagesTc);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && it1 > it0) {
      // ---- MMA issuer: A = W_down^T tile (MN-major), B = v high part, then v low part
      const uint32_t idesc = umma_idesc_bf16(kTcTile, kDnN, true);
      RingPos r;
      int m = 0;
      long long j = it0;
      bool ok = true;
      while (ok && j < it1) {
        const long long tile = j / n_kb;
        const long long seg_end = min(it1, (tile + 1) * n_kb);
        const int a = m & 1;
        if (m >= 2 && !tc_wait(&acce[a], ((m >> 1) - 1) & 1, p, &s_abort)) break;
        tc_fence_after();
        const uint32_t dbase = tmem + (uint32_t)a * kDnAccCols;
        for (long long jj = j; jj < seg_end; ++jj) {
          if (!tc_wait(&full[r.slot], r.round & 1, p, &s_abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + (size_t)r.slot * kDnStage);
#pragma unroll
          for (int k = 0; k < kTcKB / 16; ++k) {
            const uint64_t aw = umma_desc_mn(sb + 2048u * k, kDnBox);
            umma_bf16(dbase + (uint32_t)kDnN * (k & 1), aw, umma_desc_k(sb + kDnWBytesTc + 32u * k), idesc,
                      (jj == j && k < 2) ? 0u : 1u);
          }
          umma_commit(&empty[r.slot]);
          r.next(kDnStagesTc);
        }
        if (!ok) break;
        umma_commit(&accf[a]);
        ++m;
        j = seg_end;
      }
      umma_commit(&drain);
      mbar_wait_drain(&drain, 0, p.err);
    }
  } else {
    // ---- epilogue: warps 2..5, one output column per thread
    const int et = threadIdx.x - 2 * kWarp;
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    pdl_wait_prior();
    if constexpr (NB > 0) {
      // the compaction needs only the flags and kept activations of the finished gate/up kernel
      FusedArgs f{};
      f.h = h;
      f.B = B;
      f.flags = p.flags;
      f.afull = p.afull;
      f.cand_idx = nullptr;
      f.idx = p.idx;
      f.count = p.count;
      f.a_val = p.a_val;
      compact_flags<NB>(f, h, s_cnt, et, 2);
    }
    int m = 0;
    long long j = it0;
    while (j < it1) {
      const long long tile = j / n_kb;
      const long long tile_it0 = tile * n_kb, tile_it1 = tile_it0 + n_kb;
      const long long seg_end = min(it1, tile_it1);
      const int a = m & 1;
      // every epilogue warp leaves together (the split-tile protocol meets at a named barrier)
      if (!named_all(3, 4 * kWarp, tc_wait(&accf[a], (m >> 1) & 1, p, &s_abort))) break;
      tc_fence_after();
      float acc[16], part[3][16];  // tokens 0..15 of this column: high / low parts, even / odd k-steps
      tmem_ld16(lane_base + (uint32_t)a * kDnAccCols, acc);
      tmem_ld16(lane_base + (uint32_t)a * kDnAccCols + 16u, part[0]);
      tmem_ld16(lane_base + (uint32_t)a * kDnAccCols + 32u, part[1]);
      tmem_ld16(lane_base + (uint32_t)a * kDnAccCols + 48u, part[2]);
      tmem_ld_wait();
#pragma unroll
      for (int v = 0; v < 16; ++v) acc[v] = (acc[v] + part[1][v]) + (part[0][v] + part[2][v]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[a]);
      bool fin = j == tile_it0 && seg_end == tile_it1;
      if (!fin)
        fin = finish_split_tile<16>(acc, p, ctr + tile, et, tile_it0, tile_it1, j, (int)(seg_end - j), n_kb, n_it,
                                    &s_flag);
      if (fin) {
        const int col = (int)tile * kTcTile + row;
        if (col < d) {
#pragma unroll
          for (int b = 0; b < kTcN; ++b) {
            if (b < B) {
              const size_t o = (size_t)b * d + col;
              if (p.out_mode == CSFFN_OUT_BF16)
                reinterpret_cast<bf16*>(p.out)[o] = __float2bfloat16_rn(acc[b]);
              else if (p.out_mode == CSFFN_OUT_F32)
                reinterpret_cast<float*>(p.out)[o] = acc[b];
              else
                reinterpret_cast<float*>(p.out)[o] += acc[b];
            }
          }
        }
      }
      ++m;
      j = seg_end;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kDnTmemCols);
  }
}

// ---------------------------------------------------------------------------------------------
// Launcher
// ---------------------------------------------------------------------------------------------
bool tc_ffn_supported(int d, int h, int B, int wdtype) {
  return wdtype == CSFFN_BF16 && B >= 1 && B <= kTcN && d >= kTcKB && d % kTcKB == 0 && d <= CSFFN_MAX_D &&
         h >= 8 && h % 8 == 0;
}

namespace {

bool encode_2d(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
               uint32_t box_outer) {
  TensorMapEncodeFn encode = tensor_map_encoder();
  if (!encode) return false;
  const cuuint64_t dim[2] = {inner, outer};
  const cuuint64_t stride[1] = {inner * 2};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t ones[2] = {1, 1};
  return encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dim, stride, box, ones,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename K>
cudaError_t set_smem(K kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

template <int NB>
cudaError_t launch_down_t(const TcArgs& a, cudaLaunchConfig_t cfg, const CUtensorMap& tm_w, const CUtensorMap& tm_v) {
  auto kern = tc_down_kernel<NB>;
  cudaError_t e = set_smem(kern, kDnSmem);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, kern, a, tm_w, tm_v);
}

}  // namespace

cudaError_t launch_tc_ffn(const TcArgs& a, cudaStream_t s) {
  if (!tc_ffn_supported(a.d, a.h, a.B, CSFFN_BF16)) return cudaErrorInvalidValue;
  CUtensorMap tm_g, tm_u, tm_x, tm_w, tm_v;
  if (!encode_2d(&tm_g, a.W_gate, a.d, a.h, kTcKB, kTcTile) || !encode_2d(&tm_u, a.W_up, a.d, a.h, kTcKB, kTcTile) ||
      !encode_2d(&tm_x, a.x, a.d, a.B, kTcKB, kTcN) || !encode_2d(&tm_w, a.W_down_t, a.d, a.h, 64, kTcKB))
    return cudaErrorInvalidValue;
  {
    // v as [2 parts][B tokens][h neurons]: boxes of 64 neurons x 16 tokens x 2 parts (tokens past B read as zeros)
    TensorMapEncodeFn encode = tensor_map_encoder();
    const cuuint64_t dim[3] = {(cuuint64_t)a.h, (cuuint64_t)a.B, 2};
    const cuuint64_t stride[2] = {(cuuint64_t)a.h * 2, (cuuint64_t)a.B * a.h * 2};
    const cuuint32_t box[3] = {kTcKB, kTcN, 2};
    const cuuint32_t ones[3] = {1, 1, 1};
    if (encode(&tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.v, dim, stride, box, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const int sms = sm_count() < kTcMaxCtas ? sm_count() : kTcMaxCtas;
  const long long it_gu = (long long)((a.h + kTcTile - 1) / kTcTile) * (a.d / kTcKB);
  const long long it_dn = (long long)((a.d + kTcTile - 1) / kTcTile) * ((a.h + kTcKB - 1) / kTcKB);

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kTcThreads);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;

  cfg.gridDim = dim3((unsigned)(it_gu < sms ? it_gu : sms));
  cfg.dynamicSmemBytes = kGuSmem;
  cudaError_t e;
  if (a.masked) {
    e = set_smem(tc_gate_up_kernel<true>, kGuSmem);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, tc_gate_up_kernel<true>, a, tm_g, tm_u, tm_x);
  } else {
    e = set_smem(tc_gate_up_kernel<false>, kGuSmem);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, tc_gate_up_kernel<false>, a, tm_g, tm_u, tm_x);
  }
  if (e != cudaSuccess) return e;

  cfg.gridDim = dim3((unsigned)(it_dn < sms ? it_dn : sms));
  cfg.dynamicSmemBytes = kDnSmem;
  if (!a.masked) return launch_down_t<0>(a, cfg, tm_w, tm_v);
  switch (batch_tier(a.B)) {
    case 1: return launch_down_t<1>(a, cfg, tm_w, tm_v);
    case 2: return launch_down_t<2>(a, cfg, tm_w, tm_v);
    case 4: return launch_down_t<4>(a, cfg, tm_w, tm_v);
    case 8: return launch_down_t<8>(a, cfg, tm_w, tm_v);
    default: return launch_down_t<16>(a, cfg, tm_w, tm_v);
  }
}

}  // namespace csffn
