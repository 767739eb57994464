// Shared device helpers and the workspace layout of libcsffn.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/csffn.h"

namespace csffn {

typedef __nv_bfloat16 bf16;

constexpr int kWarp = 32;

// Device error bits recorded in the workspace error word.
constexpr uint32_t kDevErrTimeout = 1u;

// ------------------------------------------------------------------------------------------
// Workspace layout.  The control region (counters, status words) must be zero before the first
// call (csffn_workspace_init); every kernel that uses a counter leaves it at zero when it ends.
// ------------------------------------------------------------------------------------------
struct Control {           // one per compaction user, 64 bytes apart
  uint32_t epoch;          // bumped by the last CTA of every compaction launch
  uint32_t ticket;         // dynamic chunk tickets
  uint32_t done;           // CTAs finished
  uint32_t pad[13];
};

constexpr int kCtlGate = 0;     // csffn_gate_mask
constexpr int kCtlPred = 1;     // csffn_predict_lowrank
constexpr int kCtlFused = 2;    // csffn_cats_ffn_forward (tile and exit counters)
constexpr int kNumCtl = 4;
constexpr int kMaxSlices = 128;  // column slices of the down projection (d / slice width)
constexpr int kMaxRowRanges = 64;
constexpr int kSliceUsers = 2;  // sparse forward, dense forward

struct WsLayout {
  size_t ctl;        // Control[kNumCtl]
  size_t err;        // uint32 error word (+ pad)
  size_t slice_ctr;  // uint32 [kSliceUsers][kMaxSlices]
  size_t tickets;    // uint32 [64][32]                 chunk-ticket counters, 128 B apart (fused path)
  size_t facc;       // fp32 [kFusedAccCopies][kFusedMaxBatch][CSFFN_MAX_D] out accumulators (fused path)
  size_t status;     // uint64 [kNumCtl][max_chunks]   look-back status words
  size_t tcctr;      // uint32 [tc_counters(h)]         k-blocks done per tile (tensor-core FFN)
  size_t control_end;
  size_t vbuf;       // fp32 [max_batch][h]            v = a * u (sparse) or act(z)*u (dense)
  size_t afull;      // fp32 [max_batch][h]            per-neuron kept activations (fused path)
  size_t flags;      // uint8 [h]                      per-neuron keep flags (fused path)
  size_t partial;    // fp32 [partial_rows(max_batch)][d]
  size_t tcpart;     // fp32 [kTcMaxCtas][2][32][128]    split tiles' partial accumulators (tensor-core FFN)
  size_t svdcnt;     // uint32 [kTcMaxCtas]              kept rows per CTA (SVD step)
  size_t ybuf;       // fp32 [max_batch][max_rank]     predictor y = x U_r
  size_t hx;         // [max_batch][d] (4 B each)      tokens staged from host memory (host entry point)
  size_t hout;       // fp32 [max_batch][d]            output staged for the copy back to host memory
  size_t total;
  int max_chunks;
};

constexpr int kChunkRows = 16;  // rows per compaction chunk (one ballot)
constexpr int kFusedMaxBatch = 4;
constexpr int kFusedAccCopies = 8;  // fused step: CTA k adds into accumulator k % kFusedAccCopies

// Tensor-core FFN (tc_ffn.cu): tiles of 128 neurons (gate/up) or 128 output columns (down); at most
// kTcMaxCtas CTAs, each with two partial-accumulator slots of 32 x 128 floats.
constexpr int kTcTile = 128;
constexpr int kTcMaxCtas = 160;
__host__ __device__ inline int tc_counters(int h) { return (h + kTcTile - 1) / kTcTile + CSFFN_MAX_D / kTcTile; }

// Rows of d floats in the partial region (one per row range of the sparse/dense forward).
__host__ __device__ inline int partial_rows(int max_batch) { return kMaxRowRanges * max_batch; }

__host__ __device__ inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline WsLayout ws_layout(int d, int h, int max_batch, int max_rank) {
  WsLayout L;
  size_t o = 0;
  L.ctl = o;        o += sizeof(Control) * kNumCtl;
  L.err = o;        o += 64;
  L.slice_ctr = o;  o += sizeof(uint32_t) * kSliceUsers * kMaxSlices;
  o = align_up(o, 128);
  L.tickets = o;    o += sizeof(uint32_t) * 64 * 32;
  o = align_up(o, 256);
  L.facc = o;       o += sizeof(float) * (size_t)kFusedAccCopies * kFusedMaxBatch * CSFFN_MAX_D;
  o = align_up(o, 256);
  L.max_chunks = (h + kChunkRows - 1) / kChunkRows;
  L.status = o;     o += sizeof(uint64_t) * (size_t)kNumCtl * L.max_chunks;
  o = align_up(o, 256);
  L.tcctr = o;      o += sizeof(uint32_t) * (size_t)tc_counters(h);
  o = align_up(o, 256);
  L.control_end = o;
  L.vbuf = o;       o += sizeof(float) * (size_t)max_batch * h;
  o = align_up(o, 256);
  L.afull = o;      o += sizeof(float) * (size_t)max_batch * h;
  o = align_up(o, 256);
  L.flags = o;      o += align_up((size_t)h, 16);
  o = align_up(o, 256);
  // partials: one per row range of the sparse/dense forward
  L.partial = o;    o += sizeof(float) * (size_t)partial_rows(max_batch) * d;
  o = align_up(o, 256);
  L.tcpart = o;     o += sizeof(float) * (size_t)kTcMaxCtas * 2 * 32 * kTcTile;
  o = align_up(o, 256);
  L.svdcnt = o;     o += sizeof(uint32_t) * (size_t)kTcMaxCtas;
  o = align_up(o, 256);
  L.ybuf = o;       o += sizeof(float) * (size_t)max_batch * (max_rank > 0 ? max_rank : 1);
  o = align_up(o, 256);
  L.hx = o;         o += align_up(sizeof(float) * (size_t)max_batch * d, 256);
  L.hout = o;       o += align_up(sizeof(float) * (size_t)max_batch * d, 256);
  L.total = o;
  return L;
}

// The layout is recomputed from (d, h, B, rank) on every call.  The control region's offsets
// depend on h only, so counters persist correctly across calls with different batch sizes; the
// scratch regions after it are per call.  Each entry point checks ws_bytes against its needs.

// ------------------------------------------------------------------------------------------
// Loads and conversions
// ------------------------------------------------------------------------------------------

// Streaming 16-byte load of read-once weights: read-only path, no L1 allocation.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// Asynchronous 16-byte global -> shared copy by this thread (cp.async, cached in L2 only).  The
// data is this thread's own: it waits for it with cp_async_wait<N> and nothing else is needed.
// `after` is a value the copy must not be issued before (a register dependency that orders the
// copy after the thread's earlier reads of the same shared memory).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src, uint32_t after) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(src), "r"(after)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <typename T> struct Vec;
template <> struct Vec<bf16> { static constexpr int N = 8; };
template <> struct Vec<float> { static constexpr int N = 4; };

// 16 bytes of weights -> N floats.
__device__ __forceinline__ void unpack(const uint4& w, float (&f)[8]) {
  f[0] = bf16lo(w.x); f[1] = bf16hi(w.x); f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
  f[4] = bf16lo(w.z); f[5] = bf16hi(w.z); f[6] = bf16lo(w.w); f[7] = bf16hi(w.w);
}
__device__ __forceinline__ void unpack(const uint4& w, float (&f)[4]) {
  f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y);
  f[2] = __uint_as_float(w.z); f[3] = __uint_as_float(w.w);
}

// N consecutive x values from shared memory (16-byte aligned), as floats.
template <int N>
__device__ __forceinline__ void load_x(const bf16* p, float (&f)[N]) {
  static_assert(N == 8, "bf16 x pairs with bf16 weights");
  uint4 v = *reinterpret_cast<const uint4*>(p);
  unpack(v, f);
}
template <int N>
__device__ __forceinline__ void load_x(const float* p, float (&f)[N]) {
  if constexpr (N == 8) {
    float4 a = reinterpret_cast<const float4*>(p)[0];
    float4 b = reinterpret_cast<const float4*>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  } else {
    float4 a = reinterpret_cast<const float4*>(p)[0];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  }
}

// 16 bytes of token values (same element type as the weights) -> floats.
template <typename T>
__device__ __forceinline__ void unpack_x(const uint4& v, float (&f)[Vec<T>::N]) {
  unpack(v, f);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// SwiGLU / ReGLU gate activation.  SiLU(z) = z / (1 + e^-z), with CUDA's expf.
__device__ __forceinline__ float gate_act(float z, int act) {
  return act == CSFFN_ACT_SILU ? z / (1.0f + expf(-z)) : fmaxf(z, 0.0f);
}

// ------------------------------------------------------------------------------------------
// Cross-CTA status words.  A status word carries only a count that the reader adds up; no other
// data written by the publishing CTA is read through it inside the kernel (outputs are consumed
// by later launches), so single-copy-atomic relaxed accesses at GPU scope suffice and the
// publishing thread pays no fence.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint64_t ld_status(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_status(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Look-back status word: [epoch:32 | flag:2 | value:30].
constexpr uint64_t kFlagAggregate = 1, kFlagInclusive = 2;
__device__ __forceinline__ uint64_t status_word(uint32_t epoch, uint64_t flag, uint32_t value) {
  return ((uint64_t)epoch << 32) | (flag << 30) | (uint64_t)value;
}

// Polls before a bounded wait gives up: 2^22 polls with ~128 ns sleeps (about half a second),
// far beyond any wait on a CTA that is running.
constexpr uint32_t kSpinLimit = 1u << 22;

// Bounded wait on a 64-bit status word: polls *p until ready(value) holds or `limit`
// polls have failed.  On success returns true with the word in *out; on give-up records
// kDevErrTimeout in *err and returns false.  Every device-side wait in the library uses this.
template <typename Ready>
__device__ __forceinline__ bool bounded_wait(const uint64_t* p, uint32_t limit, uint32_t* err,
                                             Ready ready, uint64_t* out) {
  for (uint32_t spins = 0;; ++spins) {
    const uint64_t v = ld_status(p);
    if (ready(v)) {
      *out = v;
      return true;
    }
    if (spins >= limit) {
      atomicOr(err, kDevErrTimeout);
      return false;
    }
    __nanosleep(128);
  }
}

__device__ __forceinline__ uint32_t warp_sum_u32(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint64_t globaltimer_now() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Decoupled look-back for chunk c, run by one full warp (all 32 lanes call it).
//
// Publishes the chunk's aggregate `agg`, then reads the status words of 32 predecessors at once
// (lane l reads chunk base-l; positions before chunk 0 count as an inclusive prefix of 0).  As
// soon as every predecessor up to the nearest inclusive prefix is published in this epoch, it sums
// them and stops; if all 32 are published and none is inclusive, it adds the window's aggregates
// and moves 32 chunks further back.  Publishes the chunk's inclusive prefix and returns the
// exclusive one (the same in every lane).  A window that stays unusable for a second records
// kDevErrTimeout in *err and ends the walk early (the caller keeps every write in bounds).
// With agg_published the caller has already published the chunk's aggregate (chunk 0: its
// inclusive prefix), so only the walk and the inclusive publication remain.
__device__ __forceinline__ uint32_t warp_lookback(uint64_t* status, int c, uint32_t epoch, uint32_t agg,
                                                  uint32_t* err, int lane, bool agg_published = false) {
  if (c == 0) {
    if (lane == 0 && !agg_published) st_status(&status[0], status_word(epoch, kFlagInclusive, agg));
    return 0;
  }
  if (lane == 0 && !agg_published) st_status(&status[c], status_word(epoch, kFlagAggregate, agg));
  uint32_t prefix = 0;
  uint64_t t0 = 0;
  bool started = false;
  for (int base = c - 1;;) {
    const int j = base - lane;
    const uint64_t s = j >= 0 ? ld_status(&status[j]) : status_word(epoch, kFlagInclusive, 0);
    const bool ready = (uint32_t)(s >> 32) == epoch && ((s >> 30) & 3u) != 0;
    const uint32_t ready_m = __ballot_sync(0xffffffffu, ready);
    const uint32_t incl_m = __ballot_sync(0xffffffffu, ready && ((s >> 30) & 3u) == kFlagInclusive);
    const int first_wait = ready_m == 0xffffffffu ? kWarp : __ffs(~ready_m) - 1;
    const int first_incl = incl_m ? __ffs(incl_m) - 1 : kWarp;
    const uint32_t val = (uint32_t)(s & 0x3FFFFFFFu);
    if (first_incl < first_wait) {  // everything up to the nearest inclusive prefix is known
      prefix += warp_sum_u32(lane <= first_incl ? val : 0u);
      break;
    }
    if (first_wait == kWarp) {  // a full window of aggregates: add it and look further back
      prefix += warp_sum_u32(val);
      base -= kWarp;
      started = false;
      continue;
    }
    if (!started) {
      t0 = globaltimer_now();
      started = true;
    } else if (globaltimer_now() - t0 > 1000000000ull) {
      if (lane == 0) atomicOr(err, kDevErrTimeout);
      break;
    }
    __nanosleep(32);
  }
  if (lane == 0) st_status(&status[c], status_word(epoch, kFlagInclusive, prefix + agg));
  return prefix;
}

}  // namespace csffn
