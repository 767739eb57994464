// Host-side launchers of libcsffn's kernels (internal; the public surface is include/csffn.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace csffn {

struct Control;

// Token-capacity tier used to instantiate the GEMV kernels: 1, 2, 4, 8 or 16.
inline int batch_tier(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : B <= 8 ? 8 : 16; }

enum GateMode { kModeCats = 0, kModePred = 1 };

// Fused row GEMV + activation/compare + union over tokens + ascending compaction.
struct GateArgs {
  const void* W;              // [h, K] rows (W_gate, or V_r for the predictor)
  const void* x;              // [B, K] tokens: weight dtype (CATS) or fp32 (predictor y)
  int K, h, B;
  const float* bias;          // [h] or NULL
  float t;                    // CATS threshold on |act(z)|
  const float* tau;           // [h] per-neuron thresholds on z (predictor mode)
  int act;                    // csffn_act
  const int32_t* cand_idx;    // NULL = rows 0..h-1
  const int32_t* cand_count;
  int32_t* idx;
  int32_t* count;
  float* a_val;               // [B, h] (CATS mode)
  Control* ctl;
  uint64_t* status;
  uint32_t* err;
};
cudaError_t launch_gate_compact(const GateArgs& a, int wdtype, bool x_f32, int mode, cudaStream_t s);
// Streaming version with an asynchronous compaction warp (gate_stream.cu); needs the staged tokens
// to fit in shared memory.
bool gate_stream_supported(int K, int B, int wdtype, bool x_f32);
cudaError_t launch_gate_stream(const GateArgs& a, int wdtype, bool x_f32, int mode, cudaStream_t s);
// Picks the streaming kernel when the shape allows it, else the chunk-synchronous one.
inline cudaError_t launch_gate(const GateArgs& a, int wdtype, bool x_f32, int mode, cudaStream_t s) {
  return gate_stream_supported(a.K, a.B, wdtype, x_f32) ? launch_gate_stream(a, wdtype, x_f32, mode, s)
                                                        : launch_gate_compact(a, wdtype, x_f32, mode, s);
}

// v[b*h + j] = a_val[b*h + j] * (x_b . W_up[idx[j]]) for j < *count.
struct UpArgs {
  const void* W_up;
  const void* x;
  int d, h, B;
  const int32_t* idx;
  const int32_t* count;
  const float* a_val;
  float* v;
  uint32_t* err;  // device error word (for kernels with bounded waits)
};
cudaError_t launch_up_gather(const UpArgs& a, int wdtype, cudaStream_t s);
inline cudaError_t launch_up(const UpArgs& a, int wdtype, cudaStream_t s) { return launch_up_gather(a, wdtype, s); }

// v[b*h + i] = act(x_b . W_gate[i] + beta_i) * (x_b . W_up[i]) for all i < h.
struct DenseGateUpArgs {
  const void* W_gate;
  const void* W_up;
  const void* x;
  int d, h, B;
  const float* bias;
  int act;
  float* v;
};
cudaError_t launch_dense_gate_up(const DenseGateUpArgs& a, int wdtype, cudaStream_t s);

// out[b, :] (=|+=) sum_{j < n} v[b*h + j] * W_down^T[idx ? idx[j] : j, :]
struct DownArgs {
  const void* W_down_t;
  int d, h, B;
  const int32_t* idx;     // NULL = identity
  const int32_t* count;   // NULL = n_host
  int n_host;
  const float* v;
  float* partial;         // [row_ranges][B][d]
  uint32_t* slice_ctr;    // [slices]
  void* out;
  int out_mode;
  uint32_t* err;  // device error word (for kernels with bounded waits)
};
cudaError_t launch_down_gather(const DownArgs& a, int wdtype, cudaStream_t s);
inline cudaError_t launch_down(const DownArgs& a, int wdtype, cudaStream_t s) { return launch_down_gather(a, wdtype, s); }

// y[b*rank + k] = x_b . U_r^T[k]  (plain GEMV, fp32 out)
struct RowGemvArgs {
  const void* W;      // [rows, K]
  const void* x;      // [B, K] weight dtype
  int rows, K, B;
  float* y;           // [B, rows]   (y[b*y_stride + row])
  int y_stride;
  const float* bias;  // [rows] or NULL, added
  int act;            // -1 = none, else csffn_act
  int abs_out;        // write |value|
  int transpose_out;  // write y[row*y_stride + b] instead
};
cudaError_t launch_row_gemv(const RowGemvArgs& a, int wdtype, bool x_f32, cudaStream_t s);

// Dense FFN of up to 16 tokens on the tensor cores (dense_mma.cu): gate/up into v, then the down
// projection over all h neurons (DownArgs with idx = count = NULL, n_host = h).
constexpr int kDenseMmaMinBatch = 8;  // from this many tokens on, FMA throughput would bound the dense FFN
bool dense_mma_supported(int d, int h, int B, int wdtype);
cudaError_t launch_dense_gate_up_mma(const DenseGateUpArgs& a, cudaStream_t s);
cudaError_t launch_down_mma(const DownArgs& a, int max_ranges, cudaStream_t s);

// One-launch CATS decode step (cats_fused.cu): gate + threshold + up + down in one pass over
// dynamically assigned row chunks, a grid-wide count, the cross-CTA sum and the compaction of
// idx / a_val / count.
struct FusedArgs {
  const void* W_gate;
  const void* W_up;
  const void* W_down_t;
  const void* x;
  int d, h, B;
  const float* bias;
  float t;
  int act;
  const int32_t* cand_idx;    // rows to consider (ascending neurons), or NULL = all h neurons
  const int32_t* cand_count;  // device count of cand_idx
  const void* u_rt;           // predictor mode (non-NULL): U_r^T [rank, d], V_r [h, rank], tau [h]
  const void* v_r;
  const float* tau;
  int rank;
  float* ybuf;                // [B, rank] scratch: y = x U_r
  float* afull;      // [B, h] scratch: kept activation per row position
  uint8_t* flags;    // [h] scratch: keep flag per row position (16-byte aligned)
  float* facc;      // fp32 [kFusedAccCopies][B, d] accumulators of out, zero between launches
  uint32_t* ctl;     // fused control words (arrival counter, generation), zero before first use
  uint32_t* tickets; // [32 * 32] chunk-ticket counters and dry flags, 128 bytes apart
  uint32_t* svd_counts;  // [kTcMaxCtas] SVD step: kept rows per CTA
  uint32_t* err;
  int32_t* idx;
  int32_t* count;
  float* a_val;
  void* out;
  int out_mode;
};
bool cats_fused_supported(int d, int B, int wdtype, int rank = 0);
cudaError_t launch_cats_fused(const FusedArgs& a, int wdtype, cudaStream_t s);
// The same step (CATS or candidate mode, not the predictor mode) on a shared-memory ring fed by
// bulk copies from one producer warp (ring.cu): one CTA per SM.
bool cats_ring_supported(int d, int B, int wdtype);
cudaError_t launch_cats_ring(const FusedArgs& a, int wdtype, cudaStream_t s);
// Copy of `bytes` (a multiple of 16, both pointers 16-byte aligned) from src (device-accessible, e.g.
// mapped host memory) to dst, as a programmatic dependent of the kernel before it on the stream.
cudaError_t launch_stage_tokens(const void* src, void* dst, size_t bytes, cudaStream_t s);

// SVD-predicted step of up to 4 tokens in one cooperative launch (svd_step.cu): y = x U_r, one
// grid-wide count, then predictor, gate, up, down and the end phase; `parallel` fetches W_up with
// W_gate for the predicted rows.
bool svd_step_supported(int d, int h, int B, int wdtype, int rank);
cudaError_t launch_svd_step(const FusedArgs& a, int wdtype, bool parallel, cudaStream_t s);

// Gated FFN of up to 16 tokens on the fifth-generation tensor cores (tc_ffn.cu): a gate/up kernel
// (tcgen05.mma, operands staged by TMA tensor copies, fp32 accumulators in TMEM) writes v = act(z +
// beta) * u as bf16 high and low parts, then a down kernel (the same machinery, W_down^T read
// MN-major) writes out.  Both split their work evenly over the SMs as contiguous runs of 64-element
// k-blocks (a tile split between CTAs is finished by the last one to arrive).  Masked mode is the
// CATS step: v and the kept activations are zero where |act(z + beta)| <= t, the keep flags are
// written, and the down kernel also compacts idx / a_val / count.
struct TcArgs {
  const void* W_gate;
  const void* W_up;
  const void* W_down_t;
  const void* x;      // [B, d] bf16
  int d, h, B;
  const float* bias;  // [h] or NULL
  int act;
  int masked;         // CATS step (flags, afull, idx / a_val / count written)
  float t;
  uint16_t* v;        // [2][B][h] bf16 bits: high parts, then low parts
  float* afull;       // [B, h] kept activations (masked)
  uint8_t* flags;     // [h] keep flags (masked)
  float* part;        // [kTcMaxCtas][2][32][128] partial accumulators
  uint32_t* ctr;      // [tc_counters(h)]: gate/up tiles, then down column tiles; zero between launches
  uint32_t* err;
  int32_t* idx;       // masked: the compacted union (as csffn_cats_ffn_forward)
  int32_t* count;
  float* a_val;
  void* out;
  int out_mode;
};
bool tc_ffn_supported(int d, int h, int B, int wdtype);
cudaError_t launch_tc_ffn(const TcArgs& a, cudaStream_t s);

// Radix selection and per-neuron selection (calibration).
size_t kth_state_bytes();
cudaError_t launch_kth_smallest(const float* values, int64_t n, int64_t k, float* out, void* state,
                                cudaStream_t s);
cudaError_t launch_rows_kth(const float* values, int rows, int n, int k, float* out, cudaStream_t s);
// Per-neuron thresholds for a target recall of the active set (rows of P^T and Z^T, n vectors each).
cudaError_t launch_rows_recall(const float* pt, const float* zt, int rows, int n, float recall, float* out,
                               cudaStream_t s);
cudaError_t launch_fill(float* p, float v, int n, cudaStream_t s);

cudaError_t launch_rmsnorm_bf16(const float* h, int B, int d, float eps, void* xn, cudaStream_t s);

cudaError_t launch_timeout_selftest(uint64_t* flag, uint32_t* err, int spin_limit, cudaStream_t s);

int sm_count();

}  // namespace csffn
