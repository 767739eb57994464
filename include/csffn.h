/*
 * csffn -- contextually sparse gated FFN at decode time, for NVIDIA B200 (sm_100a).
 *
 * C ABI of libcsffn.so.  Plain pointers and sizes only.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument named x, w_*, idx, count, a_val, out, t_out, tau,
 *    u_rt, v_r, values, ws is a DEVICE pointer owned by the caller.  The library
 *    keeps no pointer after the call returns and allocates no device memory on
 *    any path: scratch space comes from a caller workspace (`ws`) whose size is
 *    queried up front (csffn_sparse_ffn_forward_static instead uses one fixed
 *    library-owned device array, see its comment).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Every call is asynchronous on that stream; nothing synchronises except
 *    csffn_check_status.  Index counts (`count`, `cand_count`) stay in device
 *    memory, so a whole decode step can be captured in a CUDA graph.
 *  - Arguments are validated on the host before anything is launched; a
 *    rejected call launches nothing and returns the error.  Nothing throws.
 *  - Device-side errors (a bounded wait that ran out) are recorded in an error
 *    word inside the workspace and reported by csffn_check_status.
 *  - One workspace must not be used by two streams at once: calls that share a
 *    workspace must be ordered on one stream.
 *  - Weights are neuron-major: W_gate and W_up are [h, d] (row i = neuron i's
 *    input weights, the nn.Linear [out, in] layout) and W_down^T is [h, d]
 *    (row i = neuron i's output weights, i.e. the down projection [d, h]
 *    transposed).  Skipping a neuron therefore skips whole contiguous rows.
 *  - Token vectors x are [B, d] row-major in the weight dtype.
 *  - Alignment: d % 8 == 0 for bf16, d % 4 == 0 for fp32; every weight, x and
 *    out pointer 16-byte aligned; otherwise CSFFN_ERR_ALIGNMENT.
 *  - Index lists (idx, cand_idx) are int32, unique and ascending.
 *  - Batch limits: 1 <= B <= CSFFN_MAX_BATCH (B == 0 is an empty call, see each
 *    function).  Shape limits: 1 <= h <= CSFFN_MAX_H, 8 <= d <= CSFFN_MAX_D.
 *
 * Sources (page titles; figure/section on each page):
 *  [CATS]   "CATS: Contextually-Aware Thresholding for Sparsity in Large Language
 *           Models", abstract -- thresholded SiLU gate activation; a GPU kernel
 *           fusing the gate GEMV with the compare and a flag-gated GEMV.
 *  [SVDP]   "SVD Contextual Sparsity Predictors for Fast LLM Inference", abstract,
 *           Fig. 1 (offline SVD predictors + calibrated per-neuron thresholds run
 *           ahead of each FFN), Fig. 3 (ReGLU: gate then up run sequentially on the
 *           predicted-active neurons), Table 3 ("+ Bias calibration").
 *  [SIRIUS] "Sirius: Contextual Sparsity with Correction for Efficient LLMs",
 *           abstract and its summary page, "Approach" -- sparse and full model
 *           share weights; the full model verifies a chunk of tokens in parallel.
 */
#ifndef CSFFN_H
#define CSFFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define CSFFN_VERSION 1
#define CSFFN_MAX_BATCH 16
#define CSFFN_MAX_D 16384
#define CSFFN_MAX_H (1 << 24)
#define CSFFN_MAX_RANK 4096
#define CSFFN_MAX_CALIB 8192

typedef enum {
  CSFFN_OK = 0,
  CSFFN_ERR_INVALID_ARG = 1,       /* NULL pointer, bad enum, B/n/k/rank out of range */
  CSFFN_ERR_UNSUPPORTED_SHAPE = 2, /* d/h/B combination the library does not run */
  CSFFN_ERR_ALIGNMENT = 3,         /* d not a multiple of the vector width, or pointer not 16-B aligned */
  CSFFN_ERR_WORKSPACE = 4,         /* ws NULL or ws_bytes below the queried size */
  CSFFN_ERR_CUDA = 5,              /* a CUDA runtime call or kernel launch failed */
  CSFFN_ERR_TIMEOUT = 6            /* a bounded device-side wait ran out (see csffn_check_status) */
} csffn_status;

typedef enum { CSFFN_BF16 = 0, CSFFN_F32 = 1 } csffn_dtype;

/* Output modes of the forward calls: write bf16, write fp32, or add into an fp32
 * buffer (out += FFN(x), the residual update of a transformer block). */
typedef enum { CSFFN_OUT_BF16 = 0, CSFFN_OUT_F32 = 1, CSFFN_OUT_F32_ACCUMULATE = 2 } csffn_out_mode;

/* SILU: SwiGLU gate a = SiLU(z); RELU: ReGLU gate a = max(z, 0).  z = x.W_gate[i] + beta_i. */
typedef enum { CSFFN_ACT_SILU = 0, CSFFN_ACT_RELU = 1 } csffn_act;

typedef enum {
  CSFFN_CAL_GLOBAL_ABS_ACT = 0,  /* one scalar t: quantile of |a| over calibration set x neurons [CATS] */
  CSFFN_CAL_PER_NEURON_PRED = 1, /* tau[h]: per-neuron quantile of the SVD predictor output [SVDP] Fig. 1 */
  CSFFN_CAL_PER_NEURON_RECALL = 2 /* tau[h]: per-neuron target recall of {z > 0} [SVDP] Table 3, Fig. 2 */
} csffn_cal_mode;

/* One gated FFN layer.  wdtype applies to w_gate, w_up, w_down_t and to x. */
typedef struct {
  int32_t d;              /* model (hidden) width */
  int32_t h;              /* FFN intermediate width = number of neurons */
  int32_t wdtype;         /* csffn_dtype */
  int32_t act;            /* csffn_act */
  const void* w_gate;     /* [h, d] */
  const void* w_up;       /* [h, d] */
  const void* w_down_t;   /* [h, d] */
  const float* gate_bias; /* [h] fp32 added to z, or NULL */
} csffn_layer;

/* Library version (CSFFN_VERSION). */
int csffn_version(void);

/* Static string for a status code. */
const char* csffn_status_string(int status);

/* Bytes of workspace the decode-path calls need for this layer at batch
 * <= max_batch and predictor rank <= max_rank (0 if no predictor is used).
 * Returns 0 if the arguments are invalid. */
size_t csffn_workspace_size(const csffn_layer* layer, int max_batch, int max_rank);

/* Zero the workspace's control region (counters, the one-launch step's output
 * accumulators); required once before first use and after a CSFFN_ERR_TIMEOUT.
 * Asynchronous on `stream`. */
csffn_status csffn_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, then read and clear the device-side error word of `ws`.
 * Returns CSFFN_OK, CSFFN_ERR_TIMEOUT (a bounded wait ran out: re-initialise the
 * workspace with csffn_workspace_init before reuse) or CSFFN_ERR_CUDA. */
csffn_status csffn_check_status(void* ws, void* stream);

/* Gate GEMV + activation + threshold + active-index compaction (one kernel).
 * [CATS] abstract (fused gate GEMV + compare + flag); [SVDP] Fig. 3 (gate on the
 * predicted set).
 *   z[b,i] = x_b . W_gate[i,:] + beta_i,  a = act(z),  token b keeps neuron i iff |a[b,i]| > t.
 *   Rows considered: all h neurons if cand_idx == NULL, else cand_idx[0 .. *cand_count).
 *   Outputs: idx[0 .. *count) = ascending indices of neurons kept by ANY token (the
 *   union over the batch); a_val[b*h + j] = a[b, idx[j]] if token b keeps idx[j],
 *   else 0 (per-token values, union rows).  idx: int32 [h]; count: int32 [1];
 *   a_val: fp32 [B, h] (row stride h; entries j >= *count are untouched).
 *   With act = RELU and t = 0 the kept set is {z > 0}.  t may be negative (keeps all).
 *   B == 0: writes *count = 0 and nothing else. */
csffn_status csffn_gate_mask(const csffn_layer* layer, const void* x, int B, float t,
                             const int32_t* cand_idx, const int32_t* cand_count,
                             int32_t* idx, int32_t* count, float* a_val,
                             void* ws, size_t ws_bytes, void* stream);

/* Gathered up- and down-projection over the active rows.  [CATS] abstract
 * (flag-gated GEMV); [SVDP] Fig. 3 (up and down only on the active set).
 *   out[b,:] = sum_{j < *count} a_val[b*h + j] * (x_b . W_up[idx[j],:]) * W_down^T[idx[j],:]
 *   Reads only rows idx[0 .. *count) of W_up and W_down^T.  *count is read on the
 *   device.  out: [B, d] in the dtype of out_mode (ACCUMULATE adds into fp32 out).
 *   *count == 0 gives out = 0 (or leaves an accumulated out unchanged).  B == 0: no-op. */
csffn_status csffn_sparse_ffn_forward(const csffn_layer* layer, const void* x, int B,
                                      const int32_t* idx, const int32_t* count, const float* a_val,
                                      void* out, int out_mode, void* ws, size_t ws_bytes, void* stream);

/* One CATS decode step: everything csffn_gate_mask followed by csffn_sparse_ffn_forward computes,
 * with the same outputs (idx, *count, a_val as gate_mask; out as sparse_ffn_forward).  [CATS]
 * abstract: the gate GEMV, the compare and the flag-gated GEMV of one FFN layer.  The path depends on
 * the batch:
 *   - B <= 2 (and B <= 4 for the shapes the tensor-core path below does not take): a streaming
 *     kernel runs the gate, the threshold and the up and down projections of the kept rows in one
 *     pass over dynamically assigned neuron rows, the CTAs adding their partial outputs into fp32
 *     accumulators in the workspace; a short finishing kernel, launched as its programmatic
 *     dependent, turns the accumulators into out (clearing them for the next call) and compacts
 *     idx / a_val / count.  Where that kernel does not fit (d, dtype), a one-launch cooperative
 *     kernel or the two-call path inside this call computes the same.
 *   - B >= 3 for bf16 layers with d % 64 == 0 and h % 8 == 0 (no cand_idx): the union of the tokens'
 *     masks covers most neurons, so the tensor-core FFN of csffn_dense_ffn_forward runs with the
 *     activations at or below the threshold zeroed, and its down kernel also compacts the keep flags.
 *   - other shapes: the two-call path inside this call.
 * The mask and a_val are bit-for-bit repeatable; out may differ from launch to launch in the last
 * bits on the streaming paths (rows reach CTAs dynamically and the CTAs' fp32 partial sums are added
 * in arrival order).  cand_idx / cand_count (both or neither): as in csffn_gate_mask, only the
 * listed neurons (ascending, device count) are considered, e.g. the set csffn_predict_lowrank
 * predicts ([SVDP] Fig. 3: the gate runs on the predicted set; with act = RELU and t = 0 the kept set
 * is {z > 0} within it).  ws sized by csffn_workspace_size for this layer and batch.  B == 0: writes
 * *count = 0. */
csffn_status csffn_cats_ffn_forward(const csffn_layer* layer, const void* x, int B, float t,
                                    const int32_t* cand_idx, const int32_t* cand_count,
                                    int32_t* idx, int32_t* count, float* a_val,
                                    void* out, int out_mode, void* ws, size_t ws_bytes, void* stream);

/* csffn_cats_ffn_forward with the tokens x_host [B, d] (weight dtype) and the output out_host [B, d]
 * (bf16 or fp32; out_mode CSFFN_OUT_BF16 or CSFFN_OUT_F32) in host memory, asynchronously on
 * `stream`.  When both are page-locked host memory mapped into the device's address space
 * (cudaHostAlloc, cudaMallocHost or cudaHostRegister under unified addressing) and 16-byte aligned,
 * a small kernel stages x into the workspace over the host link and the step writes out there
 * directly: no copy-engine work, and consecutive steps on the stream stay chained like
 * device-memory steps.  Otherwise x is copied into the workspace, the step runs there, and out is
 * copied back (pageable memory makes those copies synchronous).  idx,
 * count and a_val stay in device memory as in csffn_cats_ffn_forward.  The host buffers must stay
 * valid, and x_host unchanged, until the step has completed on the stream.  ws sized by
 * csffn_workspace_size for this layer and batch (it holds the staged tokens and output).  B == 0:
 * writes *count = 0. */
csffn_status csffn_cats_ffn_forward_host(const csffn_layer* layer, const void* x_host, int B, float t,
                                         int32_t* idx, int32_t* count, float* a_val,
                                         void* out_host, int out_mode, void* ws, size_t ws_bytes, void* stream);

/* Dense gated FFN over all h neurons (the full model that verifies a chunk of
 * sparse-drafted tokens, [SIRIUS] "Approach"; also the speed-up baseline).
 *   out = (act(x W_gate^T + beta) * (x W_up^T)) W_down.  B == 0: no-op.
 *   bf16 layers with d % 64 == 0 and h % 8 == 0 run on the fifth-generation tensor cores for any
 *   1 <= B <= 16 (tcgen05 MMA with fp32 accumulators in tensor memory, operands staged by TMA, one
 *   pass over the weights for all tokens; a gate/up kernel, then a down kernel); the down
 *   projection takes the fp32 activations as a bf16 high part plus a bf16 low part, so about 16 of
 *   their mantissa bits reach the product.  The result is bit-for-bit repeatable.  Other bf16 layers
 *   with 8 <= B <= 16 and d % 128 == 0 use an mma.sync path; the rest runs on the CUDA cores (fp32
 *   FMA). */
csffn_status csffn_dense_ffn_forward(const csffn_layer* layer, const void* x, int B,
                                     void* out, int out_mode, void* ws, size_t ws_bytes, void* stream);

/* SVD low-rank predictor + per-neuron compare + compaction.  [SVDP] Fig. 1.
 *   y = x U_r (u_rt is U_r^T, [rank, d], row k = sigma_k * k-th left singular vector),
 *   p[b,i] = y_b . V_r[i,:] + beta_i (v_r: [h, rank]; beta = layer->gate_bias or 0),
 *   neuron i is a candidate iff p[b,i] > tau[i] for ANY token b.
 *   cand_idx[0 .. *cand_count) = ascending candidates (int32 [h]; count int32 [1]).
 *   u_rt, v_r in layer->wdtype; rank % (8 for bf16, 4 for fp32) == 0.
 *   B == 0: writes *cand_count = 0. */
csffn_status csffn_predict_lowrank(const csffn_layer* layer, const void* x, int B, int rank,
                                   const void* u_rt, const void* v_r, const float* tau,
                                   int32_t* cand_idx, int32_t* cand_count,
                                   void* ws, size_t ws_bytes, void* stream);

/* The predictor pipeline of one decode step ([SVDP] Fig. 1 and Fig. 3): csffn_predict_lowrank
 * followed by csffn_cats_ffn_forward on the predicted set computes the same.
 *   y = x U_r; neuron i is predicted iff p[b,i] = y_b . V_r[i,:] + beta_i > tau[i] for some token b;
 *   a predicted neuron's gate runs (z = x W_gate[i] + beta_i, a = act(z), token b keeps it iff
 *   |a| > t: with act = RELU and t = 0, A = {z > 0} within the predicted set), and the kept rows'
 *   up and down projections give out.  idx[0 .. *count) = ascending kept neurons, a_val as in
 *   csffn_gate_mask, out as in csffn_sparse_ffn_forward.  The predicted set itself is not written.
 *   u_rt [rank, d], v_r [h, rank] in layer->wdtype, rank % (8 for bf16, 4 for fp32) == 0.
 *   1 <= B <= 4: two kernels, y = x U_r, then the rest of the step, chained so that the second
 *   stages its V_r rows while the first runs (for layers with h <= 256 x the SM count whose V_r rows,
 *   tokens and a few weight rows fit in shared memory; other shapes take one launch where
 *   csffn_cats_ffn_forward would).  Other shapes and B > 4 return CSFFN_ERR_UNSUPPORTED_SHAPE (use
 *   csffn_predict_lowrank, then csffn_cats_ffn_forward on the predicted set).  The
 *   mask and a_val are bit-for-bit repeatable; out may differ from launch to launch in the last
 *   bits (the CTAs' partial outputs meet in L2 in arrival order).  ws sized by
 *   csffn_workspace_size(layer, B, rank).  B == 0: writes *count = 0. */
csffn_status csffn_svd_ffn_forward(const csffn_layer* layer, const void* x, int B, int rank, const void* u_rt,
                                   const void* v_r, const float* tau, float t, int32_t* idx, int32_t* count,
                                   float* a_val, void* out, int out_mode, void* ws, size_t ws_bytes, void* stream);

/* The same step with the parallel pipeline ([SVDP] Table 3, "Parallel pipeline"; Table 2, "r=1024
 * parallel"): W_up is read with W_gate for every predicted neuron, so the up projection does not
 * wait for the gate's decision; the down projection still reads only the kept rows.  The outputs
 * are those of csffn_svd_ffn_forward (v is zero outside the kept set either way); the difference is
 * which rows are read.  Runs for the two-kernel shapes above (1 <= B <= 4); other shapes return
 * CSFFN_ERR_UNSUPPORTED_SHAPE. */
csffn_status csffn_svd_ffn_forward_parallel(const csffn_layer* layer, const void* x, int B, int rank,
                                            const void* u_rt, const void* v_r, const float* tau, float t,
                                            int32_t* idx, int32_t* count, float* a_val, void* out, int out_mode,
                                            void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes for csffn_calibrate_threshold with n calibration vectors. */
size_t csffn_calibrate_workspace_size(const csffn_layer* layer, int n, int mode, int rank);

/* Offline threshold calibration.  [CATS] abstract (contextually-aware threshold);
 * [SVDP] Fig. 1, Table 3 ("bias calibration").
 *   GLOBAL_ABS_ACT: M = n*h values |act(z)| over x_cal [n, d]; k = ceil(s*M) with s
 *     taken as this float and the product evaluated exactly; *t_out = v_(k)
 *     (k-th smallest, 1-indexed), or 0 when k == 0.
 *   PER_NEURON_PRED: p as in csffn_predict_lowrank for each calibration vector;
 *     k = ceil(s*n); t_out[i] = k-th smallest of {p_i(x_n)} (t_out is [h]), or
 *     -inf when k == 0.
 *   PER_NEURON_RECALL: s is the target recall R.  p as above and z = x.W_gate[i] + beta_i for
 *     each calibration vector; with A_i = {n : z_i(x_n) > 0}, m_i = |A_i| and c_i = ceil(R*m_i)
 *     (exact), t_out[i] = the largest float below the c_i-th largest of {p_i(x_n) : n in A_i}, so
 *     that p_i > t_out[i] predicts at least c_i of them; +inf when c_i == 0 (never predicted).
 *     Needs w_gate (and gate_bias when the layer has one).
 *   1 <= n <= CSFFN_MAX_CALIB, 0 <= s <= 1. */
csffn_status csffn_calibrate_threshold(const csffn_layer* layer, const void* x_cal, int n,
                                       float target_sparsity, int mode,
                                       const void* u_rt, const void* v_r, int rank,
                                       float* t_out, void* ws, size_t ws_bytes, void* stream);

/* Exact k-th smallest (1 <= k <= n) of n finite fp32 values by radix selection on
 * their order-preserving bit keys; *out receives the selected value bit-exactly.
 * Building block of GLOBAL_ABS_ACT calibration.  ws: csffn_kth_workspace_size(). */
size_t csffn_kth_workspace_size(void);
csffn_status csffn_kth_smallest(const float* values, int64_t n, int64_t k, float* out,
                                void* ws, size_t ws_bytes, void* stream);

/* RMSNorm with unit gain, rounded to bf16: xn[b,:] = bf16(h[b,:] / sqrt(mean(h[b,:]^2) + eps)).
 * h: fp32 [B, d]; xn: bf16 [B, d].  The input step of each block of an FFN stack
 * (h <- h + FFN(RMSNorm(h)) with out_mode ACCUMULATE). */
csffn_status csffn_rmsnorm_bf16(const float* h, int B, int d, float eps, void* xn, void* stream);

/* Failure-detection self-test: launches one tiny kernel that waits, with the same
 * bounded wait the look-back compaction uses, on a workspace flag that nothing
 * sets.  After `spin_limit` polls it records CSFFN_ERR_TIMEOUT in the workspace
 * error word and returns; csffn_check_status then reports it.  The context stays
 * usable.  Run csffn_workspace_init afterwards. */
csffn_status csffn_selftest_timeout(void* ws, size_t ws_bytes, int spin_limit, void* stream);

/* Allocation-free variant of csffn_sparse_ffn_forward.  The pages have no counterpart: this is a
 * deployment convenience of this library.
 *   For callers that cannot allocate device memory at all, and so cannot create the workspace the
 *   other entry points take: custom operators or plugins hosted by a framework that owns every
 *   device allocation, and latency-critical loops that must not allocate after start-up.  The
 *   caller still owns x, idx, count, a_val and out; the scratch of the gathered up/down projection
 *   is a library-owned device array of CSFFN_STATIC_SCRATCH_BYTES, held by every GPU that loads
 *   the library until the process exits.
 *   Computes exactly what csffn_sparse_ffn_forward computes, with the same kernels.
 *   Size limit: B*h*4 + 64*B*d*4 + 512 bytes (each term rounded up to 256) must fit in
 *   CSFFN_STATIC_SCRATCH_BYTES, e.g. B <= 4 at d = 4096 and B <= 2 at d = 8192; larger calls
 *   return CSFFN_ERR_UNSUPPORTED_SHAPE and launch nothing.
 *   All calls share the one array: calls that overlap on the GPU (other streams, other host
 *   threads) race, so order them on one stream.  The reduction counters are cleared on `stream`
 *   before each launch; the rest of the array is fully rewritten before it is read.
 *   The first call on each device looks up the array's device address (cudaGetSymbolAddress with
 *   that device current); make that first call before any stream capture that includes it.  The
 *   address is kept per device and CUDA context, so after a device reset the next call (again
 *   outside a capture) looks it up anew.
 *   Other arguments, layouts and errors as csffn_sparse_ffn_forward. */
#define CSFFN_STATIC_SCRATCH_BYTES (8u << 20)
csffn_status csffn_sparse_ffn_forward_static(const csffn_layer* layer, const void* x, int B,
                                             const int32_t* idx, const int32_t* count, const float* a_val,
                                             void* out, int out_mode, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CSFFN_H */
