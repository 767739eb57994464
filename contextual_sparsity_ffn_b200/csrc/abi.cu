// C entry points of libcsffn: argument validation, workspace carving and kernel dispatch.
// Every step of the decode path runs in this library's kernels; nothing here touches the data.
#include <cmath>
#include <cstring>

#include "common.cuh"
#include "kernels.h"

using namespace csffn;

namespace {

constexpr size_t kMaxDynSmem = 200 * 1024;  // shared memory budget for staged token vectors

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }
inline int vec_elems(int wdtype) { return wdtype == CSFFN_BF16 ? 8 : 4; }
inline size_t esize(int wdtype) { return wdtype == CSFFN_BF16 ? 2 : 4; }
inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }
inline csffn_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CSFFN_OK : CSFFN_ERR_CUDA; }

csffn_status check_layer_shape(const csffn_layer* L) {
  if (!L) return CSFFN_ERR_INVALID_ARG;
  if (L->wdtype != CSFFN_BF16 && L->wdtype != CSFFN_F32) return CSFFN_ERR_INVALID_ARG;
  if (L->act != CSFFN_ACT_SILU && L->act != CSFFN_ACT_RELU) return CSFFN_ERR_INVALID_ARG;
  if (L->d < 8 || L->d > CSFFN_MAX_D || L->h < 1 || L->h > CSFFN_MAX_H) return CSFFN_ERR_UNSUPPORTED_SHAPE;
  if (L->d % vec_elems(L->wdtype) != 0) return CSFFN_ERR_ALIGNMENT;
  if (L->gate_bias && ((uintptr_t)L->gate_bias & 3u)) return CSFFN_ERR_ALIGNMENT;
  return CSFFN_OK;
}

csffn_status check_weights(const csffn_layer* L, bool gate, bool up, bool down) {
  if ((gate && !L->w_gate) || (up && !L->w_up) || (down && !L->w_down_t)) return CSFFN_ERR_INVALID_ARG;
  if ((gate && !aligned16(L->w_gate)) || (up && !aligned16(L->w_up)) || (down && !aligned16(L->w_down_t)))
    return CSFFN_ERR_ALIGNMENT;
  return CSFFN_OK;
}

csffn_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws || ws_bytes < need || !aligned16(ws)) return CSFFN_ERR_WORKSPACE;
  return CSFFN_OK;
}

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(reinterpret_cast<char*>(ws) + off); }

// k = ceil(s * m) for a float s in [0, 1], evaluated exactly: s = mant * 2^(e - 24).
long long exact_rank(float s, long long m) {
  if (!(s > 0.f)) return 0;
  int e = 0;
  const double f = std::frexp((double)s, &e);  // s = f * 2^e, f in [0.5, 1)
  const unsigned long long mant = (unsigned long long)std::ldexp(f, 24);  // exact: s has 24 bits
  const int sh = 24 - e;  // s = mant / 2^sh, sh >= 24 for s <= 1
  const unsigned __int128 prod = (unsigned __int128)mant * (unsigned long long)m;
  unsigned __int128 k;
  if (sh <= 0) {
    k = prod << (-sh);
  } else if (sh >= 127) {
    k = prod ? 1 : 0;
  } else {
    k = (prod + (((unsigned __int128)1 << sh) - 1)) >> sh;
  }
  if (k > (unsigned __int128)m) k = m;
  return (long long)k;
}

}  // namespace

extern "C" {

int csffn_version(void) { return CSFFN_VERSION; }

const char* csffn_status_string(int status) {
  switch (status) {
    case CSFFN_OK: return "ok";
    case CSFFN_ERR_INVALID_ARG: return "invalid argument";
    case CSFFN_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case CSFFN_ERR_ALIGNMENT: return "misaligned size or pointer";
    case CSFFN_ERR_WORKSPACE: return "workspace missing or too small";
    case CSFFN_ERR_CUDA: return "CUDA error";
    case CSFFN_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

size_t csffn_workspace_size(const csffn_layer* layer, int max_batch, int max_rank) {
  if (check_layer_shape(layer) != CSFFN_OK) return 0;
  if (max_batch < 1 || max_batch > CSFFN_MAX_BATCH || max_rank < 0 || max_rank > CSFFN_MAX_RANK) return 0;
  return ws_layout(layer->d, layer->h, max_batch, max_rank).total;
}

csffn_status csffn_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < 1024 || !aligned16(ws)) return CSFFN_ERR_WORKSPACE;
  // Zero the whole control region: counters, error word and look-back status words.  Its end
  // depends on h, which is not known here, so clear the smaller of the buffer and a bound that
  // covers every h the library accepts at the smallest scratch size.
  const size_t bound = ws_layout(8, CSFFN_MAX_H, 1, 0).control_end;
  const size_t n = ws_bytes < bound ? ws_bytes : bound;
  return cuda_status(cudaMemsetAsync(ws, 0, n, as_stream(stream)));
}

csffn_status csffn_check_status(void* ws, void* stream) {
  if (!ws) return CSFFN_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  uint32_t err = 0;
  const WsLayout L = ws_layout(8, 1, 1, 0);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return CSFFN_ERR_CUDA;
  e = cudaMemcpyAsync(&err, at<uint32_t>(ws, L.err), sizeof(err), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return CSFFN_ERR_CUDA;
  if (err) {
    e = cudaMemsetAsync(at<uint32_t>(ws, L.err), 0, sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return CSFFN_ERR_CUDA;
    return CSFFN_ERR_TIMEOUT;
  }
  return CSFFN_OK;
}

csffn_status csffn_gate_mask(const csffn_layer* layer, const void* x, int B, float t,
                             const int32_t* cand_idx, const int32_t* cand_count,
                             int32_t* idx, int32_t* count, float* a_val,
                             void* ws, size_t ws_bytes, void* stream) {
  csffn_status st = check_layer_shape(layer);
  if (st != CSFFN_OK) return st;
  if (B < 0 || B > CSFFN_MAX_BATCH) return CSFFN_ERR_INVALID_ARG;
  if (!count) return CSFFN_ERR_INVALID_ARG;
  if (B == 0) return cuda_status(cudaMemsetAsync(count, 0, sizeof(int32_t), as_stream(stream)));
  if (!x || !idx || !a_val || (cand_idx == nullptr) != (cand_count == nullptr) || std::isnan(t))
    return CSFFN_ERR_INVALID_ARG;
  if ((st = check_weights(layer, true, false, false)) != CSFFN_OK) return st;
  if (!aligned16(x)) return CSFFN_ERR_ALIGNMENT;
  if ((size_t)batch_tier(B) * layer->d * esize(layer->wdtype) > kMaxDynSmem) return CSFFN_ERR_UNSUPPORTED_SHAPE;
  const WsLayout L = ws_layout(layer->d, layer->h, B, 0);
  if ((st = check_ws(ws, ws_bytes, L.control_end)) != CSFFN_OK) return st;

  GateArgs a{};
  a.W = layer->w_gate;
  a.x = x;
  a.K = layer->d;
  a.h = layer->h;
  a.B = B;
  a.bias = layer->gate_bias;
  a.t = t;
  a.tau = nullptr;
  a.act = layer->act;
  a.cand_idx = cand_idx;
  a.cand_count = cand_count;
  a.idx = idx;
  a.count = count;
  a.a_val = a_val;
  a.ctl = at<Control>(ws, L.ctl) + kCtlGate;
  a.status = at<uint64_t>(ws, L.status) + (size_t)kCtlGate * L.max_chunks;
  a.err = at<uint32_t>(ws, L.err);
  return cuda_status(launch_gate(a, layer->wdtype, false, kModeCats, as_stream(stream)));
}

csffn_status csffn_sparse_ffn_forward(const csffn_layer* layer, const void* x, int B,
                                      const int32_t* idx, const int32_t* count, const float* a_val,
                                      void* out, int out_mode, void* ws, size_t ws_bytes, void* stream) {
  csffn_status st = check_layer_shape(layer);
  if (st != CSFFN_OK) return st;
  if (B < 0 || B > CSFFN_MAX_BATCH) return CSFFN_ERR_INVALID_ARG;
  if (out_mode != CSFFN_OUT_BF16 && out_mode != CSFFN_OUT_F32 && out_mode != CSFFN_OUT_F32_ACCUMULATE)
    return CSFFN_ERR_INVALID_ARG;
  if (B == 0) return CSFFN_OK;
  if (!x || !idx || !count || !a_val || !out) return CSFFN_ERR_INVALID_ARG;
  if ((st = check_weights(layer, false, true, true)) != CSFFN_OK) return st;
  if (!aligned16(x) || !aligned16(out)) return CSFFN_ERR_ALIGNMENT;
  if ((size_t)batch_tier(B) * layer->d * esize(layer->wdtype) > kMaxDynSmem) return CSFFN_ERR_UNSUPPORTED_SHAPE;
  const WsLayout L = ws_layout(layer->d, layer->h, B, 0);
  if ((st = check_ws(ws, ws_bytes, L.ybuf)) != CSFFN_OK) return st;
  cudaStream_t s = as_stream(stream);

  UpArgs u{};
  u.W_up = layer->w_up;
  u.x = x;
  u.d = layer->d;
  u.h = layer->h;
  u.B = B;
  u.idx = idx;
  u.count = count;
  u.a_val = a_val;
  u.v = at<float>(ws, L.vbuf);
  u.err = at<uint32_t>(ws, L.err);
  cudaError_t e = launch_up(u, layer->wdtype, s);
  if (e != cudaSuccess) return CSFFN_ERR_CUDA;

  DownArgs dn{};
  dn.W_down_t = layer->w_down_t;
  dn.d = layer->d;
  dn.h = layer->h;
  dn.B = B;
  dn.idx = idx;
  dn.count = count;
  dn.n_host = 0;
  dn.v = u.v;
  dn.partial = at<float>(ws, L.partial);
  dn.slice_ctr = at<uint32_t>(ws, L.slice_ctr);
  dn.out = out;
  dn.out_mode = out_mode;
  dn.err = at<uint32_t>(ws, L.err);
  return cuda_status(launch_down(dn, layer->wdtype, s));
}

namespace {

// Arguments of the tensor-core FFN (tc_ffn.cu) for this layer, tokens and workspace.
TcArgs tc_args(const csffn_layer* layer, const void* x, int B, const WsLayout& L, void* ws) {
  TcArgs a{};
  a.W_gate = layer->w_gate;
  a.W_up = layer->w_up;
  a.W_down_t = layer->w_down_t;
  a.x = x;
  a.d = layer->d;
  a.h = layer->h;
  a.B = B;
  a.bias = layer->gate_bias;
  a.act = layer->act;
  a.v = at<uint16_t>(ws, L.vbuf);
  a.afull = at<float>(ws, L.afull);
  a.flags = at<uint8_t>(ws, L.flags);
  a.part = at<float>(ws, L.tcpart);
  a.ctr = at<uint32_t>(ws, L.tcctr);
  a.err = at<uint32_t>(ws, L.err);
  return a;
}

// Every check of a CATS step with 1 <= B <= CSFFN_MAX_BATCH, whichever path runs it (the one-launch
// kernel, or the gate mask then the gathered up/down), so that a rejected call launches nothing.
csffn_status check_cats_step(const csffn_layer* layer, const void* x, int B, float t, const int32_t* idx,
                             const float* a_val, const void* out, void* ws, size_t ws_bytes) {
  if (!x || !idx || !a_val || !out || std::isnan(t)) return CSFFN_ERR_INVALID_ARG;
  csffn_status st = check_weights(layer, true, true, true);
  if (st != CSFFN_OK) return st;
  if (!aligned16(x) || !aligned16(out)) return CSFFN_ERR_ALIGNMENT;
  if (!cats_ring_supported(layer->d, B, layer->wdtype) && !cats_fused_supported(layer->d, B, layer->wdtype) &&
      !tc_ffn_supported(layer->d, layer->h, B, layer->wdtype) &&
      (size_t)batch_tier(B) * layer->d * esize(layer->wdtype) > kMaxDynSmem)
    return CSFFN_ERR_UNSUPPORTED_SHAPE;
  return check_ws(ws, ws_bytes, ws_layout(layer->d, layer->h, B, 0).ybuf);
}

}  // namespace

csffn_status csffn_cats_ffn_forward(const csffn_layer* layer, const void* x, int B, float t,
                                    const int32_t* cand_idx, const int32_t* cand_count,
                                    int32_t* idx, int32_t* count, float* a_val,
                                    void* out, int out_mode, void* ws, size_t ws_bytes, void* stream) {
  csffn_status st = check_layer_shape(layer);
  if (st != CSFFN_OK) return st;
  if (B < 0 || B > CSFFN_MAX_BATCH) return CSFFN_ERR_INVALID_ARG;
  if (out_mode != CSFFN_OUT_BF16 && out_mode != CSFFN_OUT_F32 && out_mode != CSFFN_OUT_F32_ACCUMULATE)
    return CSFFN_ERR_INVALID_ARG;
  if (!count) return CSFFN_ERR_INVALID_ARG;
  if ((cand_idx == nullptr) != (cand_count == nullptr)) return CSFFN_ERR_INVALID_ARG;
  if (B == 0) return cuda_status(cudaMemsetAsync(count, 0, sizeof(int32_t), as_stream(stream)));
  if ((st = check_cats_step(layer, x, B, t, idx, a_val, out, ws, ws_bytes)) != CSFFN_OK) return st;
  // From three tokens on, the union of the tokens' masks covers most neurons (about 1 - s^B of them
  // at sparsity s), so every row is read once by the tensor cores with the rejected activations
  // zeroed; that takes no longer than the streaming step even at 90% sparsity.
  const bool tc = !cand_idx && tc_ffn_supported(layer->d, layer->h, B, layer->wdtype);
  const bool ring = cats_ring_supported(layer->d, B, layer->wdtype) && !(tc && batch_tier(B) >= 4);
  if (!ring && tc) {
    const WsLayout L = ws_layout(layer->d, layer->h, B, 0);
    TcArgs a = tc_args(layer, x, B, L, ws);
    a.masked = 1;
    a.t = t;
    a.idx = idx;
    a.count = count;
    a.a_val = a_val;
    a.out = out;
    a.out_mode = out_mode;
    return cuda_status(launch_tc_ffn(a, as_stream(stream)));
  }
  if (!ring && !cats_fused_supported(layer->d, B, layer->wdtype)) {
    st = csffn_gate_mask(layer, x, B, t, cand_idx, cand_count, idx, count, a_val, ws, ws_bytes, stream);
    if (st != CSFFN_OK) return st;
    return csffn_sparse_ffn_forward(layer, x, B, idx, count, a_val, out, out_mode, ws, ws_bytes, stream);
  }
  const WsLayout L = ws_layout(layer->d, layer->h, B, 0);
  FusedArgs a{};
  a.W_gate = layer->w_gate;
  a.W_up = layer->w_up;
  a.W_down_t = layer->w_down_t;
  a.x = x;
  a.d = layer->d;
  a.h = layer->h;
  a.B = B;
  a.bias = layer->gate_bias;
  a.t = t;
  a.act = layer->act;
  a.cand_idx = cand_idx;
  a.cand_count = cand_count;
  a.afull = at<float>(ws, L.afull);
  a.flags = at<uint8_t>(ws, L.flags);
  a.facc = at<float>(ws, L.facc);
  a.ctl = reinterpret_cast<uint32_t*>(at<Control>(ws, L.ctl) + kCtlFused);
  a.tickets = at<uint32_t>(ws, L.tickets);
  a.err = at<uint32_t>(ws, L.err);
  a.idx = idx;
  a.count = count;
  a.a_val = a_val;
  a.out = out;
  a.out_mode = out_mode;
  return cuda_status(ring ? launch_cats_ring(a, layer->wdtype, as_stream(stream))
                          : launch_cats_fused(a, layer->wdtype, as_stream(stream)));
}

namespace {

csffn_status svd_forward(const csffn_layer* layer, const void* x, int B, int rank, const void* u_rt, const void* v_r,
                         const float* tau, float t, bool parallel, int32_t* idx, int32_t* count, float* a_val,
                         void* out, int out_mode, void* ws, size_t ws_bytes, void* stream) {
  csffn_status st = check_layer_shape(layer);
  if (st != CSFFN_OK) return st;
  if (B < 0 || B > CSFFN_MAX_BATCH) return CSFFN_ERR_INVALID_ARG;
  if (out_mode != CSFFN_OUT_BF16 && out_mode != CSFFN_OUT_F32 && out_mode != CSFFN_OUT_F32_ACCUMULATE)
    return CSFFN_ERR_INVALID_ARG;
  if (!count) return CSFFN_ERR_INVALID_ARG;
  if (B == 0) return cuda_status(cudaMemsetAsync(count, 0, sizeof(int32_t), as_stream(stream)));
  if (!x || !u_rt || !v_r || !tau || !idx || !a_val || !out || std::isnan(t)) return CSFFN_ERR_INVALID_ARG;
  if (rank < 1 || rank > CSFFN_MAX_RANK) return CSFFN_ERR_INVALID_ARG;
  if (rank % vec_elems(layer->wdtype) != 0) return CSFFN_ERR_ALIGNMENT;
  if ((st = check_weights(layer, true, true, true)) != CSFFN_OK) return st;
  if (!aligned16(x) || !aligned16(out) || !aligned16(u_rt) || !aligned16(v_r)) return CSFFN_ERR_ALIGNMENT;
  const bool two = svd_step_supported(layer->d, layer->h, B, layer->wdtype, rank);
  if (!two && (parallel || !cats_fused_supported(layer->d, B, layer->wdtype, rank)))
    return CSFFN_ERR_UNSUPPORTED_SHAPE;
  const WsLayout L = ws_layout(layer->d, layer->h, B, rank);
  if ((st = check_ws(ws, ws_bytes, L.hx)) != CSFFN_OK) return st;
  FusedArgs a{};
  a.W_gate = layer->w_gate;
  a.W_up = layer->w_up;
  a.W_down_t = layer->w_down_t;
  a.x = x;
  a.d = layer->d;
  a.h = layer->h;
  a.B = B;
  a.bias = layer->gate_bias;
  a.t = t;
  a.act = layer->act;
  a.u_rt = u_rt;
  a.v_r = v_r;
  a.tau = tau;
  a.rank = rank;
  a.ybuf = at<float>(ws, L.ybuf);
  a.afull = at<float>(ws, L.afull);
  a.flags = at<uint8_t>(ws, L.flags);
  a.facc = at<float>(ws, L.facc);
  a.ctl = reinterpret_cast<uint32_t*>(at<Control>(ws, L.ctl) + kCtlFused);
  a.tickets = at<uint32_t>(ws, L.tickets);
  a.svd_counts = at<uint32_t>(ws, L.svdcnt);
  a.err = at<uint32_t>(ws, L.err);
  a.idx = idx;
  a.count = count;
  a.a_val = a_val;
  a.out = out;
  a.out_mode = out_mode;
  if (two) return cuda_status(launch_svd_step(a, layer->wdtype, parallel, as_stream(stream)));
  return cuda_status(launch_cats_fused(a, layer->wdtype, as_stream(stream)));
}

}  // namespace

csffn_status csffn_svd_ffn_forward(const csffn_layer* layer, const void* x, int B, int rank, const void* u_rt,
                                   const void* v_r, const float* tau, float t, int32_t* idx, int32_t* count,
                                   float* a_val, void* out, int out_mode, void* ws, size_t ws_bytes, void* stream) {
  return svd_forward(layer, x, B, rank, u_rt, v_r, tau, t, false, idx, count, a_val, out, out_mode, ws, ws_bytes,
                     stream);
}

csffn_status csffn_svd_ffn_forward_parallel(const csffn_layer* layer, const void* x, int B, int rank,
                                            const void* u_rt, const void* v_r, const float* tau, float t,
                                            int32_t* idx, int32_t* count, float* a_val, void* out, int out_mode,
                                            void* ws, size_t ws_bytes, void* stream) {
  return svd_forward(layer, x, B, rank, u_rt, v_r, tau, t, true, idx, count, a_val, out, out_mode, ws, ws_bytes,
                     stream);
}

// The device address of page-locked host memory mapped into the current device's address space
// (cudaHostAlloc / cudaMallocHost / cudaHostRegister with unified addressing), or nullptr for any
// other pointer (pageable memory included).
static void* mapped_host_ptr(const void* p) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

csffn_status csffn_cats_ffn_forward_host(const csffn_layer* layer, const void* x_host, int B, float t,
                                         int32_t* idx, int32_t* count, float* a_val,
                                         void* out_host, int out_mode, void* ws, size_t ws_bytes, void* stream) {
  csffn_status st = check_layer_shape(layer);
  if (st != CSFFN_OK) return st;
  if (B < 0 || B > CSFFN_MAX_BATCH) return CSFFN_ERR_INVALID_ARG;
  if (out_mode != CSFFN_OUT_BF16 && out_mode != CSFFN_OUT_F32) return CSFFN_ERR_INVALID_ARG;
  if (!count) return CSFFN_ERR_INVALID_ARG;
  if (B == 0) return cuda_status(cudaMemsetAsync(count, 0, sizeof(int32_t), as_stream(stream)));
  if (!x_host || !out_host) return CSFFN_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(layer->d, layer->h, B, 0);
  if ((st = check_ws(ws, ws_bytes, L.total)) != CSFFN_OK) return st;
  cudaStream_t s = as_stream(stream);
  void* xd = at<char>(ws, L.hx);
  void* od = at<char>(ws, L.hout);
  // the step's own checks, on the staging buffers, before the first copy is issued
  if ((st = check_cats_step(layer, xd, B, t, idx, a_val, od, ws, ws_bytes)) != CSFFN_OK) return st;
  const size_t xbytes = (size_t)B * layer->d * esize(layer->wdtype);
  const size_t obytes = (size_t)B * layer->d * (out_mode == CSFFN_OUT_BF16 ? 2 : 4);
  // Mapped page-locked buffers: a kernel stages the tokens into the workspace over the host link and
  // the step writes out there directly, so the stream holds only kernels (a step may then start
  // while the previous one ends).
  void* xm = mapped_host_ptr(x_host);
  void* om = xm ? mapped_host_ptr(out_host) : nullptr;
  if (xm && om && aligned16(xm) && aligned16(om)) {
    if (launch_stage_tokens(xm, xd, xbytes, s) != cudaSuccess) return CSFFN_ERR_CUDA;
    return csffn_cats_ffn_forward(layer, xd, B, t, nullptr, nullptr, idx, count, a_val, om, out_mode, ws, ws_bytes,
                                  stream);
  }
  if (cudaMemcpyAsync(xd, x_host, xbytes, cudaMemcpyHostToDevice, s) != cudaSuccess) return CSFFN_ERR_CUDA;
  st = csffn_cats_ffn_forward(layer, xd, B, t, nullptr, nullptr, idx, count, a_val, od, out_mode, ws, ws_bytes,
                              stream);
  if (st != CSFFN_OK) return st;
  return cuda_status(cudaMemcpyAsync(out_host, od, obytes, cudaMemcpyDeviceToHost, s));
}

csffn_status csffn_dense_ffn_forward(const csffn_layer* layer, const void* x, int B,
                                     void* out, int out_mode, void* ws, size_t ws_bytes, void* stream) {
  csffn_status st = check_layer_shape(layer);
  if (st != CSFFN_OK) return st;
  if (B < 0 || B > CSFFN_MAX_BATCH) return CSFFN_ERR_INVALID_ARG;
  if (out_mode != CSFFN_OUT_BF16 && out_mode != CSFFN_OUT_F32 && out_mode != CSFFN_OUT_F32_ACCUMULATE)
    return CSFFN_ERR_INVALID_ARG;
  if (B == 0) return CSFFN_OK;
  if (!x || !out) return CSFFN_ERR_INVALID_ARG;
  if ((st = check_weights(layer, true, true, true)) != CSFFN_OK) return st;
  if (!aligned16(x) || !aligned16(out)) return CSFFN_ERR_ALIGNMENT;
  const WsLayout L = ws_layout(layer->d, layer->h, B, 0);
  if ((st = check_ws(ws, ws_bytes, L.ybuf)) != CSFFN_OK) return st;
  cudaStream_t s = as_stream(stream);

  if (tc_ffn_supported(layer->d, layer->h, B, layer->wdtype)) {  // fifth-generation tensor cores
    TcArgs a = tc_args(layer, x, B, L, ws);
    a.out = out;
    a.out_mode = out_mode;
    return cuda_status(launch_tc_ffn(a, s));
  }
  if (dense_mma_supported(layer->d, layer->h, B, layer->wdtype)) {  // tensor cores, one pass
    DenseGateUpArgs g{};
    g.W_gate = layer->w_gate;
    g.W_up = layer->w_up;
    g.x = x;
    g.d = layer->d;
    g.h = layer->h;
    g.B = B;
    g.bias = layer->gate_bias;
    g.act = layer->act;
    g.v = at<float>(ws, L.vbuf);
    cudaError_t e = launch_dense_gate_up_mma(g, s);
    if (e != cudaSuccess) return CSFFN_ERR_CUDA;
    DownArgs dn{};
    dn.W_down_t = layer->w_down_t;
    dn.d = layer->d;
    dn.h = layer->h;
    dn.B = B;
    dn.n_host = layer->h;
    dn.v = g.v;
    dn.partial = at<float>(ws, L.partial);
    dn.slice_ctr = at<uint32_t>(ws, L.slice_ctr) + kMaxSlices;
    dn.out = out;
    dn.out_mode = out_mode;
    dn.err = at<uint32_t>(ws, L.err);
    return cuda_status(launch_down_mma(dn, partial_rows(B) / B, s));
  }

  // Token groups small enough to stage in shared memory (the whole batch when it fits).
  int group = B;
  while (group > 1 && (size_t)batch_tier(group) * layer->d * esize(layer->wdtype) > kMaxDynSmem) group = (group + 1) / 2;
  if ((size_t)batch_tier(group) * layer->d * esize(layer->wdtype) > kMaxDynSmem) return CSFFN_ERR_UNSUPPORTED_SHAPE;
  float* v = at<float>(ws, L.vbuf);
  for (int b0 = 0; b0 < B; b0 += group) {
    DenseGateUpArgs g{};
    g.W_gate = layer->w_gate;
    g.W_up = layer->w_up;
    g.x = reinterpret_cast<const char*>(x) + (size_t)b0 * layer->d * esize(layer->wdtype);
    g.d = layer->d;
    g.h = layer->h;
    g.B = (B - b0) < group ? (B - b0) : group;
    g.bias = layer->gate_bias;
    g.act = layer->act;
    g.v = v + (size_t)b0 * layer->h;
    cudaError_t e = launch_dense_gate_up(g, layer->wdtype, s);
    if (e != cudaSuccess) return CSFFN_ERR_CUDA;
  }
  DownArgs dn{};
  dn.W_down_t = layer->w_down_t;
  dn.d = layer->d;
  dn.h = layer->h;
  dn.B = B;
  dn.idx = nullptr;
  dn.count = nullptr;
  dn.n_host = layer->h;
  dn.v = v;
  dn.partial = at<float>(ws, L.partial);
  dn.slice_ctr = at<uint32_t>(ws, L.slice_ctr) + kMaxSlices;
  dn.out = out;
  dn.out_mode = out_mode;
  dn.err = at<uint32_t>(ws, L.err);
  return cuda_status(launch_down(dn, layer->wdtype, s));
}

csffn_status csffn_predict_lowrank(const csffn_layer* layer, const void* x, int B, int rank,
                                   const void* u_rt, const void* v_r, const float* tau,
                                   int32_t* cand_idx, int32_t* cand_count,
                                   void* ws, size_t ws_bytes, void* stream) {
  csffn_status st = check_layer_shape(layer);
  if (st != CSFFN_OK) return st;
  if (B < 0 || B > CSFFN_MAX_BATCH) return CSFFN_ERR_INVALID_ARG;
  if (!cand_count) return CSFFN_ERR_INVALID_ARG;
  if (B == 0) return cuda_status(cudaMemsetAsync(cand_count, 0, sizeof(int32_t), as_stream(stream)));
  if (!x || !u_rt || !v_r || !tau || !cand_idx) return CSFFN_ERR_INVALID_ARG;
  if (rank < 1 || rank > CSFFN_MAX_RANK) return CSFFN_ERR_INVALID_ARG;
  if (rank % vec_elems(layer->wdtype) != 0) return CSFFN_ERR_ALIGNMENT;
  if (!aligned16(x) || !aligned16(u_rt) || !aligned16(v_r)) return CSFFN_ERR_ALIGNMENT;
  if ((size_t)batch_tier(B) * layer->d * esize(layer->wdtype) > kMaxDynSmem ||
      (size_t)batch_tier(B) * rank * sizeof(float) > kMaxDynSmem)
    return CSFFN_ERR_UNSUPPORTED_SHAPE;
  const WsLayout L = ws_layout(layer->d, layer->h, B, rank);
  if ((st = check_ws(ws, ws_bytes, L.total)) != CSFFN_OK) return st;
  cudaStream_t s = as_stream(stream);

  RowGemvArgs g{};
  g.W = u_rt;
  g.x = x;
  g.rows = rank;
  g.K = layer->d;
  g.B = B;
  g.y = at<float>(ws, L.ybuf);
  g.y_stride = rank;
  g.bias = nullptr;
  g.act = -1;
  cudaError_t e = launch_row_gemv(g, layer->wdtype, false, s);
  if (e != cudaSuccess) return CSFFN_ERR_CUDA;

  GateArgs a{};
  a.W = v_r;
  a.x = g.y;
  a.K = rank;
  a.h = layer->h;
  a.B = B;
  a.bias = layer->gate_bias;
  a.tau = tau;
  a.act = layer->act;
  a.idx = cand_idx;
  a.count = cand_count;
  a.ctl = at<Control>(ws, L.ctl) + kCtlPred;
  a.status = at<uint64_t>(ws, L.status) + (size_t)kCtlPred * L.max_chunks;
  a.err = at<uint32_t>(ws, L.err);
  return cuda_status(launch_gate(a, layer->wdtype, layer->wdtype == CSFFN_BF16, kModePred, s));
}

// Calibration workspace: [header 512 B, error word at the decode layout's offset][kth state]
// [values n*h, or P^T h*n][y n*rank]
namespace {
constexpr size_t kHeaderBytes = 512;
struct CalLayout {
  size_t kth, values, y, zt, total;
};
CalLayout cal_layout(const csffn_layer* L, int n, int mode, int rank) {
  CalLayout c;
  const bool pred = mode == CSFFN_CAL_PER_NEURON_PRED || mode == CSFFN_CAL_PER_NEURON_RECALL;
  size_t o = kHeaderBytes;
  c.kth = o;    o += kth_state_bytes();
  c.values = o; o += align_up(sizeof(float) * (size_t)n * L->h, 256);
  c.y = o;      o += pred ? align_up(sizeof(float) * (size_t)n * rank, 256) : 0;
  c.zt = o;     o += mode == CSFFN_CAL_PER_NEURON_RECALL ? align_up(sizeof(float) * (size_t)n * L->h, 256) : 0;
  c.total = o;
  return c;
}

bool cal_mode_ok(int mode) {
  return mode == CSFFN_CAL_GLOBAL_ABS_ACT || mode == CSFFN_CAL_PER_NEURON_PRED || mode == CSFFN_CAL_PER_NEURON_RECALL;
}
}  // namespace

size_t csffn_calibrate_workspace_size(const csffn_layer* layer, int n, int mode, int rank) {
  if (check_layer_shape(layer) != CSFFN_OK || n < 1 || n > CSFFN_MAX_CALIB) return 0;
  if (!cal_mode_ok(mode)) return 0;
  if (mode != CSFFN_CAL_GLOBAL_ABS_ACT && (rank < 1 || rank > CSFFN_MAX_RANK)) return 0;
  return cal_layout(layer, n, mode, rank).total;
}

csffn_status csffn_calibrate_threshold(const csffn_layer* layer, const void* x_cal, int n,
                                       float target_sparsity, int mode,
                                       const void* u_rt, const void* v_r, int rank,
                                       float* t_out, void* ws, size_t ws_bytes, void* stream) {
  csffn_status st = check_layer_shape(layer);
  if (st != CSFFN_OK) return st;
  if (!x_cal || !t_out || n < 1 || n > CSFFN_MAX_CALIB) return CSFFN_ERR_INVALID_ARG;
  if (!(target_sparsity >= 0.f && target_sparsity <= 1.f)) return CSFFN_ERR_INVALID_ARG;
  if (!cal_mode_ok(mode)) return CSFFN_ERR_INVALID_ARG;
  if (!aligned16(x_cal)) return CSFFN_ERR_ALIGNMENT;
  const int group_cap = CSFFN_MAX_BATCH;
  int group = group_cap;
  while (group > 1 && (size_t)batch_tier(group) * layer->d * esize(layer->wdtype) > kMaxDynSmem) group /= 2;
  cudaStream_t s = as_stream(stream);
  const size_t xrow = (size_t)layer->d * esize(layer->wdtype);

  if (mode == CSFFN_CAL_GLOBAL_ABS_ACT) {
    if ((st = check_weights(layer, true, false, false)) != CSFFN_OK) return st;
    const CalLayout C = cal_layout(layer, n, mode, 0);
    if ((st = check_ws(ws, ws_bytes, C.total)) != CSFFN_OK) return st;
    const long long M = (long long)n * layer->h;
    const long long k = exact_rank(target_sparsity, M);
    if (k == 0) return cuda_status(launch_fill(t_out, 0.f, 1, s));
    float* vals = at<float>(ws, C.values);
    for (int b0 = 0; b0 < n; b0 += group) {
      RowGemvArgs g{};
      g.W = layer->w_gate;
      g.x = reinterpret_cast<const char*>(x_cal) + (size_t)b0 * xrow;
      g.rows = layer->h;
      g.K = layer->d;
      g.B = (n - b0) < group ? (n - b0) : group;
      g.y = vals + (size_t)b0 * layer->h;
      g.y_stride = layer->h;
      g.bias = layer->gate_bias;
      g.act = layer->act;
      g.abs_out = 1;
      if (launch_row_gemv(g, layer->wdtype, false, s) != cudaSuccess) return CSFFN_ERR_CUDA;
    }
    return cuda_status(launch_kth_smallest(vals, M, k, t_out, at<void>(ws, C.kth), s));
  }

  // PER_NEURON_PRED and PER_NEURON_RECALL
  const bool recall = mode == CSFFN_CAL_PER_NEURON_RECALL;
  if (!u_rt || !v_r) return CSFFN_ERR_INVALID_ARG;
  if (rank < 1 || rank > CSFFN_MAX_RANK) return CSFFN_ERR_INVALID_ARG;
  if (rank % vec_elems(layer->wdtype) != 0) return CSFFN_ERR_ALIGNMENT;
  if (!aligned16(u_rt) || !aligned16(v_r)) return CSFFN_ERR_ALIGNMENT;
  if (recall && (st = check_weights(layer, true, false, false)) != CSFFN_OK) return st;
  const CalLayout C = cal_layout(layer, n, mode, rank);
  if ((st = check_ws(ws, ws_bytes, C.total)) != CSFFN_OK) return st;
  const long long k = exact_rank(target_sparsity, n);
  if (!recall && k == 0) return cuda_status(launch_fill(t_out, -INFINITY, layer->h, s));
  float* y = at<float>(ws, C.y);
  float* pt = at<float>(ws, C.values);  // P^T [h][n]
  int pgroup = group;
  while (pgroup > 1 && (size_t)batch_tier(pgroup) * rank * sizeof(float) > kMaxDynSmem) pgroup /= 2;
  for (int b0 = 0; b0 < n; b0 += group) {
    RowGemvArgs g{};
    g.W = u_rt;
    g.x = reinterpret_cast<const char*>(x_cal) + (size_t)b0 * xrow;
    g.rows = rank;
    g.K = layer->d;
    g.B = (n - b0) < group ? (n - b0) : group;
    g.y = y + (size_t)b0 * rank;
    g.y_stride = rank;
    g.act = -1;
    if (launch_row_gemv(g, layer->wdtype, false, s) != cudaSuccess) return CSFFN_ERR_CUDA;
  }
  for (int b0 = 0; b0 < n; b0 += pgroup) {
    RowGemvArgs g{};
    g.W = v_r;
    g.x = y + (size_t)b0 * rank;
    g.rows = layer->h;
    g.K = rank;
    g.B = (n - b0) < pgroup ? (n - b0) : pgroup;
    g.y = pt + b0;
    g.y_stride = n;
    g.bias = layer->gate_bias;
    g.act = -1;
    g.transpose_out = 1;
    if (launch_row_gemv(g, layer->wdtype, layer->wdtype == CSFFN_BF16, s) != cudaSuccess) return CSFFN_ERR_CUDA;
  }
  if (!recall) return cuda_status(launch_rows_kth(pt, layer->h, n, (int)k, t_out, s));
  float* zt = at<float>(ws, C.zt);  // Z^T [h][n]: the gate pre-activations
  for (int b0 = 0; b0 < n; b0 += group) {
    RowGemvArgs g{};
    g.W = layer->w_gate;
    g.x = reinterpret_cast<const char*>(x_cal) + (size_t)b0 * xrow;
    g.rows = layer->h;
    g.K = layer->d;
    g.B = (n - b0) < group ? (n - b0) : group;
    g.y = zt + b0;
    g.y_stride = n;
    g.bias = layer->gate_bias;
    g.act = -1;
    g.transpose_out = 1;
    if (launch_row_gemv(g, layer->wdtype, false, s) != cudaSuccess) return CSFFN_ERR_CUDA;
  }
  return cuda_status(launch_rows_recall(pt, zt, layer->h, n, target_sparsity, t_out, s));
}

size_t csffn_kth_workspace_size(void) { return kHeaderBytes + kth_state_bytes(); }

csffn_status csffn_kth_smallest(const float* values, int64_t n, int64_t k, float* out,
                                void* ws, size_t ws_bytes, void* stream) {
  if (!values || !out || n < 1 || n > 0x7FFFFFFFLL || k < 1 || k > n) return CSFFN_ERR_INVALID_ARG;
  csffn_status st = check_ws(ws, ws_bytes, csffn_kth_workspace_size());
  if (st != CSFFN_OK) return st;
  return cuda_status(launch_kth_smallest(values, n, k, out, at<void>(ws, kHeaderBytes), as_stream(stream)));
}

csffn_status csffn_rmsnorm_bf16(const float* h, int B, int d, float eps, void* xn, void* stream) {
  if (B < 0 || B > 65535 || d < 1 || d > CSFFN_MAX_D || !(eps >= 0.f)) return CSFFN_ERR_INVALID_ARG;
  if (B == 0) return CSFFN_OK;
  if (!h || !xn) return CSFFN_ERR_INVALID_ARG;
  return cuda_status(launch_rmsnorm_bf16(h, B, d, eps, xn, as_stream(stream)));
}

csffn_status csffn_selftest_timeout(void* ws, size_t ws_bytes, int spin_limit, void* stream) {
  const WsLayout L = ws_layout(8, 1, 1, 0);
  if (!ws || ws_bytes < L.control_end || !aligned16(ws)) return CSFFN_ERR_WORKSPACE;
  if (spin_limit < 1) return CSFFN_ERR_INVALID_ARG;
  // The flag is the 8-byte word after the error word, which no kernel ever writes.
  uint64_t* flag = at<uint64_t>(ws, L.err + 8);
  return cuda_status(launch_timeout_selftest(flag, at<uint32_t>(ws, L.err), spin_limit, as_stream(stream)));
}

}  // extern "C"
