// Allocation-free variant of csffn_sparse_ffn_forward.
//
// Who needs it: callers that cannot allocate device memory at all, so they cannot create the
// workspace the other entry points take.  Examples are custom operators or plugins hosted by a
// framework that owns every device allocation and forbids raw cudaMalloc, and latency-critical
// loops that must not allocate after start-up (cudaMalloc can synchronise the device and can
// fail under fragmentation).  Such a caller still owns the inputs and the output; only the
// scratch of the gathered up/down projection moves into the library.
//
// The scratch is one file-scope device array of CSFFN_STATIC_SCRATCH_BYTES.  Every GPU that
// loads libcsffn holds it until the process exits.  Every call uses the same array, so calls that
// overlap on the GPU (on different streams, or from different host threads) race; order them on
// one stream.  The array keeps the previous call's contents: the per-slice reduction counters,
// the only part that must start at zero, are cleared on the caller's stream before each launch.
//
// Host code cannot use the array's name as a device address (in host code it names a host-side
// stand-in), so the device address is looked up with cudaGetSymbolAddress, with the device
// current, on the first call made on it.  Because that first call does this set-up, it should
// come before any stream capture that includes the entry point.  The address is remembered per
// device together with the CUDA context it belongs to: after a device reset (a new context, where
// the array may sit at another address) the next call looks it up again instead of using the old
// one.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

using namespace csffn;

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[CSFFN_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
struct ScratchAddress {
  CUcontext ctx;  // the context the address was looked up in
  void* ptr;
};
ScratchAddress g_scratch[kMaxDevices] = {};

// cuCtxGetCurrent from the driver, through the runtime (no link against libcuda).
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_getter() {
  static CtxGetCurrentFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrentFn>(nullptr);
    return reinterpret_cast<CtxGetCurrentFn>(ptr);
  }();
  return fn;
}

CUcontext current_context() {
  CUcontext c = nullptr;
  CtxGetCurrentFn get = ctx_getter();
  if (!get || get(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_static_scratch on the current device: looked up once per device and
// context, with the device current.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  CUcontext ctx = current_context();
  if (g_scratch[dev].ptr == nullptr || ctx == nullptr || g_scratch[dev].ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);  // makes the device's context current if none was
    if (e != cudaSuccess) return e;
    g_scratch[dev].ptr = p;
    g_scratch[dev].ctx = current_context();
  }
  *out = g_scratch[dev].ptr;
  return cudaSuccess;
}

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" csffn_status csffn_sparse_ffn_forward_static(const csffn_layer* layer, const void* x, int B,
                                                       const int32_t* idx, const int32_t* count,
                                                       const float* a_val, void* out, int out_mode,
                                                       void* stream) {
  if (!layer) return CSFFN_ERR_INVALID_ARG;
  if (layer->wdtype != CSFFN_BF16 && layer->wdtype != CSFFN_F32) return CSFFN_ERR_INVALID_ARG;
  if (layer->act != CSFFN_ACT_SILU && layer->act != CSFFN_ACT_RELU) return CSFFN_ERR_INVALID_ARG;
  if (layer->d < 8 || layer->d > CSFFN_MAX_D || layer->h < 1 || layer->h > CSFFN_MAX_H)
    return CSFFN_ERR_UNSUPPORTED_SHAPE;
  const int epv = layer->wdtype == CSFFN_BF16 ? 8 : 4;
  const size_t es = layer->wdtype == CSFFN_BF16 ? 2 : 4;
  if (layer->d % epv != 0) return CSFFN_ERR_ALIGNMENT;
  if (B < 0 || B > CSFFN_MAX_BATCH) return CSFFN_ERR_INVALID_ARG;
  if (out_mode != CSFFN_OUT_BF16 && out_mode != CSFFN_OUT_F32 && out_mode != CSFFN_OUT_F32_ACCUMULATE)
    return CSFFN_ERR_INVALID_ARG;
  if (B == 0) return CSFFN_OK;
  if (!x || !idx || !count || !a_val || !out || !layer->w_up || !layer->w_down_t) return CSFFN_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out) || !aligned16(layer->w_up) || !aligned16(layer->w_down_t))
    return CSFFN_ERR_ALIGNMENT;
  if ((size_t)batch_tier(B) * layer->d * es > 200 * 1024) return CSFFN_ERR_UNSUPPORTED_SHAPE;

  // Carve the static array: [slice counters][v: B*h fp32][partials: row ranges * B * d fp32].
  const size_t ctr_bytes = align_up(sizeof(uint32_t) * kMaxSlices, 256);
  const size_t v_bytes = align_up(sizeof(float) * (size_t)B * layer->h, 256);
  const size_t part_bytes = align_up(sizeof(float) * (size_t)kMaxRowRanges * B * layer->d, 256);
  if (ctr_bytes + v_bytes + part_bytes > (size_t)CSFFN_STATIC_SCRATCH_BYTES) return CSFFN_ERR_UNSUPPORTED_SHAPE;

  void* base = nullptr;
  if (scratch_address(&base) != cudaSuccess) return CSFFN_ERR_CUDA;
  char* s = reinterpret_cast<char*>(base);
  uint32_t* ctr = reinterpret_cast<uint32_t*>(s);
  float* v = reinterpret_cast<float*>(s + ctr_bytes);
  float* partial = reinterpret_cast<float*>(s + ctr_bytes + v_bytes);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  if (cudaMemsetAsync(ctr, 0, ctr_bytes, st) != cudaSuccess) return CSFFN_ERR_CUDA;

  UpArgs u{};
  u.W_up = layer->w_up;
  u.x = x;
  u.d = layer->d;
  u.h = layer->h;
  u.B = B;
  u.idx = idx;
  u.count = count;
  u.a_val = a_val;
  u.v = v;
  if (launch_up_gather(u, layer->wdtype, st) != cudaSuccess) return CSFFN_ERR_CUDA;

  DownArgs dn{};
  dn.W_down_t = layer->w_down_t;
  dn.d = layer->d;
  dn.h = layer->h;
  dn.B = B;
  dn.idx = idx;
  dn.count = count;
  dn.n_host = 0;
  dn.v = v;
  dn.partial = partial;
  dn.slice_ctr = ctr;
  dn.out = out;
  dn.out_mode = out_mode;
  return launch_down_gather(dn, layer->wdtype, st) == cudaSuccess ? CSFFN_OK : CSFFN_ERR_CUDA;
}
