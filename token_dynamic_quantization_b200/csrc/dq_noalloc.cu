// dq_ada_layernorm_quant_noalloc: AdaLayerNormQuant with its scratch table in
// a fixed device array instead of a caller-provided workspace.
//
// The AdaLayerNormQuant path needs batch * hidden pairs of fp32 (the folded
// affine table A, B that the row kernel reads). The regular entry point takes
// that scratch from the caller. Some callers have no device allocator to get
// it from: a plain C host program that links only this library, or a hook
// that runs where allocating would re-enter the caller's own allocator (for
// example inside an out-of-memory handler). This entry point serves them: the
// table lives in a file-scope __device__ array of DQ_ADA_NOALLOC_MAX_TABLE
// entries (8 bytes each, 1 MiB), and the call allocates nothing, neither
// through CUDA nor through any library.
//
// Set-up: the array's device address is looked up with cudaGetSymbolAddress
// on the first call made while a device is current, and cached together with
// the identity of that device's current context. A later call that finds a
// different context (the device was reset with cudaDeviceReset, which
// reloads the library's device code) repeats the look-up; every other call
// only reads the cache. A call that does the look-up should come before any
// stream capture.
//
// Nothing in the array has to start at zero: every call writes each table
// entry it reads (when the row kernel reads the table from global memory, the
// table kernel writes it first on the same stream and the row kernel waits
// for it; otherwise the row kernel folds the table in shared memory and the
// array is not touched). The array is shared by all calls on a device, so two
// calls whose executions overlap (different streams, or different host
// threads) race on it; such callers use the regular entry point with
// separate workspaces.

#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "dq.h"

namespace {

// The array has one instance per device (each device loads its own copy of
// the module); its address is therefore looked up per device.
static __device__ __align__(256) float2 g_ada_noalloc_table[DQ_ADA_NOALLOC_MAX_TABLE];

constexpr int kMaxDevices = 64;

struct Cached {
  void* addr;
  unsigned long long ctx_id;  // 0: not set up
};
Cached g_table[kMaxDevices];
std::mutex g_setup_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (never 0), or 0 when the
// driver cannot report one; then the cached address is kept as it is.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    cudaGetLastError();
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id + 1;  // keep 0 for "unknown"
}

// Device address of this device's table (set up on first use, and again
// after the device's context has changed).
dq_status noalloc_table(void** addr) {
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) {
    cudaGetLastError();
    return DQ_ERR_CUDA;
  }
  if (device < 0 || device >= kMaxDevices) return DQ_ERR_UNSUPPORTED;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  Cached& c = g_table[device];
  if (c.addr == nullptr || (ctx != 0 && c.ctx_id != ctx)) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ada_noalloc_table) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return DQ_ERR_CUDA;
    }
    c.addr = p;
    c.ctx_id = ctx;
  }
  *addr = c.addr;
  return DQ_OK;
}

}  // namespace

extern "C" dq_status dq_ada_layernorm_quant_noalloc(const void* x, dq_dtype x_dtype, int64_t batch, int64_t seq,
                                                    int64_t hidden, const void* ada_scale, const void* ada_shift,
                                                    const void* weight, const void* bias, const void* smooth,
                                                    dq_dtype param_dtype, float epsilon, int8_t* out,
                                                    float* quant_scale, cudaStream_t stream) {
  // the checks of dq_ada_layernorm_quant, in its order, with the array's
  // size limit in place of its workspace check
  size_t needed = 0;
  const dq_status st = dq_ada_layernorm_quant_get_workspace_size(batch, seq, hidden, x_dtype, param_dtype, &needed);
  if (st != DQ_OK) return st;
  if (!(epsilon >= 0.0f) || epsilon == INFINITY) return DQ_ERR_BAD_ARGUMENT;  // NaN, negative or infinite
  if (needed == 0) return DQ_OK;  // batch * seq == 0: nothing to do, no set-up
  if (x == nullptr || ada_scale == nullptr || ada_shift == nullptr || out == nullptr || quant_scale == nullptr)
    return DQ_ERR_NULL_POINTER;
  if (batch > DQ_ADA_NOALLOC_MAX_TABLE / hidden) return DQ_ERR_UNSUPPORTED;  // table larger than the array
  void* table = nullptr;
  const dq_status ts = noalloc_table(&table);
  if (ts != DQ_OK) return ts;
  return dq_ada_layernorm_quant(x, x_dtype, batch, seq, hidden, ada_scale, ada_shift, weight, bias, smooth,
                                param_dtype, epsilon, out, quant_scale, table,
                                sizeof(float2) * static_cast<size_t>(DQ_ADA_NOALLOC_MAX_TABLE), stream);
}
