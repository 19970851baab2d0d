// attend_static.cu -- isoquant_attend_decode_static: decode attention that
// allocates nothing and needs no workspace from the caller.
//
// Some callers cannot hand this library a workspace or let it allocate one:
// an inference server or plugin host whose memory pool owns every byte of
// device memory and forbids allocations outside it, or a latency-critical
// decode loop that must not pay for cudaMalloc/cudaFree (which can
// synchronise the whole device) in the middle of a step.  For them, the
// partial records of the split-context attention live in a fixed array
// compiled into the library.
//
// The array is a file-scope __device__ variable of kScratchBytes (16 MiB):
// every GPU that loads the library holds it until the process exits.  In
// host code its name is only a host-side stand-in, so the device address is
// looked up with cudaGetSymbolAddress, once per device and CUDA context,
// with that device current, on the first call made on it; make that first
// call before any stream capture begins.  The address is remembered with the
// context's unique id: after cudaDeviceReset (which destroys the context and
// the array with it) the next call sees a new context and looks the address
// up again, so it never passes a stale pointer; that call is again a first
// call and must precede any capture.  All calls on a device share the one array and
// leave their records in it: two calls whose kernels overlap on the GPU (on
// different streams, say) race on it and must be serialised by the caller.
// Nothing in it has to start at zero: every record the combine step reads is
// written earlier in the same call.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "isoquant_internal.cuh"
#include "trace.cuh"

namespace isoquant {
namespace {

constexpr size_t kScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // id of the context the address belongs to

// The current CUDA context's unique id (driver entry points, resolved once
// through the runtime so that the library links only cudart).
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);
CtxGetCurrentFn g_ctx_current = nullptr;
CtxGetIdFn g_ctx_id = nullptr;
int current_context_id(unsigned long long *id) {
  if (g_ctx_current == nullptr || g_ctx_id == nullptr) {
    void *a = nullptr, *b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) != cudaSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) != cudaSuccess ||
        qa != cudaDriverEntryPointSuccess || qb != cudaDriverEntryPointSuccess)
      return ISOQUANT_ERR_CUDA;
    g_ctx_current = reinterpret_cast<CtxGetCurrentFn>(a);
    g_ctx_id = reinterpret_cast<CtxGetIdFn>(b);
  }
  CUcontext c = nullptr;
  if (g_ctx_current(&c) != CUDA_SUCCESS || c == nullptr || g_ctx_id(c, id) != CUDA_SUCCESS) return ISOQUANT_ERR_CUDA;
  return ISOQUANT_OK;
}

// Device address of g_scratch on `device` (which must be current), looked up
// again whenever the current context is not the one it was found in.
int scratch_for(int device, void **out) {
  if (device < 0 || device >= kMaxDevices) return ISOQUANT_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  unsigned long long id = 0;
  const int st = current_context_id(&id);
  if (st != ISOQUANT_OK) return st;
  if (g_scratch_ptr[device] == nullptr || g_scratch_ctx[device] != id) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || p == nullptr) return ISOQUANT_ERR_CUDA;
    g_scratch_ptr[device] = p;
    g_scratch_ctx[device] = id;
  }
  *out = g_scratch_ptr[device];
  return ISOQUANT_OK;
}

}  // namespace
}  // namespace isoquant

using namespace isoquant;

extern "C" int isoquant_attend_decode_static(isoquant_ctx *ctx, const isoquant_cache *cache, const float *q_rot,
                                             int batch, int nq, int num_q_heads, const int32_t *page_table,
                                             int max_pages, const int32_t *seq_lens, int causal, float scale,
                                             float *out, void *stream) {
  ISOQUANT_TRACE("isoquant_attend_decode_static");
  if (ctx == nullptr) return ISOQUANT_ERR_INVALID_ARG;
  ctx->last_launches = 0;
  if (num_q_heads < 1 || nq < 1 || batch < 0 || num_q_heads % ctx->num_kv_heads != 0)
    return ISOQUANT_ERR_INVALID_ARG;
  // the records of one of the shape's plans must fit the fixed array (the
  // tcgen05 kernel's when they fit, else the mma.sync kernel's)
  size_t need = 0;
  int st = attend_workspace_min(ctx, batch, nq, num_q_heads, &need);
  if (st != ISOQUANT_OK) return st;
  if (need > kScratchBytes) return ISOQUANT_ERR_WORKSPACE;
  if (batch == 0) return ISOQUANT_OK;
  int device = -1;
  if (cudaGetDevice(&device) != cudaSuccess) return ISOQUANT_ERR_CUDA;
  if (device != ctx->device) return ISOQUANT_ERR_INVALID_ARG;
  void *scratch = nullptr;
  st = scratch_for(device, &scratch);
  if (st != ISOQUANT_OK) return st;
  return isoquant_attend_decode(ctx, cache, q_rot, batch, nq, num_q_heads, page_table, max_pages, seq_lens, causal,
                                scale, scratch, kScratchBytes, out, stream);
}
