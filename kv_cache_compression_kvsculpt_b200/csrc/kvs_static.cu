// kvs_loss_grad_static: the loss/gradient call for callers that cannot
// allocate device memory.
//
// Some callers of this library cannot call cudaMalloc (or any allocator) to
// provide the workspace that kvs_loss_grad needs: code embedded in a host
// application that owns every byte of device memory through its own pool and
// forbids side allocations, or a service that must fix its device footprint
// when it loads the library so that no request can later fail for lack of
// memory.  This entry point takes its scratch from one array compiled into the
// library instead, so such a caller only passes its inputs and outputs.
//
// The array is KVS_STATIC_WS_BYTES bytes of device memory on every GPU that
// loads the library, held until the process exits.  Batches whose workspace
// (kvs_workspace_bytes) exceeds it are rejected with KVS_EWORKSPACE.
#include <cuda.h>

#include <mutex>

#include "kvs_common.cuh"

#define KVS_STATIC_WS_BYTES (32u << 20)
#define KVS_STATIC_MAX_DEVICES 64

static __device__ __align__(256) unsigned char g_static_ws[KVS_STATIC_WS_BYTES];

namespace {

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

std::mutex g_static_mu;
struct Cached {
  CUcontext ctx;  // the context the address belongs to
  void *ptr;
};
Cached g_static[KVS_STATIC_MAX_DEVICES];

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void *p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of g_static_ws in the current device's current context.  The
// host-side name of the array is only a handle: the address must come from
// cudaGetSymbolAddress with that device current.  It is looked up once per
// device and again whenever the current context is not the one it was looked
// up in (after cudaDeviceReset, or under another driver context).
int static_workspace(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    kvs::set_cuda_error(e, "cudaGetDevice");
    return KVS_ECUDA;
  }
  if (dev < 0 || dev >= KVS_STATIC_MAX_DEVICES) return KVS_ENOTSUP;
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return KVS_ECUDA;
  // null before the runtime's first call on this thread has made a context current
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return KVS_ECUDA;
  std::lock_guard<std::mutex> lock(g_static_mu);
  Cached &c = g_static[dev];
  if (!c.ptr || !ctx || c.ctx != ctx) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_ws);  // makes the device's context current
    if (e != cudaSuccess) {
      kvs::set_cuda_error(e, "cudaGetSymbolAddress(g_static_ws)");
      return KVS_ECUDA;
    }
    if (get(&ctx) != CUDA_SUCCESS || !ctx) return KVS_ECUDA;
    c.ctx = ctx;
    c.ptr = p;
  }
  *out = c.ptr;
  return KVS_OK;
}

}  // namespace

extern "C" int kvs_loss_grad_static(const kvs_batch *batch, const float *Q, const float *Kc,
                                    const float *Vc, const float *Y, const float *lse,
                                    float w_out, float w_lse, float *loss, float *parts,
                                    float *dKc, void *stream) {
  const size_t need = kvs_workspace_bytes(batch, nullptr);
  if (need == 0) return KVS_EINVAL;
  if (need > KVS_STATIC_WS_BYTES) return KVS_EWORKSPACE;
  void *ws = nullptr;
  int rc = static_workspace(&ws);
  if (rc) return rc;
  return kvs_loss_grad(batch, Q, Kc, Vc, Y, lse, w_out, w_lse, loss, parts, dKc, ws,
                       KVS_STATIC_WS_BYTES, stream);
}
