// isd_accept_resample_static: the accept / resample step with its scratch
// in a buffer compiled into the library, for callers that cannot allocate
// device memory.
//
// Who needs it: a host program that links the C ABI directly and has no
// device allocator of its own (no framework caching allocator), where a
// cudaMalloc per call would synchronise the device and fragment memory,
// or a serving process whose framework has already reserved the device
// memory pool, so that no workspace can be carved out for this call.
//
// The scratch is a file-scope __device__ array of ISD_ACCEPT_STATIC_SCRATCH
// bytes.  Every GPU that loads the library holds one copy of it until the
// process exits.  Host code cannot pass the array's name to a kernel (on the
// host that name is only a stand-in, not a device address), so the first
// call on each device looks up the array's device address with
// cudaGetSymbolAddress, with that device current, and remembers it for the
// current CUDA context; that first call should be made before any stream
// capture begins.  All calls on
// a device share the one array and it keeps the previous call's contents:
// nothing in it needs to start at zero, because every scratch word the
// kernels read is written earlier in the same call, but calls whose work
// overlaps on the GPU (different streams, no ordering) race on it and must
// not be issued.  Nothing here allocates or frees device memory.
#include <mutex>

#include "common.cuh"

namespace isd {
size_t accept_workspace_bytes(int B, int N, int K, int V);
int accept_validate(const isd_accept_args* a);
}

namespace {

__device__ __align__(256) unsigned char g_accept_scratch[ISD_ACCEPT_STATIC_SCRATCH];

// The address is remembered per CUDA context (the module, and so the array,
// is loaded once per context); a different current context on a device,
// such as the primary context recreated after cudaDeviceReset under a new
// handle, triggers a fresh look-up.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
  }
  return fn;
}

constexpr int kMaxDevices = 64;
struct Slot {
  CUcontext ctx;
  void* addr;
};
Slot g_scratch[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array in the current context (set-up on
// first use per device, with that device current).  nullptr on a CUDA error.
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nullptr;
  CtxGetCurrentFn get = ctx_get_current();
  if (!get) return nullptr;
  // Null until the runtime has bound a context on this thread.
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  Slot& s = g_scratch[dev];
  if (ctx && s.addr && s.ctx == ctx) return s.addr;
  void* ptr = nullptr;   // the look-up binds the primary context if needed
  if (cudaGetSymbolAddress(&ptr, g_accept_scratch) != cudaSuccess)
    return nullptr;
  if (!ctx && (get(&ctx) != CUDA_SUCCESS || !ctx)) return nullptr;
  s.ctx = ctx;
  s.addr = ptr;
  return s.addr;
}

}  // namespace

extern "C" int isd_accept_resample_static(const isd_accept_args* a,
                                          void* stream) {
  // The same argument checks, in the same order, as isd_accept_resample;
  // then the size limit in place of the workspace check.
  const int rc = isd::accept_validate(a);
  if (rc != ISD_OK) return rc;
  const size_t need = isd::accept_workspace_bytes(a->B, a->N, a->K, a->V);
  if (need > (size_t)ISD_ACCEPT_STATIC_SCRATCH) return ISD_ERR_WORKSPACE;
  void* ptr = scratch_address();
  if (!ptr) return ISD_ERR_CUDA;
  isd_accept_args b = *a;
  b.workspace = ptr;
  b.workspace_bytes = (size_t)ISD_ACCEPT_STATIC_SCRATCH;
  return isd_accept_resample(&b, stream);
}
