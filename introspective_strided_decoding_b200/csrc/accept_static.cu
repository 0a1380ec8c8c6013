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
// cudaGetSymbolAddress, with that device current, and remembers it; that
// first call should be made before any stream capture begins.  All calls on
// a device share the one array and it keeps the previous call's contents:
// nothing in it needs to start at zero, because every scratch word the
// kernels read is written earlier in the same call, but calls whose work
// overlaps on the GPU (different streams, no ordering) race on it and must
// not be issued.  Nothing here allocates or frees device memory.
#include <mutex>

#include "common.cuh"

namespace isd {
size_t accept_workspace_bytes(int B, int N, int K, int V);
}

namespace {

__device__ __align__(256) unsigned char g_accept_scratch[ISD_ACCEPT_STATIC_SCRATCH];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (set-up on
// first use per device).  Returns nullptr on a CUDA error.
void* scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_accept_scratch) != cudaSuccess)
      return nullptr;
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" int isd_accept_resample_static(const isd_accept_args* a,
                                          void* stream) {
  if (!a) return ISD_ERR_INVALID_ARG;
  const size_t need = isd_accept_workspace_bytes(a);
  if (need == 0) return isd_accept_resample(a, stream);  // its own error
  if (need > (size_t)ISD_ACCEPT_STATIC_SCRATCH) return ISD_ERR_WORKSPACE;
  void* ptr = scratch_address();
  if (!ptr) return ISD_ERR_CUDA;
  isd_accept_args b = *a;
  b.workspace = ptr;
  b.workspace_bytes = (size_t)ISD_ACCEPT_STATIC_SCRATCH;
  return isd_accept_resample(&b, stream);
}
