// lcb_noalloc.cu -- IKBO-LCB for callers that cannot allocate device memory.
//
// rocs_lcb_forward() needs a caller-provided device workspace (status word, per-request
// ready flags and the fp32 request contributions Z).  Some callers have no way to provide
// one: for example a plugin running inside a serving process whose device memory is entirely
// reserved up front by the host framework's own pool, with no allocator exposed to plugins,
// or a latency-critical path where a cudaMalloc (which can synchronise the device and must
// find room in an already fully reserved pool) is not permitted.  rocs_lcb_forward_noalloc()
// serves them: it runs the same kernel with the same launch configuration, but its scratch
// lives in a fixed-size array in device global memory that the library itself declares, so
// the call allocates nothing.  The caller still passes its inputs and outputs.
//
// Costs of this convenience, stated for the user:
//   * every GPU that loads this library holds kNoallocScratchBytes of device memory for the
//     array until the process exits;
//   * all calls share the one array per device: calls that can overlap on the GPU (different
//     streams, or different host threads without ordering) race on it and must be serialised
//     by the caller;
//   * the array keeps whatever the last call left in it; each call clears the parts that must
//     start at zero (status word and ready flags) before its kernel runs;
//   * the first call on a device looks up the array's device address (cudaGetSymbolAddress,
//     once per device, with that device current).  Make that first call before any stream
//     capture begins.  cudaDeviceReset() unloads the library's device code, so the looked-up
//     address is stale afterwards: do not call this entry point after resetting a device that
//     it has already run on;
//   * device-side status (a bounded wait that expired, a bad device offset) is recorded in the
//     array's own header; rocs_lcb_noalloc_read_status() reads it without allocating.  Host-side
//     validation errors are returned as usual.
#include <atomic>

#include "lcb_sm100.h"

namespace rocs {
int lcb_validate_ext(const rocs_lcb_args* a, int64_t* C);
int lcb_run_ext(const rocs_lcb_args* a, int64_t C, WsHeader* hdr, uint8_t* body, cudaStream_t st, int* launches);
size_t lcb_body_bytes_ext(int64_t R, int64_t o_c, int64_t d);
void set_last_launches(int n);
}  // namespace rocs

using namespace rocs;

namespace {

constexpr size_t kNoallocScratchBytes = ROCS_LCB_NOALLOC_SCRATCH_BYTES;
static_assert(kNoallocScratchBytes % 256 == 0, "scratch size is a multiple of 256 bytes");

// The scratch array.  In host code its name is only a host-side stand-in for the symbol, never
// a device address: the address passed to kernels comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_lcb_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
// One slot per device ordinal.  Atomic, so host threads that make their first call at the same time
// may both look the address up, but each reads and publishes a complete pointer (the same one).
std::atomic<void*> g_scratch_addr[kMaxDevices];

// Device address of the array on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return ROCS_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return ROCS_ERR_UNSUPPORTED;
  void* p = g_scratch_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    if (cudaGetSymbolAddress(&p, g_lcb_noalloc_scratch) != cudaSuccess || p == nullptr) return ROCS_ERR_CUDA;
    g_scratch_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return ROCS_OK;
}

}  // namespace

extern "C" int rocs_lcb_forward_noalloc(const rocs_lcb_args* a, rocs_stream_t stream) {
  int64_t C = 0;
  int rc = lcb_validate_ext(a, &C);
  if (rc) return rc;
  const size_t need = sizeof(WsHeader) + lcb_body_bytes_ext(a->R, a->o_c, a->d);
  if (need > kNoallocScratchBytes) return ROCS_ERR_WORKSPACE;  // too many requests for the fixed array
  void* scratch = nullptr;
  rc = scratch_address(&scratch);
  if (rc) return rc;
  WsHeader* hdr = static_cast<WsHeader*>(scratch);
  int launches = 0;
  rc = lcb_run_ext(a, C, hdr, reinterpret_cast<uint8_t*>(hdr + 1), reinterpret_cast<cudaStream_t>(stream), &launches);
  if (rc == ROCS_OK) set_last_launches(launches);
  return rc;
}

extern "C" int rocs_lcb_noalloc_read_status(rocs_stream_t stream, int32_t* device_code, int32_t* detail) {
  if (!device_code) return ROCS_ERR_INVALID_ARG;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc) return rc;
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t h[2] = {0, 0};  // code and detail: the first 8 bytes of the header at the start of the array
  if (cudaMemcpyAsync(h, scratch, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return ROCS_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return ROCS_ERR_CUDA;
  *device_code = h[0];
  if (detail) *detail = h[1];
  return ROCS_OK;
}
