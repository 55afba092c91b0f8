// fp8mlp_w2_fp8_cache_refresh_noalloc: the transposed FP8 W2 cache refresh
// for callers that cannot hand the library any device memory of its own.
//
// Some callers cannot allocate device memory at the point where they call
// the library: code running inside another framework's operator hook that
// owns all device memory through its own pool and exposes no workspace, or
// a runtime that forbids cudaMalloc/cudaFree on its hot path because those
// calls can synchronise the whole device.  This entry point therefore takes
// no workspace argument.  Its scratch -- one partial maximum of |W2| per
// reduction block -- lives in the fixed array below, which every GPU that
// loads the library holds until the process exits.  It runs the same two
// kernels as fp8mlp_w2_fp8_cache_refresh, with the array's address in place
// of the workspace, so the two entry points give the same bits.
//
// The array is shared by every call on a device and keeps what the last
// call wrote.  Nothing in it has to start at zero: each call writes every
// entry it later reads.  Calls that overlap on the GPU (two streams, or two
// host threads enqueueing at once) use the same entries and race.
//
// The first call on a device looks up the array's device address
// (cudaGetSymbolAddress) with that device current, and caches it; make that
// first call before any stream capture.
#include <mutex>
#include <string>

#include "internal.h"

namespace fp8mlp {
namespace {

constexpr int kScratchEntries = 2048;  // partial maxima the array holds
// one partial maximum per kW2ElemsPerBlock (8192) elements of W2, as in the
// workspace version, whose two kernels this entry point launches
constexpr long long kMaxElems = static_cast<long long>(kScratchEntries) * kW2ElemsPerBlock;  // 16,777,216
static_assert(kMaxElems == 16777216, "the documented limit");

static __device__ __align__(256) unsigned int g_w2_partial_amax[kScratchEntries];

constexpr int kMaxDev = 64;
unsigned int* g_partial_ptr[kMaxDev] = {};
std::mutex g_setup_mutex;

int noalloc_fail(int code, const char* what) {
  set_error_detail(what);
  return code;
}

}  // namespace
}  // namespace fp8mlp

using namespace fp8mlp;

extern "C" int fp8mlp_w2_fp8_cache_refresh_noalloc(int h, int d, const uint16_t* W2, uint8_t* W2q_t,
                                                   float* w2_scale_inv, fp8mlp_stream_t stream) {
  set_error_detail("");
  if (d < 16 || h < 16 || d % 16 != 0 || h % 16 != 0)
    return noalloc_fail(FP8MLP_ERR_UNSUPPORTED_SHAPE, "d and h must be multiples of 16 and >= 16");
  if (static_cast<long long>(h) * d > kMaxElems)
    return noalloc_fail(FP8MLP_ERR_UNSUPPORTED_SHAPE,
                        "h*d exceeds the no-allocation scratch limit of 16777216 elements "
                        "(use fp8mlp_w2_fp8_cache_refresh with a workspace)");
  if (W2 == nullptr || W2q_t == nullptr || w2_scale_inv == nullptr)
    return noalloc_fail(FP8MLP_ERR_INVALID_ARG, "W2, W2q_t and w2_scale_inv must not be NULL");
  if ((reinterpret_cast<uintptr_t>(W2) & 15u) || (reinterpret_cast<uintptr_t>(W2q_t) & 15u) ||
      (reinterpret_cast<uintptr_t>(w2_scale_inv) & 3u))
    return noalloc_fail(FP8MLP_ERR_INVALID_ARG, "W2 / W2q_t must be 16-byte aligned, w2_scale_inv 4-byte aligned");
  DeviceInfo* di = nullptr;
  const int rc = current_device(&di);
  if (rc != FP8MLP_OK) return rc;
  const int dev = di->device;
  if (dev < 0 || dev >= kMaxDev) return noalloc_fail(FP8MLP_ERR_NO_DEVICE, "device index out of range");
  unsigned int* partial = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_partial_ptr[dev] == nullptr) {
      // the array's name is only a host-side stand-in: ask the runtime for its
      // address on this device (the current one)
      void* p = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&p, g_w2_partial_amax);
      if (e != cudaSuccess) {
        cudaGetLastError();
        return noalloc_fail(FP8MLP_ERR_CUDA, "cudaGetSymbolAddress of the no-allocation scratch failed");
      }
      g_partial_ptr[dev] = static_cast<unsigned int*>(p);
    }
    partial = g_partial_ptr[dev];
  }
  // the two kernels of fp8mlp_w2_fp8_cache_refresh, with the fixed array in
  // place of the caller's workspace: the results are the same bits
  const cudaError_t e = launch_w2_cache(h, d, W2, W2q_t, w2_scale_inv, partial, di->status, di->num_sms, stream);
  if (e != cudaSuccess) return noalloc_fail(FP8MLP_ERR_CUDA, cudaGetErrorString(e));
  return FP8MLP_OK;
}
