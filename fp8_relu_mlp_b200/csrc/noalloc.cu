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
// loads the library holds until the process exits.
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

using namespace dev;

constexpr int kScratchEntries = 2048;          // partial maxima the array holds
constexpr int kElemsPerBlock = 8192;           // W2 elements one reduction block covers
constexpr long long kMaxElems = static_cast<long long>(kScratchEntries) * kElemsPerBlock;  // 16,777,216

static __device__ __align__(256) unsigned int g_w2_partial_amax[kScratchEntries];

constexpr int kMaxDev = 64;
unsigned int* g_partial_ptr[kMaxDev] = {};
std::mutex g_setup_mutex;

// Block b writes max |W2| (as BF16 magnitude bits, whose integer order is
// the value order, NaN above infinity) over elements [b*8192, (b+1)*8192).
__global__ void __launch_bounds__(256) noalloc_w2_block_amax(const uint4* __restrict__ W, long long n_vec,
                                                             unsigned int* __restrict__ partial) {
  __shared__ unsigned int wmax[8];
  const long long base = static_cast<long long>(blockIdx.x) * (kElemsPerBlock / 8);
  unsigned int m = 0;
#pragma unroll
  for (int k = 0; k < kElemsPerBlock / 8 / 256; ++k) {
    const long long i = base + k * 256 + threadIdx.x;
    if (i < n_vec) {
      const uint4 v = W[i];
      const unsigned int w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        m = max(m, w4[j] & 0x7FFFu);
        m = max(m, (w4[j] >> 16) & 0x7FFFu);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned int r = 0;
    for (int w = 0; w < 8; ++w) r = max(r, wmax[w]);
    partial[blockIdx.x] = r;
  }
}

// Every block reduces the partial maxima to s_w, then writes its 64x64 tile
// of W2q_t[j, i] = e4m3(W2[i, j] * s_w).
__global__ void __launch_bounds__(256) noalloc_w2_quant_t(int h, int d, const uint16_t* __restrict__ W2,
                                                          uint8_t* __restrict__ W2q_t, float* w2_scale_inv,
                                                          const unsigned int* __restrict__ partial, int nparts,
                                                          unsigned int* status) {
  __shared__ float tile[64][65];
  __shared__ unsigned int wmax[8];
  unsigned int m = 0;
  for (int i = threadIdx.x; i < nparts; i += 256) m = max(m, partial[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  m = 0;
  for (int w = 0; w < 8; ++w) m = max(m, wmax[w]);
  const float a = __uint_as_float(m << 16);
  const bool ok = isfinite(a) && a > 0.f;
  const float s_w = ok ? __fdiv_rn(FP8MLP_E4M3_MAX, a) : 1.f;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    w2_scale_inv[0] = __fdiv_rn(1.f, s_w);
    if (!ok) atomicOr(status, STATUS_W2_DEGENERATE);
  }
  const int i0 = blockIdx.y * 64;  // rows of W2 (h)
  const int j0 = blockIdx.x * 64;  // columns of W2 (d)
  for (int t = threadIdx.x; t < 64 * 8; t += 256) {
    const int r = t >> 3, c8 = (t & 7) * 8;
    const int i = i0 + r, j = j0 + c8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (i < h && j < d) v = *reinterpret_cast<const uint4*>(W2 + static_cast<size_t>(i) * d + j);
    const unsigned int w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      tile[r][c8 + 2 * k] = bf16lo_to_f32(w4[k]);
      tile[r][c8 + 2 * k + 1] = bf16hi_to_f32(w4[k]);
    }
  }
  __syncthreads();
  for (int t = threadIdx.x; t < 64 * 16; t += 256) {
    const int jr = t >> 4, i4 = (t & 15) * 4;
    const int j = j0 + jr, i = i0 + i4;
    if (j < d && i < h) {
      const uint32_t lo = pack_e4m3x2(__fmul_rn(tile[i4][jr], s_w), __fmul_rn(tile[i4 + 1][jr], s_w));
      const uint32_t hi = pack_e4m3x2(__fmul_rn(tile[i4 + 2][jr], s_w), __fmul_rn(tile[i4 + 3][jr], s_w));
      *reinterpret_cast<uint32_t*>(W2q_t + static_cast<size_t>(j) * h + i) = lo | (hi << 16);
    }
  }
}

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
  const long long n = static_cast<long long>(h) * d;
  const int nparts = static_cast<int>((n + kElemsPerBlock - 1) / kElemsPerBlock);
  cudaStream_t s = stream;
  noalloc_w2_block_amax<<<nparts, 256, 0, s>>>(reinterpret_cast<const uint4*>(W2), n / 8, partial);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return noalloc_fail(FP8MLP_ERR_CUDA, cudaGetErrorString(e));
  dim3 grid((d + 63) / 64, (h + 63) / 64);
  noalloc_w2_quant_t<<<grid, 256, 0, s>>>(h, d, W2, W2q_t, w2_scale_inv, partial, nparts, di->status);
  count_launches(1);
  e = cudaGetLastError();
  if (e != cudaSuccess) return noalloc_fail(FP8MLP_ERR_CUDA, cudaGetErrorString(e));
  return FP8MLP_OK;
}
