// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "fp8mlp.h"
#include "gemm_sm100.cuh"

namespace fp8mlp {

// GEMM variants (one template instantiation each)
enum class GemmKind : int {
  Up = 0,       // K1: x . W1^T -> post, post_fp8, partial amax (BF16, K-major A/B)
  Down8 = 1,    // K2: q . W2q_t^T -> out (e4m3, K-major A/B)
  Bf16MnB = 2,  // post . W2 (eval) and dPre . W1 (dX): BF16, K-major A, MN-major B
  DPre = 3,     // K5: dOut . W2^T -> dPre with the 2 sqrt(post) epilogue
  DW = 4,       // K7/K8: dPre^T . x and post^T . dOut (BF16, MN-major A/B), fp32 out
  UpQ = 5,      // K1 on e4m3 x and W1 (dequantised in the epilogue)
  CeFwd = 6,    // LM head x . W^T -> softcapped cross-entropy partial sums (BF16)
  CeFwd8 = 7,   // the same on e4m3 x and W
  CeBwd = 8,    // LM head x . W^T recomputed -> BF16 dlogits (BF16)
  CeBwd8 = 9,   // the same on e4m3 x and W
};
constexpr int kGemmBM = 128;  // accumulator rows per CTA
constexpr int kGemmBN = 256;  // output tile columns
constexpr int kLinearSplitRows = 64;  // the linear dW's token split falls on a k-block (64 BF16 rows)

// rows of one output tile of `kind` (128 per CTA times the CTA-group size)
int gemm_tile_m(GemmKind kind);
// columns of post covered by one partial-amax entry
int up_partial_cols();

struct DeviceInfo {
  int device = -1;
  int num_sms = 0;
  unsigned int* status = nullptr;  // device status word
};

// Checks that the current device is compute capability 10.0; fills `info`.
int current_device(DeviceInfo** info);

cudaError_t launch_gemm(GemmKind kind, const GemmParams& p, int num_tiles, int num_sms, cudaStream_t s);

// small kernels
cudaError_t launch_state_init(fp8mlp_scale_state* st, float margin, float s0, cudaStream_t s);
cudaError_t launch_add_f32(size_t n, float* dst, const float* src, int num_sms, cudaStream_t s);
cudaError_t launch_amax_scale(const float* pa, int n, fp8mlp_scale_state* st, unsigned int* status, cudaStream_t s);
// the W2 cache refresh reduces |W2| in blocks of kW2ElemsPerBlock elements,
// one partial maximum per block in the caller's workspace
constexpr int kW2ElemsPerBlock = 8192;
cudaError_t launch_w2_cache(int h, int d, const uint16_t* W2, uint8_t* W2q_t, float* w2_scale_inv,
                            unsigned int* partial, unsigned int* status, int num_sms, cudaStream_t s);
cudaError_t launch_rmsnorm_fwd(int M, int d, const uint16_t* r, uint16_t* x, float* rstd, int num_sms,
                               cudaStream_t s);
cudaError_t launch_rmsnorm_fwd_quant(int M, int d, const uint16_t* r, uint16_t* x, float* rstd,
                                     const fp8mlp_scale_state* st_x, uint8_t* x_fp8, float* row_amax, int num_sms,
                                     cudaStream_t s);
cudaError_t launch_rmsnorm_bwd(int M, int d, const uint16_t* r, const float* rstd, const uint16_t* dx,
                               const uint16_t* dr_in, uint16_t* dr_out, int num_sms, cudaStream_t s);
cudaError_t launch_residual_add(int M, int d, const uint16_t* r, const uint16_t* out, uint16_t* r_next,
                                int num_sms, cudaStream_t s);

// set the text returned by fp8mlp_last_error_detail() on this thread
void set_error_detail(const char* what);

// number of kernels this library has launched (all devices, all threads)
void count_launches(unsigned long long n);

// programmatic dependent launch on/off (fp8mlp_set_programmatic_launch)
bool pdl_enabled();

// Launch `k` with the programmatic stream-serialisation attribute (when
// enabled): the kernel may start while the previous kernel on the stream
// finishes, and waits for it with pdl_wait() before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, static_cast<KArgs>(args)...);
}

// e4m3 copies of x (delayed scale) and W1 (exact scale) for the FP8 up-projection
constexpr int kXElemsPerBlock = 8192;  // elements of x per partial max |x|
cudaError_t launch_quantize_x(long long n, const uint16_t* x, const fp8mlp_scale_state* st, uint8_t* xq,
                              float* partial, cudaStream_t s);
cudaError_t launch_w1_cache(int h, int d, const uint16_t* W1, uint8_t* W1q, float* w1_scale_inv,
                            unsigned int* partial, unsigned int* status, cudaStream_t s);

// softcapped cross-entropy: rows -> lse, row loss and per-block sums; then
// the block sums -> {sum, weight, mean}, both in a fixed order
constexpr int kCeRowsPerBlock = 32;
constexpr int kCeSlices = 8;  // threads per row in the row pass
int ce_partial_cols();        // vocabulary columns covered by one partial sum
cudaError_t launch_ce_finalize(int M, int nparts, int T, int V, const int* targets, const float* w, float cap,
                               const float* partial, const float* ztgt, float* lse, float* row_loss,
                               double* block_sums, float* loss, cudaStream_t s);

// status word symbol address on the current device
cudaError_t status_word_address(unsigned int** ptr);

}  // namespace fp8mlp
