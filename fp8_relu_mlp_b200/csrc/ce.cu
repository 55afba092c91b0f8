// Softcapped cross-entropy: the two small passes after the LM-head GEMM.
//
// The GEMM epilogue (Epi::CeFwd) leaves, for every row m and every group of
// 128 vocabulary columns j, S_j[m] = sum over the group of exp(z - c), where
// z = c tanh(y/c) is the softcapped logit, and z - c at each valid target.
// Because |z| <= c, every term lies in [e^-2c, 1], so no running maximum is
// needed: lse = c + ln(sum_j S_j).  These passes turn that into lse, the row
// losses and the reduced loss, summing in double and in a fixed order, so
// the result does not depend on the launch.
#include "internal.h"

namespace fp8mlp {
namespace {

using namespace dev;

// Block = kCeRowsPerBlock rows x kCeSlices threads per row.  Warp s sums the
// partials j = s, s + kCeSlices, ... of 32 consecutive rows (coalesced: the
// partials are stored [j][m]).
__global__ void __launch_bounds__(kCeRowsPerBlock* kCeSlices)
    ce_rows_kernel(int M, int nparts, int T, int V, const int* __restrict__ targets, float4 w, float cap,
                   const float* __restrict__ partial, const float* __restrict__ ztgt, float* __restrict__ lse,
                   float* __restrict__ row_loss, double* __restrict__ block_sums) {
  static_assert(kCeRowsPerBlock == 32, "one row per lane");
  __shared__ double part[kCeSlices][kCeRowsPerBlock];
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch_dependents();
  const int r = threadIdx.x & 31;
  const int slice = threadIdx.x >> 5;
  const int m = blockIdx.x * kCeRowsPerBlock + r;
  double s = 0.0;
  if (m < M) {
    for (int j = slice; j < nparts; j += kCeSlices) s += partial[static_cast<size_t>(j) * M + m];
  }
  part[slice][r] = s;
  __syncthreads();
  if (slice != 0) return;
  double loss = 0.0, wsum = 0.0;
  if (m < M) {
    double S = 0.0;
#pragma unroll
    for (int k = 0; k < kCeSlices; ++k) S += part[k][r];
    const double lnS = log(S);  // lse - c
    lse[m] = static_cast<float>(static_cast<double>(cap) + lnS);
    const float wt[4] = {w.x, w.y, w.z, w.w};
    for (int t = 0; t < T; ++t) {
      const int tv = targets[static_cast<size_t>(m) * T + t];
      if (tv >= 0 && tv < V) {
        // lse - z = (lse - c) - (z - c)
        loss += static_cast<double>(wt[t]) * (lnS - static_cast<double>(ztgt[static_cast<size_t>(m) * T + t]));
        wsum += wt[t];
      }
    }
    if (row_loss != nullptr) row_loss[m] = static_cast<float>(loss);
  }
  // the block's 32 rows, in a fixed butterfly order
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    loss += __shfl_xor_sync(0xffffffffu, loss, o);
    wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  }
  if (r == 0) {
    block_sums[2 * blockIdx.x] = loss;
    block_sums[2 * blockIdx.x + 1] = wsum;
  }
}

// One block: {sum, weight, mean} of the per-block sums, in a fixed order.
__global__ void __launch_bounds__(256) ce_total_kernel(int nblk, const double* __restrict__ block_sums,
                                                       float* __restrict__ loss) {
  __shared__ double sl[256], sw[256];
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch_dependents();
  double a = 0.0, b = 0.0;
  for (int i = threadIdx.x; i < nblk; i += 256) {
    a += block_sums[2 * i];
    b += block_sums[2 * i + 1];
  }
  sl[threadIdx.x] = a;
  sw[threadIdx.x] = b;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      sl[threadIdx.x] += sl[threadIdx.x + o];
      sw[threadIdx.x] += sw[threadIdx.x + o];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    loss[0] = static_cast<float>(sl[0]);
    loss[1] = static_cast<float>(sw[0]);
    loss[2] = sw[0] > 0.0 ? static_cast<float>(sl[0] / sw[0]) : 0.f;
  }
}

}  // namespace

cudaError_t launch_ce_finalize(int M, int nparts, int T, int V, const int* targets, const float* w, float cap,
                               const float* partial, const float* ztgt, float* lse, float* row_loss,
                               double* block_sums, float* loss, cudaStream_t s) {
  const int nblk = (M + kCeRowsPerBlock - 1) / kCeRowsPerBlock;
  const float4 w4 = make_float4(w[0], w[1], w[2], w[3]);
  cudaError_t e = launch_pdl(ce_rows_kernel, dim3(nblk), dim3(kCeRowsPerBlock * kCeSlices), 0, s, M, nparts, T, V,
                             targets, w4, cap, partial, ztgt, lse, row_loss, block_sums);
  count_launches(1);
  if (e != cudaSuccess) return e;
  e = launch_pdl(ce_total_kernel, dim3(1), dim3(256), 0, s, nblk, static_cast<const double*>(block_sums), loss);
  count_launches(1);
  return e;
}

}  // namespace fp8mlp
