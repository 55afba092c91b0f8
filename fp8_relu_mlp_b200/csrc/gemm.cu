// Instantiations of the tcgen05 GEMM for the five roles of the MLP block.
#include "internal.h"

namespace fp8mlp {

using CfgUp = GemmCfg<kGemmBN, 4, false, false, false, Epi::UpFused>;
using CfgDown8 = GemmCfg<kGemmBN, 4, true, false, false, Epi::DownScaled>;
using CfgBf16MnB = GemmCfg<kGemmBN, 4, false, false, true, Epi::StoreBf16>;
using CfgDPre = GemmCfg<kGemmBN, 3, false, false, false, Epi::DPre>;
using CfgDW = GemmCfg<kGemmBN, 4, false, true, true, Epi::StoreF32>;

namespace {

constexpr int kMaxDevices = 64;

template <class C>
cudaError_t launch_one(const GemmParams& p, int num_tiles, int num_sms, cudaStream_t s) {
  static bool attr_done[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < kMaxDevices && !attr_done[dev]) {
    e = cudaFuncSetAttribute(gemm_sm100_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const int grid = num_tiles < num_sms ? num_tiles : num_sms;
  if (grid <= 0) return cudaSuccess;
  gemm_sm100_kernel<C><<<grid, 192, C::SMEM_BYTES, s>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(GemmKind kind, const GemmParams& p, int num_tiles, int num_sms, cudaStream_t s) {
  switch (kind) {
    case GemmKind::Up:
      return launch_one<CfgUp>(p, num_tiles, num_sms, s);
    case GemmKind::Down8:
      return launch_one<CfgDown8>(p, num_tiles, num_sms, s);
    case GemmKind::Bf16MnB:
      return launch_one<CfgBf16MnB>(p, num_tiles, num_sms, s);
    case GemmKind::DPre:
      return launch_one<CfgDPre>(p, num_tiles, num_sms, s);
    case GemmKind::DW:
      return launch_one<CfgDW>(p, num_tiles, num_sms, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace fp8mlp
