// Instantiations of the tcgen05 GEMM for the roles of the MLP block, the FP8
// linear layer and the softcapped cross-entropy head.
#include <atomic>

#include "internal.h"

namespace fp8mlp {

// 2-CTA UMMA (cluster pairs, 256x256 tiles): each SM streams its 128 rows of
// A and half of B, a third less operand traffic per FLOP than 1-CTA tiles
// up-projection: the MMA waits on operand stages far more often than on the
// epilogue, so one staging slot per epilogue warp pays for a sixth stage
using CfgUp = GemmCfg<2, kGemmBN, 6, false, false, false, Epi::UpFused, 8, 4, 1>;
using CfgDown8 = GemmCfg<2, kGemmBN, 6, true, false, false, Epi::DownScaled>;
using CfgBf16MnB = GemmCfg<2, kGemmBN, 6, false, false, true, Epi::StoreBf16>;
// e4m3 up-projection: the mainloop is twice as fast, so the epilogue sets the
// pace; 16 epilogue warps (96 registers each, one staging slot)
using CfgUpQ = GemmCfg<2, kGemmBN, 5, true, false, false, Epi::UpFused, 16, 4, 1>;
// dPre: 16 epilogue warps (two 32-column chunks each per tile) with a
// one-chunk post ring and one staging slot, which leaves room for a fifth
// operand stage
using CfgDPre = GemmCfg<2, kGemmBN, 5, false, false, false, Epi::DPre, 16, 1, 1>;
// dW: one long tile per CTA pair, so a light epilogue (4 warps) and more stages
using CfgDW = GemmCfg<2, kGemmBN, 6, false, true, true, Epi::StoreF32, 4>;
// LM head with the softcapped cross-entropy in the epilogue; the forward
// stores no tile, so its shared memory all goes to the operand ring
using CfgCeF = GemmCfg<2, kGemmBN, 6, false, false, false, Epi::CeFwd, 16>;
using CfgCeF8 = GemmCfg<2, kGemmBN, 6, true, false, false, Epi::CeFwd, 16>;
using CfgCeB = GemmCfg<2, kGemmBN, 5, false, false, false, Epi::CeBwd, 16>;
using CfgCeB8 = GemmCfg<2, kGemmBN, 5, true, false, false, Epi::CeBwd, 16>;

namespace {

constexpr int kMaxDevices = 64;

template <class C>
cudaError_t launch_one(const GemmParams& p, int num_tiles, int num_sms, cudaStream_t s) {
  // the attribute is set once per device; two threads racing here both set
  // the same value, which CUDA allows
  static std::atomic<bool> attr_done[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices || !attr_done[dev].load(std::memory_order_acquire)) {
    e = cudaFuncSetAttribute(gemm_sm100_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < kMaxDevices) attr_done[dev].store(true, std::memory_order_release);
  }
  // persistent: one CTA (pair) per SM (pair), never more than the tiles
  const int units = num_sms / C::CG;
  const int pairs = num_tiles < units ? num_tiles : units;
  if (pairs <= 0) return cudaSuccess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pairs * C::CG, 1, 1);
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C::CG;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = pdl_enabled() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, gemm_sm100_kernel<C>, p);
  count_launches(1);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

int up_partial_cols() {
  // fp8mlp_partial_amax_shape serves both up-projections: blocks of 32 rows
  // x 64 columns, whatever their epilogue warp counts
  static_assert(CfgUp::PA_PER_TILE == CfgUpQ::PA_PER_TILE && CfgUp::BN == CfgUpQ::BN &&
                    CfgUp::TILE_M == CfgUpQ::TILE_M,
                "the BF16 and e4m3 up-projections share one partial-amax layout");
  return CfgUp::BN / CfgUp::PA_PER_TILE;
}

int ce_partial_cols() {
  static_assert(CfgCeF::BN / CfgCeF::EPI_SPLIT == CfgCeF8::BN / CfgCeF8::EPI_SPLIT, "same partial layout");
  return CfgCeF::BN / CfgCeF::EPI_SPLIT;
}

int gemm_tile_m(GemmKind kind) {
  switch (kind) {
    case GemmKind::Up:
      return CfgUp::TILE_M;
    case GemmKind::Down8:
      return CfgDown8::TILE_M;
    case GemmKind::Bf16MnB:
      return CfgBf16MnB::TILE_M;
    case GemmKind::DPre:
      return CfgDPre::TILE_M;
    case GemmKind::DW:
      return CfgDW::TILE_M;
    case GemmKind::UpQ:
      return CfgUpQ::TILE_M;
    case GemmKind::CeFwd:
      return CfgCeF::TILE_M;
    case GemmKind::CeFwd8:
      return CfgCeF8::TILE_M;
    case GemmKind::CeBwd:
      return CfgCeB::TILE_M;
    case GemmKind::CeBwd8:
      return CfgCeB8::TILE_M;
  }
  return 128;
}

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
    case GemmKind::UpQ:
      return launch_one<CfgUpQ>(p, num_tiles, num_sms, s);
    case GemmKind::CeFwd:
      return launch_one<CfgCeF>(p, num_tiles, num_sms, s);
    case GemmKind::CeFwd8:
      return launch_one<CfgCeF8>(p, num_tiles, num_sms, s);
    case GemmKind::CeBwd:
      return launch_one<CfgCeB>(p, num_tiles, num_sms, s);
    case GemmKind::CeBwd8:
      return launch_one<CfgCeB8>(p, num_tiles, num_sms, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace fp8mlp
