// Warp-specialised, persistent tcgen05 GEMM with fused epilogues.
//
//   D[m, n] = sum_k A[m, k] * B[n, k]      (fp32 accumulate in TMEM)
//
// One CTA per SM (64 + 32*NEPI threads); with CG = 2 the CTAs of a cluster
// pair share a 2-CTA UMMA over a 256-row tile (each CTA loads its 128 rows of
// A and half of B; the leader issues the UMMA; each CTA drains its own 128
// TMEM lanes):
//   warp 0      TMA producer: streams A/B k-blocks into a STAGES-deep smem ring
//   warp 1      allocates 512 TMEM columns (two 256-column accumulators) and
//               issues the UMMAs from one thread
//   warps 2..   NEPI epilogue warps (4, 8 or 16): TMEM -> registers -> fused
//               math -> swizzled smem -> TMA store, 32 columns at a time; warp
//               w owns TMEM lanes 32*(w%4) .. +31 (tile rows 32*(w%4) .. +31)
//               and one of NEPI/4 column groups of the tile, so NEPI/4 warps
//               share each SM sub-partition
// The two accumulators let the epilogue of tile i overlap the mainloop of
// tile i+1.  Operands are BF16 (kind::f16) or e4m3 (kind::f8f6f4), each
// K-major or MN-major, staged with 128-byte swizzle.  TMA zero-fills rows and
// columns past the tensor edges and clips stores, so any M, N, K work.
#pragma once

#include "fp8mlp.h"
#include "sm100.cuh"

namespace fp8mlp {

enum class Epi : int {
  UpFused = 0,     // post = bf16(relu(pre)^2), q = e4m3(post*s), partial amax;
                   // pre = acc (BF16 inputs) or acc * s_x^-1 * s_w1^-1 (e4m3 inputs)
  DownScaled = 1,  // out = bf16(acc * s^-1 * s_w^-1)
  StoreBf16 = 2,   // out = bf16(acc)
  DPre = 3,        // dPre = bf16(2 sqrt(post) * acc), post read by TMA (hardware sqrt.approx)
  StoreF32 = 4,    // out = acc (fp32)
  CeFwd = 5,       // softcapped cross-entropy, forward: per row and column group the
                   // sum of exp(z - c), z = c tanh(y/c), and z at the row's targets;
                   // nothing [M,V] is written
  CeBwd = 6,       // softcapped cross-entropy, backward: dlogits = bf16(dL/dy)
};

struct alignas(64) GemmParams {
  CUtensorMap tmA[2];
  CUtensorMap tmB[2];
  CUtensorMap tmOut[2];
  CUtensorMap tmOut2;  // UpFused: post_fp8
  CUtensorMap tmAux;   // DPre: post
  int M, N, K;
  int tiles_m, tiles_n;
  int num_groups;
  int write_q;
  int pad0;
  float* partial_amax;
  float* pre_debug;
  const fp8mlp_scale_state* st;
  const float* w2_scale_inv;
  const fp8mlp_scale_state* st_in;  // UpFused on e4m3 inputs: x's delayed scale
  const float* w_in_scale_inv;      // UpFused on e4m3 inputs: 1 / s_w1
  unsigned int* status;
  unsigned long long timeout_ns;
  int debug_flags;
  int launch_flags;  // FP8MLP_LAUNCH_OVERLAP_PREVIOUS: wait for the previous grid only before finishing
  int n_major;       // tile order: 0 = row blocks outer (consecutive tiles share A), 1 = column blocks outer
  // softcapped cross-entropy (CeFwd / CeBwd); the logits are y = acc (BF16
  // inputs) or acc * s_x^-1 * s_w^-1 (e4m3 inputs, scales in st_in / w_in_scale_inv)
  int ce_T;                  // targets per row (1..4)
  int ce_mean;               // CeBwd: the reduced loss is the mean over the valid weights
  const int* ce_targets;     // [M, ce_T]; outside [0, N) = ignored
  float ce_w[4];             // target weights
  float ce_cap;              // c
  float ce_k;                // -2 log2(e) / c
  float ce_cl2;              // c log2(e)
  float* ce_partial;         // CeFwd: [tiles_n * EPI_SPLIT][M] sums of exp(z - c)
  float* ce_ztgt;            // CeFwd: [M, ce_T] z - c at each valid target
  const float* ce_lse;       // CeBwd: [M]
  const float* ce_loss;      // CeBwd: {sum, weight, mean} of the forward
  const float* ce_dloss;     // CeBwd: gradient of the reduced loss (NULL = 1)
};

template <int CG_, int BN_, int STAGES_, bool FP8_, bool A_MN_, bool B_MN_, Epi EPI_, int NEPI_ = 8,
          int AUX_RING_ = 4, int NSLOT_ = 2>
struct GemmCfg {
  static constexpr int CG = CG_;           // CTAs per UMMA (1, or 2 = the pair of a cluster)
  static constexpr int BM = 128;           // accumulator rows per CTA (TMEM lanes)
  static constexpr int TILE_M = BM * CG;   // rows of one output tile
  static constexpr int BN = BN_;           // columns of one output tile
  static constexpr int B_ROWS = BN / CG;   // rows of B (N) each CTA loads
  static constexpr int STAGES = STAGES_;
  static constexpr bool FP8 = FP8_;
  static constexpr bool A_MN = A_MN_;
  static constexpr bool B_MN = B_MN_;
  static constexpr Epi EPI = EPI_;
  static_assert(CG == 1 || CG == 2, "CTA group");
  static_assert(!(FP8 && (A_MN || B_MN)), "MN-major operands are BF16 only here");
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256 && B_ROWS % 64 == 0, "BN");
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int BK = 128 / ELEM;     // K elements per stage (one 128-byte swizzle row)
  static constexpr int UMMA_K = 32 / ELEM;  // K per UMMA instruction (32 bytes)
  static constexpr int A_BYTES = BM * BK * ELEM;
  static constexpr int B_BYTES = B_ROWS * BK * ELEM;
  static constexpr int STAGE_TX = CG * (A_BYTES + B_BYTES);  // bytes landing on the leader's barrier per stage
  // descriptor strides: K-major: 8-row groups 1024 B apart (LBO unused);
  // MN-major: 64-element MN atoms BK*128 B apart (LBO), 8-k-row groups 1024 B apart
  static constexpr uint32_t A_LBO = A_MN ? BK * 128 : 16;
  static constexpr uint32_t B_LBO = B_MN ? BK * 128 : 16;
  static constexpr uint32_t SBO = 1024;
  static constexpr uint32_t A_KSTEP = A_MN ? UMMA_K * 128 : UMMA_K * ELEM;
  static constexpr uint32_t B_KSTEP = B_MN ? UMMA_K * 128 : UMMA_K * ELEM;
  static constexpr uint32_t IDESC = dev::instr_desc(FP8 ? dev::FMT_E4M3 : dev::FMT_BF16,
                                                    FP8 ? dev::FMT_E4M3 : dev::FMT_BF16, A_MN, B_MN, TILE_M, BN);
  static constexpr int ECOLS = 32;
  static constexpr int NCHUNK = BN / ECOLS;      // 32-column chunks per tile row block
  static constexpr int NEPI = NEPI_;             // epilogue warps: NEPI/4 per TMEM lane quarter
  static constexpr int EPI_SPLIT = NEPI / 4;     // column groups per lane quarter
  static constexpr int NCH_W = NCHUNK / EPI_SPLIT;  // chunks per epilogue warp per tile
  static constexpr int THREADS = 64 + 32 * NEPI;
  static_assert(NEPI % 4 == 0 && NCHUNK % EPI_SPLIT == 0, "chunks per warp");
  // up-projection: partial-amax entries per tile row block of 32 (one per 64
  // columns: two chunks of one warp)
  static constexpr int PA_PER_TILE = BN / 64;
  static_assert(EPI != Epi::UpFused || NCH_W % 2 == 0, "whole 64-column blocks per warp");
  static constexpr bool STORES = EPI != Epi::CeFwd;  // the epilogue writes a tile with TMA
  static constexpr int OUT_BUF = !STORES ? 0 : 32 * ECOLS * (EPI == Epi::StoreF32 ? 4 : 2);
  static constexpr int OUT2_BUF = EPI == Epi::UpFused ? 32 * ECOLS : 0;
  static constexpr int SLOT = OUT_BUF + OUT2_BUF;  // one output staging slot
  // staging slots per epilogue warp: with 2 a chunk is written while the
  // previous chunk's store still reads the other slot; 1 leaves that shared
  // memory to the operand ring
  static constexpr int NSLOT = NSLOT_;
  static_assert(NSLOT == 1 || NSLOT == 2, "staging slots");
  static_assert(SLOT % 1024 == 0, "slot alignment");
  // DPre: each epilogue warp streams its 32x32 blocks of post through a ring
  // of NAUX slots of its own, loaded NAUX chunks ahead of use
  static constexpr int AUX_CHUNK = EPI == Epi::DPre ? 32 * ECOLS * 2 : 0;
  static constexpr int NAUX = EPI == Epi::DPre ? AUX_RING_ : 0;  // ring slots per warp
  static constexpr int AUX_WARP = AUX_CHUNK * NAUX;
  static_assert(NAUX == 0 || (NAUX <= NCH_W && NCH_W % (NAUX > 0 ? NAUX : 1) == 0), "post ring");
  static constexpr int TMEM_COLS = 512;
  static_assert(2 * BN <= TMEM_COLS, "two accumulators");
  static constexpr int NUM_BARS = 2 * STAGES + 4 + NEPI * NAUX + 1;
  static constexpr int SMEM_BYTES = 1024 /*alignment slack*/ + STAGES * (A_BYTES + B_BYTES) + NSLOT * NEPI * SLOT +
                                    NEPI * AUX_WARP + NUM_BARS * 8 + 16;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

namespace dev {

// Bounded wait that ignores the abort flag (used to drain in-flight copies).
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity, unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return;
  const unsigned long long t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit_ns) return;
  }
}

template <int ROWB>
__device__ __forceinline__ void store_row_bf16(uint32_t base, int lane, const uint32_t (&pk)[16]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    st_shared_v4(base + swz<3>(lane * 64 + j * 16), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
}

// Softcap z = c tanh(y/c), t = tanh(y/c), from e = exp(-2|y|/c) in (0, 1]
// and r = 1/(1+e):
//   t - 1 = -2 s r  with s = e (y >= 0) or 1 (y < 0),     1 - t^2 = 4 e r^2,
// so neither z - c = c (t - 1) nor the derivative loses digits to
// cancellation.  kd = -2 log2(e) / c times the dequantising factor of the
// accumulator (y = acc * dq, dq > 0), so e = 2^(kd |acc|).
// r is computed on the FMA pipe (the special-function unit, which also runs
// both exponentials, is the epilogue's bottleneck): a quadratic start with
// relative error < 1.02e-2 on e in [0, 1] and two Newton-Raphson steps
// r <- r + r (1 - (1+e) r), relative error < 1.4e-7 in fp32.
__device__ __forceinline__ void softcap_er(float acc, float kd, float& e, float& r) {
  e = ex2_approx(kd * fabsf(acc));
  const float x = 1.f + e;
  r = fmaf(fmaf(0.32321758f, e, -0.80804528f), e, 0.98988505f);
  r = fmaf(r, fmaf(-x, r, 1.f), r);
  r = fmaf(r, fmaf(-x, r, 1.f), r);
}

// softcap_er on the two accumulators (a0, a1) at once, packed: returns
// e = (e0, e1) and r = (r0, r1) as fp32 pairs; kd2 = (kd, kd)
__device__ __forceinline__ void softcap_er2(float a0, float a1, uint64_t kd2, uint64_t& e, uint64_t& r) {
  const uint64_t one = f2_pack(1.f, 1.f), m1 = f2_pack(-1.f, -1.f);
  float t0, t1;
  f2_unpack(f2_mul(f2_pack(fabsf(a0), fabsf(a1)), kd2), t0, t1);
  e = f2_pack(ex2_approx(t0), ex2_approx(t1));
  const uint64_t nx = f2_fma(e, m1, m1);  // -(1 + e)
  r = f2_fma(f2_fma(f2_pack(0.32321758f, 0.32321758f), e, f2_pack(-0.80804528f, -0.80804528f)), e,
             f2_pack(0.98988505f, 0.98988505f));
  r = f2_fma(r, f2_fma(nx, r, one), r);
  r = f2_fma(r, f2_fma(nx, r, one), r);
}

// s r of the pair, s = e (accumulator >= 0) or 1: t - 1 = -2 s r
__device__ __forceinline__ uint64_t softcap_sr2(float a0, float a1, uint64_t e, uint64_t r) {
  float e0, e1;
  f2_unpack(e, e0, e1);
  return f2_mul(f2_pack(a0 >= 0.f ? e0 : 1.f, a1 >= 0.f ? e1 : 1.f), r);
}

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace dev

// (row block, column block) of tile tt within its group.  With n_major the
// CTA pairs working at the same time share a column block, i.e. one B tile,
// which then leaves DRAM once even while a large output stream runs through
// L2; otherwise they share row blocks (A tiles).
__device__ __forceinline__ void tile_coords(const GemmParams& p, int tt, int& mb, int& nb) {
  if (p.n_major) {
    nb = tt / p.tiles_m;
    mb = tt - nb * p.tiles_m;
  } else {
    mb = tt / p.tiles_n;
    nb = tt - mb * p.tiles_n;
  }
}

template <class C>
__global__ void __launch_bounds__(C::THREADS, 1) gemm_sm100_kernel(const __grid_constant__ GemmParams p) {
  using namespace dev;
  constexpr int CG = C::CG;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint8_t* sA = smem;
  uint8_t* sB = sA + C::STAGES * C::A_BYTES;
  uint8_t* sEpi = sB + C::STAGES * C::B_BYTES;
  uint8_t* sAux = sEpi + C::NSLOT * C::NEPI * C::SLOT;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sAux + C::NEPI * C::AUX_WARP);
  uint64_t* full = bars;                // [STAGES] (the leader's are used)
  uint64_t* empty = bars + C::STAGES;   // [STAGES]
  uint64_t* tfull = bars + 2 * C::STAGES;
  uint64_t* tempty = tfull + 2;         // the leader's count both CTAs' epilogues
  uint64_t* auxb = tempty + 2;          // [NEPI warps][NAUX chunks]
  uint64_t* fin = auxb + C::NEPI * C::NAUX;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;  // position in the CTA pair
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x) / CG;
  const int npairs = static_cast<int>(gridDim.x) / CG;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], C::NEPI * CG);  // one arrival per epilogue warp of the pair
    }
    for (int i = 0; i < C::NEPI * C::NAUX; ++i) mbar_init(&auxb[i], 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc<CG>(tmem_holder, C::TMEM_COLS);
    tmem_relinquish<CG>();
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync();  // the peer's barriers are initialised
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // the set-up above overlaps the previous kernel's tail; from here on global
  // memory is read and written.  Every kernel of the library waits for its
  // predecessor before it lets its dependents launch, so when this grid
  // starts the grid two launches back has completed; a launch that reads and
  // writes nothing the previous grid writes or reads (the caller says so
  // with FP8MLP_LAUNCH_OVERLAP_PREVIOUS) can therefore run its tiles while
  // that grid drains, and waits for it only before finishing (so that
  // whatever waits for this grid also sees the previous one complete).  Such
  // a grid lets its own dependents launch only after that wait, which keeps
  // the two-launches-back guarantee for the next launch.
  const bool late_wait = (p.launch_flags & FP8MLP_LAUNCH_OVERLAP_PREVIOUS) != 0;
  if (!late_wait) {
    pdl_wait();
    if (threadIdx.x == 0) pdl_launch_dependents();
  }
  const WaitCtx w{p.status, abort_flag, p.timeout_ns};

  const int tiles_per_group = p.tiles_m * p.tiles_n;
  const int num_tiles = tiles_per_group * p.num_groups;
  const int num_kb = (p.K + C::BK - 1) / C::BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !(p.debug_flags & FP8MLP_DEBUG_STALL_PRODUCER)) {
      for (int g = 0; g < p.num_groups; ++g) {
        tma_prefetch_desc(&p.tmA[g]);
        tma_prefetch_desc(&p.tmB[g]);
      }
      uint32_t stage = 0, phase = 0;
      long long issued = 0;
      for (int t = pair; t < num_tiles; t += npairs) {
        const int g = t / tiles_per_group;
        const int tt = t - g * tiles_per_group;
        int mb, nb;
        tile_coords(p, tt, mb, nb);
        const int m0 = mb * C::TILE_M + static_cast<int>(rank) * C::BM;  // this CTA's A rows
        const int n0 = nb * C::BN + static_cast<int>(rank) * C::B_ROWS;  // this CTA's B rows
        const CUtensorMap* mA = &p.tmA[g];
        const CUtensorMap* mB = &p.tmB[g];
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, w)) {
            ok = false;
            break;
          }
          uint8_t* a = sA + stage * C::A_BYTES;
          uint8_t* b = sB + stage * C::B_BYTES;
          const int k0 = kb * C::BK;
          if constexpr (CG == 1) {
            mbar_arrive_expect_tx(&full[stage], C::STAGE_TX);
            if constexpr (C::A_MN) {
#pragma unroll
              for (int i = 0; i < C::BM / 64; ++i) tma_load_2d(a + i * C::BK * 128, mA, &full[stage], m0 + i * 64, k0);
            } else {
              tma_load_2d(a, mA, &full[stage], k0, m0);
            }
            if constexpr (C::B_MN) {
#pragma unroll
              for (int i = 0; i < C::B_ROWS / 64; ++i)
                tma_load_2d(b + i * C::BK * 128, mB, &full[stage], n0 + i * 64, k0);
            } else {
              tma_load_2d(b, mB, &full[stage], k0, n0);
            }
          } else {
            // both CTAs' copies complete on the leader's full barrier
            if (leader) mbar_arrive_expect_tx(&full[stage], C::STAGE_TX);
            const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
            if constexpr (C::A_MN) {
#pragma unroll
              for (int i = 0; i < C::BM / 64; ++i) tma_load_2d_cg2(a + i * C::BK * 128, mA, fb, m0 + i * 64, k0);
            } else {
              tma_load_2d_cg2(a, mA, fb, k0, m0);
            }
            if constexpr (C::B_MN) {
#pragma unroll
              for (int i = 0; i < C::B_ROWS / 64; ++i) tma_load_2d_cg2(b + i * C::BK * 128, mB, fb, n0 + i * 64, k0);
            } else {
              tma_load_2d_cg2(b, mB, fb, k0, n0);
            }
          }
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
      }
      // drain: the last copy into each stage must have landed before exit
      // (the leader's barrier sees both CTAs' copies)
      if (leader) {
        const long long n_drain = issued < C::STAGES ? issued : C::STAGES;
        for (long long i = 0; i < n_drain; ++i) {
          const long long n = issued - 1 - i;
          mbar_wait_drain(&full[n % C::STAGES], static_cast<uint32_t>((n / C::STAGES) & 1), p.timeout_ns);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (the pair's leader)
    if (lane == 0 && leader) {
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      for (int t = pair; t < num_tiles; t += npairs) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, w)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * C::BN;
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < C::BK / C::UMMA_K; ++k) {
            const uint64_t ad = smem_desc(a0 + k * C::A_KSTEP, C::A_LBO, C::SBO);
            const uint64_t bd = smem_desc(b0 + k * C::B_KSTEP, C::B_LBO, C::SBO);
            umma<CG, C::FP8>(d_tmem, ad, bd, C::IDESC, (kb | k) != 0 ? 1u : 0u);
          }
          if constexpr (CG == 1)
            tc_commit(&empty[stage]);
          else
            tc_commit_cg2_mc(&empty[stage], 0x3);  // frees the stage in both CTAs
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if constexpr (CG == 1)
          tc_commit(&tfull[acc]);
        else
          tc_commit_cg2_mc(&tfull[acc], 0x3);  // accumulator ready in both CTAs
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // every UMMA this thread issued must be complete before TMEM is freed
      if constexpr (CG == 1)
        tc_commit(fin);
      else
        tc_commit_cg2(fin);
      mbar_wait_drain(fin, 0, p.timeout_ns);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter == row block of 32 within this CTA's rows
    const int e = warp - 2;  // epilogue warp index
    const int half = e / 4;  // which column group of the tile this warp drains (< EPI_SPLIT)
    const int c_begin = half * C::NCH_W;
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    // arrivals that free an accumulator go to the leader's barrier
    const uint32_t tempty_addr0 = CG == 2 ? mapa_shared(smem_u32(&tempty[0]), 0) : 0u;
    uint32_t acc = 0, acc_phase = 0, ctr = 0;
    float s_up = 0.f, comb = 1.f;
    if constexpr (C::EPI == Epi::UpFused) {
      if (p.write_q) s_up = p.st->scale;
    }
    if constexpr (C::EPI == Epi::DownScaled) comb = __fmul_rn(p.st->scale_inv, *p.w2_scale_inv);
    // e4m3 up-projection: dequantise the accumulator before relu and the square
    float dq = 1.f;
    constexpr bool kCe = C::EPI == Epi::CeFwd || C::EPI == Epi::CeBwd;
    if constexpr ((C::EPI == Epi::UpFused || kCe) && C::FP8) dq = __fmul_rn(p.st_in->scale_inv, *p.w_in_scale_inv);
    // cross-entropy: the exponent constants (the e4m3 dequantising factor
    // folded into kd) and, backward, g, the factor of every row's gradient
    const float ce_kd = kCe ? p.ce_k * dq : 0.f;
    const float ce_K = -2.f * p.ce_cl2;
    float ce_g = 0.f;
    if constexpr (C::EPI == Epi::CeBwd) {
      ce_g = p.ce_dloss != nullptr ? *p.ce_dloss : 1.f;
      if (p.ce_mean) {
        const float ws = p.ce_loss[1];
        ce_g = ws > 0.f ? __fdiv_rn(ce_g, ws) : 0.f;
      }
    }
    // DPre: this warp's post chunks, counted over its tiles (chunk q = tile
    // iter, column chunk cw: q = iter * NCH_W + cw), go through ring slot
    // q % NAUX; aux_issued = chunks whose load has been issued
    uint32_t aux_issued = 0;
    uint8_t* aux_ring = sAux + e * C::AUX_WARP;
    uint64_t* my_auxb = auxb + e * C::NAUX;
    // test hook: issue no loads of post, so that the waits for them run out
    const bool stall_aux = (p.debug_flags & FP8MLP_DEBUG_STALL_AUX) != 0;
    auto tile_rows = [&](int tile) {  // first row of this warp's 32 rows in `tile`
      int mb2, nb2;
      tile_coords(p, tile - (tile / tiles_per_group) * tiles_per_group, mb2, nb2);
      return mb2 * C::TILE_M + static_cast<int>(rank) * C::BM + q * 32;
    };
    auto tile_cols = [&](int tile) {
      int mb2, nb2;
      tile_coords(p, tile - (tile / tiles_per_group) * tiles_per_group, mb2, nb2);
      return nb2 * C::BN;
    };
    if constexpr (C::EPI == Epi::DPre) {
      if (pair < num_tiles && !stall_aux) {
        const int r0 = tile_rows(pair), c0 = tile_cols(pair);
        if (lane == 0) {
          for (int c = 0; c < C::NAUX; ++c) {
            mbar_arrive_expect_tx(&my_auxb[c], C::AUX_CHUNK);
            tma_load_2d(aux_ring + c * C::AUX_CHUNK, &p.tmAux, &my_auxb[c], c0 + (c_begin + c) * C::ECOLS, r0);
          }
        }
        aux_issued = C::NAUX;
      }
    }
    uint32_t iter = 0;  // tiles processed by this CTA

    for (int t = pair; t < num_tiles; t += npairs) {
      const int g = t / tiles_per_group;
      const int tt = t - g * tiles_per_group;
      int mb, nb;
      tile_coords(p, tt, mb, nb);
      const int row0 = tile_rows(t);
      const int n0 = nb * C::BN;
      const int next_tile = t + npairs;
      // cross-entropy: this thread's row, its valid targets, and (backward)
      // (lse - c) log2(e) and g times the row's weight
      const int ce_m = row0 + lane;
      int ce_tg[4] = {-1, -1, -1, -1};
      float ce_sum = 0.f, ce_L = 0.f, ce_gw4 = 0.f;
      if constexpr (kCe) {
        if (ce_m < p.M) {
          float wsum = 0.f;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            if (t < p.ce_T) {
              const int tv = p.ce_targets[static_cast<size_t>(ce_m) * p.ce_T + t];
              if (tv >= 0 && tv < p.N) {
                ce_tg[t] = tv;
                wsum += p.ce_w[t];
              }
            }
          }
          if constexpr (C::EPI == Epi::CeBwd) {
            ce_L = __fmul_rn(__fsub_rn(p.ce_lse[ce_m], p.ce_cap), kLog2e);
            ce_gw4 = 4.f * __fmul_rn(ce_g, wsum);
          }
        }
      }
      if (!mbar_wait(&tfull[acc], acc_phase, w)) break;
      tc_fence_after();
      float tmax = 0.f;
      bool ok = true;
#pragma unroll 1
      for (int cw = 0; cw < C::NCH_W; ++cw) {
        const int c = c_begin + cw;  // chunk within the tile
        uint32_t v[32];
        tmem_ld32(tmem_base + lane_base + acc * C::BN + c * C::ECOLS, v);
        if (cw == C::NCH_W - 1) {
          // every lane's TMEM loads of this accumulator are complete (the load
          // waits); order them before the warp's single release to the MMA
          // issuer (a cluster-scope release per lane stalls on a memory barrier)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if constexpr (CG == 1)
              mbar_arrive(&tempty[acc]);
            else
              mbar_arrive_cluster(tempty_addr0 + acc * 8u);
          }
        }
        uint8_t* slot = sEpi + (e * C::NSLOT + (C::NSLOT == 2 ? (ctr & 1u) : 0u)) * C::SLOT;
        const uint32_t sbase = smem_u32(slot);
        if constexpr (C::STORES) {
          // the store issued from this slot NSLOT chunks ago has read it
          if (lane == 0) bulk_wait_read<C::NSLOT - 1>();
          __syncwarp();
        }
        const int col0 = n0 + c * C::ECOLS;

        if constexpr (C::EPI == Epi::UpFused) {
          uint32_t pk[16], qk[8];
          if constexpr (C::FP8) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__fmul_rn(__uint_as_float(v[i]), dq));
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a = fmaxf(__uint_as_float(v[2 * i]), 0.f);
            const float bb = fmaxf(__uint_as_float(v[2 * i + 1]), 0.f);
            const float sa = __fmul_rn(a, a), sb = __fmul_rn(bb, bb);
            tmax = fmaxf(tmax, fmaxf(sa, sb));
            pk[i] = pack_bf16x2(sa, sb);
          }
          store_row_bf16<64>(sbase, lane, pk);
          if (p.write_q) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t q0 = pack_e4m3x2(__fmul_rn(bf16lo_to_f32(pk[2 * i]), s_up),
                                              __fmul_rn(bf16hi_to_f32(pk[2 * i]), s_up));
              const uint32_t q1 = pack_e4m3x2(__fmul_rn(bf16lo_to_f32(pk[2 * i + 1]), s_up),
                                              __fmul_rn(bf16hi_to_f32(pk[2 * i + 1]), s_up));
              qk[i] = q0 | (q1 << 16);
            }
            const uint32_t qb = sbase + C::OUT_BUF;
#pragma unroll
            for (int j = 0; j < 2; ++j)
              st_shared_v4(qb + swz<1>(lane * 32 + j * 16), qk[4 * j], qk[4 * j + 1], qk[4 * j + 2], qk[4 * j + 3]);
          }
          if (p.pre_debug != nullptr) {
            const int m = row0 + lane;
            if (m < p.M) {
              float* dst = p.pre_debug + static_cast<size_t>(m) * p.N;
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (col0 + i < p.N) dst[col0 + i] = __uint_as_float(v[i]);
            }
          }
        } else if constexpr (C::EPI == Epi::DownScaled || C::EPI == Epi::StoreBf16) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float a = __uint_as_float(v[2 * i]), bb = __uint_as_float(v[2 * i + 1]);
            if constexpr (C::EPI == Epi::DownScaled) {
              a = __fmul_rn(a, comb);
              bb = __fmul_rn(bb, comb);
            }
            pk[i] = pack_bf16x2(a, bb);
          }
          store_row_bf16<64>(sbase, lane, pk);
        } else if constexpr (C::EPI == Epi::DPre) {
          // post of this chunk was loaded NAUX chunks ahead of its use into
          // ring slot q_aux % NAUX
          const uint32_t q_aux = iter * C::NCH_W + cw;
          const int slot_aux = static_cast<int>(q_aux % C::NAUX);
          if (!mbar_wait(&my_auxb[slot_aux], (q_aux / C::NAUX) & 1u, w)) {
            ok = false;
          } else {
            const uint32_t ab = smem_u32(aux_ring + slot_aux * C::AUX_CHUNK);
            uint32_t pp[16], pk[16];
#pragma unroll
            for (int j = 0; j < 4; ++j)
              ld_shared_v4(ab + swz<3>(lane * 64 + j * 16), pp[4 * j], pp[4 * j + 1], pp[4 * j + 2], pp[4 * j + 3]);
            __syncwarp();
            // the slot is free again: fetch chunk q + NAUX into it (column
            // chunk cw + NAUX of this tile, or of the next one)
            const int cw_n = cw + C::NAUX;
            const int t_n = cw_n < C::NCH_W ? t : next_tile;
            if (t_n < num_tiles && !stall_aux) {
              const int cn = cw_n < C::NCH_W ? cw_n : cw_n - C::NCH_W;
              if (lane == 0) {
                mbar_arrive_expect_tx(&my_auxb[slot_aux], C::AUX_CHUNK);
                tma_load_2d(aux_ring + slot_aux * C::AUX_CHUNK, &p.tmAux, &my_auxb[slot_aux],
                            tile_cols(t_n) + (c_begin + cn) * C::ECOLS, tile_rows(t_n));
              }
              aux_issued = q_aux + C::NAUX + 1;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float r0 = 2.f * sqrt_approx(bf16lo_to_f32(pp[i]));
              const float r1 = 2.f * sqrt_approx(bf16hi_to_f32(pp[i]));
              pk[i] = pack_bf16x2(__fmul_rn(r0, __uint_as_float(v[2 * i])), __fmul_rn(r1, __uint_as_float(v[2 * i + 1])));
            }
            store_row_bf16<64>(sbase, lane, pk);
          }
        } else if constexpr (C::EPI == Epi::CeFwd) {
          // sum over the chunk's columns inside the vocabulary of exp(z - c) =
          // 2^(c log2(e) (t - 1)) = 2^(K s r), K = -2 c log2(e); |z| <= c keeps
          // every term in [e^-2c, 1]
          // (pairs of columns in packed fp32)
          const uint64_t kd2 = f2_pack(ce_kd, ce_kd), K2 = f2_pack(ce_K, ce_K);
          uint64_t csum2 = f2_pack(0.f, 0.f);
          if (col0 + 32 <= p.N) {
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float a0 = __uint_as_float(v[i]), a1 = __uint_as_float(v[i + 1]);
              uint64_t e2, r2;
              softcap_er2(a0, a1, kd2, e2, r2);
              float g0, g1;
              f2_unpack(f2_mul(softcap_sr2(a0, a1, e2, r2), K2), g0, g1);
              csum2 = f2_add(csum2, f2_pack(ex2_approx(g0), ex2_approx(g1)));
            }
          } else {  // the vocabulary's last, partial chunk
            const int nvalid = p.N - col0;
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float a0 = __uint_as_float(v[i]), a1 = __uint_as_float(v[i + 1]);
              uint64_t e2, r2;
              softcap_er2(a0, a1, kd2, e2, r2);
              float g0, g1;
              f2_unpack(f2_mul(softcap_sr2(a0, a1, e2, r2), K2), g0, g1);
              csum2 = f2_add(csum2, f2_pack(i < nvalid ? ex2_approx(g0) : 0.f, i + 1 < nvalid ? ex2_approx(g1) : 0.f));
            }
          }
          float cs0, cs1;
          f2_unpack(csum2, cs0, cs1);
          ce_sum += cs0 + cs1;
          // z - c = -2c s r at the row's targets that fall in this chunk (one
          // thread in the grid owns each (row, target))
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int off = ce_tg[t] - col0;
            if (off >= 0 && off < 32) {
              float av = 0.f;
#pragma unroll
              for (int i = 0; i < 32; ++i) av = i == off ? __uint_as_float(v[i]) : av;
              float ee, rr;
              softcap_er(av, ce_kd, ee, rr);
              p.ce_ztgt[static_cast<size_t>(ce_m) * p.ce_T + t] = (-2.f * p.ce_cap) * ((av >= 0.f ? ee : 1.f) * rr);
            }
          }
        } else if constexpr (C::EPI == Epi::CeBwd) {
          // dL/dy = g (W_m softmax(z) - sum_t w_t onehot(tgt_t)) (1 - t^2),
          // softmax(z) = 2^(K s r - (lse - c) log2(e)),  1 - t^2 = 4 e r^2
          // (pairs of columns in packed fp32)
          float dy[32];
          const uint64_t kd2 = f2_pack(ce_kd, ce_kd), K2 = f2_pack(ce_K, ce_K);
          const uint64_t nL2 = f2_pack(-ce_L, -ce_L), gw2 = f2_pack(ce_gw4, ce_gw4);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float a0 = __uint_as_float(v[i]), a1 = __uint_as_float(v[i + 1]);
            uint64_t e2, r2;
            softcap_er2(a0, a1, kd2, e2, r2);
            float g0, g1;
            f2_unpack(f2_fma(K2, softcap_sr2(a0, a1, e2, r2), nL2), g0, g1);
            const uint64_t prob = f2_pack(ex2_approx(g0), ex2_approx(g1));  // exp(z - lse)
            const uint64_t der = f2_mul(f2_mul(e2, r2), r2);                // (1 - t^2) / 4
            f2_unpack(f2_mul(f2_mul(gw2, prob), der), dy[i], dy[i + 1]);
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int off = ce_tg[t] - col0;
            if (off >= 0 && off < 32) {
              float av = 0.f;
#pragma unroll
              for (int i = 0; i < 32; ++i) av = i == off ? __uint_as_float(v[i]) : av;
              float ee, rr;
              softcap_er(av, ce_kd, ee, rr);
              const float sub = (4.f * ce_g * p.ce_w[t]) * ((ee * rr) * rr);
#pragma unroll
              for (int i = 0; i < 32; ++i) dy[i] = i == off ? dy[i] - sub : dy[i];
            }
          }
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(dy[2 * i], dy[2 * i + 1]);
          store_row_bf16<64>(sbase, lane, pk);
        } else {  // StoreF32
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(sbase + swz<7>(lane * 128 + j * 16), v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
        if (!ok) break;
        if constexpr (C::STORES) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&p.tmOut[g], slot, col0, row0);
            if constexpr (C::EPI == Epi::UpFused) {
              if (p.write_q) tma_store_2d(&p.tmOut2, slot + C::OUT_BUF, col0, row0);
            }
            bulk_commit();
          }
        }
        if constexpr (C::EPI == Epi::UpFused) {
          if (cw & 1) {
            // this warp's 32 rows x 64 columns of post are complete: one
            // partial-amax entry (row block of 32, column block of 64)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
            if (lane == 0)
              p.partial_amax[((mb * CG + static_cast<int>(rank)) * 4 + q) * (p.tiles_n * C::PA_PER_TILE) +
                             nb * C::PA_PER_TILE + (c >> 1)] = round_bf16(tmax);
            tmax = 0.f;
          }
        }
        ++ctr;
      }
      if (!ok) break;
      if constexpr (C::EPI == Epi::CeFwd) {
        if (ce_m < p.M) p.ce_partial[static_cast<size_t>(nb * C::EPI_SPLIT + half) * p.M + ce_m] = ce_sum;
      }
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
      ++iter;
    }
    if (lane == 0) {
      if constexpr (C::EPI == Epi::DPre) {
        // the last load issued into each ring slot must have landed before exit
        for (uint32_t c = 0; c < static_cast<uint32_t>(C::NAUX); ++c) {
          if (aux_issued > c) {
            const uint32_t q_last = c + ((aux_issued - 1u - c) / C::NAUX) * C::NAUX;  // last chunk in slot c
            mbar_wait_drain(&my_auxb[c], (q_last / C::NAUX) & 1u, p.timeout_ns);
          }
        }
      }
      bulk_wait<0>();
    }
    __syncwarp();
  }

  __syncwarp();
  if (late_wait && threadIdx.x == 0) {
    pdl_wait();
    pdl_launch_dependents();
  }
  __syncthreads();
  // no CTA of a pair leaves while its peer may still read its shared memory
  // or arrive on its barriers; TMEM is freed by both CTAs together
  if constexpr (CG == 2) cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc<CG>(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace fp8mlp
