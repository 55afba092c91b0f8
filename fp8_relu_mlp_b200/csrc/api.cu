// C-ABI entry points: argument checks on the host, tensor-map encoding, and
// the launches.  See include/fp8mlp.h for the contract of each call.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "internal.h"

#define FP8MLP_VERSION_STRING "fp8mlp 0.1.0 (sm_100a)"

namespace fp8mlp {
namespace {

thread_local std::string g_detail;
std::atomic<unsigned long long> g_launches{0};
std::atomic<unsigned long long> g_timeout_ns{2000000000ull};
std::atomic<int> g_debug_flags{0};
std::atomic<int> g_pdl{1};

int fail(int code, const std::string& what) {
  g_detail = what;
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  g_detail = std::string(where) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")";
  return FP8MLP_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE_PTR(p)                                                                     \
  do {                                                                                     \
    if ((p) == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, #p " is NULL");                \
    if (!aligned16(p)) return fail(FP8MLP_ERR_INVALID_ARG, #p " is not 16-byte aligned"); \
  } while (0)

int check_launch_flags(int flags) {
  if (flags & ~FP8MLP_LAUNCH_OVERLAP_PREVIOUS) return fail(FP8MLP_ERR_INVALID_ARG, "unknown launch flags");
  return FP8MLP_OK;
}

int check_dims(int M, int d, int h) {
  if (M < 0) return fail(FP8MLP_ERR_INVALID_ARG, "M < 0");
  if (d < 16 || h < 16) return fail(FP8MLP_ERR_UNSUPPORTED_SHAPE, "d and h must be >= 16");
  if (d % 16 != 0 || h % 16 != 0) return fail(FP8MLP_ERR_UNSUPPORTED_SHAPE, "d and h must be multiples of 16");
  return FP8MLP_OK;
}

// ---- device info --------------------------------------------------------
constexpr int kMaxDevices = 64;
// filled once per device under g_dev_mutex; g_dev_ok (release / acquire)
// lets later calls from any thread read the entry without the lock
DeviceInfo g_dev[kMaxDevices];
std::atomic<bool> g_dev_ok[kMaxDevices] = {};
std::mutex g_dev_mutex;

// ---- tensor maps ---------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D row-major tensor [outer, inner] of `esize`-byte elements, dense rows.
int map2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, uint64_t inner, uint64_t outer,
          uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz, const char* what) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(FP8MLP_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * static_cast<uint64_t>(esize)};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    char buf[160];
    snprintf(buf, sizeof(buf), "tensor map for %s failed (CUresult %d)", what, static_cast<int>(r));
    return fail(FP8MLP_ERR_CUDA, buf);
  }
  return FP8MLP_OK;
}

constexpr CUtensorMapDataType BF16 = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
constexpr CUtensorMapDataType U8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
constexpr CUtensorMapDataType F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
constexpr CUtensorMapSwizzle SW128 = CU_TENSOR_MAP_SWIZZLE_128B;
constexpr CUtensorMapSwizzle SW64 = CU_TENSOR_MAP_SWIZZLE_64B;
constexpr CUtensorMapSwizzle SW32 = CU_TENSOR_MAP_SWIZZLE_32B;

// operand maps: K-major [rows, K] or MN-major [K, cols]
int map_kmajor(CUtensorMap* m, const void* p, CUtensorMapDataType dt, int esize, int rows, int K, int box_rows,
               const char* what) {
  return map2d(m, p, dt, esize, K, rows, 128 / esize, box_rows, SW128, what);
}
int map_mnmajor(CUtensorMap* m, const void* p, int K, int cols, const char* what) {
  return map2d(m, p, BF16, 2, cols, K, 64, 64, SW128, what);
}
// 32x32 output/aux tiles of an [rows, cols] tensor
int map_tile32(CUtensorMap* m, const void* p, CUtensorMapDataType dt, int esize, int rows, int cols,
               const char* what) {
  const CUtensorMapSwizzle swz = esize == 4 ? SW128 : (esize == 2 ? SW64 : SW32);
  return map2d(m, p, dt, esize, cols, rows, 32, 32, swz, what);
}

#define TRY(x)                           \
  do {                                   \
    const int rc_ = (x);                 \
    if (rc_ != FP8MLP_OK) return rc_;    \
  } while (0)

int cdiv(int a, int b) { return (a + b - 1) / b; }

void fill_common(GemmParams& p, GemmKind kind, const DeviceInfo* di, int M, int N, int K, int groups) {
  p.M = M;
  p.N = N;
  p.K = K;
  p.tiles_m = cdiv(M, gemm_tile_m(kind));
  p.tiles_n = cdiv(N, kGemmBN);
  p.num_groups = groups;
  p.status = di->status;
  p.timeout_ns = g_timeout_ns.load();
  p.debug_flags = g_debug_flags.load();
}

int launch(GemmKind k, const GemmParams& p, const DeviceInfo* di, cudaStream_t s, const char* what) {
  const cudaError_t e = launch_gemm(k, p, p.tiles_m * p.tiles_n * p.num_groups, di->num_sms, s);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return FP8MLP_OK;
}

}  // namespace

void count_launches(unsigned long long n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

void set_error_detail(const char* what) { g_detail = what; }

bool pdl_enabled() { return g_pdl.load(std::memory_order_relaxed) != 0; }

int current_device(DeviceInfo** info) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(FP8MLP_ERR_NO_DEVICE, std::string("no CUDA device: ") + cudaGetErrorString(e));
  }
  if (dev < 0 || dev >= kMaxDevices) return fail(FP8MLP_ERR_NO_DEVICE, "device index out of range");
  if (!g_dev_ok[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (g_dev_ok[dev].load(std::memory_order_relaxed)) {
      *info = &g_dev[dev];
      return FP8MLP_OK;
    }
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      cudaGetLastError();
      return fail(FP8MLP_ERR_NO_DEVICE, "cannot query the current device");
    }
    if (major != 10 || minor != 0) {
      char buf[96];
      snprintf(buf, sizeof(buf), "device %d has compute capability %d.%d; sm_100a (10.0) is required", dev, major,
               minor);
      return fail(FP8MLP_ERR_NO_DEVICE, buf);
    }
    unsigned int* st = nullptr;
    e = status_word_address(&st);
    if (e != cudaSuccess) return cuda_fail(e, "status word");
    g_dev[dev].device = dev;
    g_dev[dev].num_sms = sms;
    g_dev[dev].status = st;
    g_dev_ok[dev].store(true, std::memory_order_release);
  }
  *info = &g_dev[dev];
  return FP8MLP_OK;
}

}  // namespace fp8mlp

using namespace fp8mlp;

namespace {

// ---- softcapped cross-entropy: workspace layout and shared checks ----------
struct CeLayout {
  int nblk = 0;    // row blocks of the row pass
  int nparts = 0;  // partial sums per row (128-column groups, whole tiles)
  size_t off_partial = 0, off_ztgt = 0, total = 0;
};

CeLayout ce_layout(int M, int V, int T) {
  auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  CeLayout L;
  L.nblk = cdiv(M, kCeRowsPerBlock);
  L.nparts = cdiv(V, kGemmBN) * (kGemmBN / ce_partial_cols());
  // [block sums: 2 doubles per row block][partials: nparts x M][z - c at targets: M x T]
  L.off_partial = al(sizeof(double) * 2 * static_cast<size_t>(L.nblk));
  L.off_ztgt = L.off_partial + al(sizeof(float) * static_cast<size_t>(L.nparts) * M);
  L.total = L.off_ztgt + al(sizeof(float) * static_cast<size_t>(M) * T);
  return L;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

#define REQUIRE_PTR4(p)                                                                   \
  do {                                                                                    \
    if ((p) == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, #p " is NULL");               \
    if (!aligned4(p)) return fail(FP8MLP_ERR_INVALID_ARG, #p " is not 4-byte aligned");  \
  } while (0)

// shape, cap and weight checks; fills p's cross-entropy fields
int ce_setup(int M, int d, int V, int T, const int32_t* targets, const float* target_weights, float softcap,
             GemmParams* p) {
  TRY(check_dims(M, d, V));
  if (T < 1 || T > 4) return fail(FP8MLP_ERR_INVALID_ARG, "T (targets per row) must be 1..4");
  if (!(softcap > 0.f && softcap <= 40.f)) return fail(FP8MLP_ERR_INVALID_ARG, "softcap must be in (0, 40]");
  for (int t = 0; t < 4; ++t) {
    const float w = t >= T ? 0.f : (target_weights != nullptr ? target_weights[t] : 1.f);
    if (!std::isfinite(w)) return fail(FP8MLP_ERR_INVALID_ARG, "target weights must be finite");
    p->ce_w[t] = w;
  }
  if (M > 0) REQUIRE_PTR4(targets);
  p->ce_T = T;
  p->ce_targets = targets;
  p->ce_cap = softcap;
  const double log2e = 1.4426950408889634;
  p->ce_k = static_cast<float>(-2.0 * log2e / softcap);
  p->ce_cl2 = static_cast<float>(softcap * log2e);
  return FP8MLP_OK;
}

int ce_fwd_impl(bool fp8, int M, int d, int V, int T, const void* x, const void* W, const fp8mlp_scale_state* st_x,
                const float* w_scale_inv, const int32_t* targets, const float* target_weights, float softcap,
                float* lse, float* row_loss, float* loss, void* workspace, cudaStream_t stream) {
  GemmParams p{};
  TRY(ce_setup(M, d, V, T, targets, target_weights, softcap, &p));
  REQUIRE_PTR4(loss);
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  if (M == 0) {
    const cudaError_t e = cudaMemsetAsync(loss, 0, 3 * sizeof(float), stream);
    return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "ce_fwd memset");
  }
  REQUIRE_PTR(x);
  REQUIRE_PTR(W);
  REQUIRE_PTR(workspace);
  REQUIRE_PTR4(lse);
  if (row_loss != nullptr) REQUIRE_PTR4(row_loss);
  const GemmKind kind = fp8 ? GemmKind::CeFwd8 : GemmKind::CeFwd;
  const CUtensorMapDataType dt = fp8 ? U8 : BF16;
  const int es = fp8 ? 1 : 2;
  if (fp8) {
    REQUIRE_PTR(st_x);
    if (w_scale_inv == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "w_scale_inv is NULL");
    p.st_in = st_x;
    p.w_in_scale_inv = w_scale_inv;
  }
  TRY(map_kmajor(&p.tmA[0], x, dt, es, M, d, kGemmBM, "x"));
  TRY(map_kmajor(&p.tmB[0], W, dt, es, V, d, kGemmBN * kGemmBM / gemm_tile_m(kind), "W"));
  fill_common(p, kind, di, M, V, d, 1);
  const CeLayout L = ce_layout(M, V, T);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.ce_partial = reinterpret_cast<float*>(ws + L.off_partial);
  p.ce_ztgt = reinterpret_cast<float*>(ws + L.off_ztgt);
  TRY(launch(kind, p, di, stream, "ce_fwd launch"));
  const cudaError_t e = launch_ce_finalize(M, L.nparts, T, V, targets, p.ce_w, softcap, p.ce_partial, p.ce_ztgt,
                                           lse, row_loss, reinterpret_cast<double*>(ws), loss, stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "ce_fwd finalize launch");
}

int ce_bwd_impl(bool fp8, int M, int d, int V, int T, const void* x, const void* W, const fp8mlp_scale_state* st_x,
                const float* w_scale_inv, const int32_t* targets, const float* target_weights, float softcap,
                const float* lse, const float* loss, const float* dloss, int reduction, uint16_t* dlogits,
                cudaStream_t stream) {
  GemmParams p{};
  TRY(ce_setup(M, d, V, T, targets, target_weights, softcap, &p));
  if (reduction != FP8MLP_CE_SUM && reduction != FP8MLP_CE_MEAN)
    return fail(FP8MLP_ERR_INVALID_ARG, "reduction must be FP8MLP_CE_SUM or FP8MLP_CE_MEAN");
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(x);
  REQUIRE_PTR(W);
  REQUIRE_PTR(dlogits);
  REQUIRE_PTR4(lse);
  REQUIRE_PTR4(loss);
  if (dloss != nullptr) REQUIRE_PTR4(dloss);
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const GemmKind kind = fp8 ? GemmKind::CeBwd8 : GemmKind::CeBwd;
  const CUtensorMapDataType dt = fp8 ? U8 : BF16;
  const int es = fp8 ? 1 : 2;
  if (fp8) {
    REQUIRE_PTR(st_x);
    if (w_scale_inv == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "w_scale_inv is NULL");
    p.st_in = st_x;
    p.w_in_scale_inv = w_scale_inv;
  }
  TRY(map_kmajor(&p.tmA[0], x, dt, es, M, d, kGemmBM, "x"));
  TRY(map_kmajor(&p.tmB[0], W, dt, es, V, d, kGemmBN * kGemmBM / gemm_tile_m(kind), "W"));
  TRY(map_tile32(&p.tmOut[0], dlogits, BF16, 2, M, V, "dlogits"));
  fill_common(p, kind, di, M, V, d, 1);
  // the pairs at work share one vocabulary tile of the head, which then stays
  // in L2 while the dlogits stream passes through
  p.n_major = 1;
  p.ce_lse = lse;
  p.ce_loss = loss;
  p.ce_dloss = dloss;
  p.ce_mean = reduction == FP8MLP_CE_MEAN ? 1 : 0;
  return launch(kind, p, di, stream, "ce_bwd_dlogits launch");
}

}  // namespace

extern "C" {

int fp8mlp_partial_amax_shape(int M, int h, int* row_blocks, int* col_blocks, int* block_rows, int* block_cols) {
  if (M < 0 || h < 0) return fail(FP8MLP_ERR_INVALID_ARG, "negative size");
  const int tm = gemm_tile_m(GemmKind::Up);
  if (row_blocks) *row_blocks = (tm / 32) * cdiv(M, tm);
  const int pc = up_partial_cols();
  if (col_blocks) *col_blocks = cdiv(h, kGemmBN) * (kGemmBN / pc);
  if (block_rows) *block_rows = kGemmBM / 4;
  if (block_cols) *block_cols = pc;
  return FP8MLP_OK;
}

int fp8mlp_partial_amax_count(int M, int h) {
  if (M < 0 || h < 0) return 0;
  int rb = 0, cb = 0;
  fp8mlp_partial_amax_shape(M, h, &rb, &cb, nullptr, nullptr);
  return rb * cb;
}

size_t fp8mlp_workspace_size(int M, int d, int h) {
  (void)M;
  if (d <= 0 || h <= 0) return 256;
  // W2 cache refresh: one 4-byte partial maximum per kW2ElemsPerBlock elements
  const long long n = static_cast<long long>(h) * d;
  const size_t need = 4 * static_cast<size_t>((n + kW2ElemsPerBlock - 1) / kW2ElemsPerBlock);
  return need < 256 ? 256 : ((need + 255) / 256) * 256;
}

int fp8mlp_up_proj_fused(int M, int d, int h, const uint16_t* x, const uint16_t* W1, const fp8mlp_scale_state* st,
                         uint16_t* post, uint8_t* post_fp8, float* partial_amax, float* pre_debug, int flags,
                         fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, h));
  if (flags & ~(FP8MLP_FWD_EVAL_BF16 | FP8MLP_FWD_CALIBRATE)) return fail(FP8MLP_ERR_INVALID_ARG, "unknown flags");
  const bool write_q = (flags & (FP8MLP_FWD_EVAL_BF16 | FP8MLP_FWD_CALIBRATE)) == 0;
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(x);
  REQUIRE_PTR(W1);
  REQUIRE_PTR(post);
  if (partial_amax == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "partial_amax is NULL");
  if (reinterpret_cast<uintptr_t>(partial_amax) & 3u) return fail(FP8MLP_ERR_INVALID_ARG, "partial_amax misaligned");
  if (write_q) {
    REQUIRE_PTR(post_fp8);
    REQUIRE_PTR(st);
  }
  if (pre_debug != nullptr && (reinterpret_cast<uintptr_t>(pre_debug) & 3u))
    return fail(FP8MLP_ERR_INVALID_ARG, "pre_debug misaligned");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  GemmParams p{};
  TRY(map_kmajor(&p.tmA[0], x, BF16, 2, M, d, kGemmBM, "x"));
  TRY(map_kmajor(&p.tmB[0], W1, BF16, 2, h, d, kGemmBN * kGemmBM / gemm_tile_m(GemmKind::Up), "W1"));
  TRY(map_tile32(&p.tmOut[0], post, BF16, 2, M, h, "post"));
  if (write_q) TRY(map_tile32(&p.tmOut2, post_fp8, U8, 1, M, h, "post_fp8"));
  fill_common(p, GemmKind::Up, di, M, h, d, 1);
  p.write_q = write_q ? 1 : 0;
  p.partial_amax = partial_amax;
  p.pre_debug = pre_debug;
  p.st = st;
  return launch(GemmKind::Up, p, di, stream, "up_proj_fused launch");
}

int fp8mlp_down_proj_fp8(int M, int d, int h, const uint8_t* post_fp8, const uint8_t* W2q_t,
                         const float* w2_scale_inv, const fp8mlp_scale_state* st, uint16_t* out,
                         fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, h));
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(post_fp8);
  REQUIRE_PTR(W2q_t);
  REQUIRE_PTR(out);
  REQUIRE_PTR(st);
  if (w2_scale_inv == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "w2_scale_inv is NULL");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  GemmParams p{};
  TRY(map_kmajor(&p.tmA[0], post_fp8, U8, 1, M, h, kGemmBM, "post_fp8"));
  TRY(map_kmajor(&p.tmB[0], W2q_t, U8, 1, d, h, kGemmBN * kGemmBM / gemm_tile_m(GemmKind::Down8), "W2q_t"));
  TRY(map_tile32(&p.tmOut[0], out, BF16, 2, M, d, "out"));
  fill_common(p, GemmKind::Down8, di, M, d, h, 1);
  p.st = st;
  p.w2_scale_inv = w2_scale_inv;
  return launch(GemmKind::Down8, p, di, stream, "down_proj_fp8 launch");
}

int fp8mlp_down_proj_bf16(int M, int d, int h, const uint16_t* post, const uint16_t* W2, uint16_t* out,
                          fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, h));
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(post);
  REQUIRE_PTR(W2);
  REQUIRE_PTR(out);
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  GemmParams p{};
  TRY(map_kmajor(&p.tmA[0], post, BF16, 2, M, h, kGemmBM, "post"));
  TRY(map_mnmajor(&p.tmB[0], W2, h, d, "W2"));
  TRY(map_tile32(&p.tmOut[0], out, BF16, 2, M, d, "out"));
  fill_common(p, GemmKind::Bf16MnB, di, M, d, h, 1);
  return launch(GemmKind::Bf16MnB, p, di, stream, "down_proj_bf16 launch");
}

int fp8mlp_mlp_fwd(int M, int d, int h, const uint16_t* x, const uint16_t* W1, const uint8_t* W2q_t,
                   const float* w2_scale_inv, const uint16_t* W2, const fp8mlp_scale_state* st, uint16_t* post,
                   uint8_t* post_fp8, float* partial_amax, uint16_t* out, float* pre_debug, int flags,
                   fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, h));
  if ((flags & FP8MLP_FWD_EVAL_BF16) && (flags & FP8MLP_FWD_CALIBRATE))
    return fail(FP8MLP_ERR_INVALID_ARG, "EVAL_BF16 and CALIBRATE are exclusive");
  if (M == 0) return FP8MLP_OK;
  // check the down-projection's arguments before anything is enqueued
  if (flags & FP8MLP_FWD_EVAL_BF16) {
    REQUIRE_PTR(W2);
    REQUIRE_PTR(out);
  } else if (!(flags & FP8MLP_FWD_CALIBRATE)) {
    REQUIRE_PTR(W2q_t);
    REQUIRE_PTR(out);
    if (w2_scale_inv == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "w2_scale_inv is NULL");
  }
  TRY(fp8mlp_up_proj_fused(M, d, h, x, W1, st, post, post_fp8, partial_amax, pre_debug, flags, stream));
  if (flags & FP8MLP_FWD_CALIBRATE) return FP8MLP_OK;
  if (flags & FP8MLP_FWD_EVAL_BF16) return fp8mlp_down_proj_bf16(M, d, h, post, W2, out, stream);
  return fp8mlp_down_proj_fp8(M, d, h, post_fp8, W2q_t, w2_scale_inv, st, out, stream);
}

int fp8mlp_scale_state_init(fp8mlp_scale_state* st, float margin, float initial_scale, fp8mlp_stream_t stream) {
  g_detail.clear();
  REQUIRE_PTR(st);
  if (!(margin > 0.f) || !std::isfinite(margin)) return fail(FP8MLP_ERR_INVALID_ARG, "margin must be finite and > 0");
  if (!(initial_scale > 0.f) || !std::isfinite(initial_scale))
    return fail(FP8MLP_ERR_INVALID_ARG, "initial_scale must be finite and > 0");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const cudaError_t e = launch_state_init(st, margin, initial_scale, stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "scale_state_init launch");
}

int fp8mlp_amax_reduce_update_scale(const float* partial_amax, int n, fp8mlp_scale_state* st,
                                    fp8mlp_stream_t stream) {
  g_detail.clear();
  if (n < 0) return fail(FP8MLP_ERR_INVALID_ARG, "n < 0");
  REQUIRE_PTR(st);
  if (n > 0 && partial_amax == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "partial_amax is NULL");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const cudaError_t e = launch_amax_scale(partial_amax, n, st, di->status, stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "amax_reduce_update_scale launch");
}

int fp8mlp_w2_fp8_cache_refresh(int h, int d, const uint16_t* W2, uint8_t* W2q_t, float* w2_scale_inv,
                                void* workspace, fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(0, d, h));
  REQUIRE_PTR(W2);
  REQUIRE_PTR(W2q_t);
  REQUIRE_PTR(workspace);
  if (w2_scale_inv == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "w2_scale_inv is NULL");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const cudaError_t e = launch_w2_cache(h, d, W2, W2q_t, w2_scale_inv, static_cast<unsigned int*>(workspace),
                                        di->status, di->num_sms, stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "w2_fp8_cache_refresh launch");
}

int fp8mlp_x_partial_amax_count(int M, int d) {
  if (M < 0 || d < 0) return 0;
  const long long n = static_cast<long long>(M) * d;
  return static_cast<int>((n + kXElemsPerBlock - 1) / kXElemsPerBlock);
}

int fp8mlp_quantize_x(int M, int d, const uint16_t* x, const fp8mlp_scale_state* st_x, uint8_t* x_fp8,
                      float* partial_amax_x, fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, 16));
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(x);
  REQUIRE_PTR(st_x);
  REQUIRE_PTR(x_fp8);
  if (partial_amax_x == nullptr || (reinterpret_cast<uintptr_t>(partial_amax_x) & 3u))
    return fail(FP8MLP_ERR_INVALID_ARG, "partial_amax_x is NULL or misaligned");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const cudaError_t e = launch_quantize_x(static_cast<long long>(M) * d, x, st_x, x_fp8, partial_amax_x, stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "quantize_x launch");
}

int fp8mlp_weight_fp8_cache_refresh(int N, int K, const uint16_t* W, uint8_t* Wq, float* w_scale_inv,
                                    void* workspace, fp8mlp_stream_t stream) {
  return fp8mlp_w1_fp8_cache_refresh(N, K, W, Wq, w_scale_inv, workspace, stream);
}

int fp8mlp_w1_fp8_cache_refresh(int h, int d, const uint16_t* W1, uint8_t* W1q, float* w1_scale_inv,
                                void* workspace, fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(0, d, h));
  REQUIRE_PTR(W1);
  REQUIRE_PTR(W1q);
  REQUIRE_PTR(workspace);
  if (w1_scale_inv == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "w1_scale_inv is NULL");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const cudaError_t e = launch_w1_cache(h, d, W1, W1q, w1_scale_inv, static_cast<unsigned int*>(workspace),
                                        di->status, stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "w1_fp8_cache_refresh launch");
}

int fp8mlp_up_proj_fused_fp8(int M, int d, int h, const uint8_t* x_fp8, const uint8_t* W1q,
                             const float* w1_scale_inv, const fp8mlp_scale_state* st_x, const fp8mlp_scale_state* st,
                             uint16_t* post, uint8_t* post_fp8, float* partial_amax, float* pre_debug, int flags,
                             fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, h));
  if (flags & ~(FP8MLP_FWD_EVAL_BF16 | FP8MLP_FWD_CALIBRATE)) return fail(FP8MLP_ERR_INVALID_ARG, "unknown flags");
  const bool write_q = (flags & (FP8MLP_FWD_EVAL_BF16 | FP8MLP_FWD_CALIBRATE)) == 0;
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(x_fp8);
  REQUIRE_PTR(W1q);
  REQUIRE_PTR(st_x);
  REQUIRE_PTR(post);
  if (w1_scale_inv == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "w1_scale_inv is NULL");
  if (partial_amax == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "partial_amax is NULL");
  if (reinterpret_cast<uintptr_t>(partial_amax) & 3u) return fail(FP8MLP_ERR_INVALID_ARG, "partial_amax misaligned");
  if (write_q) {
    REQUIRE_PTR(post_fp8);
    REQUIRE_PTR(st);
  }
  if (pre_debug != nullptr && (reinterpret_cast<uintptr_t>(pre_debug) & 3u))
    return fail(FP8MLP_ERR_INVALID_ARG, "pre_debug misaligned");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  GemmParams p{};
  TRY(map_kmajor(&p.tmA[0], x_fp8, U8, 1, M, d, kGemmBM, "x_fp8"));
  TRY(map_kmajor(&p.tmB[0], W1q, U8, 1, h, d, kGemmBN * kGemmBM / gemm_tile_m(GemmKind::UpQ), "W1q"));
  TRY(map_tile32(&p.tmOut[0], post, BF16, 2, M, h, "post"));
  if (write_q) TRY(map_tile32(&p.tmOut2, post_fp8, U8, 1, M, h, "post_fp8"));
  fill_common(p, GemmKind::UpQ, di, M, h, d, 1);
  p.write_q = write_q ? 1 : 0;
  p.partial_amax = partial_amax;
  p.pre_debug = pre_debug;
  p.st = st;
  p.st_in = st_x;
  p.w_in_scale_inv = w1_scale_inv;
  return launch(GemmKind::UpQ, p, di, stream, "up_proj_fused_fp8 launch");
}

int fp8mlp_linear_fwd_fp8(int M, int K, int N, const uint8_t* x_fp8, const uint8_t* Wq, const float* w_scale_inv,
                          const fp8mlp_scale_state* st_x, uint16_t* y, fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, N, K));
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(x_fp8);
  REQUIRE_PTR(Wq);
  REQUIRE_PTR(st_x);
  REQUIRE_PTR(y);
  if (w_scale_inv == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "w_scale_inv is NULL");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  GemmParams p{};
  TRY(map_kmajor(&p.tmA[0], x_fp8, U8, 1, M, K, kGemmBM, "x_fp8"));
  TRY(map_kmajor(&p.tmB[0], Wq, U8, 1, N, K, kGemmBN * kGemmBM / gemm_tile_m(GemmKind::Down8), "Wq"));
  TRY(map_tile32(&p.tmOut[0], y, BF16, 2, M, N, "y"));
  fill_common(p, GemmKind::Down8, di, M, N, K, 1);
  p.st = st_x;
  p.w2_scale_inv = w_scale_inv;
  return launch(GemmKind::Down8, p, di, stream, "linear_fwd_fp8 launch");
}

size_t fp8mlp_linear_bwd_workspace_size(int M, int K, int N) {
  if (M < 2 * kLinearSplitRows || K <= 0 || N <= 0) return 0;
  return sizeof(float) * static_cast<size_t>(N) * K;
}

int fp8mlp_linear_bwd(int M, int K, int N, const uint16_t* x, const uint16_t* W, const uint16_t* dY, uint16_t* dX,
                      float* dW, void* workspace, int flags, fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, N, K));
  TRY(check_launch_flags(flags));
  REQUIRE_PTR(dW);
  if (M == 0) {
    DeviceInfo* di = nullptr;
    TRY(current_device(&di));
    const cudaError_t e = cudaMemsetAsync(dW, 0, sizeof(float) * static_cast<size_t>(N) * K, stream);
    return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "linear_bwd memset");
  }
  REQUIRE_PTR(x);
  REQUIRE_PTR(W);
  REQUIRE_PTR(dY);
  if (dX != nullptr) REQUIRE_PTR(dX);
  if (workspace != nullptr && (reinterpret_cast<uintptr_t>(workspace) & 15u))
    return fail(FP8MLP_ERR_INVALID_ARG, "workspace misaligned");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  // both launches are set up (and their tensor maps checked) before either
  // is enqueued
  // dX[M,K] = dY[M,N] . W[N,K]: contraction over N, W as an MN-major B operand
  GemmParams px{};
  if (dX != nullptr) {
    TRY(map_kmajor(&px.tmA[0], dY, BF16, 2, M, N, kGemmBM, "dY"));
    TRY(map_mnmajor(&px.tmB[0], W, N, K, "W"));
    TRY(map_tile32(&px.tmOut[0], dX, BF16, 2, M, K, "dX"));
    fill_common(px, GemmKind::Bf16MnB, di, M, K, N, 1);
    px.launch_flags = flags;
  }
  // dW[N,K] = dY^T . x: contraction over the M tokens, both operands MN-major.
  // With few output tiles (a third of the CTA pairs for 768 -> 2304) and a
  // workspace, the tokens are split in two: rows [0, M0) accumulate into dW,
  // rows [M0, M) into the workspace (the second group of one launch), and
  // the workspace is added to dW afterwards, in that order
  GemmParams p{};
  const int tiles = cdiv(N, kGemmBN) * cdiv(K, kGemmBN);
  const bool split = workspace != nullptr && M >= 2 * kLinearSplitRows && 2 * tiles <= di->num_sms / 2;
  const int M0 = split ? cdiv(cdiv(M, 2), kLinearSplitRows) * kLinearSplitRows : M;
  TRY(map_mnmajor(&p.tmA[0], dY, M0, N, "dY"));
  TRY(map_mnmajor(&p.tmB[0], x, M0, K, "x"));
  TRY(map_tile32(&p.tmOut[0], dW, F32, 4, N, K, "dW"));
  if (split) {
    TRY(map_mnmajor(&p.tmA[1], dY + static_cast<size_t>(M0) * N, M - M0, N, "dY"));
    TRY(map_mnmajor(&p.tmB[1], x + static_cast<size_t>(M0) * K, M - M0, K, "x"));
    TRY(map_tile32(&p.tmOut[1], workspace, F32, 4, N, K, "workspace"));
  }
  fill_common(p, GemmKind::DW, di, N, K, M0, split ? 2 : 1);
  // dW neither reads dX nor writes what dX reads: it may overlap its tail
  p.launch_flags = dX != nullptr ? FP8MLP_LAUNCH_OVERLAP_PREVIOUS : flags;
  if (dX != nullptr) TRY(launch(GemmKind::Bf16MnB, px, di, stream, "linear_bwd dX launch"));
  TRY(launch(GemmKind::DW, p, di, stream, "linear_bwd dW launch"));
  if (!split) return FP8MLP_OK;
  const cudaError_t e =
      launch_add_f32(static_cast<size_t>(N) * K, dW, static_cast<const float*>(workspace), di->num_sms, stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "linear_bwd dW add");
}

size_t fp8mlp_ce_workspace_size(int M, int V, int T) {
  if (M <= 0 || V <= 0 || T <= 0) return 0;
  return ce_layout(M, V, T).total;
}

int fp8mlp_ce_fwd(int M, int d, int V, int T, const uint16_t* x, const uint16_t* W, const int32_t* targets,
                  const float* target_weights, float softcap, float* lse, float* row_loss, float* loss,
                  void* workspace, fp8mlp_stream_t stream) {
  g_detail.clear();
  return ce_fwd_impl(false, M, d, V, T, x, W, nullptr, nullptr, targets, target_weights, softcap, lse, row_loss, loss,
                     workspace, stream);
}

int fp8mlp_ce_fwd_fp8(int M, int d, int V, int T, const uint8_t* x_fp8, const fp8mlp_scale_state* st_x,
                      const uint8_t* Wq, const float* w_scale_inv, const int32_t* targets,
                      const float* target_weights, float softcap, float* lse, float* row_loss, float* loss,
                      void* workspace, fp8mlp_stream_t stream) {
  g_detail.clear();
  return ce_fwd_impl(true, M, d, V, T, x_fp8, Wq, st_x, w_scale_inv, targets, target_weights, softcap, lse, row_loss,
                     loss, workspace, stream);
}

int fp8mlp_ce_bwd_dlogits(int M, int d, int V, int T, const uint16_t* x, const uint16_t* W, const int32_t* targets,
                          const float* target_weights, float softcap, const float* lse, const float* loss,
                          const float* dloss, int reduction, uint16_t* dlogits, fp8mlp_stream_t stream) {
  g_detail.clear();
  return ce_bwd_impl(false, M, d, V, T, x, W, nullptr, nullptr, targets, target_weights, softcap, lse, loss, dloss,
                     reduction, dlogits, stream);
}

int fp8mlp_ce_bwd_dlogits_fp8(int M, int d, int V, int T, const uint8_t* x_fp8, const fp8mlp_scale_state* st_x,
                              const uint8_t* Wq, const float* w_scale_inv, const int32_t* targets,
                              const float* target_weights, float softcap, const float* lse, const float* loss,
                              const float* dloss, int reduction, uint16_t* dlogits, fp8mlp_stream_t stream) {
  g_detail.clear();
  return ce_bwd_impl(true, M, d, V, T, x_fp8, Wq, st_x, w_scale_inv, targets, target_weights, softcap, lse, loss,
                     dloss, reduction, dlogits, stream);
}

int fp8mlp_bwd_dpre(int M, int d, int h, const uint16_t* dOut, const uint16_t* W2, const uint16_t* post,
                    uint16_t* dPre, int flags, fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, h));
  TRY(check_launch_flags(flags));
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(dOut);
  REQUIRE_PTR(W2);
  REQUIRE_PTR(post);
  REQUIRE_PTR(dPre);
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  GemmParams p{};
  TRY(map_kmajor(&p.tmA[0], dOut, BF16, 2, M, d, kGemmBM, "dOut"));
  TRY(map_kmajor(&p.tmB[0], W2, BF16, 2, h, d, kGemmBN * kGemmBM / gemm_tile_m(GemmKind::DPre), "W2"));
  TRY(map_tile32(&p.tmOut[0], dPre, BF16, 2, M, h, "dPre"));
  TRY(map_tile32(&p.tmAux, post, BF16, 2, M, h, "post"));
  fill_common(p, GemmKind::DPre, di, M, h, d, 1);
  p.launch_flags = flags;
  return launch(GemmKind::DPre, p, di, stream, "bwd_dpre launch");
}

int fp8mlp_bwd_dx(int M, int d, int h, const uint16_t* dPre, const uint16_t* W1, uint16_t* dX,
                  fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, h));
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(dPre);
  REQUIRE_PTR(W1);
  REQUIRE_PTR(dX);
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  GemmParams p{};
  TRY(map_kmajor(&p.tmA[0], dPre, BF16, 2, M, h, kGemmBM, "dPre"));
  TRY(map_mnmajor(&p.tmB[0], W1, h, d, "W1"));
  TRY(map_tile32(&p.tmOut[0], dX, BF16, 2, M, d, "dX"));
  fill_common(p, GemmKind::Bf16MnB, di, M, d, h, 1);
  return launch(GemmKind::Bf16MnB, p, di, stream, "bwd_dx launch");
}

int fp8mlp_bwd_dw(int M, int d, int h, const uint16_t* x, const uint16_t* dPre, const uint16_t* post,
                  const uint16_t* dOut, float* dW1, float* dW2, int flags, fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, h));
  TRY(check_launch_flags(flags));
  REQUIRE_PTR(dW1);
  REQUIRE_PTR(dW2);
  if (M == 0) {
    // an empty batch contributes zero gradient
    DeviceInfo* di = nullptr;
    TRY(current_device(&di));
    cudaError_t e = cudaMemsetAsync(dW1, 0, sizeof(float) * h * d, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(dW2, 0, sizeof(float) * h * d, stream);
    return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "bwd_dw memset");
  }
  REQUIRE_PTR(x);
  REQUIRE_PTR(dPre);
  REQUIRE_PTR(post);
  REQUIRE_PTR(dOut);
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  GemmParams p{};
  // group 0: dW1[i,j] = sum_m dPre[m,i] x[m,j];  group 1: dW2[i,j] = sum_m post[m,i] dOut[m,j]
  TRY(map_mnmajor(&p.tmA[0], dPre, M, h, "dPre"));
  TRY(map_mnmajor(&p.tmB[0], x, M, d, "x"));
  TRY(map_tile32(&p.tmOut[0], dW1, F32, 4, h, d, "dW1"));
  TRY(map_mnmajor(&p.tmA[1], post, M, h, "post"));
  TRY(map_mnmajor(&p.tmB[1], dOut, M, d, "dOut"));
  TRY(map_tile32(&p.tmOut[1], dW2, F32, 4, h, d, "dW2"));
  fill_common(p, GemmKind::DW, di, h, d, M, 2);
  p.launch_flags = flags;
  return launch(GemmKind::DW, p, di, stream, "bwd_dw launch");
}

int fp8mlp_mlp_bwd(int M, int d, int h, const uint16_t* x, const uint16_t* W1, const uint16_t* W2,
                   const uint16_t* post, const uint16_t* dOut, uint16_t* dPre, uint16_t* dX, float* dW1,
                   float* dW2, fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, h));
  if (M > 0) {
    REQUIRE_PTR(x);
    REQUIRE_PTR(W1);
    REQUIRE_PTR(W2);
    REQUIRE_PTR(post);
    REQUIRE_PTR(dOut);
    REQUIRE_PTR(dPre);
    REQUIRE_PTR(dX);
  }
  REQUIRE_PTR(dW1);
  REQUIRE_PTR(dW2);
  TRY(fp8mlp_bwd_dpre(M, d, h, dOut, W2, post, dPre, 0, stream));
  TRY(fp8mlp_bwd_dx(M, d, h, dPre, W1, dX, stream));
  // dW reads nothing dX writes and writes nothing dX reads: it may start
  // while the dX GEMM finishes its last wave
  return fp8mlp_bwd_dw(M, d, h, x, dPre, post, dOut, dW1, dW2, M > 0 ? FP8MLP_LAUNCH_OVERLAP_PREVIOUS : 0,
                       stream);
}

}  // extern "C"

namespace {
// the second stream and the events of fp8mlp_mlp_train_step, one set per
// device, created at the first call on it; a call enqueues its whole
// sequence (event records and waits included) under the device's lock
struct StepStreams {
  cudaStream_t side = nullptr;
  cudaEvent_t ev[4] = {nullptr, nullptr, nullptr, nullptr};
};
StepStreams g_step[kMaxDevices];
std::mutex g_step_mutex[kMaxDevices];

int step_streams(int dev, StepStreams** out) {
  StepStreams& ss = g_step[dev];
  if (ss.side == nullptr) {
    cudaStream_t side = nullptr;
    cudaError_t e = cudaStreamCreateWithFlags(&side, cudaStreamNonBlocking);
    if (e != cudaSuccess) return cuda_fail(e, "train_step: second stream");
    cudaEvent_t ev[4] = {nullptr, nullptr, nullptr, nullptr};
    for (int i = 0; i < 4; ++i) {
      e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
      if (e != cudaSuccess) {
        for (int j = 0; j < i; ++j) cudaEventDestroy(ev[j]);
        cudaStreamDestroy(side);
        return cuda_fail(e, "train_step: events");
      }
    }
    for (int i = 0; i < 4; ++i) ss.ev[i] = ev[i];
    ss.side = side;
  }
  *out = &ss;
  return FP8MLP_OK;
}
}  // namespace

extern "C" {

int fp8mlp_mlp_train_step(int M, int d, int h, const uint16_t* x, const uint16_t* W1, const uint16_t* W2,
                          const uint16_t* dOut, uint8_t* W2q_t, float* w2_scale_inv, fp8mlp_scale_state* st,
                          uint16_t* post, uint8_t* post_fp8, float* partial_amax, uint16_t* out, uint16_t* dPre,
                          uint16_t* dX, float* dW1, float* dW2, void* workspace, fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, h));
  REQUIRE_PTR(W1);
  REQUIRE_PTR(W2);
  REQUIRE_PTR(W2q_t);
  REQUIRE_PTR(st);
  REQUIRE_PTR(dW1);
  REQUIRE_PTR(dW2);
  REQUIRE_PTR(workspace);
  if (w2_scale_inv == nullptr || (reinterpret_cast<uintptr_t>(w2_scale_inv) & 3u))
    return fail(FP8MLP_ERR_INVALID_ARG, "w2_scale_inv is NULL or misaligned");
  if (M > 0) {
    REQUIRE_PTR(x);
    REQUIRE_PTR(dOut);
    REQUIRE_PTR(post);
    REQUIRE_PTR(post_fp8);
    REQUIRE_PTR(out);
    REQUIRE_PTR(dPre);
    REQUIRE_PTR(dX);
    if (partial_amax == nullptr || (reinterpret_cast<uintptr_t>(partial_amax) & 3u))
      return fail(FP8MLP_ERR_INVALID_ARG, "partial_amax is NULL or misaligned");
  }
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const int npa = fp8mlp_partial_amax_count(M, h);
  if (M == 0) {
    // nothing to overlap: the cache, zero weight gradients, the kept scale
    TRY(fp8mlp_w2_fp8_cache_refresh(h, d, W2, W2q_t, w2_scale_inv, workspace, stream));
    TRY(fp8mlp_mlp_bwd(0, d, h, x, W1, W2, post, dOut, dPre, dX, dW1, dW2, stream));
    return fp8mlp_amax_reduce_update_scale(partial_amax, 0, st, stream);
  }
  std::lock_guard<std::mutex> lock(g_step_mutex[di->device]);
  StepStreams* ss = nullptr;
  TRY(step_streams(di->device, &ss));
  cudaStream_t s = stream, side = ss->side;
#define TRY_CUDA(call, what)                    \
  do {                                          \
    const cudaError_t e_ = (call);              \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)
  // the W2 cache refresh (from the current W2) beside the up-projection,
  // which does not read the cache; joined before the down-projection
  TRY_CUDA(cudaEventRecord(ss->ev[0], s), "train_step: fork");
  TRY_CUDA(cudaStreamWaitEvent(side, ss->ev[0], 0), "train_step: fork");
  TRY(fp8mlp_w2_fp8_cache_refresh(h, d, W2, W2q_t, w2_scale_inv, workspace, side));
  TRY_CUDA(cudaEventRecord(ss->ev[1], side), "train_step: join");
  TRY(fp8mlp_up_proj_fused(M, d, h, x, W1, st, post, post_fp8, partial_amax, nullptr, 0, s));
  TRY_CUDA(cudaStreamWaitEvent(s, ss->ev[1], 0), "train_step: join");
  TRY(fp8mlp_down_proj_fp8(M, d, h, post_fp8, W2q_t, w2_scale_inv, st, out, s));
  // dPre reads nothing the down-projection writes: it may start in its last wave
  TRY(fp8mlp_bwd_dpre(M, d, h, dOut, W2, post, dPre, FP8MLP_LAUNCH_OVERLAP_PREVIOUS, s));
  // the delayed-scale update beside dX and dW, which do not read the scale
  TRY_CUDA(cudaEventRecord(ss->ev[2], s), "train_step: fork");
  TRY_CUDA(cudaStreamWaitEvent(side, ss->ev[2], 0), "train_step: fork");
  TRY(fp8mlp_amax_reduce_update_scale(partial_amax, npa, st, side));
  TRY_CUDA(cudaEventRecord(ss->ev[3], side), "train_step: join");
  TRY(fp8mlp_bwd_dx(M, d, h, dPre, W1, dX, s));
  // dW reads nothing dX writes: it may start in dX's last wave
  TRY(fp8mlp_bwd_dw(M, d, h, x, dPre, post, dOut, dW1, dW2, FP8MLP_LAUNCH_OVERLAP_PREVIOUS, s));
  TRY_CUDA(cudaStreamWaitEvent(s, ss->ev[3], 0), "train_step: join");
#undef TRY_CUDA
  return FP8MLP_OK;
}

int fp8mlp_rmsnorm_fwd_quant(int M, int d, const uint16_t* r, uint16_t* x, float* rstd,
                             const fp8mlp_scale_state* st_x, uint8_t* x_fp8, float* row_amax,
                             fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, 16));
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(r);
  REQUIRE_PTR(x);
  REQUIRE_PTR(st_x);
  REQUIRE_PTR(x_fp8);
  if (rstd == nullptr || (reinterpret_cast<uintptr_t>(rstd) & 3u)) return fail(FP8MLP_ERR_INVALID_ARG, "rstd");
  if (row_amax == nullptr || (reinterpret_cast<uintptr_t>(row_amax) & 3u))
    return fail(FP8MLP_ERR_INVALID_ARG, "row_amax");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const cudaError_t e = launch_rmsnorm_fwd_quant(M, d, r, x, rstd, st_x, x_fp8, row_amax, di->num_sms, stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "rmsnorm_fwd_quant launch");
}

int fp8mlp_rmsnorm_fwd(int M, int d, const uint16_t* r, uint16_t* x, float* rstd, fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, 16));
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(r);
  REQUIRE_PTR(x);
  if (rstd == nullptr || (reinterpret_cast<uintptr_t>(rstd) & 3u)) return fail(FP8MLP_ERR_INVALID_ARG, "rstd");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const cudaError_t e = launch_rmsnorm_fwd(M, d, r, x, rstd, di->num_sms, stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "rmsnorm_fwd launch");
}

int fp8mlp_rmsnorm_bwd(int M, int d, const uint16_t* r, const float* rstd, const uint16_t* dx,
                       const uint16_t* dr_in, uint16_t* dr_out, fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, 16));
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(r);
  REQUIRE_PTR(dx);
  REQUIRE_PTR(dr_in);
  REQUIRE_PTR(dr_out);
  if (rstd == nullptr || (reinterpret_cast<uintptr_t>(rstd) & 3u)) return fail(FP8MLP_ERR_INVALID_ARG, "rstd");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const cudaError_t e = launch_rmsnorm_bwd(M, d, r, rstd, dx, dr_in, dr_out, di->num_sms, stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "rmsnorm_bwd launch");
}

int fp8mlp_residual_add(int M, int d, const uint16_t* r, const uint16_t* out, uint16_t* r_next,
                        fp8mlp_stream_t stream) {
  g_detail.clear();
  TRY(check_dims(M, d, 16));
  if (M == 0) return FP8MLP_OK;
  REQUIRE_PTR(r);
  REQUIRE_PTR(out);
  REQUIRE_PTR(r_next);
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const cudaError_t e = launch_residual_add(M, d, r, out, r_next, di->num_sms, stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "residual_add launch");
}

int fp8mlp_get_device_status(unsigned int* status, fp8mlp_stream_t stream) {
  g_detail.clear();
  if (status == nullptr) return fail(FP8MLP_ERR_INVALID_ARG, "status is NULL");
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  cudaError_t e = cudaMemcpyAsync(status, di->status, sizeof(unsigned int), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "get_device_status");
}

int fp8mlp_clear_device_status(fp8mlp_stream_t stream) {
  g_detail.clear();
  DeviceInfo* di = nullptr;
  TRY(current_device(&di));
  const cudaError_t e = cudaMemsetAsync(di->status, 0, sizeof(unsigned int), stream);
  return e == cudaSuccess ? FP8MLP_OK : cuda_fail(e, "clear_device_status");
}

int fp8mlp_set_wait_timeout_ns(unsigned long long ns) {
  if (ns == 0) return fail(FP8MLP_ERR_INVALID_ARG, "timeout must be > 0");
  g_timeout_ns.store(ns);
  return FP8MLP_OK;
}

int fp8mlp_set_programmatic_launch(int enable) {
  g_pdl.store(enable ? 1 : 0);
  return FP8MLP_OK;
}

int fp8mlp_set_debug_flags(int flags) {
  if (flags & ~(FP8MLP_DEBUG_STALL_PRODUCER | FP8MLP_DEBUG_STALL_AUX))
    return fail(FP8MLP_ERR_INVALID_ARG, "unknown debug flags");
  g_debug_flags.store(flags);
  return FP8MLP_OK;
}

const char* fp8mlp_error_string(int code) {
  switch (code) {
    case FP8MLP_OK:
      return "ok";
    case FP8MLP_ERR_INVALID_ARG:
      return "invalid argument";
    case FP8MLP_ERR_UNSUPPORTED_SHAPE:
      return "unsupported shape";
    case FP8MLP_ERR_CUDA:
      return "CUDA error";
    case FP8MLP_ERR_TIMEOUT:
      return "device wait timed out";
    case FP8MLP_ERR_NO_DEVICE:
      return "no sm_100a device";
    default:
      return "unknown error code";
  }
}

const char* fp8mlp_last_error_detail(void) { return g_detail.c_str(); }

const char* fp8mlp_version(void) { return FP8MLP_VERSION_STRING; }

unsigned long long fp8mlp_kernel_launch_count(void) { return g_launches.load(); }

}  // extern "C"
