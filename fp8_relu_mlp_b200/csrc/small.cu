// The small kernels of the block: scale-state init, partial-amax reduction
// with the delayed-scale update, the transposed FP8 W2 cache refresh, and the
// RMSNorm / residual helpers of the layer stack.  All memory-bound or tiny.
#include <cuda_bf16.h>

#include "internal.h"

namespace fp8mlp {

__device__ unsigned int g_status_word = 0;

cudaError_t status_word_address(unsigned int** ptr) {
  return cudaGetSymbolAddress(reinterpret_cast<void**>(ptr), g_status_word);
}

namespace {

using namespace dev;

__global__ void state_init_kernel(fp8mlp_scale_state* st, float margin, float s0) {
  pdl_wait();
  pdl_launch_dependents();
  st->amax_prev = 0.f;
  st->scale = s0;
  st->scale_inv = __fdiv_rn(1.f, s0);
  st->margin = margin;
  st->step = 0;
  st->flags = 0;
  st->pad[0] = 0;
  st->pad[1] = 0;
}

// A = max(partial amax); s = 448 / (margin * A); see fp8mlp_amax_reduce_update_scale.
__global__ void __launch_bounds__(1024) amax_scale_kernel(const float* __restrict__ pa, int n,
                                                          fp8mlp_scale_state* st, unsigned int* status) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float smax[32];
  __shared__ int snan[32];
  float m = 0.f;
  int nan = 0;
  // eight independent loads in flight per thread per round (the partials are
  // a few thousand floats: latency, not bandwidth, is the cost)
  for (int base = 0; base < n; base += 8 * 1024) {
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int i = base + k * 1024 + threadIdx.x;
      v[k] = i < n ? __ldg(pa + i) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      nan |= (v[k] != v[k]);
      m = fmaxf(m, v[k]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    nan |= __shfl_xor_sync(0xffffffffu, nan, o);
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    smax[w] = m;
    snan[w] = nan;
  }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    m = l < nw ? smax[l] : 0.f;
    nan = l < nw ? snan[l] : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      nan |= __shfl_xor_sync(0xffffffffu, nan, o);
    }
    if (l == 0) {
      const float A = nan ? __int_as_float(0x7fc00000) : m;
      st->amax_prev = A;
      st->step += 1;
      if (isfinite(A) && A > 0.f) {
        const float den = __fmul_rn(st->margin, A);
        const float s = __fdiv_rn(FP8MLP_E4M3_MAX, den);
        if (isfinite(s) && s > 0.f) {
          st->scale = s;
          st->scale_inv = __fdiv_rn(1.f, s);
          st->flags &= ~FP8MLP_STATE_KEPT_SCALE;
          return;
        }
      }
      st->flags |= FP8MLP_STATE_KEPT_SCALE;
      if (!isfinite(A)) atomicOr(status, STATUS_NONFINITE_AMAX);
    }
  }
}

// max |W2| over BF16 bit patterns: the magnitude bits order like the values
// (NaN patterns above infinity), so an integer max is exact.  Block b covers
// elements [b*kW2ElemsPerBlock, (b+1)*kW2ElemsPerBlock) and writes its max to
// partial[b]; the quantising kernel reduces the partials.
__global__ void __launch_bounds__(256) w2_amax_kernel(const uint4* __restrict__ W, long long n_vec,
                                                      unsigned int* __restrict__ partial) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ unsigned int wmax[8];
  const long long base = static_cast<long long>(blockIdx.x) * (kW2ElemsPerBlock / 8);
  unsigned int m = 0;
#pragma unroll
  for (int k = 0; k < kW2ElemsPerBlock / 8 / 256; ++k) {
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

__device__ __forceinline__ float w2_scale_from(unsigned int amax_bits, bool* degenerate) {
  const float a = __uint_as_float(amax_bits << 16);
  if (isfinite(a) && a > 0.f) {
    *degenerate = false;
    return __fdiv_rn(FP8MLP_E4M3_MAX, a);
  }
  *degenerate = true;
  return 1.f;
}

// W2q_t[j, i] = e4m3(W2[i, j] * s_w); 64x64 tiles through shared memory.
__global__ void __launch_bounds__(256) w2_quant_t_kernel(int h, int d, const uint16_t* __restrict__ W2,
                                                         uint8_t* __restrict__ W2q_t, float* w2_scale_inv,
                                                         const unsigned int* __restrict__ partial, int nparts,
                                                         unsigned int* status) {
  __shared__ float tile[64][65];
  pdl_wait();
  pdl_launch_dependents();
  __shared__ unsigned int wmax[8];
  const int i0 = blockIdx.y * 64;  // rows of W2 (h)
  const int j0 = blockIdx.x * 64;  // cols of W2 (d)
  unsigned int am = 0;
  for (int i = threadIdx.x; i < nparts; i += 256) am = max(am, partial[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = am;
  __syncthreads();
  am = 0;
  for (int w = 0; w < 8; ++w) am = max(am, wmax[w]);
  bool degenerate;
  const float s_w = w2_scale_from(am, &degenerate);
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
    w2_scale_inv[0] = __fdiv_rn(1.f, s_w);
    if (degenerate) atomicOr(status, STATUS_W2_DEGENERATE);
  }
  // load: 64 rows x 64 bf16; each thread loads 8 consecutive bf16 (16 B)
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
  // store: W2q_t rows j (64 of them), 64 bytes each; each thread writes 4 codes
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

// One warp per row.  d is a multiple of 16; each lane handles 8-element groups.
__global__ void rmsnorm_fwd_kernel(int M, int d, const uint16_t* __restrict__ r, uint16_t* __restrict__ x,
                                   float* __restrict__ rstd) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  for (int row = blockIdx.x * warps + (threadIdx.x >> 5); row < M; row += gridDim.x * warps) {
    const uint16_t* rr = r + static_cast<size_t>(row) * d;
    float ss = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 v = *reinterpret_cast<const uint4*>(rr + c);
      const unsigned int w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float a = bf16lo_to_f32(w4[k]), b = bf16hi_to_f32(w4[k]);
        ss = fmaf(a, a, ss);
        ss = fmaf(b, b, ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rs = __fdiv_rn(1.f, __fsqrt_rn(__fdiv_rn(ss, static_cast<float>(d)) + 1e-6f));
    if (lane == 0) rstd[row] = rs;
    uint16_t* xr = x + static_cast<size_t>(row) * d;
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 v = *reinterpret_cast<const uint4*>(rr + c);
      const unsigned int w4[4] = {v.x, v.y, v.z, v.w};
      unsigned int o4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        o4[k] = pack_bf16x2(__fmul_rn(bf16lo_to_f32(w4[k]), rs), __fmul_rn(bf16hi_to_f32(w4[k]), rs));
      *reinterpret_cast<uint4*>(xr + c) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
  }
}

// RMSNorm forward that also writes the e4m3 copy of x for an FP8
// up-projection: x_fp8 = e4m3(fp32(x_bf16 * s_x)) under the delayed x-scale,
// and row_amax[m] = max |x_bf16[m,:]| (the amax that drives the next scale).
__global__ void rmsnorm_fwd_quant_kernel(int M, int d, const uint16_t* __restrict__ r, uint16_t* __restrict__ x,
                                         float* __restrict__ rstd, const fp8mlp_scale_state* st_x,
                                         uint2* __restrict__ xq, float* __restrict__ row_amax) {
  pdl_wait();
  pdl_launch_dependents();
  const float s = st_x->scale;
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  for (int row = blockIdx.x * warps + (threadIdx.x >> 5); row < M; row += gridDim.x * warps) {
    const uint16_t* rr = r + static_cast<size_t>(row) * d;
    float ss = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 v = *reinterpret_cast<const uint4*>(rr + c);
      const unsigned int w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float a = bf16lo_to_f32(w4[k]), b = bf16hi_to_f32(w4[k]);
        ss = fmaf(a, a, ss);
        ss = fmaf(b, b, ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float rs = __fdiv_rn(1.f, __fsqrt_rn(__fdiv_rn(ss, static_cast<float>(d)) + 1e-6f));
    if (lane == 0) rstd[row] = rs;
    uint16_t* xr = x + static_cast<size_t>(row) * d;
    uint2* qr = xq + static_cast<size_t>(row) * (d / 8);
    unsigned int m = 0;  // max |x| as BF16 magnitude bits (integer order = value order)
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 v = *reinterpret_cast<const uint4*>(rr + c);
      const unsigned int w4[4] = {v.x, v.y, v.z, v.w};
      unsigned int o4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        o4[k] = pack_bf16x2(__fmul_rn(bf16lo_to_f32(w4[k]), rs), __fmul_rn(bf16hi_to_f32(w4[k]), rs));
        m = max(m, o4[k] & 0x7FFFu);
        m = max(m, (o4[k] >> 16) & 0x7FFFu);
      }
      *reinterpret_cast<uint4*>(xr + c) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
      uint32_t q[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint32_t a = pack_e4m3x2(__fmul_rn(bf16lo_to_f32(o4[2 * j]), s), __fmul_rn(bf16hi_to_f32(o4[2 * j]), s));
        const uint32_t b = pack_e4m3x2(__fmul_rn(bf16lo_to_f32(o4[2 * j + 1]), s),
                                       __fmul_rn(bf16hi_to_f32(o4[2 * j + 1]), s));
        q[j] = a | (b << 16);
      }
      qr[c / 8] = make_uint2(q[0], q[1]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) row_amax[row] = __uint_as_float(m << 16);
  }
}

__global__ void rmsnorm_bwd_kernel(int M, int d, const uint16_t* __restrict__ r, const float* __restrict__ rstd,
                                   const uint16_t* __restrict__ dx, const uint16_t* dr_in, uint16_t* dr_out) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  for (int row = blockIdx.x * warps + (threadIdx.x >> 5); row < M; row += gridDim.x * warps) {
    const size_t base = static_cast<size_t>(row) * d;
    const float rs = rstd[row];
    float dot = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 vr = *reinterpret_cast<const uint4*>(r + base + c);
      const uint4 vg = *reinterpret_cast<const uint4*>(dx + base + c);
      const unsigned int a4[4] = {vr.x, vr.y, vr.z, vr.w}, g4[4] = {vg.x, vg.y, vg.z, vg.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        dot = fmaf(bf16lo_to_f32(g4[k]), bf16lo_to_f32(a4[k]) * rs, dot);
        dot = fmaf(bf16hi_to_f32(g4[k]), bf16hi_to_f32(a4[k]) * rs, dot);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    dot = dot / static_cast<float>(d);
    for (int c = lane * 8; c < d; c += 256) {
      const uint4 vr = *reinterpret_cast<const uint4*>(r + base + c);
      const uint4 vg = *reinterpret_cast<const uint4*>(dx + base + c);
      const uint4 vi = *reinterpret_cast<const uint4*>(dr_in + base + c);
      const unsigned int a4[4] = {vr.x, vr.y, vr.z, vr.w}, g4[4] = {vg.x, vg.y, vg.z, vg.w},
                         i4[4] = {vi.x, vi.y, vi.z, vi.w};
      unsigned int o4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float x0 = bf16lo_to_f32(a4[k]) * rs, x1 = bf16hi_to_f32(a4[k]) * rs;
        const float d0 = bf16lo_to_f32(i4[k]) + rs * (bf16lo_to_f32(g4[k]) - x0 * dot);
        const float d1 = bf16hi_to_f32(i4[k]) + rs * (bf16hi_to_f32(g4[k]) - x1 * dot);
        o4[k] = pack_bf16x2(d0, d1);
      }
      *reinterpret_cast<uint4*>(dr_out + base + c) = make_uint4(o4[0], o4[1], o4[2], o4[3]);
    }
  }
}

__global__ void residual_add_kernel(size_t n_vec, const uint4* __restrict__ r, const uint4* __restrict__ o,
                                    uint4* __restrict__ rn) {
  pdl_wait();
  pdl_launch_dependents();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n_vec;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 a = r[i], b = o[i];
    const unsigned int a4[4] = {a.x, a.y, a.z, a.w}, b4[4] = {b.x, b.y, b.z, b.w};
    unsigned int c4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      c4[k] = pack_bf16x2(bf16lo_to_f32(a4[k]) + bf16lo_to_f32(b4[k]), bf16hi_to_f32(a4[k]) + bf16hi_to_f32(b4[k]));
    rn[i] = make_uint4(c4[0], c4[1], c4[2], c4[3]);
  }
}

// dst += src over n fp32 values (n a multiple of 4): the second half of a
// weight gradient split over the tokens, added in a fixed order
__global__ void add_f32_kernel(size_t n4, float4* __restrict__ dst, const float4* __restrict__ src) {
  pdl_wait();
  pdl_launch_dependents();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 a = dst[i], b = __ldcs(src + i);
    dst[i] = make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z), __fadd_rn(a.w, b.w));
  }
}

// x_q = e4m3(fp32(x * s_x)) with s_x = st->scale; block b also writes the
// max |x| over its kXElemsPerBlock elements (BF16 magnitude bits: integer
// order = value order) as the partial amax of x's delayed scale.
__global__ void __launch_bounds__(256) quantize_x_kernel(const uint4* __restrict__ x, long long n_vec,
                                                         const fp8mlp_scale_state* st, uint2* __restrict__ xq,
                                                         float* __restrict__ partial) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ unsigned int wmax[8];
  const float s = st->scale;
  const long long base = static_cast<long long>(blockIdx.x) * (kXElemsPerBlock / 8);
  unsigned int m = 0;
#pragma unroll
  for (int k = 0; k < kXElemsPerBlock / 8 / 256; ++k) {
    const long long i = base + k * 256 + threadIdx.x;
    if (i < n_vec) {
      const uint4 v = x[i];
      const unsigned int w4[4] = {v.x, v.y, v.z, v.w};
      uint32_t q[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const uint32_t a = pack_e4m3x2(__fmul_rn(bf16lo_to_f32(w4[2 * j]), s), __fmul_rn(bf16hi_to_f32(w4[2 * j]), s));
        const uint32_t b = pack_e4m3x2(__fmul_rn(bf16lo_to_f32(w4[2 * j + 1]), s),
                                       __fmul_rn(bf16hi_to_f32(w4[2 * j + 1]), s));
        q[j] = a | (b << 16);
      }
      xq[i] = make_uint2(q[0], q[1]);
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
    partial[blockIdx.x] = __uint_as_float(r << 16);
  }
}

// W1q = e4m3(fp32(W1 * s_w1)), s_w1 = 448 / max|W1| from the partial maxima;
// flat (W1 [h,d] is already K-major for the up-projection).
__global__ void __launch_bounds__(256) w1_quant_kernel(long long n_vec, const uint4* __restrict__ W1,
                                                       uint2* __restrict__ W1q, float* w1_scale_inv,
                                                       const unsigned int* __restrict__ partial, int nparts,
                                                       unsigned int* status) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ unsigned int wmax[8];
  unsigned int am = 0;
  for (int i = threadIdx.x; i < nparts; i += 256) am = max(am, partial[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = max(am, __shfl_xor_sync(0xffffffffu, am, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = am;
  __syncthreads();
  am = 0;
  for (int w = 0; w < 8; ++w) am = max(am, wmax[w]);
  bool degenerate;
  const float s = w2_scale_from(am, &degenerate);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    w1_scale_inv[0] = __fdiv_rn(1.f, s);
    if (degenerate) atomicOr(status, STATUS_W2_DEGENERATE);
  }
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n_vec; i += static_cast<long long>(gridDim.x) * 256) {
    const uint4 v = W1[i];
    const unsigned int w4[4] = {v.x, v.y, v.z, v.w};
    uint32_t q[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const uint32_t a = pack_e4m3x2(__fmul_rn(bf16lo_to_f32(w4[2 * j]), s), __fmul_rn(bf16hi_to_f32(w4[2 * j]), s));
      const uint32_t b = pack_e4m3x2(__fmul_rn(bf16lo_to_f32(w4[2 * j + 1]), s),
                                     __fmul_rn(bf16hi_to_f32(w4[2 * j + 1]), s));
      q[j] = a | (b << 16);
    }
    W1q[i] = make_uint2(q[0], q[1]);
  }
}

int grid_for(size_t work, int per_block, int num_sms, int blocks_per_sm) {
  size_t g = (work + per_block - 1) / per_block;
  const size_t cap = static_cast<size_t>(num_sms) * blocks_per_sm;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

}  // namespace

cudaError_t launch_add_f32(size_t n, float* dst, const float* src, int num_sms, cudaStream_t s) {
  const size_t n4 = n / 4;
  const cudaError_t e = launch_pdl(add_f32_kernel, dim3(grid_for(n4, 256, num_sms, 4)), dim3(256), 0, s, n4,
                                   reinterpret_cast<float4*>(dst), reinterpret_cast<const float4*>(src));
  count_launches(1);
  return e;
}

cudaError_t launch_state_init(fp8mlp_scale_state* st, float margin, float s0, cudaStream_t s) {
  const cudaError_t e = launch_pdl(state_init_kernel, dim3(1), dim3(1), 0, s, st, margin, s0);
  count_launches(1);
  return e;
}

cudaError_t launch_amax_scale(const float* pa, int n, fp8mlp_scale_state* st, unsigned int* status, cudaStream_t s) {
  const cudaError_t e = launch_pdl(amax_scale_kernel, dim3(1), dim3(1024), 0, s, pa, n, st, status);
  count_launches(1);
  return e;
}

cudaError_t launch_w2_cache(int h, int d, const uint16_t* W2, uint8_t* W2q_t, float* w2_scale_inv,
                            unsigned int* partial, unsigned int* status, int num_sms, cudaStream_t s) {
  (void)num_sms;
  const long long n = static_cast<long long>(h) * d;
  const int nparts = static_cast<int>((n + kW2ElemsPerBlock - 1) / kW2ElemsPerBlock);
  cudaError_t e = launch_pdl(w2_amax_kernel, dim3(nparts), dim3(256), 0, s, reinterpret_cast<const uint4*>(W2),
                             n / 8, partial);
  count_launches(1);
  if (e != cudaSuccess) return e;
  dim3 grid((d + 63) / 64, (h + 63) / 64);
  e = launch_pdl(w2_quant_t_kernel, grid, dim3(256), 0, s, h, d, W2, W2q_t, w2_scale_inv,
                 static_cast<const unsigned int*>(partial), nparts, status);
  count_launches(1);
  return e;
}

cudaError_t launch_quantize_x(long long n, const uint16_t* x, const fp8mlp_scale_state* st, uint8_t* xq,
                              float* partial, cudaStream_t s) {
  const int nparts = static_cast<int>((n + kXElemsPerBlock - 1) / kXElemsPerBlock);
  const cudaError_t e = launch_pdl(quantize_x_kernel, dim3(nparts), dim3(256), 0, s,
                                   reinterpret_cast<const uint4*>(x), n / 8, st, reinterpret_cast<uint2*>(xq), partial);
  count_launches(1);
  return e;
}

cudaError_t launch_w1_cache(int h, int d, const uint16_t* W1, uint8_t* W1q, float* w1_scale_inv,
                            unsigned int* partial, unsigned int* status, cudaStream_t s) {
  const long long n = static_cast<long long>(h) * d;
  const int nparts = static_cast<int>((n + kW2ElemsPerBlock - 1) / kW2ElemsPerBlock);
  cudaError_t e = launch_pdl(w2_amax_kernel, dim3(nparts), dim3(256), 0, s, reinterpret_cast<const uint4*>(W1), n / 8,
                             partial);
  count_launches(1);
  if (e != cudaSuccess) return e;
  e = launch_pdl(w1_quant_kernel, dim3(nparts), dim3(256), 0, s, n / 8, reinterpret_cast<const uint4*>(W1),
                 reinterpret_cast<uint2*>(W1q), w1_scale_inv, static_cast<const unsigned int*>(partial), nparts, status);
  count_launches(1);
  return e;
}

cudaError_t launch_rmsnorm_fwd_quant(int M, int d, const uint16_t* r, uint16_t* x, float* rstd,
                                     const fp8mlp_scale_state* st_x, uint8_t* x_fp8, float* row_amax, int num_sms,
                                     cudaStream_t s) {
  const cudaError_t e = launch_pdl(rmsnorm_fwd_quant_kernel, dim3(grid_for(static_cast<size_t>(M), 8, num_sms, 8)),
                                   dim3(256), 0, s, M, d, r, x, rstd, st_x, reinterpret_cast<uint2*>(x_fp8), row_amax);
  count_launches(1);
  return e;
}

cudaError_t launch_rmsnorm_fwd(int M, int d, const uint16_t* r, uint16_t* x, float* rstd, int num_sms,
                               cudaStream_t s) {
  const cudaError_t e = launch_pdl(rmsnorm_fwd_kernel, dim3(grid_for(static_cast<size_t>(M), 8, num_sms, 8)),
                                   dim3(256), 0, s, M, d, r, x, rstd);
  count_launches(1);
  return e;
}

cudaError_t launch_rmsnorm_bwd(int M, int d, const uint16_t* r, const float* rstd, const uint16_t* dx,
                               const uint16_t* dr_in, uint16_t* dr_out, int num_sms, cudaStream_t s) {
  const cudaError_t e = launch_pdl(rmsnorm_bwd_kernel, dim3(grid_for(static_cast<size_t>(M), 8, num_sms, 8)),
                                   dim3(256), 0, s, M, d, r, rstd, dx, dr_in, dr_out);
  count_launches(1);
  return e;
}

cudaError_t launch_residual_add(int M, int d, const uint16_t* r, const uint16_t* out, uint16_t* r_next,
                                int num_sms, cudaStream_t s) {
  const size_t n_vec = static_cast<size_t>(M) * d / 8;
  const cudaError_t e =
      launch_pdl(residual_add_kernel, dim3(grid_for(n_vec, 256, num_sms, 8)), dim3(256), 0, s, n_vec,
                 reinterpret_cast<const uint4*>(r), reinterpret_cast<const uint4*>(out), reinterpret_cast<uint4*>(r_next));
  count_launches(1);
  return e;
}

}  // namespace fp8mlp
