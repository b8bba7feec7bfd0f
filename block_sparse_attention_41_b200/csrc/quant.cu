// 8-bit QK^T operands of the low-precision variant (the review page of the Sol Video Inference
// Engine paper, "five acceleration techniques": SageAttention's 8-bit attention with outlier
// smoothing; Sol-Engine README news: fused 8-bit compute).
//
//   mu_c       = sum_j n_j k_bar_jc / L                   the head's mean key (from the pooled keys)
//   Q tile     : symmetric int8, one scale amax/127 per 128-row query block
//   K tile     : K - mu, symmetric int8, one scale per 128-row key block
//   pooled tile: k_bar - mu, symmetric int8, one scale per chunk of 128 pooled keys
// A code is round-to-nearest-even of x * (127 / amax) in fp32, clamped to [-127, 127]; an all-zero
// tile gets scale 1 and zero codes. The scale is one factor per score tile, so the fused kernel
// folds scale_q * scale_k into the softmax scale.
//
// HBM-bound: each input element is read once and each code written once. One CTA quantizes one
// 128-row tile of one head: a thread owns a 16-byte column slice of every (256 / (d / VEC))-th
// row, keeps the tile's values in registers between the amax pass and the code pass, and writes
// 8 (bf16 input) or 4 (fp32 input) codes at a time.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "device_common.cuh"
#include "launchers.h"

namespace sol {

namespace {

constexpr int kQThreads = 256;
constexpr int kTileRows = 128;

// The head's mean key from the pooled keys: mu[bh][c] = sum_j n_j kbar[bh][j][c] / L, the blocks
// taken in order with fp32 fused multiply-adds.
__global__ void __launch_bounds__(128) sol_key_mean_kernel(const float* __restrict__ kbar, float* __restrict__ mu,
                                                           int L, int nkb, int block, int d) {
  const int bh = blockIdx.x;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float s = 0.f;
    for (int j = 0; j < nkb; ++j) {
      const int n = min(block, L - j * block);
      s = fmaf(__ldg(kbar + (static_cast<size_t>(bh) * nkb + j) * d + c), static_cast<float>(n), s);
    }
    mu[static_cast<size_t>(bh) * d + c] = s / static_cast<float>(L);
  }
}

template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static void unpack(const uint4& v, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = __uint_as_float(w[k] << 16);
      x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
};
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void unpack(const uint4& v, float (&x)[4]) {
    x[0] = __uint_as_float(v.x);
    x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z);
    x[3] = __uint_as_float(v.w);
  }
};

__device__ __forceinline__ uint32_t code4(const float* x, float inv) {
  uint32_t r = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    int c = __float2int_rn(x[k] * inv);
    c = max(-127, min(127, c));
    r |= (static_cast<uint32_t>(c) & 0xffu) << (8 * k);
  }
  return r;
}

// One 128-row tile of `rows` valid rows: src [rows, D] (row stride D) minus `mu` (or nothing),
// codes to dst [rows, D] int8 and the tile scale to *scale.
template <typename T, int D>
__global__ void __launch_bounds__(kQThreads)
    sol_quant_tile_kernel(const T* __restrict__ src, const float* __restrict__ mu, int8_t* __restrict__ dst,
                          float* __restrict__ scale, int rows_total, int n_tiles) {
  constexpr int VEC = Vec<T>::N;
  constexpr int LPR = D / VEC;          // lanes per row
  constexpr int RG = kQThreads / LPR;   // row groups
  constexpr int RPT = kTileRows / RG;   // rows per thread
  __shared__ float s_red[kQThreads / 32];
  const int tile = blockIdx.x, bh = blockIdx.y, tid = threadIdx.x;
  const int c = tid % LPR, rg = tid / LPR;
  const int r0 = tile * kTileRows;
  const int rows = min(kTileRows, rows_total - r0);
  const T* base = src + (static_cast<size_t>(bh) * rows_total + r0) * D + c * VEC;
  float m[VEC];
#pragma unroll
  for (int k = 0; k < VEC; ++k) m[k] = mu != nullptr ? __ldg(mu + static_cast<size_t>(bh) * D + c * VEC + k) : 0.f;
  float x[RPT][VEC];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int r = rg + i * RG;
    if (r < rows) {
      Vec<T>::unpack(__ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(r) * D)), x[i]);
#pragma unroll
      for (int k = 0; k < VEC; ++k) {
        x[i][k] -= m[k];
        amax = fmaxf(amax, fabsf(x[i][k]));
      }
    } else {
#pragma unroll
      for (int k = 0; k < VEC; ++k) x[i][k] = 0.f;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((tid & 31) == 0) s_red[tid >> 5] = amax;
  __syncthreads();
  amax = s_red[0];
#pragma unroll
  for (int w = 1; w < kQThreads / 32; ++w) amax = fmaxf(amax, s_red[w]);
  const float inv = amax > 0.f ? 127.0f / amax : 0.f;
  if (tid == 0) scale[static_cast<size_t>(bh) * n_tiles + tile] = amax > 0.f ? amax / 127.0f : 1.0f;
  int8_t* out = dst + (static_cast<size_t>(bh) * rows_total + r0) * D + c * VEC;
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int r = rg + i * RG;
    if (r < rows) {
      if constexpr (VEC == 8) {
        const uint2 v = make_uint2(code4(x[i], inv), code4(x[i] + 4, inv));
        *reinterpret_cast<uint2*>(out + static_cast<size_t>(r) * D) = v;
      } else {
        *reinterpret_cast<uint32_t*>(out + static_cast<size_t>(r) * D) = code4(x[i], inv);
      }
    }
  }
}

template <int D>
cudaError_t launch_quant_d(const QuantArgs& a, cudaStream_t stream) {
  const int nqb = (a.L + kTileRows - 1) / kTileRows;
  const int nkb = nqb;
  const int nchunks = (nkb + kTileRows - 1) / kTileRows;
  sol_key_mean_kernel<<<a.BH, 128, 0, stream>>>(a.kbar, a.mu, a.L, nkb, kTileRows, D);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sol_quant_tile_kernel<__nv_bfloat16, D><<<dim3(nqb, a.BH), kQThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(a.Q), nullptr, a.q8, a.q_scale, a.L, nqb);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sol_quant_tile_kernel<__nv_bfloat16, D><<<dim3(nkb, a.BH), kQThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(a.K), a.mu, a.k8, a.k_scale, a.L, nkb);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sol_quant_tile_kernel<float, D><<<dim3(nchunks, a.BH), kQThreads, 0, stream>>>(a.kbar, a.mu, a.kb8, a.kb_scale,
                                                                                 nkb, nchunks);
  return cudaGetLastError();
}

// ---- 8-bit PV values: V and v_bar as E4M3 with one scale per channel (d = 128) -----------------
// SageAttention's FP8 PV layout: s_c = amax_c / 448 over the head's L tokens (1 for an all-zero
// channel); a code is E4M3(x / s_c), round to nearest even, saturating at +-448. The codes are
// stored transposed, [d][keys] per head (keys contiguous), the K-major layout of the PV product's
// B operand; keys past L (and pooled blocks past N_kb) get code 0. v_bar takes V's scales.

constexpr int kVD = 128;

// Per-(head, channel) amax of V over one 128-key block, merged into amax[] with atomicMax on the
// float bits (non-negative floats order as their bit patterns).
__global__ void __launch_bounds__(256) sol_v_amax_kernel(const __nv_bfloat16* __restrict__ V,
                                                         unsigned int* __restrict__ amax, int L) {
  __shared__ float s_m[16][kVD];  // [row group][channel]
  const int j = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int cg = t & 15, rg = t >> 4;  // channels [8 cg, 8 cg + 8), rows rg, rg + 16, ...
  const int n = min(kTileRows, L - j * kTileRows);
  const __nv_bfloat16* base = V + (static_cast<size_t>(bh) * L + static_cast<size_t>(j) * kTileRows) * kVD + cg * 8;
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = 0.f;
  for (int r = rg; r < n; r += 16) {
    float x[8];
    Vec<__nv_bfloat16>::unpack(__ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(r) * kVD)), x);
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = fmaxf(m[k], fabsf(x[k]));
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) s_m[rg][cg * 8 + k] = m[k];
  __syncthreads();
  if (t < kVD) {
    float a = 0.f;
#pragma unroll
    for (int g = 0; g < 16; ++g) a = fmaxf(a, s_m[g][t]);
    atomicMax(amax + static_cast<size_t>(bh) * kVD + t, __float_as_uint(a));
  }
}

__device__ __forceinline__ float channel_scale(unsigned int amax_bits) {
  const float a = __uint_as_float(amax_bits);
  return a > 0.f ? a / 448.f : 1.f;
}

// Codes of 128 rows (tokens or pooled blocks) of one head, written transposed: out[c][col0 + r].
// T = bf16 (V, 8 channels per 16-byte load) or float (v_bar, 4 per load).
template <typename T>
__global__ void __launch_bounds__(256) sol_v_codes_kernel(const T* __restrict__ src, const unsigned int* __restrict__ amax,
                                                          uint8_t* __restrict__ out, int rows, int out_pitch) {
  constexpr int VEC = Vec<T>::N;
  constexpr int CG = kVD / VEC;     // channel groups per row
  constexpr int RG = 256 / CG;      // row groups
  __shared__ uint8_t s_codes[kVD][kTileRows + 16];  // [channel][row], rows padded to 144 B
  __shared__ float s_scale[kVD];
  const int jb = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  if (t < kVD) s_scale[t] = channel_scale(__ldg(amax + static_cast<size_t>(bh) * kVD + t));
  __syncthreads();
  const int cg = t % CG, rg = t / CG;
  const int n = min(kTileRows, rows - jb * kTileRows);
  const T* base = src + (static_cast<size_t>(bh) * rows + static_cast<size_t>(jb) * kTileRows) * kVD + cg * VEC;
  for (int r = rg; r < kTileRows; r += RG) {
    float x[VEC];
    if (r < n) {
      Vec<T>::unpack(__ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(r) * kVD)), x);
    } else {
#pragma unroll
      for (int k = 0; k < VEC; ++k) x[k] = 0.f;
    }
#pragma unroll
    for (int k = 0; k < VEC; ++k) {
      const int c = cg * VEC + k;
      s_codes[c][r] = static_cast<uint8_t>(__nv_cvt_float_to_fp8(__fdiv_rn(x[k], s_scale[c]), __NV_SATFINITE, __NV_E4M3));
    }
  }
  __syncthreads();
  // thread t writes 64 codes (keys or pooled blocks [64 h, 64 h + 64)) of channel t / 2
  const int c = t >> 1, h = t & 1;
  uint8_t* dst = out + (static_cast<size_t>(bh) * kVD + c) * out_pitch + static_cast<size_t>(jb) * kTileRows + 64 * h;
#pragma unroll
  for (int i = 0; i < 4; ++i)
    *reinterpret_cast<uint4*>(dst + 16 * i) = *reinterpret_cast<const uint4*>(&s_codes[c][64 * h + 16 * i]);
}

// amax bits -> scales, in place
__global__ void __launch_bounds__(kVD) sol_v_scale_kernel(unsigned int* amax_then_scale) {
  const size_t i = static_cast<size_t>(blockIdx.x) * kVD + threadIdx.x;
  amax_then_scale[i] = __float_as_uint(channel_scale(amax_then_scale[i]));
}

}  // namespace

cudaError_t launch_quant_qk8(const QuantArgs& a, cudaStream_t stream) {
  if (a.d == 64) return launch_quant_d<64>(a, stream);
  if (a.d == 128) return launch_quant_d<128>(a, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_quant_v8(const QuantV8Args& a, cudaStream_t stream) {
  if (a.d != kVD) return cudaErrorInvalidValue;
  const int nkb = (a.L + kTileRows - 1) / kTileRows;
  const int nchunks = (nkb + kTileRows - 1) / kTileRows;
  unsigned int* amax = reinterpret_cast<unsigned int*>(a.v_scale);
  cudaError_t e = cudaMemsetAsync(amax, 0, static_cast<size_t>(a.BH) * kVD * 4, stream);
  if (e != cudaSuccess) return e;
  sol_v_amax_kernel<<<dim3(nkb, a.BH), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(a.V), amax, a.L);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sol_v_codes_kernel<__nv_bfloat16><<<dim3(nkb, a.BH), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(a.V), amax,
                                                                         a.v8t, a.L, nkb * kTileRows);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sol_v_codes_kernel<float><<<dim3(nchunks, a.BH), 256, 0, stream>>>(a.vbar, amax, a.vb8t, nkb, nchunks * kTileRows);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  sol_v_scale_kernel<<<a.BH, kVD, 0, stream>>>(amax);
  return cudaGetLastError();
}

}  // namespace sol
