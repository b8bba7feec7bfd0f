// Key/value block pooling: k_bar_j, v_bar_j = mean over the valid tokens of key block j.
// (Sol-Attn project page, Abstract: the routing proxy and the skipped-block correction read
// pooled block vectors.)
//
// HBM-bound: every K and V element is read exactly once with 16-byte vector loads; the output
// is 1/block of the input. One CTA pools one key block of one tensor (K or V) of one head.
// Each thread owns a 16-byte column slice and sums every `rows_per_pass`-th row in fp32. The row
// groups that share a warp are then added with warp shuffles, and the warps' sums through shared
// memory, always in the same order, so the result is deterministic.
#include <cuda_bf16.h>

#include "device_common.cuh"
#include "launchers.h"

namespace sol {

namespace {

constexpr int kPoolThreads = 256;

template <typename T>
__device__ __forceinline__ void add_vec(float (&acc)[16 / sizeof(T)], const uint4& raw);

template <>
__device__ __forceinline__ void add_vec<__nv_bfloat16>(float (&acc)[8], const uint4& raw) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}

template <>
__device__ __forceinline__ void add_vec<float>(float (&acc)[4], const uint4& raw) {
  acc[0] += __uint_as_float(raw.x);
  acc[1] += __uint_as_float(raw.y);
  acc[2] += __uint_as_float(raw.z);
  acc[3] += __uint_as_float(raw.w);
}

template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
    sol_pool_kernel(const T* __restrict__ K, const T* __restrict__ V, int L, int d, int block, int nkb,
                    float* __restrict__ kbar, float* __restrict__ vbar, __nv_bfloat16* __restrict__ kbar_lp,
                    __nv_bfloat16* __restrict__ vbar_lp) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int kWarps = kPoolThreads / 32;
  __shared__ float partial[kWarps][256];  // d <= 256 (bf16) or 128 (fp32)

  const int j = blockIdx.x;
  const int bh = blockIdx.y;
  const bool is_v = blockIdx.z != 0;
  const T* src = (is_v ? V : K) + (static_cast<size_t>(bh) * L + static_cast<size_t>(j) * block) * d;
  const int n = min(block, L - j * block);

  const int lanes_per_row = d / VEC;
  const int rows_per_pass = kPoolThreads / lanes_per_row;
  const int tid = threadIdx.x;
  const int c = tid % lanes_per_row;
  const int r0 = tid / lanes_per_row;

  float acc[VEC];
#pragma unroll
  for (int v = 0; v < VEC; ++v) acc[v] = 0.f;

  {
    const uint4* base = reinterpret_cast<const uint4*>(src) + c;
    const size_t row_stride = static_cast<size_t>(lanes_per_row);  // in uint4
    int r = r0;
    // four independent 16-byte loads in flight per thread
    for (; r + 3 * rows_per_pass < n; r += 4 * rows_per_pass) {
      uint4 x0 = __ldg(base + static_cast<size_t>(r) * row_stride);
      uint4 x1 = __ldg(base + static_cast<size_t>(r + rows_per_pass) * row_stride);
      uint4 x2 = __ldg(base + static_cast<size_t>(r + 2 * rows_per_pass) * row_stride);
      uint4 x3 = __ldg(base + static_cast<size_t>(r + 3 * rows_per_pass) * row_stride);
      add_vec<T>(acc, x0);
      add_vec<T>(acc, x1);
      add_vec<T>(acc, x2);
      add_vec<T>(acc, x3);
    }
    for (; r < n; r += rows_per_pass) add_vec<T>(acc, __ldg(base + static_cast<size_t>(r) * row_stride));
  }
  // the row groups inside a warp sit lanes_per_row lanes apart (lanes_per_row = d / VEC divides 32)
  for (int o = lanes_per_row; o < 32; o <<= 1) {
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] += __shfl_xor_sync(0xffffffffu, acc[v], o);
  }
  const int warp = tid >> 5, lane = tid & 31;
  if (lane < lanes_per_row) {
#pragma unroll
    for (int v = 0; v < VEC; ++v) partial[warp][c * VEC + v] = acc[v];
  }
  __syncthreads();

  float* out = (is_v ? vbar : kbar) + (static_cast<size_t>(bh) * nkb + j) * d;
  __nv_bfloat16* out_lp = is_v ? vbar_lp : kbar_lp;
  for (int col = tid; col < d; col += kPoolThreads) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += partial[w][col];
    const float mean = s / static_cast<float>(n);
    out[col] = mean;
    if (out_lp != nullptr) out_lp[(static_cast<size_t>(bh) * nkb + j) * d + col] = __float2bfloat16_rn(mean);
  }
}

}  // namespace

cudaError_t launch_pool(const void* K, const void* V, bool bf16, int BH, int L, int d, int block, float* kbar,
                        float* vbar, void* kbar_lp, void* vbar_lp, cudaStream_t stream) {
  const int nkb = (L + block - 1) / block;
  dim3 grid(nkb, BH, 2);
  if (bf16) {
    sol_pool_kernel<__nv_bfloat16><<<grid, kPoolThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(K), static_cast<const __nv_bfloat16*>(V), L, d, block, nkb, kbar, vbar,
        static_cast<__nv_bfloat16*>(kbar_lp), static_cast<__nv_bfloat16*>(vbar_lp));
  } else {
    sol_pool_kernel<float><<<grid, kPoolThreads, 0, stream>>>(static_cast<const float*>(K),
                                                               static_cast<const float*>(V), L, d, block, nkb,
                                                               kbar, vbar, nullptr, nullptr);
  }
  return cudaGetLastError();
}

}  // namespace sol
