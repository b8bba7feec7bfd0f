// Fused QK-norm + rotary embedding + block pooling, the step before the sparse attention
// (Sol-Engine README, "The five acceleration methods": kernel fusion of the memory-bound DiT glue,
// QK-norm + RoPE; news list: "fused QK+RoPE").
//
// One CTA per (key block, head). For each of the block's valid tokens t and for Q and K:
//   y   = x / sqrt(mean(x^2) + eps) * gain             (RMS norm over the head dimension)
//   y'  = pairs (y_2i, y_2i+1) turned by the angle of cos/sin[t, i]
// and the rotated rows are stored in bf16. The same pass sums the stored (bf16-rounded) keys and
// the values of the block into the pooled vectors the sparse attention routes and corrects with,
// so the keys are not read back from HBM by a separate pooling pass. Optionally it also writes the
// mean of the block's stored query rows (q_bar, the routing proxy's query side), so the routing
// pass need not read Q again either.
//
// Layout: a lane owns 8 consecutive columns (16 bytes, four whole pairs) of one row; D/8 lanes
// cover a row, so a warp covers 32 / (D/8) rows at once and the row's sum of squares is reduced
// over those lanes only. HBM-bound: every byte is read or written once. The grid runs the heads
// of one token range next to each other (head = blockIdx.x), so the cos/sin rows of that range
// come from L2 for all but the first head.
#include <cmath>

#include "device_common.cuh"
#include "launchers.h"

namespace sol {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kBlocksPerCta = 4;  // consecutive key blocks per CTA: amortises launch and the final reduction

struct RopePoolParams {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const float* gq;   // [D]
  const float* gk;   // [D]
  const float* cs;   // cos [L, D/2]
  const float* sn;   // sin [L, D/2]
  __nv_bfloat16* Qo;
  __nv_bfloat16* Ko;
  float* kbar;             // [BH, nkb, D]
  float* vbar;             // [BH, nkb, D]
  __nv_bfloat16* kbar_lp;  // [BH, nkb, D]
  __nv_bfloat16* vbar_lp;  // [BH, nkb, D]
  float* qbar;             // [BH, nkb, D] query-block means, or null
  int L, nkb, block;
  float eps;
};

__device__ __forceinline__ void unpack8(const uint4 v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    x[2 * k] = __uint_as_float(w[k] << 16);
    x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
  }
}

// Norm, rotate and store (unless dst is null) one 8-column chunk of a row; returns the stored
// values (as fp32) in x. All lanes of the warp must call it together.
template <int LPR>
__device__ __forceinline__ void norm_rope_chunk(float (&x)[8], const float* gain, const float* cs, const float* sn,
                                                int c0, float inv_d, float eps, __nv_bfloat16* dst) {
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) ss = fmaf(x[k], x[k], ss);
#pragma unroll
  for (int o = LPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = 1.0f / sqrtf(ss * inv_d + eps);
  const float4 g0 = *reinterpret_cast<const float4*>(gain + c0);
  const float4 g1 = *reinterpret_cast<const float4*>(gain + c0 + 4);
  const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
  const float4 c = *reinterpret_cast<const float4*>(cs + c0 / 2);
  const float4 s = *reinterpret_cast<const float4*>(sn + c0 / 2);
  const float cc[4] = {c.x, c.y, c.z, c.w}, ssn[4] = {s.x, s.y, s.z, s.w};
  uint32_t pk[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = x[2 * i] * inv * g[2 * i];
    const float b = x[2 * i + 1] * inv * g[2 * i + 1];
    const float ra = fmaf(a, cc[i], -b * ssn[i]);
    const float rb = fmaf(a, ssn[i], b * cc[i]);
    pk[i] = pack_bf16x2(ra, rb);
    x[2 * i] = __uint_as_float(pk[i] << 16);
    x[2 * i + 1] = __uint_as_float(pk[i] & 0xffff0000u);
  }
  if (dst != nullptr) *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
}

template <int D>
__global__ void __launch_bounds__(kThreads) sol_qknorm_rope_pool_kernel(const __grid_constant__ RopePoolParams p) {
  constexpr int LPR = D / 8;          // lanes per row
  constexpr int RPW = 32 / LPR;       // rows per warp step
  constexpr int RG = kWarps * RPW;    // row groups per CTA
  __shared__ float s_part[3][RG][D];  // per row group partial sums of the stored keys / the values / the stored queries

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const int cl = lane % LPR, sub = lane / LPR;
  const int c0 = cl * 8;
  const int rg = warp * RPW + sub;
  const float inv_d = 1.0f / static_cast<float>(D);
  const int jb_end = min(p.nkb, (static_cast<int>(blockIdx.y) + 1) * kBlocksPerCta);
  for (int jb = blockIdx.y * kBlocksPerCta; jb < jb_end; ++jb) {
    const int row0 = jb * p.block;
    const int n = min(p.block, p.L - row0);
    const size_t base = (static_cast<size_t>(bh) * p.L + row0) * D + c0;

    float ak[8], av[8], aq[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) ak[k] = av[k] = aq[k] = 0.f;
    // the loop runs the same number of times in every lane of a warp (the norm's shuffles need the
    // whole warp); lanes past the block's last row carry zeros and store nothing
    for (int rbase = warp * RPW; rbase < n; rbase += RG) {
      const int r = rbase + sub;
      const bool valid = r < n;
      const size_t off = base + static_cast<size_t>(valid ? r : 0) * D;
      const int t = row0 + (valid ? r : 0);
      const float* cs = p.cs + static_cast<size_t>(t) * (D / 2);
      const float* sn = p.sn + static_cast<size_t>(t) * (D / 2);
      float xq[8], xk[8], xv[8];
      const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
      unpack8(valid ? __ldg(reinterpret_cast<const uint4*>(p.Q + off)) : zero, xq);
      unpack8(valid ? __ldg(reinterpret_cast<const uint4*>(p.K + off)) : zero, xk);
      unpack8(valid ? __ldg(reinterpret_cast<const uint4*>(p.V + off)) : zero, xv);
      norm_rope_chunk<LPR>(xq, p.gq, cs, sn, c0, inv_d, p.eps, valid ? p.Qo + off : nullptr);
      norm_rope_chunk<LPR>(xk, p.gk, cs, sn, c0, inv_d, p.eps, valid ? p.Ko + off : nullptr);
      if (valid) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          ak[k] += xk[k];
          av[k] += xv[k];
          aq[k] += xq[k];
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      s_part[0][rg][c0 + k] = ak[k];
      s_part[1][rg][c0 + k] = av[k];
      s_part[2][rg][c0 + k] = aq[k];
    }
    __syncthreads();
    // index i < 3 D: column i % D of the keys, the values or the queries (i / D = 0, 1, 2)
    const int nsum = p.qbar != nullptr ? 3 * D : 2 * D;
    for (int i = tid; i < nsum; i += kThreads) {
      const int which = i / D, c = i % D;
      float sum = 0.f;
#pragma unroll 4
      for (int k = 0; k < RG; ++k) sum += s_part[which][k][c];
      const float mean = sum / static_cast<float>(n);
      const size_t o = (static_cast<size_t>(bh) * p.nkb + jb) * D + c;
      if (which == 0) {
        p.kbar[o] = mean;
        p.kbar_lp[o] = __float2bfloat16_rn(mean);
      } else if (which == 1) {
        p.vbar[o] = mean;
        p.vbar_lp[o] = __float2bfloat16_rn(mean);
      } else {
        p.qbar[o] = mean;
      }
    }
    __syncthreads();  // s_part is reused by the next block
  }
}

template <int D>
cudaError_t launch_t(const RopePoolArgs& a, cudaStream_t stream) {
  RopePoolParams p;
  p.Q = static_cast<const __nv_bfloat16*>(a.Q);
  p.K = static_cast<const __nv_bfloat16*>(a.K);
  p.V = static_cast<const __nv_bfloat16*>(a.V);
  p.gq = a.gain_q;
  p.gk = a.gain_k;
  p.cs = a.cos;
  p.sn = a.sin;
  p.Qo = static_cast<__nv_bfloat16*>(a.Qout);
  p.Ko = static_cast<__nv_bfloat16*>(a.Kout);
  p.kbar = a.kbar;
  p.vbar = a.vbar;
  p.kbar_lp = static_cast<__nv_bfloat16*>(a.kbar_lp);
  p.vbar_lp = static_cast<__nv_bfloat16*>(a.vbar_lp);
  p.qbar = a.qbar;
  p.L = a.L;
  p.block = a.block;
  p.nkb = (a.L + a.block - 1) / a.block;
  p.eps = a.eps;
  const dim3 grid(a.BH, (p.nkb + kBlocksPerCta - 1) / kBlocksPerCta);
  sol_qknorm_rope_pool_kernel<D><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qknorm_rope_pool(const RopePoolArgs& a, cudaStream_t stream) {
  if (a.d == 64) return launch_t<64>(a, stream);
  if (a.d == 128) return launch_t<128>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sol
