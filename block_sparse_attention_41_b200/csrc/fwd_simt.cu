// fp32 Sol-Attn forward on CUDA cores (one CTA per query block of one head).
//
// Same method as the tensor-core kernel (Sol-Attn project page, Abstract: threshold routing,
// exact attention on kept blocks, correction of skipped blocks, one online softmax), in fp32
// throughout. tf32 tensor-core inputs would round Q and K to 10 mantissa bits, which is too
// coarse for a 1e-4 absolute tolerance, so this path stays on FMA units. It serves fp32 inputs
// (small head counts / sequence lengths); bf16 inputs take the tcgen05 kernel.
//
// Thread layout: TPR = D/32 threads per query row, each owning 32 consecutive channels of q
// and of the output accumulator. The TPR partial dot products are combined with xor shuffles,
// which add the same pairs in every lane, so all TPR lanes hold bitwise-identical logits and
// softmax state.
#include <cmath>

#include "device_common.cuh"
#include "launchers.h"

namespace sol {

namespace {

struct SimtParams {
  const float* Q;
  const float* K;
  const float* V;
  const float* kbar;
  const float* vbar;
  float* O;
  uint8_t* kept_mask;
  float* density;
  uint32_t* ws;
  int BH, H, L, nqb, nkb, n_force;
  float inv_sqrt_d;
  float tau[kMaxHeads];
};

template <int D, int BLK>
struct SimtCfg {
  static constexpr int TPR = D / 32;
  static constexpr int NT = BLK * TPR;
  static constexpr int NW = NT / 32;
  static constexpr int R0_FLOATS = (BLK > 64 ? BLK : 64) * D;  // Q rows, later 32 K + 32 V rows
  static constexpr size_t SMEM = sizeof(float) * (R0_FLOATS + D + kMaxKeyBlocks + 64) + kMaxKeyBlocks;
};

// Online-softmax merge of one term: weight w, logit x (natural base), value slice v[32].
__device__ __forceinline__ void merge_term(float x, float w, const float* v, float& m, float& l, float (&acc)[32]) {
  if (x > m) {
    const float c = expf(m - x);
    l = fmaf(l, c, w);
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = fmaf(acc[i], c, w * v[i]);
    m = x;
  } else {
    const float e = w * expf(x - m);
    l += e;
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = fmaf(e, v[i], acc[i]);
  }
}

template <int TPR>
__device__ __forceinline__ float row_allreduce(float v) {
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int D, int BLK>
__global__ void __launch_bounds__(SimtCfg<D, BLK>::NT)
    sol_fwd_simt_kernel(const __grid_constant__ SimtParams p) {
  using C = SimtCfg<D, BLK>;
  extern __shared__ float sm[];
  float* R0 = sm;
  float* qbar = R0 + C::R0_FLOATS;
  float* sbar = qbar + D;
  float* red = sbar + kMaxKeyBlocks;  // 32 floats + 32 ints
  int* ired = reinterpret_cast<int*>(red + 32);
  uint8_t* keep = reinterpret_cast<uint8_t*>(red + 64);

  const int unit = blockIdx.x;
  const int bh = unit / p.nqb, qb = unit % p.nqb, h = bh % p.H;
  const int tid = threadIdx.x, row = tid / C::TPR, part = tid % C::TPR;
  const int lane = tid & 31, warp = tid >> 5;
  const int L = p.L, nkb = p.nkb;
  const int m_i = min(BLK, L - qb * BLK);
  const size_t head_off = static_cast<size_t>(bh) * L * D;

  if (tid == 0) ired[0] = 0;

  // 1. this thread's 32 channels of its query row (zeros past the valid rows)
  float q[32];
  {
    const bool valid = row < m_i;
    const float4* src = reinterpret_cast<const float4*>(p.Q + head_off + static_cast<size_t>(qb * BLK + row) * D +
                                                        part * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 v = valid ? __ldg(src + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      q[4 * i] = v.x; q[4 * i + 1] = v.y; q[4 * i + 2] = v.z; q[4 * i + 3] = v.w;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) R0[row * D + part * 32 + i] = q[i];
  }
  __syncthreads();

  // 2. q_bar: mean of the valid query rows of this block
  for (int c = tid; c < D; c += C::NT) {
    float s = 0.f;
    for (int r = 0; r < m_i; ++r) s += R0[r * D + c];
    qbar[c] = s / static_cast<float>(m_i);
  }
  __syncthreads();

  // 3. routing: s_bar_j = q_bar . k_bar_j / sqrt(d), kept iff >= max - tau (or forced)
  const float* kb = p.kbar + static_cast<size_t>(bh) * nkb * D;
  float wmax = -INFINITY;
  for (int j = warp; j < nkb; j += C::NW) {
    float dot = 0.f;
#pragma unroll
    for (int c = lane; c < D; c += 32) dot = fmaf(qbar[c], __ldg(kb + static_cast<size_t>(j) * D + c), dot);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    const float s = dot * p.inv_sqrt_d;
    if (lane == 0) sbar[j] = s;
    wmax = fmaxf(wmax, s);
  }
  if (lane == 0) red[warp] = wmax;
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < C::NW; ++w) M = fmaxf(M, red[w]);
  const float thr = M - p.tau[h];
  int cnt = 0;
  for (int j = tid; j < nkb; j += C::NT) {
    const uint8_t k = (sbar[j] >= thr) || (j < p.n_force);
    keep[j] = k;
    cnt += k;
    if (p.kept_mask != nullptr) p.kept_mask[(static_cast<size_t>(bh) * p.nqb + qb) * nkb + j] = k;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) atomicAdd(&ired[0], cnt);
  __syncthreads();
  if (tid == 0) atomicAdd(&p.ws[WS_COUNTS + bh], static_cast<uint32_t>(ired[0]));

  // 4. one online-softmax pass over kept tokens and pooled skipped blocks, in block order
  float m = -INFINITY, l = 0.f, acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = 0.f;
  const float* Kh = p.K + head_off;
  const float* Vh = p.V + head_off;
  const float* vb = p.vbar + static_cast<size_t>(bh) * nkb * D;
  float* Ks = R0;
  float* Vs = R0 + 32 * D;
  for (int j = 0; j < nkb; ++j) {
    const int n_j = min(BLK, L - j * BLK);
    if (keep[j]) {
      for (int kc = 0; kc < n_j; kc += 32) {
        const int nk = min(32, n_j - kc);
        __syncthreads();
        const float4* ksrc = reinterpret_cast<const float4*>(Kh + static_cast<size_t>(j * BLK + kc) * D);
        const float4* vsrc = reinterpret_cast<const float4*>(Vh + static_cast<size_t>(j * BLK + kc) * D);
        for (int e = tid; e < nk * D / 4; e += C::NT) {
          reinterpret_cast<float4*>(Ks)[e] = __ldg(ksrc + e);
          reinterpret_cast<float4*>(Vs)[e] = __ldg(vsrc + e);
        }
        __syncthreads();
        for (int t = 0; t < nk; ++t) {
          const float* kt = Ks + t * D + part * 32;
          float dot = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) dot = fmaf(q[i], kt[i], dot);
          dot = row_allreduce<C::TPR>(dot);
          merge_term(dot * p.inv_sqrt_d, 1.f, Vs + t * D + part * 32, m, l, acc);
        }
      }
    } else {
      const float* kbj = kb + static_cast<size_t>(j) * D + part * 32;
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) dot = fmaf(q[i], __ldg(kbj + i), dot);
      dot = row_allreduce<C::TPR>(dot);
      float vv[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) vv[i] = __ldg(vb + static_cast<size_t>(j) * D + part * 32 + i);
      merge_term(dot * p.inv_sqrt_d, static_cast<float>(n_j), vv, m, l, acc);
    }
  }

  // 5. epilogue
  if (row < m_i) {
    const float inv = 1.f / l;
    float4* dst = reinterpret_cast<float4*>(p.O + head_off + static_cast<size_t>(qb * BLK + row) * D + part * 32);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      dst[i] = make_float4(acc[4 * i] * inv, acc[4 * i + 1] * inv, acc[4 * i + 2] * inv, acc[4 * i + 3] * inv);
  }

  // 6. the last CTA to finish turns kept-block counts into per-head densities
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    ired[1] = (atomicAdd(&p.ws[WS_DONE], 1u) == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (ired[1] && p.density != nullptr) {
    __threadfence();
    const double denom = static_cast<double>(p.nqb) * static_cast<double>(nkb);
    for (int i = tid; i < p.BH; i += C::NT)
      p.density[i] = static_cast<float>(static_cast<double>(atomicAdd(&p.ws[WS_COUNTS + i], 0u)) / denom);
  }
}

template <int D, int BLK>
cudaError_t launch_simt_t(const FwdArgs& a, cudaStream_t stream) {
  using C = SimtCfg<D, BLK>;
  SimtParams p;
  p.Q = static_cast<const float*>(a.Q);
  p.K = static_cast<const float*>(a.K);
  p.V = static_cast<const float*>(a.V);
  p.kbar = a.kbar;
  p.vbar = a.vbar;
  p.O = static_cast<float*>(a.O);
  p.kept_mask = a.kept_mask;
  p.density = a.density;
  p.ws = a.ws;
  p.BH = a.B * a.H;
  p.H = a.H;
  p.L = a.L;
  p.nqb = (a.L + BLK - 1) / BLK;
  p.nkb = p.nqb;
  p.n_force = a.n_force;
  p.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  for (int h = 0; h < kMaxHeads; ++h) p.tau[h] = h < a.H ? a.tau[h] : 0.f;
  cudaError_t e = cudaFuncSetAttribute(sol_fwd_simt_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::SMEM));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(p.BH) * static_cast<unsigned>(p.nqb);
  sol_fwd_simt_kernel<D, BLK><<<grid, C::NT, C::SMEM, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdArgs& a, cudaStream_t stream) {
  switch (a.d * 1000 + a.block) {
    case 32032: return launch_simt_t<32, 32>(a, stream);
    case 32064: return launch_simt_t<32, 64>(a, stream);
    case 32128: return launch_simt_t<32, 128>(a, stream);
    case 64032: return launch_simt_t<64, 32>(a, stream);
    case 64064: return launch_simt_t<64, 64>(a, stream);
    case 64128: return launch_simt_t<64, 128>(a, stream);
    case 128032: return launch_simt_t<128, 32>(a, stream);
    case 128064: return launch_simt_t<128, 64>(a, stream);
    case 128128: return launch_simt_t<128, 128>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace sol
