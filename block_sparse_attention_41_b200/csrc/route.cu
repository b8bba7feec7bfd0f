// Routing pass of the bf16 Sol-Attn forward (Sol-Attn project page, Abstract: the kept key blocks of
// each query block are chosen on the fly by a query-dependent threshold on a cheap proxy score).
//
// For a run of R query blocks of one head, one CTA computes
//   q_bar_i  = mean of the valid query rows of block i          (from Q in global memory)
//   s_bar_ij = q_bar_i . k_bar_j / sqrt(d) for every key block j  (fp32, shared memory only)
//   keep_ij  = s_bar_ij >= max_j s_bar_ij - tau[h]  or  j < n_force
// and writes only the keep bits (one u32 word per 32 key blocks), the optional uint8 mask, and the
// per-head kept-block count. The proxy scores never leave shared memory.
//
// Doing this for R query blocks at once reads each head's pooled keys once per R units instead of
// once per unit; the fused forward then only turns the bits into its tile lists.
#include <cmath>

#include "device_common.cuh"
#include "launchers.h"

namespace sol {

namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kRows = 128;

struct RouteParams {
  const __nv_bfloat16* Q;  // [BH, L, D]
  const float* kbar;       // [BH, nkb, D] fp32
  uint32_t* bits;          // [BH, nqb, nwords]
  uint8_t* kept_mask;      // [BH, nqb, nkb] or null
  uint32_t* counts;        // [BH] kept blocks per head (accumulated)
  int BH, H, L, nqb, nkb, nwords, n_force;
  float inv_sqrt_d;
  float tau[kMaxHeads];
};

// Sum each of the N values of a lane over the 32 lanes, with N - 1 + (5 - log2 N) shuffles instead
// of 5 N: at every butterfly step a lane keeps half of its values and receives the partner's
// copies of that half, until one value is left. The additions follow the same pairwise tree as
// the plain xor reduction (a lane adds its own value and its partner's at every level), so the
// sums are bit-identical to it. On return v[0] holds the total of value r = lane >> (5 - log2 N):
// the first step decides the top bit of r from lane bit 4, the next from lane bit 3, and so on.
template <int N, int O = 16>
__device__ __forceinline__ void butterfly_sum(float (&v)[N], int lane) {
  if constexpr (O >= 1) {
    if constexpr (N > 1) {
      constexpr int H = N / 2;
      const bool hi = (lane & O) != 0;
#pragma unroll
      for (int k = 0; k < H; ++k) {
        const float send = hi ? v[k] : v[H + k];
        const float keep = hi ? v[H + k] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, O);
      }
      float (&w)[H] = *reinterpret_cast<float (*)[H]>(&v[0]);
      butterfly_sum<H, O / 2>(w, lane);
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], O);
      butterfly_sum<1, O / 2>(v, lane);
    }
  }
}

template <int D, int R>
__global__ void __launch_bounds__(kRouteThreads) sol_route_kernel(const __grid_constant__ RouteParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* s_qbar = reinterpret_cast<float*>(smem_raw);  // [R][D]
  float* s_sc = s_qbar + R * D;                         // [R][nkb]; its start also holds the q_bar partials
  __shared__ uint32_t s_cnt;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int qb0 = blockIdx.x * R;
  const int nr = min(R, p.nqb - qb0);
  const int nkb = p.nkb;
  if (tid == 0) s_cnt = 0;

  // (1) q_bar of each of the nr query blocks, four blocks at a time: thread t sums a 16-byte chunk
  // (8 columns) of each over a strided set of rows (the same rows, in the same order, as the fused
  // kernel's own routing); partial sums meet in shared memory
  {
    constexpr int CH = D / 8;
    constexpr int RG = kRouteThreads / CH;
    constexpr int NB = 4;
    const int c8 = tid % CH, rg = tid / CH;
    float* part = s_sc;  // [NB][RG][D]
    for (int r0 = 0; r0 < nr; r0 += NB) {
      float a[NB][8];
      int m[NB];
#pragma unroll
      for (int rb = 0; rb < NB; ++rb) {
        m[rb] = (r0 + rb < nr) ? min(kRows, p.L - (qb0 + r0 + rb) * kRows) : 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) a[rb][k] = 0.f;
      }
      const __nv_bfloat16* qrow = p.Q + (static_cast<size_t>(bh) * p.L + static_cast<size_t>(qb0 + r0) * kRows) * D + c8 * 8;
#pragma unroll 2
      for (int rr = rg; rr < kRows; rr += RG) {
        uint4 v[NB];
#pragma unroll
        for (int rb = 0; rb < NB; ++rb)
          if (rr < m[rb]) v[rb] = __ldg(reinterpret_cast<const uint4*>(qrow + static_cast<size_t>(rb * kRows + rr) * D));
#pragma unroll
        for (int rb = 0; rb < NB; ++rb) {
          if (rr < m[rb]) {
            const uint32_t wv[4] = {v[rb].x, v[rb].y, v[rb].z, v[rb].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              a[rb][2 * k] += __uint_as_float(wv[k] << 16);
              a[rb][2 * k + 1] += __uint_as_float(wv[k] & 0xffff0000u);
            }
          }
        }
      }
#pragma unroll
      for (int rb = 0; rb < NB; ++rb)
#pragma unroll
        for (int k = 0; k < 8; ++k) part[(rb * RG + rg) * D + c8 * 8 + k] = a[rb][k];
      __syncthreads();
      for (int idx = tid; idx < NB * D; idx += kRouteThreads) {
        const int rb = idx / D, c = idx % D;
        if (r0 + rb < nr) {
          float q = 0.f;
          for (int k = 0; k < RG; ++k) q += part[(rb * RG + k) * D + c];
          s_qbar[(r0 + rb) * D + c] = q / static_cast<float>(m[rb]);
        }
      }
      __syncthreads();
    }
  }

  // (2) proxy scores: warp w takes key blocks w, w + 8, ...; lane l holds components [l DPL, (l+1) DPL)
  {
    constexpr int DPL = D / 32;
    const float* kb = p.kbar + static_cast<size_t>(bh) * nkb * D + lane * DPL;
    constexpr int U = 4;  // key blocks in flight per warp
    for (int j0 = warp; j0 < nkb; j0 += kRouteWarps * U) {
      float kv[U][DPL];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + kRouteWarps * u;
#pragma unroll
        for (int k = 0; k < DPL; ++k) kv[u][k] = 0.f;
        if (j < nkb) {
          if constexpr (DPL == 4) {
            const float4 v = __ldg(reinterpret_cast<const float4*>(kb + static_cast<size_t>(j) * D));
            kv[u][0] = v.x; kv[u][1] = v.y; kv[u][2] = v.z; kv[u][3] = v.w;
          } else {
            const float2 v = __ldg(reinterpret_cast<const float2*>(kb + static_cast<size_t>(j) * D));
            kv[u][0] = v.x; kv[u][1] = v.y;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + kRouteWarps * u;
        float dot[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          // the same fp32 operation order as the fused kernel's own routing, so both give the
          // same keep bits
          if constexpr (DPL == 4) {
            const float4 qv = *reinterpret_cast<const float4*>(s_qbar + r * D + lane * DPL);
            dot[r] = fmaf(qv.x, kv[u][0], fmaf(qv.y, kv[u][1], fmaf(qv.z, kv[u][2], qv.w * kv[u][3])));
          } else {
            const float2 qv = *reinterpret_cast<const float2*>(s_qbar + r * D + lane * DPL);
            dot[r] = fmaf(qv.x, kv[u][0], qv.y * kv[u][1]);
          }
        }
        butterfly_sum<R>(dot, lane);
        // lane l now holds the total of query block r(l); the lanes that agree on r hold the same value
        constexpr int LOGR = R == 16 ? 4 : (R == 8 ? 3 : 2);
        const int r = lane >> (5 - LOGR);
        if ((lane & ((32 >> LOGR) - 1)) == 0 && j < nkb && r < nr) s_sc[r * nkb + j] = dot[0] * p.inv_sqrt_d;
      }
    }
  }
  __syncthreads();

  // (3) per query block: max, threshold, keep bits, mask bytes, count (warp w takes blocks w, w + 8, ...)
  {
    const float tau = p.tau[bh % p.H];
    uint32_t kept = 0;
    for (int r = warp; r < nr; r += kRouteWarps) {
      const float* sc = s_sc + r * nkb;
      float M = -INFINITY;
      for (int j = lane; j < nkb; j += 32) M = fmaxf(M, sc[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      const float thr = M - tau;
      const size_t unit = static_cast<size_t>(bh) * p.nqb + qb0 + r;
      uint32_t* bw = p.bits + unit * p.nwords;
      uint8_t* mrow = p.kept_mask != nullptr ? p.kept_mask + unit * nkb : nullptr;
      for (int i = 0; i < p.nwords; ++i) {
        const int j = 32 * i + lane;
        const bool k = j < nkb && (sc[j] >= thr || j < p.n_force);
        const uint32_t m = __ballot_sync(0xffffffffu, k);
        if (lane == 0) bw[i] = m;
        if (mrow != nullptr && j < nkb) mrow[j] = k ? 1 : 0;
        kept += __popc(m);
      }
    }
    if (lane == 0 && kept) atomicAdd(&s_cnt, kept);
  }
  __syncthreads();
  if (tid == 0 && s_cnt) atomicAdd(&p.counts[bh], s_cnt);
}

template <int D, int R>
cudaError_t launch_route_t(const FwdArgs& a, cudaStream_t stream) {
  RouteParams p;
  p.Q = static_cast<const __nv_bfloat16*>(a.Q);
  p.kbar = a.kbar;
  p.bits = a.route_bits;
  p.kept_mask = a.kept_mask;
  p.counts = a.ws + WS_COUNTS;
  p.BH = a.B * a.H;
  p.H = a.H;
  p.L = a.L;
  p.nqb = (a.L + kRows - 1) / kRows;
  p.nkb = p.nqb;
  p.nwords = (p.nkb + 31) / 32;
  p.n_force = a.n_force;
  p.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  for (int h = 0; h < kMaxHeads; ++h) p.tau[h] = h < a.H ? a.tau[h] : 0.f;
  constexpr int RG = kRouteThreads / (D / 8);
  const size_t part_floats = static_cast<size_t>(4) * RG * D;  // q_bar partial sums of four blocks
  const size_t sc_floats = static_cast<size_t>(R) * p.nkb > part_floats ? static_cast<size_t>(R) * p.nkb : part_floats;
  const size_t smem = (static_cast<size_t>(R) * D + sc_floats) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(sol_route_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid((p.nqb + R - 1) / R, p.BH);
  sol_route_kernel<D, R><<<grid, kRouteThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_route_d(const FwdArgs& a, cudaStream_t stream) {
  const int nkb = (a.L + kRows - 1) / kRows;
  // keep the score buffer (R x N_kb floats) within 64 KB
  if (nkb <= 1024) return launch_route_t<D, 16>(a, stream);
  if (nkb <= 2048) return launch_route_t<D, 8>(a, stream);
  return launch_route_t<D, 4>(a, stream);
}

}  // namespace

cudaError_t launch_route(const FwdArgs& a, cudaStream_t stream) {
  if (a.d == 64) return launch_route_d<64>(a, stream);
  if (a.d == 128) return launch_route_d<128>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sol
