// Routing pass of the bf16 Sol-Attn forward (Sol-Attn project page, Abstract: the kept key blocks of
// each query block are chosen on the fly by a query-dependent threshold on a cheap proxy score).
//
// Two kernels. The first, sol_qbar_kernel, streams Q once at full HBM bandwidth and writes
//   q_bar_i  = mean of the valid query rows of block i          (fp32, into the workspace)
// for every query block. The second, for a run of R query blocks of one head per CTA, computes
//   s_bar_ij = q_bar_i . k_bar_j / sqrt(d) for every key block j  (fp32, shared memory only)
//   keep_ij  = s_bar_ij >= max_j s_bar_ij - tau[h]  or  j < n_force
// or, in fixed-sparsity mode, keep_ij = j among the k highest s_bar_ij (equal scores: the lower
// index first) or j < n_force, and writes only the keep bits (one u32 word per 32 key blocks), the optional uint8 mask, and the
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
  const float* qbar;       // [BH, nqb, D] fp32, from sol_qbar_kernel
  const float* kbar;       // [BH, nkb, D] fp32
  uint32_t* bits;          // [BH, nqb, nwords]
  uint8_t* kept_mask;      // [BH, nqb, nkb] or null
  uint32_t* counts;        // [BH] kept blocks per head (accumulated)
  int BH, H, L, nqb, nkb, nwords, n_force;
  int k_keep;  // 0: threshold routing; k > 0: the k highest scores
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

// A 32-bit key whose unsigned order is the order of the fp32 scores (-0 counted as +0).
__device__ __forceinline__ uint32_t ordered_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);  // -0 + 0 = +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The lowest n set bits of m.
__device__ __forceinline__ uint32_t lowest_bits(uint32_t m, int n) {
  uint32_t r = 0;
  for (int i = 0; i < n && m; ++i) {
    const uint32_t b = m & (0u - m);
    r |= b;
    m ^= b;
  }
  return r;
}

// Key of the k-th highest of the nkb scores in sc (k >= 1), and how many scores equal to it are
// among the k highest. One warp, a 256-bin histogram per 8 key bits, most significant first.
__device__ __forceinline__ void radix_select_kth(const float* sc, int nkb, int k, uint32_t* hist, int lane,
                                                 uint32_t* key_out, int* eq_out) {
  uint32_t prefix = 0, pmask = 0;
  int kk = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = lane; b < 256; b += 32) hist[b] = 0;
    __syncwarp();
    for (int j = lane; j < nkb; j += 32) {
      const uint32_t key = ordered_key(sc[j]);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncwarp();
    // lane l holds bins [8l, 8l + 8); count the candidates in higher bins, from the top
    uint32_t c[8], lsum = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      c[q] = hist[8 * lane + q];
      lsum += c[q];
    }
    uint32_t suf = lsum;  // candidates in lanes lane .. 31
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, suf, o);
      if (lane + o < 32) suf += y;
    }
    const uint32_t above = suf - lsum;
    const bool mine = above < static_cast<uint32_t>(kk) && static_cast<uint32_t>(kk) <= suf;
    const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
    int bin = 0;
    uint32_t higher = 0;
    if (mine) {
      uint32_t acc = above;
      int qsel = -1;
#pragma unroll
      for (int q = 7; q >= 0; --q) {  // the highest bin whose count reaches the k-th score
        const bool hit = qsel < 0 && acc + c[q] >= static_cast<uint32_t>(kk);
        if (hit) {
          qsel = q;
          higher = acc;
        }
        acc += c[q];
      }
      bin = 8 * lane + qsel;
    }
    bin = __shfl_sync(0xffffffffu, bin, src);
    higher = __shfl_sync(0xffffffffu, higher, src);
    prefix |= static_cast<uint32_t>(bin) << shift;
    pmask |= 255u << shift;
    kk -= static_cast<int>(higher);
    __syncwarp();
  }
  *key_out = prefix;
  *eq_out = kk;
}

// q_bar of QB query blocks of one head per CTA. Thread t sums one 16-byte chunk (8 columns) of a
// block over the rows r = rg, rg + RG, ... in ascending order (rg = t / (D / 8), RG = 256 / (D / 8)),
// then the RG partial sums of a column are added in the order rg = 0, 1, ... and divided by the
// number of valid rows. The fused kernel's own routing (from its Q tile) takes exactly these
// fp32 operations in this order, so both routing paths get the same q_bar bit for bit. All of a
// thread's loads are issued before the first addition, so each CTA keeps QB * 16 KB (d = 128) of
// Q in flight.
template <int D, int QB>
__global__ void __launch_bounds__(kRouteThreads) sol_qbar_kernel(const __nv_bfloat16* __restrict__ Q,
                                                                 float* __restrict__ qbar, int L, int nqb) {
  constexpr int CH = D / 8;
  constexpr int RG = kRouteThreads / CH;
  constexpr int RPT = kRows / RG;  // rows per thread and block
  __shared__ float part[QB][RG][D];
  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int qb0 = blockIdx.x * QB;
  const int c8 = tid % CH, rg = tid / CH;
  uint4 v[QB][RPT];
  int m[QB];
#pragma unroll
  for (int b = 0; b < QB; ++b) {
    m[b] = (qb0 + b < nqb) ? min(kRows, L - (qb0 + b) * kRows) : 0;
    const __nv_bfloat16* base = Q + (static_cast<size_t>(bh) * L + static_cast<size_t>(qb0 + b) * kRows) * D + c8 * 8;
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      const int r = rg + k * RG;
      v[b][k] = r < m[b] ? __ldg(reinterpret_cast<const uint4*>(base + static_cast<size_t>(r) * D))
                         : make_uint4(0u, 0u, 0u, 0u);
    }
  }
#pragma unroll
  for (int b = 0; b < QB; ++b) {
    float a[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] = 0.f;
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
      if (rg + k * RG < m[b]) {
        const uint32_t wv[4] = {v[b][k].x, v[b][k].y, v[b][k].z, v[b][k].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          a[2 * q] += __uint_as_float(wv[q] << 16);
          a[2 * q + 1] += __uint_as_float(wv[q] & 0xffff0000u);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) part[b][rg][c8 * 8 + k] = a[k];
  }
  __syncthreads();
  for (int idx = tid; idx < QB * D; idx += kRouteThreads) {
    const int b = idx / D, c = idx % D;
    if (m[b] > 0) {
      float q = 0.f;
#pragma unroll 8
      for (int k = 0; k < RG; ++k) q += part[b][k][c];
      qbar[(static_cast<size_t>(bh) * nqb + qb0 + b) * D + c] = q / static_cast<float>(m[b]);
    }
  }
}

template <int D, int R>
__global__ void __launch_bounds__(kRouteThreads) sol_route_kernel(const __grid_constant__ RouteParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  float* s_qbar = reinterpret_cast<float*>(smem_raw);  // [R][D]
  float* s_sc = s_qbar + R * D;                         // [R][nkb] proxy scores
  __shared__ uint32_t s_cnt;
  __shared__ uint32_t s_hist[kRouteWarps][256];  // fixed-sparsity mode: one histogram per warp

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int qb0 = blockIdx.x * R;
  const int nr = min(R, p.nqb - qb0);
  const int nkb = p.nkb;
  if (tid == 0) s_cnt = 0;

  // (1) q_bar of the nr query blocks, from the workspace
  {
    const float* src = p.qbar + (static_cast<size_t>(bh) * p.nqb + qb0) * D;
    for (int idx = tid; idx < nr * D; idx += kRouteThreads) s_qbar[idx] = src[idx];
  }
  __syncthreads();

  // (2) proxy scores: warp w takes key blocks w, w + 8, ...; lane l holds components [l DPL, (l+1) DPL)
  // of every q_bar in registers for the whole loop (re-reading them from shared memory for each key
  // block would make shared-memory bandwidth the bound)
  {
    constexpr int DPL = D / 32;
    float qv[R][DPL];
#pragma unroll
    for (int r = 0; r < R; ++r) {
#pragma unroll
      for (int k = 0; k < DPL; ++k) qv[r][k] = r < nr ? s_qbar[r * D + lane * DPL + k] : 0.f;
    }
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
            dot[r] = fmaf(qv[r][0], kv[u][0], fmaf(qv[r][1], kv[u][1], fmaf(qv[r][2], kv[u][2], qv[r][3] * kv[u][3])));
          } else {
            dot[r] = fmaf(qv[r][0], kv[u][0], qv[r][1] * kv[u][1]);
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

  // (3) per query block: max, threshold (or the k-th highest score), keep bits, mask bytes, count
  // (warp w takes blocks w, w + 8, ...)
  if (p.k_keep > 0) {
    uint32_t kept = 0;
    for (int r = warp; r < nr; r += kRouteWarps) {
      const float* sc = s_sc + r * nkb;
      uint32_t kth;
      int take;  // scores equal to the k-th one still to keep, lowest index first
      radix_select_kth(sc, nkb, p.k_keep, s_hist[warp], lane, &kth, &take);
      const size_t unit = static_cast<size_t>(bh) * p.nqb + qb0 + r;
      uint32_t* bw = p.bits + unit * p.nwords;
      uint8_t* mrow = p.kept_mask != nullptr ? p.kept_mask + unit * nkb : nullptr;
      for (int i = 0; i < p.nwords; ++i) {
        const int j = 32 * i + lane;
        const uint32_t key = j < nkb ? ordered_key(sc[j]) : 0u;
        const uint32_t gt = __ballot_sync(0xffffffffu, j < nkb && key > kth);
        const uint32_t eq = __ballot_sync(0xffffffffu, j < nkb && key == kth);
        const uint32_t eq_kept = lowest_bits(eq, take);
        take -= __popc(eq_kept);
        const uint32_t forced = __ballot_sync(0xffffffffu, j < nkb && j < p.n_force);
        const uint32_t m = gt | eq_kept | forced;
        if (lane == 0) bw[i] = m;
        if (mrow != nullptr && j < nkb) mrow[j] = static_cast<uint8_t>((m >> lane) & 1u);
        kept += __popc(m);
      }
    }
    if (lane == 0 && kept) atomicAdd(&s_cnt, kept);
  } else {
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
  p.qbar = a.qbar_in != nullptr ? a.qbar_in : a.route_qbar;
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
  p.k_keep = a.k_keep;
  p.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  for (int h = 0; h < kMaxHeads; ++h) p.tau[h] = h < a.H ? a.tau[h] : 0.f;
  cudaError_t e = cudaSuccess;
  if (a.qbar_in == nullptr) {  // else the caller's means, from the pass that stored Q
    constexpr int QB = 2;
    sol_qbar_kernel<D, QB><<<dim3((p.nqb + QB - 1) / QB, p.BH), kRouteThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a.Q), a.route_qbar, p.L, p.nqb);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t smem = (static_cast<size_t>(R) * D + static_cast<size_t>(R) * p.nkb) * sizeof(float);
  e = cudaFuncSetAttribute(sol_route_kernel<D, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
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
