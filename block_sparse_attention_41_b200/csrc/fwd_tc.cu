// bf16 Sol-Attn forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA), persistent.
//
// The method (Sol-Attn project page, Abstract) in one kernel, per work unit = one 128-row
// query block of one head:
//   1. route    : q_bar from the Q tile in shared memory, proxy scores s_bar_j = q_bar.k_bar_j/sqrt(d)
//                 against the fp32 pooled keys, threshold max - tau. The scores live only in shared
//                 memory. The outputs are a kept-block list and a bitmask.
//   2. exact    : for each kept block, S = Q K^T (tcgen05, fp32 in TMEM), online softmax on CUDA cores,
//                 P (bf16) written to TMEM, O += P V (tcgen05, A operand read from TMEM).
//   3. correct  : every 128 consecutive pooled blocks that contain at least one skipped block form a
//                 "pooled tile". The tile's keys are k_bar (bf16) and its values are v_bar (bf16).
//                 Kept columns and columns past N_kb are masked; skipped columns get the
//                 multiplicity n_j as a +log2(n_j) logit offset. These tiles run through the same
//                 MMA/softmax pipeline and the same running max, sum and accumulator.
//   4. epilogue : O / l -> bf16 -> global.
//
// Roles (256 threads): warp 0 = TMA producer, warp 1 = MMA issuer (also owns TMEM),
// warps 4..7 = router + softmax + epilogue (thread r owns query row r = TMEM lane r), warps 2..3
// idle. Units come from an atomic counter in head-major order, so CTAs running at the same
// time share one head's K/V in L2.
//
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+D) P0 [384,448) P1 [448,512).
// P has its own columns, separate from S. The next QK^T into S[b] therefore never has to wait
// for the PV MMA that reads P[b].
//
// Every mbarrier wait is bounded (sol::mbar_wait). On expiry the CTA records SOL_ETIMEOUT in the
// workspace, the other roles stop at their next wait, in-flight copies and MMAs are drained, and
// TMEM is freed before the kernel returns.
#include <cmath>

#include "device_common.cuh"
#include "launchers.h"

namespace sol {

namespace {

constexpr int kThreads = 256;
constexpr int kSoftmaxWarp0 = 4;
constexpr int kRows = 128;  // B_q = B_k
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP0 = 384, kColP1 = 448;
constexpr float kRescaleThreshold = 8.0f;  // lazy rescale: only when the row max grows by > 2^8

template <int D>
struct TcCfg {
  static constexpr int NCHUNK = D / 64;                 // 128-byte swizzle atoms per row
  static constexpr int CHUNK_BYTES = kRows * 128;       // 128 rows x 128 B
  static constexpr int TILE_BYTES = NCHUNK * CHUNK_BYTES;
  static constexpr int NSTAGE = (D == 128) ? 2 : 4;     // K/V ring depth
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE_BYTES;
  static constexpr int OFF_V = OFF_K + NSTAGE * TILE_BYTES;
  static constexpr int OFF_SBAR = OFF_V + NSTAGE * TILE_BYTES;            // float[kMaxKeyBlocks]
  static constexpr int OFF_KLIST = OFF_SBAR + kMaxKeyBlocks * 4;          // u16[kMaxKeyBlocks]
  static constexpr int OFF_BITS = OFF_KLIST + kMaxKeyBlocks * 2;          // u32[kMaxKeyBlocks/32]
  static constexpr int OFF_CLIST = OFF_BITS + kMaxKeyBlocks / 8;          // u16[kMaxKeyBlocks/128]
  static constexpr int OFF_QBAR = OFF_CLIST + (kMaxKeyBlocks / 128) * 2;  // float[D] means + float[128] partials
  static constexpr int OFF_RED = OFF_QBAR + (D + kRows) * 4;              // float[8]
  static constexpr int OFF_MISC = OFF_RED + 32;                           // int[8]
  static constexpr int OFF_BAR = OFF_MISC + 32;                           // mbarriers
  // q_full, k_full[NSTAGE], v_full[NSTAGE], kv_empty[NSTAGE], s_full[2], p_full[2],
  // o_done, o_final, list_ready, drain
  static constexpr int NBAR = 1 + 3 * NSTAGE + 2 + 2 + 4;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM + 16 + 1024;  // + slack to align the base to 1024 B
};

struct TcParams {
  const float* kbar;  // fp32 [BH, nkb, D] routing proxy
  __nv_bfloat16* O;
  uint8_t* kept_mask;
  float* density;
  uint32_t* ws;
  int BH, H, L, nqb, nkb, n_force, last_n, total_units;
  float sl2;         // log2(e) / sqrt(d)
  float inv_sqrt_d;  // 1 / sqrt(d)
  float log2_last_n;
  int drop_one_load;
  unsigned long long wait_limit_ns;
  float tau[kMaxHeads];
};

enum MiscSlot : int { MISC_UNIT = 0, MISC_NK = 1, MISC_NC = 2, MISC_ABORT = 3, MISC_LAST = 4 };

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    sol_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                      const __grid_constant__ CUtensorMap tmVb, const __grid_constant__ TcParams p) {
  using C = TcCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);

  float* s_sbar = reinterpret_cast<float*>(smem + C::OFF_SBAR);
  uint16_t* s_klist = reinterpret_cast<uint16_t*>(smem + C::OFF_KLIST);
  uint32_t* s_bits = reinterpret_cast<uint32_t*>(smem + C::OFF_BITS);
  uint16_t* s_clist = reinterpret_cast<uint16_t*>(smem + C::OFF_CLIST);
  float* s_qbar = reinterpret_cast<float*>(smem + C::OFF_QBAR);
  float* s_red = reinterpret_cast<float*>(smem + C::OFF_RED);
  volatile int* s_misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  volatile int* s_abort = s_misc + MISC_ABORT;

  const uint32_t bar_q = sb + C::OFF_BAR;
  const uint32_t bar_kfull = bar_q + 8;
  const uint32_t bar_vfull = bar_kfull + 8 * C::NSTAGE;
  const uint32_t bar_kvempty = bar_vfull + 8 * C::NSTAGE;
  const uint32_t bar_sfull = bar_kvempty + 8 * C::NSTAGE;
  const uint32_t bar_pfull = bar_sfull + 16;
  const uint32_t bar_odone = bar_pfull + 16;
  const uint32_t bar_ofinal = bar_odone + 8;
  const uint32_t bar_list = bar_ofinal + 8;
  const uint32_t bar_drain = bar_list + 8;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint64_t limit = p.wait_limit_ns;

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::NSTAGE; ++s) {
      mbar_init(bar_kfull + 8 * s, 1);
      mbar_init(bar_vfull + 8 * s, 1);
      mbar_init(bar_kvempty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_sfull + 8 * b, 1);
      mbar_init(bar_pfull + 8 * b, kRows);
    }
    mbar_init(bar_odone, 1);
    mbar_init(bar_ofinal, 1);
    mbar_init(bar_list, 1);
    mbar_init(bar_drain, 1);
    s_misc[MISC_ABORT] = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmKb);
    tma_prefetch_desc(&tmVb);
  }
  if (warp == 1) {
    tmem_alloc(sb + C::OFF_TMEM, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::OFF_TMEM);

  uint32_t tile_base = 0;  // tiles processed by this CTA before the current unit (all roles agree)
  uint32_t unit_iter = 0;  // units processed by this CTA before the current one
  // producer bookkeeping for the final drain: last load number armed on each stage, +1 (0 = none)
  uint32_t armed[C::NSTAGE];  // 1 + use index of the last load armed on each stage (0 = none)
  bool k_dropped[C::NSTAGE];
#pragma unroll
  for (int s = 0; s < C::NSTAGE; ++s) {
    armed[s] = 0;
    k_dropped[s] = false;
  }
  bool mma_issued = false;

  for (;;) {
    if (tid == 0) s_misc[MISC_UNIT] = static_cast<int>(atomicAdd(&p.ws[WS_COUNTER], 1u));
    __syncthreads();
    const int unit = s_misc[MISC_UNIT];
    if (unit >= p.total_units || *s_abort) break;
    const int bh = unit / p.nqb;
    const int qb = unit - bh * p.nqb;
    const uint32_t uphase = unit_iter & 1u;

    if (warp == 0) {
      // ------------------------------------------------------------------ TMA producer
      if (lane == 0) {
        mbar_arrive_expect_tx(bar_q, C::TILE_BYTES);
        for (int c = 0; c < C::NCHUNK; ++c)
          tma_load_3d(sb + C::OFF_Q + c * C::CHUNK_BYTES, &tmQ, bar_q, c * 64, qb * kRows, bh);
        int w = mbar_wait(bar_list, uphase, s_abort, limit);
        if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_PRODUCER);
        if (w == WAIT_OK) {
          const int nk = s_misc[MISC_NK], T = nk + s_misc[MISC_NC];
          for (int t = 0; t < T; ++t) {
            const uint32_t r = tile_base + t;
            const int s = static_cast<int>(r % C::NSTAGE);
            if (r >= static_cast<uint32_t>(C::NSTAGE)) {
              w = mbar_wait(bar_kvempty + 8 * s, ((r / C::NSTAGE) - 1u) & 1u, s_abort, limit);
              if (w != WAIT_OK) {
                if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_PRODUCER);
                break;
              }
            }
            const bool exact = t < nk;
            const void* mk = exact ? static_cast<const void*>(&tmK) : static_cast<const void*>(&tmKb);
            const void* mv = exact ? static_cast<const void*>(&tmV) : static_cast<const void*>(&tmVb);
            const int y = (exact ? static_cast<int>(s_klist[t]) : static_cast<int>(s_clist[t - nk])) * kRows;
            const bool drop = p.drop_one_load && blockIdx.x == 0 && unit_iter == 0 && t == 0;
            if (!drop) {
              mbar_arrive_expect_tx(bar_kfull + 8 * s, C::TILE_BYTES);
              for (int c = 0; c < C::NCHUNK; ++c)
                tma_load_3d(sb + C::OFF_K + s * C::TILE_BYTES + c * C::CHUNK_BYTES, mk, bar_kfull + 8 * s, c * 64,
                            y, bh);
            }
            mbar_arrive_expect_tx(bar_vfull + 8 * s, C::TILE_BYTES);
            for (int c = 0; c < C::NCHUNK; ++c)
              tma_load_3d(sb + C::OFF_V + s * C::TILE_BYTES + c * C::CHUNK_BYTES, mv, bar_vfull + 8 * s, c * 64, y,
                          bh);
            armed[s] = r / C::NSTAGE + 1u;
            k_dropped[s] = drop;
          }
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        int w = mbar_wait(bar_list, uphase, s_abort, limit);
        if (w == WAIT_OK) w = mbar_wait(bar_q, uphase, s_abort, limit);
        if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_MMA);
        if (w == WAIT_OK) {
          const int T = s_misc[MISC_NK] + s_misc[MISC_NC];
          constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
          constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
          const uint32_t q_addr = sb + C::OFF_Q;
          bool ok = true;
          for (int t = 0; t <= T && ok; ++t) {
            if (t < T) {
              const uint32_t g = tile_base + t;
              const int s = static_cast<int>(g % C::NSTAGE);
              const uint32_t b = g & 1u;
              w = mbar_wait(bar_kfull + 8 * s, (g / C::NSTAGE) & 1u, s_abort, limit);
              if (w != WAIT_OK) {
                if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_MMA);
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t k_addr = sb + C::OFF_K + s * C::TILE_BYTES;
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = (kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32;
                mma_bf16_ss(tmem + (b ? kColS1 : kColS0), smem_desc_sw128(q_addr + off, 16, 1024),
                            smem_desc_sw128(k_addr + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
              }
              mma_issued = true;
              tc_commit(bar_sfull + 8 * b);
            }
            if (t >= 1) {
              // O += P V for the previous tile
              const int tp = t - 1;
              const uint32_t g = tile_base + tp;
              const int s = static_cast<int>(g % C::NSTAGE);
              const uint32_t b = g & 1u;
              w = mbar_wait(bar_pfull + 8 * b, (g >> 1) & 1u, s_abort, limit);
              if (w == WAIT_OK) w = mbar_wait(bar_vfull + 8 * s, (g / C::NSTAGE) & 1u, s_abort, limit);
              if (w != WAIT_OK) {
                if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_MMA);
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t v_addr = sb + C::OFF_V + s * C::TILE_BYTES;
              const uint32_t p_col = tmem + (b ? kColP1 : kColP0);
#pragma unroll
              for (int kk = 0; kk < kRows / 16; ++kk) {
                mma_bf16_ts(tmem + kColO, p_col + kk * 8, smem_desc_sw128(v_addr + kk * 2048, C::CHUNK_BYTES, 1024),
                            idesc_pv, (tp > 0 || kk > 0) ? 1u : 0u);
              }
              tc_commit(bar_kvempty + 8 * s);
              tc_commit(bar_odone);
            }
          }
          if (ok) tc_commit(bar_ofinal);
        }
      }
    } else if (warp >= kSoftmaxWarp0) {
      // ------------------------------------------------------------------ router + softmax + epilogue
      const int row = tid - kSoftmaxWarp0 * 32;  // 0..127, TMEM lane
      const int wq = warp - kSoftmaxWarp0;       // TMEM lane quarter
      const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
      const int m_i = min(kRows, p.L - qb * kRows);
      const int nkb = p.nkb;
      bool alive = true;

      int w = mbar_wait(bar_q, uphase, s_abort, limit);
      if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_ROUTER);
      alive = !named_barrier_or(1, kRows, w != WAIT_OK);  // identical in all 128 threads

      // (1a) q_bar = mean of the valid query rows, read from the swizzled Q tile
      {
        constexpr int TPC = kRows / D;  // threads per column: 1 (D=128) or 2 (D=64)
        const int c = row % D, part = row / D;
        const uint8_t* qt = smem + C::OFF_Q + (c >> 6) * C::CHUNK_BYTES;
        const int cw = c & 63;
        float acc = 0.f;
        if (alive) {
          for (int r = part; r < m_i; r += TPC) {
            const uint32_t off = r * 128 + ((((cw >> 3) ^ (r & 7))) << 4) + ((cw & 7) << 1);
            acc += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(qt + off));
          }
        }
        s_qbar[D + row] = acc;
        named_barrier_sync(1, kRows);
        if (row < D) {
          float s = 0.f;
#pragma unroll
          for (int k = 0; k < TPC; ++k) s += s_qbar[D + row + k * D];
          s_qbar[row] = s / static_cast<float>(m_i);
        }
        named_barrier_sync(1, kRows);
      }

      // (1b) proxy scores s_bar_j (shared memory only) and their max
      {
        constexpr int DPL = D / 32;
        float qv[DPL];
#pragma unroll
        for (int k = 0; k < DPL; ++k) qv[k] = s_qbar[lane * DPL + k];
        const float* kb = p.kbar + static_cast<size_t>(bh) * nkb * D + lane * DPL;
        float wmax = -INFINITY;
        for (int j0 = wq; j0 < nkb; j0 += 16) {
          float dot[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = j0 + 4 * u;
            dot[u] = 0.f;
            if (j < nkb) {
              const float* src = kb + static_cast<size_t>(j) * D;
              if constexpr (DPL == 4) {
                const float4 v = __ldg(reinterpret_cast<const float4*>(src));
                dot[u] = fmaf(qv[0], v.x, fmaf(qv[1], v.y, fmaf(qv[2], v.z, qv[3] * v.w)));
              } else {
                const float2 v = __ldg(reinterpret_cast<const float2*>(src));
                dot[u] = fmaf(qv[0], v.x, qv[1] * v.y);
              }
            }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
            for (int u = 0; u < 4; ++u) dot[u] += __shfl_xor_sync(0xffffffffu, dot[u], o);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int j = j0 + 4 * u;
            if (j < nkb) {
              const float s = dot[u] * p.inv_sqrt_d;
              if (lane == 0) s_sbar[j] = s;
              wmax = fmaxf(wmax, s);
            }
          }
        }
        if (lane == 0) s_red[wq] = wmax;
        named_barrier_sync(1, kRows);
      }

      // (1c) keep bits, kept list, pooled-tile list (warp 0 of the group)
      if (wq == 0) {
        const float M = fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3]));
        const float thr = M - p.tau[bh % p.H];
        int nk = 0;
        for (int base = 0; base < nkb; base += 32) {
          const int j = base + lane;
          const bool k = j < nkb && (s_sbar[j] >= thr || j < p.n_force);
          const uint32_t m = __ballot_sync(0xffffffffu, k);
          if (lane == 0) s_bits[base >> 5] = m;
          if (k) s_klist[nk + __popc(m & ((1u << lane) - 1u))] = static_cast<uint16_t>(j);
          nk += __popc(m);
        }
        __syncwarp();
        const int nchunks = (nkb + kRows - 1) / kRows;
        int nc = 0;
        for (int cb = 0; cb < nchunks; cb += 32) {
          const int cc = cb + lane;
          bool has_skip = false;
          if (cc < nchunks) {
            const int valid = min(kRows, nkb - cc * kRows);
            int kept = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (cc * 4 + q < (nkb + 31) / 32) kept += __popc(s_bits[cc * 4 + q]);
            has_skip = kept < valid;
          }
          const uint32_t m = __ballot_sync(0xffffffffu, has_skip);
          if (has_skip) s_clist[nc + __popc(m & ((1u << lane) - 1u))] = static_cast<uint16_t>(cc);
          nc += __popc(m);
        }
        if (lane == 0) {
          s_misc[MISC_NK] = alive ? nk : 0;
          s_misc[MISC_NC] = alive ? nc : 0;
          atomicAdd(&p.ws[WS_COUNTS + bh], static_cast<uint32_t>(nk));
        }
      }
      named_barrier_sync(1, kRows);
      if (row == 0 && alive) mbar_arrive(bar_list);
      if (p.kept_mask != nullptr) {
        uint8_t* mrow = p.kept_mask + (static_cast<size_t>(bh) * p.nqb + qb) * nkb;
        for (int j = row; j < nkb; j += kRows) mrow[j] = static_cast<uint8_t>((s_bits[j >> 5] >> (j & 31)) & 1u);
      }

      // (2)+(3) online softmax over kept tiles, then pooled tiles
      const int nk = s_misc[MISC_NK];
      const int T = alive ? nk + s_misc[MISC_NC] : 0;
      float m_run = -INFINITY, l_run = 0.f;
      for (int t = 0; t < T; ++t) {
        const uint32_t g = tile_base + t;
        const uint32_t b = g & 1u;
        w = mbar_wait(bar_sfull + 8 * b, (g >> 1) & 1u, s_abort, limit);
        if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_SOFTMAX);
        if (!__all_sync(0xffffffffu, w == WAIT_OK)) {  // leave as a whole warp (tcgen05.ld is warp-wide)
          alive = false;
          break;
        }
        tc_fence_after();
        uint32_t sraw[128];
        tmem_ld_x128(tmem + lane_base + (b ? kColS1 : kColS0), sraw);
        float x[128];
        if (t < nk) {
          const int j = s_klist[t];
          const int valid = (j == nkb - 1) ? p.last_n : kRows;
#pragma unroll
          for (int c = 0; c < 128; ++c) x[c] = (c < valid) ? __uint_as_float(sraw[c]) * p.sl2 : -INFINITY;
        } else {
          const int cc = s_clist[t - nk];
          const int valid = min(kRows, nkb - cc * kRows);
          uint32_t kw[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) kw[q] = (cc * 4 + q < (nkb + 31) / 32) ? s_bits[cc * 4 + q] : 0u;
          const bool has_last = (cc * kRows + valid == nkb);
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const bool skipped = c < valid && !((kw[c >> 5] >> (c & 31)) & 1u);
            const float off = (has_last && c == valid - 1) ? p.log2_last_n : 7.0f;  // log2(n_j)
            x[c] = skipped ? fmaf(__uint_as_float(sraw[c]), p.sl2, off) : -INFINITY;
          }
        }
        float mt = x[0];
#pragma unroll
        for (int c = 1; c < 128; ++c) mt = fmaxf(mt, x[c]);
        float m_new = m_run, alpha = 1.f;
        bool need = false;
        if (t == 0) {
          m_new = mt;
        } else if (mt > m_run + kRescaleThreshold) {
          need = true;
          m_new = mt;
          alpha = ex2_approx(m_run - mt);
        }
        uint32_t pk[64];
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const float p0 = ex2_approx(x[2 * c] - m_new);
          const float p1 = ex2_approx(x[2 * c + 1] - m_new);
          rs += p0 + p1;
          pk[c] = pack_bf16x2(p0, p1);
        }
        l_run = fmaf(l_run, alpha, rs);
        m_run = m_new;
        if (__any_sync(0xffffffffu, need)) {
          // rescale O after the previous tile's PV has landed
          w = mbar_wait(bar_odone, (g - 1u) & 1u, s_abort, limit);
          if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_SOFTMAX);
          if (!__all_sync(0xffffffffu, w == WAIT_OK)) {
            alive = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t o[32];
            tmem_ld_x32(tmem + lane_base + kColO + ch * 32, o);
#pragma unroll
            for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
            tmem_st_x32(tmem + lane_base + kColO + ch * 32, o);
          }
        }
        uint32_t pk0[32], pk1[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          pk0[c] = pk[c];
          pk1[c] = pk[32 + c];
        }
        const uint32_t pcol = tmem + lane_base + (b ? kColP1 : kColP0);
        tmem_st_x32(pcol, pk0);
        tmem_st_x32(pcol + 32, pk1);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_pfull + 8 * b);
      }

      // (4) epilogue: O / l -> bf16
      if (alive && T > 0) {
        w = mbar_wait(bar_ofinal, uphase, s_abort, limit);
        if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_SOFTMAX);
        if (__all_sync(0xffffffffu, w == WAIT_OK)) {
          tc_fence_after();
          const float inv = 1.f / l_run;
          const bool store = row < m_i;
          __nv_bfloat16* dst = p.O + (static_cast<size_t>(bh) * p.L + static_cast<size_t>(qb) * kRows + row) * D;
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t o[32];
            tmem_ld_x32(tmem + lane_base + kColO + ch * 32, o);
            uint32_t pkd[16];
#pragma unroll
            for (int c = 0; c < 16; ++c)
              pkd[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv, __uint_as_float(o[2 * c + 1]) * inv);
            if (store) {
              uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 32);
#pragma unroll
              for (int v = 0; v < 4; ++v) d4[v] = make_uint4(pkd[4 * v], pkd[4 * v + 1], pkd[4 * v + 2], pkd[4 * v + 3]);
            }
          }
        }
      }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    tile_base += static_cast<uint32_t>(s_misc[MISC_NK] + s_misc[MISC_NC]);
    ++unit_iter;
  }

  // ---- drain: no copy or MMA may still be in flight when TMEM and shared memory are released
  if (warp == 1 && lane == 0 && mma_issued) {
    tc_commit(bar_drain);
    mbar_wait(bar_drain, 0, nullptr, limit);
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::NSTAGE; ++s) {
      if (armed[s] == 0) continue;
      const uint32_t use = armed[s] - 1u;
      if (!k_dropped[s]) mbar_wait(bar_kfull + 8 * s, use & 1u, nullptr, limit);
      mbar_wait(bar_vfull + 8 * s, use & 1u, nullptr, limit);
    }
    if (unit_iter > 0) mbar_wait(bar_q, (unit_iter - 1u) & 1u, nullptr, limit);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);

  // ---- the last CTA to finish turns the kept-block counts into per-head densities
  if (tid == 0) {
    __threadfence();
    s_misc[MISC_LAST] = (atomicAdd(&p.ws[WS_DONE], 1u) == gridDim.x - 1) ? 1 : 0;
  }
  __syncthreads();
  if (s_misc[MISC_LAST] && p.density != nullptr) {
    __threadfence();
    const double denom = static_cast<double>(p.nqb) * static_cast<double>(p.nkb);
    for (int i = tid; i < p.BH; i += kThreads)
      p.density[i] = static_cast<float>(static_cast<double>(atomicAdd(&p.ws[WS_COUNTS + i], 0u)) / denom);
  }
}

template <int D>
cudaError_t launch_tc_t(const FwdArgs& a, const CUtensorMap* maps, cudaStream_t stream) {
  using C = TcCfg<D>;
  TcParams p;
  p.kbar = a.kbar;
  p.O = static_cast<__nv_bfloat16*>(a.O);
  p.kept_mask = a.kept_mask;
  p.density = a.density;
  p.ws = a.ws;
  p.BH = a.B * a.H;
  p.H = a.H;
  p.L = a.L;
  p.nqb = (a.L + kRows - 1) / kRows;
  p.nkb = p.nqb;
  p.n_force = a.n_force;
  p.last_n = a.L - (p.nkb - 1) * kRows;
  p.total_units = p.BH * p.nqb;
  p.sl2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D)));
  p.inv_sqrt_d = static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  p.log2_last_n = static_cast<float>(std::log2(static_cast<double>(p.last_n)));
  p.drop_one_load = a.drop_one_load;
  p.wait_limit_ns = a.wait_limit_ns;
  for (int h = 0; h < kMaxHeads; ++h) p.tau[h] = h < a.H ? a.tau[h] : 0.f;
  cudaError_t e = cudaFuncSetAttribute(sol_fwd_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = p.total_units < a.num_sms ? p.total_units : a.num_sms;
  sol_fwd_tc_kernel<D><<<grid, kThreads, C::SMEM_BYTES, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4], p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_tc(const FwdArgs& a, const CUtensorMap* maps, cudaStream_t stream) {
  if (a.d == 64) return launch_tc_t<64>(a, maps, stream);
  if (a.d == 128) return launch_tc_t<128>(a, maps, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sol
