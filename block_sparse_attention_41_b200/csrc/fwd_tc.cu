// bf16 Sol-Attn forward on the sm_100a tensor cores (tcgen05 + TMEM + TMA), persistent.
//
// The method (Sol-Attn project page, Abstract) in one kernel, per work unit = one 128-row
// query block of one head:
//   1. route    : the unit's keep bits (one per key block), expanded into a kept-block list and a
//                 pooled-tile list. They come either from the routing pass (route.cu: one read of
//                 the pooled keys for several query blocks) or, when no bits are given, from this
//                 kernel itself: q_bar from the Q tile in shared memory, proxy scores
//                 s_bar_j = q_bar.k_bar_j/sqrt(d) against the fp32 pooled keys, threshold max - tau,
//                 with the scores kept only in shared memory and the bitmask written out. Both ways
//                 take the same fp32 operations in the same order, so they keep the same blocks.
//   2. exact    : for each kept block, S = Q K^T (tcgen05, fp32 in TMEM), online softmax on CUDA cores,
//                 P (bf16) written to TMEM, O += P V (tcgen05, A operand read from TMEM).
//   3. correct  : every 128 consecutive pooled blocks that contain at least one skipped block form a
//                 "pooled tile". The tile's keys are k_bar (bf16) and its values are v_bar (bf16).
//                 Kept columns and columns past N_kb are masked; skipped columns get the
//                 multiplicity n_j as a +log2(n_j) logit offset. These tiles run through the same
//                 MMA/softmax pipeline and the same running max, sum and accumulator.
//   4. epilogue : O / l -> bf16 -> global.
//
// Roles (384 threads): warp 0 = TMA producer, warps 1 and 11 = PV issuers of softmax groups 0
// and 1 (warp 1 also owns TMEM), warps 2..5 and 6..9 = the two softmax groups, warp 10 = QK^T
// issuer. A tcgen05.mma blocks its issuing thread for about as long as the tensor pipe takes to
// run it, so the products are issued from three threads: a group's PV starts as soon as that
// group's P is written, and waiting for one tile's PV to finish (before its S buffer is refilled)
// never delays the PV of the next tile. A warp may only touch TMEM lanes 32*(warp%4) .. +31, and any four
// consecutive warps cover all four quarters, so thread (g, r) of softmax group g owns query
// row r (TMEM lane r) and score columns [64g, 64g+64) of every tile.
//
// The two groups never synchronise inside the tile loop. Each keeps its own running max m_g and
// sum l_g over its half of the key columns and accumulates its own output O_g = sum P_g V_g in
// TMEM. That is the same softmax split into two partial sums over disjoint key sets; the
// epilogue merges them once per unit with the usual rescale,
//   O = (2^(m_0-m) O_0 + 2^(m_1-m) O_1) / (2^(m_0-m) l_0 + 2^(m_1-m) l_1),  m = max(m_0, m_1).
//
// TMEM columns: S0 [0,128) S1 [128,256) O_0 [256,256+D) O_1 [256+D,256+2D). Group g writes its
// bf16 P over S columns [64g, 64g+32) of the buffer it has just read. S is double-buffered, so
// the refill of a buffer (the QK^T of tile t+2, issued once the PV of tile t has completed) runs
// while the softmax works on tile t+1. K tiles go round a 3-deep ring (d = 128) and are released
// as soon as their QK^T completes; V tiles go round a 2-deep ring and are released after PV.
//
// Exponentials: ex2.approx on the MUFU unit. An optional path (kPolyEvery) computes some of them
// on the FMA pipe as 2^x = 2^floor(x) * p(x - floor(x)), where p is a cubic minimax fit of 2^f on
// [0, 1) (max relative error 8.6e-5, far below the bf16 rounding of P).
//
// Every mbarrier wait is bounded (sol::mbar_wait). On expiry the CTA records SOL_ETIMEOUT in the
// workspace, the other roles stop at their next wait, in-flight copies and MMAs are drained, and
// TMEM is freed before the kernel returns. Every softmax warp reaches the epilogue's named
// barrier whether or not its tile loop ended early, so no warp is left waiting there.
#include <cmath>

#include "device_common.cuh"
#include "launchers.h"

namespace sol {

namespace {

constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 2;
constexpr int kQkWarp = 10;
constexpr int kPv1Warp = 11;  // PV issuer of softmax group 1 (group 0's is warp 1)
constexpr int kSoftmaxThreads = 256;
constexpr int kGroupWarps = 4;  // warps per softmax group
constexpr int kRows = 128;      // B_q = B_k
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;    // S buffer b at kColS + 128 b
constexpr uint32_t kColO = 256;  // O_g at kColO + D g
constexpr float kRescaleThreshold = 8.0f;  // lazy rescale: only when the row max grows by > 2^8
// 8-bit PV: P is E4M3 with no scale, against an integer reference 6 below the running max; the
// lazy threshold drops to 2 so that P stays below 2^(6 + 2) = 256 < 448, and every weight above
// 2^-12 of the running max is a normal E4M3 value (its mantissa rounded, its exponent exact)
constexpr int kHeadroom8 = 6;
constexpr float kRescaleThreshold8 = 2.0f;
constexpr uint32_t kBarSoftmax = 1;       // named barrier of the 256 softmax threads

// cubic minimax fit of 2^f on [0, 1] with p(0) = 1 (relative error <= 8.6e-5)
constexpr float kExpC1 = 0.69511664f, kExpC2 = 0.22764498f, kExpC3 = 0.07706724f;
// Column pairs of a full exact tile whose exponentials take the polynomial: pair c with
// c % kPolyEvery == kPolyEvery - 1; 0 = none. Measured on B200 with this pipeline, moving work off
// MUFU costs more issue slots than it saves, so it is off.
constexpr int kPolyEvery = 0;

// QK8: Q, K and the pooled keys arrive as int8 codes (one 128-byte swizzle atom per row at d = 128)
// and QK^T runs as kind::i8 with int32 accumulation; V, P and the rest stay bf16.
// PV8 (with QK8): V and the pooled values arrive as E4M3 codes with one scale per channel, stored
// transposed ([d][keys], one 128-byte atom of keys per channel row), P is written as E4M3 against
// an integer running maximum lowered by 6, and PV runs as kind::f8f6f4; the epilogue applies the
// channel scales.
template <int D, bool QK8, bool PV8 = false>
struct TcCfg {
  static constexpr int NCHUNK = D / 64;                 // 128-byte swizzle atoms per bf16 row
  static constexpr int CHUNK_BYTES = kRows * 128;       // 128 rows x 128 B
  static constexpr int QK_CHUNKS = QK8 ? D / 128 : NCHUNK;  // swizzle atoms per Q or K row
  static constexpr int QK_TILE_BYTES = QK_CHUNKS * CHUNK_BYTES;
  static constexpr int NK = (D == 128) ? 3 : 4;         // K ring depth
  static constexpr int NV = (D == 128) ? 2 : 4;         // V ring depth
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + QK_TILE_BYTES;
  static constexpr int V_CHUNKS = PV8 ? 1 : NCHUNK;                       // swizzle atoms per V stage row
  static constexpr int V_TILE_BYTES = V_CHUNKS * CHUNK_BYTES;             // PV8: d rows x 128 key bytes
  static constexpr int OFF_V = OFF_K + NK * QK_TILE_BYTES;
  static constexpr int OFF_SBAR = OFF_V + NV * V_TILE_BYTES;              // float[kMaxKeyBlocks]
  static constexpr int OFF_KLIST = OFF_SBAR + kMaxKeyBlocks * 4;          // u16[kMaxKeyBlocks]
  static constexpr int OFF_BITS = OFF_KLIST + kMaxKeyBlocks * 2;          // u32[kMaxKeyBlocks/32]
  static constexpr int OFF_CLIST = OFF_BITS + kMaxKeyBlocks / 8;          // u16[kMaxKeyBlocks/128]
  static constexpr int OFF_QBAR = OFF_CLIST + (kMaxKeyBlocks / 128) * 2;  // float[D] + int[256] word prefixes
  static constexpr int OFF_ML = OFF_QBAR + (D + kSoftmaxThreads) * 4;     // float2[2 grp][128 rows]
  static constexpr int OFF_RED = OFF_ML + 2 * kRows * 8;                  // float[8]
  static constexpr int OFF_MISC = OFF_RED + 32;                           // int[8]
  static constexpr int OFF_BAR = OFF_MISC + 32;                           // mbarriers
  // q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[2], p_full[2 buf][2 grp],
  // pv_done[2 buf], o_final, list_ready, drain[3 issuers]
  static constexpr int NBAR = 1 + 2 * NK + 2 * NV + 2 + 4 + 2 + 1 + 1 + 3;
  static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
  static constexpr int SMEM_BYTES = OFF_TMEM + 16 + 1024;  // + slack to align the base to 1024 B
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(kMaxKeyBlocks / 32 <= kSoftmaxThreads, "word prefixes fit after q_bar");
  static_assert((kSoftmaxThreads / (D / 8)) * D <= kMaxKeyBlocks, "q_bar partial sums fit in the proxy-score buffer");
  static_assert(kColO + 2 * D <= kTmemCols, "TMEM budget");
  static_assert(!QK8 || D == 128, "8-bit QK^T needs d = 128");
  static_assert(!PV8 || QK8, "8-bit PV comes with 8-bit QK^T");
};

struct TcParams {
  const float* kbar;          // fp32 [BH, nkb, D] routing proxy
  const uint32_t* bits;       // [BH * nqb, ceil(nkb / 32)] keep bits from the routing pass, or null
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
  const float* q_scale;   // 8-bit QK^T: [BH, nqb] query-tile scales
  const float* k_scale;   // [BH, nkb] key-block scales
  const float* kb_scale;  // [BH, ceil(nkb / 128)] pooled-key chunk scales
  const float* v_scale;   // 8-bit PV: [BH, D] channel scales of V and v_bar
  unsigned long long* cta_times;  // measurement hook: [2 * cta_capacity] start/finish ns, or null
  int cta_capacity;
  float tau[kMaxHeads];
};

enum MiscSlot : int { MISC_UNIT = 0, MISC_NK = 1, MISC_NC = 2, MISC_ABORT = 3, MISC_LAST = 4 };

// 2^x for a pair, on the FMA pipe: floor by a round-down add of 1.5*2^23, cubic on the fraction,
// exponent added to the bit pattern. x must lie in [-126, 126].
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float2 t = __fadd2_rd(x, make_float2(12582912.0f, 12582912.0f));  // mantissa of t = floor(x)
  const float2 j = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __fadd2_rn(x, make_float2(-j.x, -j.y));                // in [0, 1)
  float2 q = __ffma2_rn(f, make_float2(kExpC3, kExpC3), make_float2(kExpC2, kExpC2));
  q = __ffma2_rn(f, q, make_float2(kExpC1, kExpC1));
  q = __ffma2_rn(f, q, make_float2(1.0f, 1.0f));
  const uint32_t ex = __float_as_uint(t.x) << 23, ey = __float_as_uint(t.y) << 23;  // floor(x) << 23
  return make_float2(__uint_as_float(__float_as_uint(q.x) + ex), __uint_as_float(__float_as_uint(q.y) + ey));
}

__device__ __forceinline__ float max64(const float (&s)[64]) {
  // four independent chains of three-input max over the 64 values
  float m[4] = {fmax3(s[0], s[1], s[2]), fmax3(s[3], s[4], s[5]), fmax3(s[6], s[7], s[8]), fmax3(s[9], s[10], s[11])};
#pragma unroll
  for (int c = 12; c < 60; c += 8) {
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = fmax3(m[k], s[c + 2 * k], s[c + 2 * k + 1]);
  }
  m[0] = fmax3(m[0], s[60], s[61]);
  m[1] = fmax3(m[1], s[62], s[63]);
  return fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
}

template <int D, bool QK8, bool PV8>
__global__ void __launch_bounds__(kThreads, 1)
    sol_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                      const __grid_constant__ CUtensorMap tmVb, const __grid_constant__ TcParams p) {
  using C = TcCfg<D, QK8, PV8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  float* s_sbar = reinterpret_cast<float*>(smem + C::OFF_SBAR);
  uint16_t* s_klist = reinterpret_cast<uint16_t*>(smem + C::OFF_KLIST);
  uint32_t* s_bits = reinterpret_cast<uint32_t*>(smem + C::OFF_BITS);
  uint16_t* s_clist = reinterpret_cast<uint16_t*>(smem + C::OFF_CLIST);
  float* s_qbar = reinterpret_cast<float*>(smem + C::OFF_QBAR);
  float2* s_ml = reinterpret_cast<float2*>(smem + C::OFF_ML);
  float* s_red = reinterpret_cast<float*>(smem + C::OFF_RED);
  volatile int* s_misc = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  volatile int* s_abort = s_misc + MISC_ABORT;

  const uint32_t bar_q = sb + C::OFF_BAR;
  const uint32_t bar_kfull = bar_q + 8;
  const uint32_t bar_kempty = bar_kfull + 8 * C::NK;
  const uint32_t bar_vfull = bar_kempty + 8 * C::NK;
  const uint32_t bar_vempty = bar_vfull + 8 * C::NV;
  const uint32_t bar_sfull = bar_vempty + 8 * C::NV;  // [2 buf]
  const uint32_t bar_pfull = bar_sfull + 16;          // [2 buf][2 grp]
  const uint32_t bar_pvdone = bar_pfull + 32;         // [2 buf]: the PV of a tile using S[buf] completed
  const uint32_t bar_ofinal = bar_pvdone + 16;        // completes once per unit, after its last PV
  const uint32_t bar_list = bar_ofinal + 8;
  const uint32_t bar_drain = bar_list + 8;            // [3]: PV issuers of groups 0 and 1, QK^T issuer

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint64_t limit = p.wait_limit_ns;

  if (tid == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::NK; ++s) {
      mbar_init(bar_kfull + 8 * s, 1);
      mbar_init(bar_kempty + 8 * s, 1);
    }
    for (int s = 0; s < C::NV; ++s) {
      mbar_init(bar_vfull + 8 * s, 1);
      mbar_init(bar_vempty + 8 * s, 2);  // both PV issuers commit
    }
    for (int b = 0; b < 2; ++b) mbar_init(bar_sfull + 8 * b, 1);
    for (int i = 0; i < 4; ++i) mbar_init(bar_pfull + 8 * i, kGroupWarps);  // one elected lane per warp
    for (int b = 0; b < 2; ++b) mbar_init(bar_pvdone + 8 * b, 2);  // both PV issuers commit
    mbar_init(bar_ofinal, 2);
    mbar_init(bar_list, 1);
    for (int i = 0; i < 3; ++i) mbar_init(bar_drain + 8 * i, 1);
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
  const bool stamp = p.cta_times != nullptr && static_cast<int>(blockIdx.x) < p.cta_capacity && tid == 0;
  if (stamp) p.cta_times[2 * blockIdx.x] = globaltimer_ns();

  uint32_t tile_base = 0;  // tiles processed by this CTA before the current unit (all roles agree)
  uint32_t unit_iter = 0;  // units processed by this CTA before the current one
  // producer bookkeeping for the final drain: 1 + use index of the last load armed per stage
  uint32_t k_armed[C::NK], v_armed[C::NV];
#pragma unroll
  for (int s = 0; s < C::NK; ++s) k_armed[s] = 0;
#pragma unroll
  for (int s = 0; s < C::NV; ++s) v_armed[s] = 0;
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
        mbar_arrive_expect_tx(bar_q, C::QK_TILE_BYTES);
        for (int c = 0; c < C::QK_CHUNKS; ++c)  // a 128-byte-wide box: 64 bf16 or 128 int8 columns
          tma_load_3d(sb + C::OFF_Q + c * C::CHUNK_BYTES, &tmQ, bar_q, c * (QK8 ? 128 : 64), qb * kRows, bh);
        int w = mbar_wait(bar_list, uphase, s_abort, limit);
        if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_PRODUCER);
        if (w == WAIT_OK) {
          const int nk = s_misc[MISC_NK], T = nk + s_misc[MISC_NC];
          // K runs one tile ahead of V: K_0, K_1, V_0, K_2, V_1, ...
          for (int t = 0; t <= T; ++t) {
            if (t < T) {
              const uint32_t g = tile_base + t;
              const int s = static_cast<int>(g % C::NK);
              if (g >= static_cast<uint32_t>(C::NK)) {
                w = mbar_wait(bar_kempty + 8 * s, ((g / C::NK) - 1u) & 1u, s_abort, limit);
                if (w != WAIT_OK) {
                  if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_PRODUCER);
                  break;
                }
              }
              const bool exact = t < nk;
              const void* mk = exact ? static_cast<const void*>(&tmK) : static_cast<const void*>(&tmKb);
              const int y = (exact ? static_cast<int>(s_klist[t]) : static_cast<int>(s_clist[t - nk])) * kRows;
              const bool drop = p.drop_one_load && blockIdx.x == 0 && unit_iter == 0 && t == 0;
              if (!drop) {
                mbar_arrive_expect_tx(bar_kfull + 8 * s, C::QK_TILE_BYTES);
                for (int c = 0; c < C::QK_CHUNKS; ++c)
                  tma_load_3d(sb + C::OFF_K + s * C::QK_TILE_BYTES + c * C::CHUNK_BYTES, mk, bar_kfull + 8 * s,
                              c * (QK8 ? 128 : 64), y, bh);
                k_armed[s] = g / C::NK + 1u;
              }
            }
            if (t >= 1) {
              const int tp = t - 1;
              const uint32_t g = tile_base + tp;
              const int s = static_cast<int>(g % C::NV);
              if (g >= static_cast<uint32_t>(C::NV)) {
                w = mbar_wait(bar_vempty + 8 * s, ((g / C::NV) - 1u) & 1u, s_abort, limit);
                if (w != WAIT_OK) {
                  if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_PRODUCER);
                  break;
                }
              }
              const bool exact = tp < nk;
              const void* mv = exact ? static_cast<const void*>(&tmV) : static_cast<const void*>(&tmVb);
              const int y = (exact ? static_cast<int>(s_klist[tp]) : static_cast<int>(s_clist[tp - nk])) * kRows;
              mbar_arrive_expect_tx(bar_vfull + 8 * s, C::V_TILE_BYTES);
              if constexpr (PV8) {
                // transposed codes: the box is 128 keys (x, from the tile's first key) x d channel rows
                tma_load_3d(sb + C::OFF_V + s * C::V_TILE_BYTES, mv, bar_vfull + 8 * s, y, 0, bh);
              } else {
                for (int c = 0; c < C::NCHUNK; ++c)
                  tma_load_3d(sb + C::OFF_V + s * C::V_TILE_BYTES + c * C::CHUNK_BYTES, mv, bar_vfull + 8 * s, c * 64,
                              y, bh);
              }
              v_armed[s] = g / C::NV + 1u;
            }
          }
        }
      }
    } else if (warp == 1 || warp == kPv1Warp) {
      // ------------------------------------------------------------------ PV issuers
      // O_grp += P_grp V[64 grp .. 64 grp + 64): one thread per softmax group
      const int grp = warp == 1 ? 0 : 1;
      if (lane == 0) {
        int w = mbar_wait(bar_list, uphase, s_abort, limit);
        if (w == WAIT_OK) {
          const int T = s_misc[MISC_NK] + s_misc[MISC_NC];
          constexpr uint32_t idesc_pv = PV8 ? idesc_e4m3_f32(128, D) : idesc_bf16_f32(128, D, true);
          // base descriptor; a K-step or stage offset is added to the start-address field
          // (addresses stay below 256 KB, so the 14-bit field never carries). bf16: V rows
          // [64 grp, 64 grp + 64) start 4 grp x 2048 B in; E4M3 (K-major, 128 keys per row): keys
          // [64 grp, ...) start 64 grp B into every row
          const uint64_t vdesc0 = PV8 ? smem_desc_sw128(sb + C::OFF_V, 16, 1024) + ((64 * grp) >> 4)
                                      : smem_desc_sw128(sb + C::OFF_V, C::CHUNK_BYTES, 1024) + ((4 * grp * 2048) >> 4);
          const uint32_t o_acc = tmem + kColO + D * grp;
          for (int t = 0; t < T && w == WAIT_OK; ++t) {
            const uint32_t g = tile_base + t;
            const uint32_t b = g & 1u;
            const int s = static_cast<int>(g % C::NV);
            // V first: it lands long before P, so the wait on P is the one left on the critical path
            w = mbar_wait(bar_vfull + 8 * s, (g / C::NV) & 1u, s_abort, limit);
            if (w == WAIT_OK) w = mbar_wait(bar_pfull + 8 * (2 * b + grp), (g >> 1) & 1u, s_abort, limit);
            if (w != WAIT_OK) break;
            tc_fence_after();
            const uint64_t vd = vdesc0 + ((s * C::V_TILE_BYTES) >> 4);
            const uint32_t p_col = tmem + kColS + 128 * b + 64 * grp;
            if constexpr (PV8) {
              // 64 keys in two K = 32 steps; P: 32 E4M3 per lane = 8 TMEM columns per step
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)
                mma_f8_ts(o_acc, p_col + kk * 8, vd + kk * 2, idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
            } else {
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                mma_bf16_ts(o_acc, p_col + kk * 8, vd + ((kk * 2048) >> 4), idesc_pv, (t > 0 || kk > 0) ? 1u : 0u);
            }
            mma_issued = true;
            tc_commit(bar_vempty + 8 * s);
            tc_commit(bar_pvdone + 8 * b);
          }
          if (w == WAIT_OK) tc_commit(bar_ofinal);
        }
        if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_MMA);
      }
    } else if (warp == kQkWarp) {
      // ------------------------------------------------------------------ QK^T issuer
      if (lane == 0) {
        int w = mbar_wait(bar_list, uphase, s_abort, limit);
        if (w == WAIT_OK) w = mbar_wait(bar_q, uphase, s_abort, limit);
        if (w == WAIT_OK) {
          const int T = s_misc[MISC_NK] + s_misc[MISC_NC];
          constexpr uint32_t idesc_qk = QK8 ? idesc_s8_s32(128, 128) : idesc_bf16_f32(128, 128, false);
          const uint64_t qdesc0 = smem_desc_sw128(sb + C::OFF_Q, 16, 1024);
          const uint64_t kdesc0 = smem_desc_sw128(sb + C::OFF_K, 16, 1024);
          for (int t = 0; t < T && w == WAIT_OK; ++t) {
            const uint32_t g = tile_base + t;
            const int s = static_cast<int>(g % C::NK);
            const uint32_t b = g & 1u;
            // S[b] holds the P of tile t-2 until that tile's PV has completed. pv_done[b] completes
            // once per tile using S[b], and the PV of tile t cannot run before this QK^T, so the
            // parity wait is exact. (Tiles of the previous unit completed before the unit ended.)
            // K first (loaded well ahead), then the PV that frees this S buffer: the last wait
            w = mbar_wait(bar_kfull + 8 * s, (g / C::NK) & 1u, s_abort, limit);
            if (w == WAIT_OK && t >= 2) w = mbar_wait(bar_pvdone + 8 * b, ((g - 2u) >> 1) & 1u, s_abort, limit);
            if (w != WAIT_OK) break;
            tc_fence_after();
            const uint64_t kd = kdesc0 + ((s * C::QK_TILE_BYTES) >> 4);
            if constexpr (QK8) {
              // K = 32 int8 values (32 bytes) per MMA: four steps through the row's single atom
#pragma unroll
              for (int kk = 0; kk < D / 32; ++kk)
                mma_i8_ss(tmem + kColS + 128 * b, qdesc0 + kk * 2, kd + kk * 2, idesc_qk, kk > 0 ? 1u : 0u);
            } else {
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t off = ((kk >> 2) * C::CHUNK_BYTES + (kk & 3) * 32) >> 4;
                mma_bf16_ss(tmem + kColS + 128 * b, qdesc0 + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
              }
            }
            mma_issued = true;
            tc_commit(bar_sfull + 8 * b);
            tc_commit(bar_kempty + 8 * s);
          }
        }
        if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_MMA);
      }
    } else {
      // ------------------------------------------------------------------ router + softmax + epilogue
      const int st = tid - kSoftmaxWarp0 * 32;  // 0..255
      const int grp = st >> 7;                  // column half: warps 2..5 -> 0, warps 6..9 -> 1
      const int sw = st >> 5;                   // softmax warp 0..7
      const int wq = (warp & 3);                // TMEM lane quarter this warp may access
      const int row = wq * 32 + lane;           // query row = TMEM lane
      const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
      const int m_i = min(kRows, p.L - qb * kRows);
      const int nkb = p.nkb;

      const int nwords = (nkb + 31) / 32;
      int w = WAIT_OK;
      bool alive = true;  // same in all 256
      if (p.bits != nullptr) {
        // (1) the unit was routed by the routing pass: its keep bits
        const uint32_t* ub = p.bits + static_cast<size_t>(unit) * nwords;
        for (int i = st; i < nwords; i += kSoftmaxThreads) s_bits[i] = __ldg(ub + i);
      } else {
        w = mbar_wait(bar_q, uphase, s_abort, limit);
        if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_ROUTER);
        alive = !named_barrier_or(kBarSoftmax, kSoftmaxThreads, w != WAIT_OK);

        // (1a) q_bar = mean of the valid query rows, read from the swizzled Q tile. Thread st sums one
        // 16-byte chunk (8 columns) over a strided set of rows; the partial sums meet in shared memory
        // (the proxy-score buffer, not yet in use).
        {
          constexpr int CH = D / 8;                  // 16-byte chunks per row
          constexpr int RG = kSoftmaxThreads / CH;   // row groups: 16 (D=128) or 32 (D=64)
          const int c8 = st % CH, rg = st / CH;
          const uint8_t* qt = smem + C::OFF_Q + (c8 >> 3) * C::CHUNK_BYTES;
          const int jc = c8 & 7;
          float a[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) a[k] = 0.f;
          if (alive) {
#pragma unroll 2
            for (int r = rg; r < m_i; r += RG) {
              const uint4 v = *reinterpret_cast<const uint4*>(qt + r * 128 + ((jc ^ (r & 7)) << 4));
              const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                a[2 * k] += __uint_as_float(wv[k] << 16);
                a[2 * k + 1] += __uint_as_float(wv[k] & 0xffff0000u);
              }
            }
          }
          float* part = s_sbar;  // [RG][D]
#pragma unroll
          for (int k = 0; k < 8; ++k) part[rg * D + c8 * 8 + k] = a[k];
          named_barrier_sync(kBarSoftmax, kSoftmaxThreads);
          if (st < D) {
            float q = 0.f;
#pragma unroll 8
            for (int k = 0; k < RG; ++k) q += part[k * D + st];
            s_qbar[st] = q / static_cast<float>(m_i);
          }
          named_barrier_sync(kBarSoftmax, kSoftmaxThreads);
        }

        // (1b) proxy scores s_bar_j (shared memory only) and their max; 8 warps, 16 rows in flight
        // each (the pooled keys come from L2, so the loop is bound by how many loads are in flight)
        {
          constexpr int DPL = D / 32;
          constexpr int U = 16;
          float qv[DPL];
#pragma unroll
          for (int k = 0; k < DPL; ++k) qv[k] = s_qbar[lane * DPL + k];
          const float* kb = p.kbar + static_cast<size_t>(bh) * nkb * D + lane * DPL;
          float wmax = -INFINITY;
          for (int j0 = sw; j0 < nkb; j0 += 8 * U) {
            float dot[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
              const int j = j0 + 8 * u;
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
              for (int u = 0; u < U; ++u) dot[u] += __shfl_xor_sync(0xffffffffu, dot[u], o);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
              const int j = j0 + 8 * u;
              if (j < nkb) {
                const float sc = dot[u] * p.inv_sqrt_d;
                if (lane == 0) s_sbar[j] = sc;
                wmax = fmaxf(wmax, sc);
              }
            }
          }
          if (lane == 0) s_red[sw] = wmax;
          named_barrier_sync(kBarSoftmax, kSoftmaxThreads);
        }

        // (1c) keep bits, each warp ballots whole words
        {
          float M = s_red[0];
#pragma unroll
          for (int k = 1; k < 8; ++k) M = fmaxf(M, s_red[k]);
          const float thr = M - p.tau[bh % p.H];
          for (int i = sw; i < nwords; i += 8) {
            const int j = 32 * i + lane;
            const bool k = j < nkb && (s_sbar[j] >= thr || j < p.n_force);
            const uint32_t m = __ballot_sync(0xffffffffu, k);
            if (lane == 0) s_bits[i] = m;
          }
        }
      }  // routed in this kernel
      named_barrier_sync(kBarSoftmax, kSoftmaxThreads);

      // (1d) prefix counts of the keep words and the pooled-tile list (warp 0), then the kept list
      {
        int* s_pref = reinterpret_cast<int*>(s_qbar + D);  // [kMaxKeyBlocks / 32]: kept blocks before word i
        if (sw == 0) {
          int run = 0;
          for (int i0 = 0; i0 < nwords; i0 += 32) {
            const int i = i0 + lane;
            const int c = i < nwords ? __popc(s_bits[i]) : 0;
            int x = c;  // inclusive warp scan
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int y = __shfl_up_sync(0xffffffffu, x, o);
              if (lane >= o) x += y;
            }
            if (i < nwords) s_pref[i] = run + x - c;
            run += __shfl_sync(0xffffffffu, x, 31);
          }
          const int nk = run;
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
                if (cc * 4 + q < nwords) kept += __popc(s_bits[cc * 4 + q]);
              has_skip = kept < valid;
            }
            const uint32_t m = __ballot_sync(0xffffffffu, has_skip);
            if (has_skip) s_clist[nc + __popc(m & ((1u << lane) - 1u))] = static_cast<uint16_t>(cc);
            nc += __popc(m);
          }
          if (lane == 0) {
            s_misc[MISC_NK] = alive ? nk : 0;
            s_misc[MISC_NC] = alive ? nc : 0;
            if (p.bits == nullptr) atomicAdd(&p.ws[WS_COUNTS + bh], static_cast<uint32_t>(nk));
          }
        }
        named_barrier_sync(kBarSoftmax, kSoftmaxThreads);
        for (int i = sw; i < nwords; i += 8) {
          const uint32_t m = s_bits[i];
          if ((m >> lane) & 1u) s_klist[s_pref[i] + __popc(m & ((1u << lane) - 1u))] = static_cast<uint16_t>(32 * i + lane);
        }
      }
      named_barrier_sync(kBarSoftmax, kSoftmaxThreads);
      if constexpr (QK8) {
        // the scale of each kept tile's int32 scores: log2(e)/sqrt(d) * scale_q * scale_k. The
        // proxy-score buffer is free: 8-bit QK^T always comes with the routing pass's bits.
        const float sq = p.sl2 * __ldg(p.q_scale + unit);
        const float* ks = p.k_scale + static_cast<size_t>(bh) * nkb;
        const int nk_u = s_misc[MISC_NK];
        for (int t = st; t < nk_u; t += kSoftmaxThreads) s_sbar[t] = sq * __ldg(ks + s_klist[t]);
        named_barrier_sync(kBarSoftmax, kSoftmaxThreads);
      }
      if (st == 0 && alive) mbar_arrive(bar_list);
      if (p.kept_mask != nullptr && p.bits == nullptr) {
        uint8_t* mrow = p.kept_mask + (static_cast<size_t>(bh) * p.nqb + qb) * nkb;
        for (int j = st; j < nkb; j += kSoftmaxThreads)
          mrow[j] = static_cast<uint8_t>((s_bits[j >> 5] >> (j & 31)) & 1u);
      }

      // (2)+(3) online softmax over kept tiles, then pooled tiles; this thread: row `row`,
      // score columns [64 grp, 64 grp + 64), its own running max, sum and accumulator O_grp
      const int nk = s_misc[MISC_NK];
      const int T = alive ? nk + s_misc[MISC_NC] : 0;
      const float sl2 = p.sl2;
      // 8-bit QK^T: pooled tiles take log2(e)/sqrt(d) * scale_q * scale of their chunk of pooled keys
      const float sq2 = QK8 ? sl2 * __ldg(p.q_scale + unit) : sl2;
      const float* kbs = QK8 ? p.kb_scale + static_cast<size_t>(bh) * ((nkb + kRows - 1) / kRows) : nullptr;
      const uint32_t o_col = tmem + lane_base + kColO + D * grp;
      float m_run = -INFINITY, l_run = 0.f;
      bool bad = false;  // a wait of this warp failed inside the tile loop
      for (int t = 0; t < T; ++t) {
        const uint32_t g = tile_base + t;
        const uint32_t b = g & 1u;
        const uint32_t s_col = tmem + lane_base + kColS + 128 * b + 64 * grp;
        w = mbar_wait(bar_sfull + 8 * b, (g >> 1) & 1u, s_abort, limit);
        if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_SOFTMAX);
        if (!__all_sync(0xffffffffu, w == WAIT_OK)) {
          bad = true;
          break;
        }
        tc_fence_after();
        float s[64];
        const bool exact = t < nk;
        const int j = exact ? static_cast<int>(s_klist[t]) : 0;
        const bool full = exact && (j != nkb - 1 || p.last_n == kRows);
        // the factor that turns this tile's raw scores into log2-domain logits (> 0)
        float ts = sl2;
        if constexpr (QK8) ts = exact ? s_sbar[t] : sq2 * __ldg(kbs + s_clist[t - nk]);
        {
          uint32_t raw[64];
          tmem_ld_x64(s_col, raw);
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = QK8 ? s32_to_f32_small(raw[c]) : __uint_as_float(raw[c]);
        }
        float mx;
        if (full) {
          mx = max64(s) * ts;  // ts > 0: the max of the scaled scores
        } else {
          if (exact) {
            const int valid = p.last_n - grp * 64;  // valid columns in this half (may be <= 0)
#pragma unroll
            for (int c = 0; c < 64; ++c) s[c] = (c < valid) ? s[c] * ts : -INFINITY;
          } else {
            const int cc = s_clist[t - nk];
            const int valid = min(kRows, nkb - cc * kRows) - grp * 64;
            const int nwords = (nkb + 31) / 32;
            const uint32_t kw0 = (cc * 4 + grp * 2 < nwords) ? s_bits[cc * 4 + grp * 2] : 0u;
            const uint32_t kw1 = (cc * 4 + grp * 2 + 1 < nwords) ? s_bits[cc * 4 + grp * 2 + 1] : 0u;
            const int last_col = nkb - 1 - cc * kRows - grp * 64;  // column of the ragged last block, if here
#pragma unroll
            for (int c = 0; c < 64; ++c) {
              const uint32_t kw = c < 32 ? kw0 : kw1;
              const bool skipped = c < valid && !((kw >> (c & 31)) & 1u);
              const float off = (c == last_col) ? p.log2_last_n : 7.0f;  // log2(n_j)
              s[c] = skipped ? fmaf(s[c], ts, off) : -INFINITY;
            }
          }
          mx = max64(s);
        }
        // lazy rescale; a half row whose columns have all been masked so far keeps m = -inf and
        // P = 0, and the first finite max rescales its (zero) accumulator by 0
        float m_new = m_run, alpha = 1.f;
        bool need = false;
        if constexpr (PV8) {
          // integer reference (the oracle's e4m3_channel reading): a rescale moves it to the
          // ceiling of the new max and multiplies O by an exact power of two
          if (t == 0) {
            m_new = ceilf(mx);
          } else if (mx > m_run + kRescaleThreshold8) {
            need = true;
            m_new = ceilf(mx);
            alpha = exp2_int(m_run - m_new);
          }
        } else {
          if (t == 0) {
            m_new = mx;
          } else if (mx > m_run + kRescaleThreshold) {
            need = true;
            m_new = mx;
            alpha = ex2_approx(m_run - mx);
          }
        }
        m_run = m_new;
        if constexpr (PV8) {
          // P = 2^(x - (m - 6)) <= 2^(6 + 2) = 256 < 448: E4M3 codes, four per TMEM column; the row
          // sum adds the codes' exact values, the weights the PV product uses
          const float m_use = (m_new == -INFINITY) ? 0.f : m_new - static_cast<float>(kHeadroom8);
          uint32_t pk[16];
          float2 a2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
          for (int c4 = 0; c4 < 16; ++c4) {
            float e[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
              e[k] = ex2_approx(full ? fmaf(s[4 * c4 + k], ts, -m_use) : s[4 * c4 + k] - m_use);
            const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(e[0], e[1]), __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(e[2], e[3]), __NV_SATFINITE, __NV_E4M3);
            pk[c4] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
            a2[0] = __fadd2_rn(a2[0], e4m3x2_to_float2(lo));
            a2[1] = __fadd2_rn(a2[1], e4m3x2_to_float2(hi));
          }
          l_run = fmaf(l_run, alpha, (a2[0].x + a2[0].y) + (a2[1].x + a2[1].y));
          // P over the first 16 of this group's S columns, which are already in registers
          tmem_st_x16(s_col, pk);
        } else {
          const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
          uint32_t pk[32];
          float acc[4] = {0.f, 0.f, 0.f, 0.f};  // row sum of the bf16-rounded weights, 4 chains
          if (full) {
            const float2 scale2 = make_float2(ts, ts);
            const float2 negm2 = make_float2(-m_use, -m_use);
#pragma unroll
            for (int c2 = 0; c2 < 32; ++c2) {
              const float2 x2 = __ffma2_rn(make_float2(s[2 * c2], s[2 * c2 + 1]), scale2, negm2);
              float2 e2;
              if (kPolyEvery > 0 && (c2 % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1) {
                e2 = exp2_poly2(make_float2(fmaxf(x2.x, -126.f), fmaxf(x2.y, -126.f)));
              } else {
                e2 = make_float2(ex2_approx(x2.x), ex2_approx(x2.y));
              }
              pk[c2] = pack_bf16x2(e2.x, e2.y);
              acc[c2 & 3] = add_bf16x2(acc[c2 & 3], pk[c2]);
            }
          } else {
#pragma unroll
            for (int c2 = 0; c2 < 32; ++c2) {
              const float e0 = ex2_approx(s[2 * c2] - m_use);
              const float e1 = ex2_approx(s[2 * c2 + 1] - m_use);
              pk[c2] = pack_bf16x2(e0, e1);
              acc[c2 & 3] = add_bf16x2(acc[c2 & 3], pk[c2]);
            }
          }
          // the row sum takes the same bf16-rounded weights the PV MMA uses
          l_run = fmaf(l_run, alpha, (acc[0] + acc[1]) + (acc[2] + acc[3]));
          // P over the first 32 of this group's S columns, which are already in registers
          tmem_st_x32(s_col, pk);
        }
        if (__any_sync(0xffffffffu, need)) {
          // rescale O_grp once the previous tile's PV has landed. pv_done[buf] completes once per
          // tile using that buffer; the PV three tiles back completed before the one two tiles back
          // (same accumulators, same issuing thread), which completed before this tile's QK^T was
          // issued, and the PV of tile t+1 needs this group's next P, so the parity wait is exact.
          w = mbar_wait(bar_pvdone + 8 * ((g - 1u) & 1u), ((g - 1u) >> 1) & 1u, s_abort, limit);
          if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_SOFTMAX);
          if (__all_sync(0xffffffffu, w == WAIT_OK)) {
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < D / 32; ++ch) {
              uint32_t o[32];
              tmem_ld_x32(o_col + ch * 32, o);
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
              tmem_st_x32(o_col + ch * 32, o);
            }
          } else {
            bad = true;  // P is still published below, so the MMA issuer is not left waiting
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_pfull + 8 * (2 * b + grp));
        if (bad) break;
      }

      // (4) epilogue: merge the two groups' partial results, O / l -> bf16; group g stores
      // output columns [g D/2, (g+1) D/2)
      {
        bool ok = alive && !bad && T > 0;
        if (ok) {
          w = mbar_wait(bar_ofinal, uphase, s_abort, limit);
          if (w == WAIT_TIMEOUT) raise_timeout(s_abort, p.ws, WHERE_SOFTMAX);
          ok = __all_sync(0xffffffffu, w == WAIT_OK);
        }
        // every softmax thread reaches this barrier, whether or not its tile loop ended early
        s_ml[grp * kRows + row] = make_float2(m_run, l_run);
        const bool any_bad = named_barrier_or(kBarSoftmax, kSoftmaxThreads, !ok);
        if (!any_bad) {
          tc_fence_after();
          const float2 ml0 = s_ml[row], ml1 = s_ml[kRows + row];
          const float m = fmaxf(ml0.x, ml1.x);  // finite: every row sees at least one valid column
          // 2^-inf = 0; with integer references (8-bit PV) the factors are exact powers of two
          const float a0 = PV8 ? exp2_int(ml0.x - m) : ex2_approx(ml0.x - m);
          const float a1 = PV8 ? exp2_int(ml1.x - m) : ex2_approx(ml1.x - m);
          const float inv = 1.f / fmaf(ml0.y, a0, ml1.y * a1);
          const float c0 = a0 * inv, c1 = a1 * inv;
          const bool store = row < m_i;
          __nv_bfloat16* dst = p.O + (static_cast<size_t>(bh) * p.L + static_cast<size_t>(qb) * kRows + row) * D +
                               grp * (D / 2);
          const uint32_t o0 = tmem + lane_base + kColO + grp * (D / 2);
#pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) {
            uint32_t x0[32], x1[32];
            tmem_ld_x32(o0 + ch * 32, x0);
            tmem_ld_x32(o0 + D + ch * 32, x1);
            uint32_t pkd[16];
            if constexpr (PV8) {
              // the E4M3 values' channel scales, one per output column
              const float* vs = p.v_scale + static_cast<size_t>(bh) * D + grp * (D / 2) + ch * 32;
#pragma unroll
              for (int c = 0; c < 16; ++c) {
                const float2 sc = __ldg(reinterpret_cast<const float2*>(vs) + c);
                pkd[c] = pack_bf16x2(fmaf(__uint_as_float(x0[2 * c]), c0, __uint_as_float(x1[2 * c]) * c1) * sc.x,
                                     fmaf(__uint_as_float(x0[2 * c + 1]), c0, __uint_as_float(x1[2 * c + 1]) * c1) *
                                         sc.y);
              }
            } else {
#pragma unroll
              for (int c = 0; c < 16; ++c)
                pkd[c] = pack_bf16x2(fmaf(__uint_as_float(x0[2 * c]), c0, __uint_as_float(x1[2 * c]) * c1),
                                     fmaf(__uint_as_float(x0[2 * c + 1]), c0, __uint_as_float(x1[2 * c + 1]) * c1));
            }
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

  if (stamp) p.cta_times[2 * blockIdx.x + 1] = globaltimer_ns();

  // ---- drain: no copy or MMA may still be in flight when TMEM and shared memory are released
  if ((warp == 1 || warp == kPv1Warp || warp == kQkWarp) && lane == 0 && mma_issued) {
    const uint32_t bd = bar_drain + (warp == 1 ? 0 : (warp == kPv1Warp ? 8 : 16));
    tc_commit(bd);
    mbar_wait(bd, 0, nullptr, limit);
  }
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::NK; ++s)
      if (k_armed[s]) mbar_wait(bar_kfull + 8 * s, (k_armed[s] - 1u) & 1u, nullptr, limit);
    for (int s = 0; s < C::NV; ++s)
      if (v_armed[s]) mbar_wait(bar_vfull + 8 * s, (v_armed[s] - 1u) & 1u, nullptr, limit);
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

template <int D, bool QK8, bool PV8 = false>
cudaError_t launch_tc_t(const FwdArgs& a, const CUtensorMap* maps, cudaStream_t stream) {
  using C = TcCfg<D, QK8, PV8>;
  TcParams p;
  p.kbar = a.kbar;
  p.bits = a.route_bits;
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
  p.q_scale = QK8 ? a.qk8->q_scale : nullptr;
  p.k_scale = QK8 ? a.qk8->k_scale : nullptr;
  p.kb_scale = QK8 ? a.qk8->kb_scale : nullptr;
  p.v_scale = PV8 ? a.pv8->v_scale : nullptr;
  p.cta_times = a.cta_times;
  p.cta_capacity = a.cta_capacity;
  for (int h = 0; h < kMaxHeads; ++h) p.tau[h] = h < a.H ? a.tau[h] : 0.f;
  cudaError_t e = cudaFuncSetAttribute(sol_fwd_tc_kernel<D, QK8, PV8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int grid = p.total_units < a.num_sms ? p.total_units : a.num_sms;
  sol_fwd_tc_kernel<D, QK8, PV8><<<grid, kThreads, C::SMEM_BYTES, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4],
                                                                             p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_tc(const FwdArgs& a, const CUtensorMap* maps, cudaStream_t stream) {
  if (a.qk8 != nullptr) {
    // 8-bit QK^T: d = 128 and keep bits from the routing pass (the Q tile in shared memory holds
    // int8 codes, which the in-kernel routing cannot average); 8-bit PV only with it
    if (a.d != 128 || a.route_bits == nullptr) return cudaErrorNotSupported;
    if (a.pv8 != nullptr) return launch_tc_t<128, true, true>(a, maps, stream);
    return launch_tc_t<128, true>(a, maps, stream);
  }
  if (a.pv8 != nullptr) return cudaErrorNotSupported;
  if (a.d == 64) return launch_tc_t<64, false>(a, maps, stream);
  if (a.d == 128) return launch_tc_t<128, false>(a, maps, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sol
