// Internal launcher interface between the C ABI (sol_attn_api.cu) and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace sol {

// 8-bit QK^T operands of the forward (sol_attn_quantize_qk8): codes and per-tile scales
struct Qk8Operands {
  const int8_t* q8;        // [BH, L, d]
  const int8_t* k8;        // [BH, L, d], K - mu
  const int8_t* kb8;       // [BH, N_kb, d], k_bar - mu
  const float* q_scale;    // [BH, N_qb]
  const float* k_scale;    // [BH, N_kb]
  const float* kb_scale;   // [BH, ceil(N_kb / 128)]
};

// 8-bit PV operands of the forward (sol_attn_quantize_v8): E4M3 codes, transposed, and channel scales
struct Pv8Operands {
  const uint8_t* v8t;      // [BH, d, N_kb * 128]
  const uint8_t* vb8t;     // [BH, d, 128 * ceil(N_kb / 128)]
  const float* v_scale;    // [BH, d]
};

struct FwdArgs {
  const void* Q;
  const void* K;
  const void* V;
  const float* kbar;
  const float* vbar;
  const void* kbar_lp;
  const void* vbar_lp;
  const float* tau;  // host [H]
  bool bf16;
  int B, H, L, d, block;
  int n_force;
  void* O;
  uint8_t* kept_mask;
  float* density;
  uint32_t* ws;
  int num_sms;
  int drop_one_load;       // failure-detection test hook (bf16 path)
  uint32_t* route_bits;    // bf16 path: [B*H, N_qb, ceil(N_kb/32)] keep bits from launch_route, or null
                           // (the fused kernel then routes each unit itself)
  float* route_qbar;       // with route_bits: [B*H, N_qb, d] fp32 query-block means (workspace)
  uint64_t wait_limit_ns;  // bound on every on-device wait
  int k_keep = 0;          // routing pass: 0 = threshold max - tau; k > 0 = the k highest scores
  unsigned long long* cta_times = nullptr;  // measurement hook: [2 * cta_capacity] start/finish ns
  int cta_capacity = 0;
  const Qk8Operands* qk8 = nullptr;  // bf16 path: int8 Q, K and pooled keys for QK^T, or null
  const Pv8Operands* pv8 = nullptr;  // with qk8: E4M3 V and v_bar for PV (kind::f8f6f4), or null
  const float* qbar_in = nullptr;    // routing pass: fp32 [B*H, N_qb, d] query-block means given by the
                                     // caller (the QK-norm + RoPE pass); null = computed from Q
};

cudaError_t launch_pool(const void* K, const void* V, bool bf16, int BH, int L, int d, int block,
                        float* kbar, float* vbar, void* kbar_lp, void* vbar_lp, cudaStream_t stream);

struct RopePoolArgs {
  const void* Q;  // bf16 [BH, L, d]
  const void* K;
  const void* V;
  const float* gain_q;  // [d]
  const float* gain_k;  // [d]
  const float* cos;     // [L, d/2]
  const float* sin;     // [L, d/2]
  float eps;
  void* Qout;  // bf16 [BH, L, d]
  void* Kout;
  float* kbar;  // fp32 [BH, N_kb, d]
  float* vbar;
  void* kbar_lp;  // bf16 [BH, N_kb, d]
  void* vbar_lp;
  float* qbar = nullptr;  // out, optional: fp32 [BH, N_kb, d] means of the stored query rows per block
  int BH, L, d, block;
};

struct QuantArgs {
  const void* Q;       // bf16 [BH, L, d]
  const void* K;       // bf16 [BH, L, d]
  const float* kbar;   // fp32 [BH, N_kb, d] from the pooling pass
  float* mu;           // out: fp32 [BH, d] mean key
  int8_t* q8;          // out: int8 [BH, L, d]
  int8_t* k8;          // out: int8 [BH, L, d] codes of K - mu
  int8_t* kb8;         // out: int8 [BH, N_kb, d] codes of k_bar - mu
  float* q_scale;      // out: [BH, N_qb]
  float* k_scale;      // out: [BH, N_kb]
  float* kb_scale;     // out: [BH, ceil(N_kb / 128)]
  int BH, L, d;
};

// bf16, d in {64, 128}, blocks of 128: the mean key, then int8 codes and tile scales of Q, K - mu
// and k_bar - mu.
cudaError_t launch_quant_qk8(const QuantArgs& a, cudaStream_t stream);

// 8-bit PV values (d = 128): per-channel scales of V and the transposed E4M3 codes of V and v_bar.
struct QuantV8Args {
  const void* V;        // bf16 [BH, L, d]
  const float* vbar;    // fp32 [BH, N_kb, d] from the pooling pass
  uint8_t* v8t;         // out: E4M3 [BH, d, N_kb * 128], keys contiguous, zero past L
  uint8_t* vb8t;        // out: E4M3 [BH, d, 128 * ceil(N_kb / 128)], zero past N_kb
  float* v_scale;       // out: fp32 [BH, d] (also the amax accumulator while the pass runs)
  int BH, L, d;
};
cudaError_t launch_quant_v8(const QuantV8Args& a, cudaStream_t stream);

// bf16, d in {64, 128}: QK RMS norm + rotary embedding + K/V block pooling in one pass.
cudaError_t launch_qknorm_rope_pool(const RopePoolArgs& a, cudaStream_t stream);

// bf16, d in {64, 128}, block 128: routing pass for every unit (q_bar kernel, then the routing
// kernel); writes a.route_qbar, a.route_bits, the optional mask and the per-head kept counts
// (ws + WS_COUNTS).
cudaError_t launch_route(const FwdArgs& a, cudaStream_t stream);

// bf16, d in {64, 128}, block 128: TMA + tcgen05 persistent kernel.
cudaError_t launch_fwd_tc(const FwdArgs& a, const CUtensorMap* maps /* Q, K, V, Kbar_lp, Vbar_lp */,
                          cudaStream_t stream);

// fp32, d in {32, 64, 128}, block in {32, 64, 128}: SIMT kernel.
cudaError_t launch_fwd_simt(const FwdArgs& a, cudaStream_t stream);

}  // namespace sol
