// C ABI of the Sol-Attn forward (declared in include/sol_attn.h): argument validation on the
// host, TMA tensor-map encoding, and dispatch to the pool, fp32 SIMT and bf16 tcgen05 kernels.
// Nothing here allocates device memory; every launch goes to the caller's stream.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "device_common.cuh"
#include "launchers.h"
#include "sol_attn.h"

namespace {

thread_local std::string g_last_error;
int g_drop_one_load = 0;  // failure-detection test hook, consumed by the next bf16 launch

sol_status fail(sol_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

sol_status cuda_fail(cudaError_t e, const char* what) {
  return fail(SOL_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device checks: an sm_100 GPU is current. Returns SOL_OK and its SM count.
sol_status current_device(int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute");
  if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute");
  if (major != 10 || minor != 0)
    return fail(SOL_EUNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a (B200)", dev, major, minor);
  if ((e = cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute");
  return SOL_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link-time libcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 3-D bf16 view [BH][rows][d] with 64 x 128 x 1 boxes and 128-byte swizzle. Rows past `rows`
// (a ragged last block) are zero-filled by the copy engine.
sol_status make_map(CUtensorMap* m, const void* base, int d, int rows, int BH) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(SOL_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(rows) * d * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SOL_ECUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
  return SOL_OK;
}

bool size_ok(long long v, long long lim) { return v >= 1 && v <= lim; }

// Workspace layout: [error, where, counter, done, counts[B*H]] rounded to 256 B (the header), then
// the keep bits of the routing pass, u32[B*H][N_qb][ceil(N_kb/32)].
size_t ws_header_bytes(int B, int H) {
  const size_t words = static_cast<size_t>(sol::WS_COUNTS) + static_cast<size_t>(B) * H;
  return (words * 4 + 255) / 256 * 256;
}
size_t ws_bits_bytes(int B, int H, int L, int block) {
  const size_t nb = (static_cast<size_t>(L) + block - 1) / block;
  const size_t bytes = static_cast<size_t>(B) * H * nb * ((nb + 31) / 32) * 4;
  return (bytes + 255) / 256 * 256;
}

// ---- workspace in the library's own device memory, for sol_attn_fwd_noalloc -------------------
constexpr int kNoAllocMaxHeads = 4096;  // B * H
constexpr size_t kNoAllocWords = static_cast<size_t>(sol::WS_COUNTS) + kNoAllocMaxHeads;
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

}  // namespace

// One array per device that loads the library, alive until the process exits. In host code this
// name is only a host-side handle: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint32_t g_noalloc_ws[kNoAllocWords];

namespace {

// Device address of g_noalloc_ws on the current device, looked up once per device.
sol_status noalloc_workspace(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SOL_EUNSUPPORTED, "device index %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_ws);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static workspace)");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return SOL_OK;
}

}  // namespace

extern "C" {

const char* sol_attn_status_string(sol_status s) {
  switch (s) {
    case SOL_OK: return "SOL_OK";
    case SOL_EINVAL: return "SOL_EINVAL (invalid argument)";
    case SOL_EUNSUPPORTED: return "SOL_EUNSUPPORTED (shape/dtype not implemented)";
    case SOL_ECUDA: return "SOL_ECUDA (CUDA runtime error)";
    case SOL_ETIMEOUT: return "SOL_ETIMEOUT (bounded device wait expired)";
  }
  return "unknown sol_status";
}

const char* sol_attn_last_error(void) { return g_last_error.c_str(); }

void sol_attn_debug_drop_one_load(int mode) { g_drop_one_load = mode; }

sol_status sol_attn_pool(const void* K, const void* V, sol_dtype dt, int B, int H, int L, int d, int block_k,
                         float* kbar, float* vbar, void* kbar_lp, void* vbar_lp, void* stream) {
  g_last_error.clear();
  if (dt != SOL_F32 && dt != SOL_BF16) return fail(SOL_EINVAL, "unknown dtype %d", static_cast<int>(dt));
  if (!size_ok(B, 1 << 16) || !size_ok(H, 1 << 16) || !size_ok(L, 1 << 28) || !size_ok(d, 1 << 16) ||
      !size_ok(block_k, 1 << 20))
    return fail(SOL_EINVAL, "sizes must be positive (B=%d H=%d L=%d d=%d block_k=%d)", B, H, L, d, block_k);
  if (static_cast<long long>(B) * H > 65535) return fail(SOL_EUNSUPPORTED, "B*H must be <= 65535");
  if (K == nullptr || V == nullptr || kbar == nullptr || vbar == nullptr)
    return fail(SOL_EINVAL, "K, V, kbar and vbar must be non-null");
  if (!aligned16(K) || !aligned16(V) || !aligned16(kbar) || !aligned16(vbar))
    return fail(SOL_EINVAL, "device pointers must be 16-byte aligned");
  const bool bf16 = dt == SOL_BF16;
  if (bf16 && (kbar_lp == nullptr || vbar_lp == nullptr))
    return fail(SOL_EINVAL, "kbar_lp and vbar_lp are required for bf16 inputs");
  if (!bf16 && (kbar_lp != nullptr || vbar_lp != nullptr))
    return fail(SOL_EINVAL, "kbar_lp and vbar_lp must be NULL for fp32 inputs");
  if (bf16 && (!aligned16(kbar_lp) || !aligned16(vbar_lp)))
    return fail(SOL_EINVAL, "device pointers must be 16-byte aligned");
  if (d > 512 || d % (bf16 ? 8 : 4) != 0)
    return fail(SOL_EUNSUPPORTED, "pool needs d <= 512 and d %% %d == 0 (d=%d)", bf16 ? 8 : 4, d);
  if (block_k > 4096) return fail(SOL_EUNSUPPORTED, "pool needs block_k <= 4096");
  if ((L + block_k - 1) / block_k > 0x7fffffff / 1) return fail(SOL_EUNSUPPORTED, "too many blocks");
  int sms = 0;
  sol_status st = current_device(&sms);
  if (st != SOL_OK) return st;
  cudaError_t e = sol::launch_pool(K, V, bf16, B * H, L, d, block_k, kbar, vbar, kbar_lp, vbar_lp,
                                   static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pool kernel launch");
  return SOL_OK;
}

sol_status sol_attn_qknorm_rope_pool(const void* Q, const void* K, const void* V, const float* gain_q,
                                     const float* gain_k, const float* rope_cos, const float* rope_sin, float eps,
                                     int B, int H, int L, int d, int block_k, void* Q_out, void* K_out, float* kbar,
                                     float* vbar, void* kbar_lp, void* vbar_lp, void* stream) {
  g_last_error.clear();
  if (!size_ok(B, 1 << 16) || !size_ok(H, 1 << 16) || !size_ok(L, 1 << 28) || !size_ok(d, 1 << 16) ||
      !size_ok(block_k, 1 << 20))
    return fail(SOL_EINVAL, "sizes must be positive (B=%d H=%d L=%d d=%d block_k=%d)", B, H, L, d, block_k);
  if (!(eps > 0.f) || std::isinf(eps)) return fail(SOL_EINVAL, "eps=%g must be positive and finite", eps);
  const void* ptrs[] = {Q, K, V, gain_q, gain_k, rope_cos, rope_sin, Q_out, K_out, kbar, vbar, kbar_lp, vbar_lp};
  for (const void* ptr : ptrs) {
    if (ptr == nullptr) return fail(SOL_EINVAL, "every pointer argument must be non-null");
    if (!aligned16(ptr)) return fail(SOL_EINVAL, "device pointers must be 16-byte aligned");
  }
  if (d != 64 && d != 128) return fail(SOL_EUNSUPPORTED, "QK-norm + RoPE + pooling needs d in {64, 128} (d=%d)", d);
  if (block_k > 4096) return fail(SOL_EUNSUPPORTED, "block_k must be <= 4096");
  if (static_cast<long long>(B) * H > 65535) return fail(SOL_EUNSUPPORTED, "B*H must be <= 65535");
  int sms = 0;
  sol_status st = current_device(&sms);
  if (st != SOL_OK) return st;
  sol::RopePoolArgs a;
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.gain_q = gain_q;
  a.gain_k = gain_k;
  a.cos = rope_cos;
  a.sin = rope_sin;
  a.eps = eps;
  a.Qout = Q_out;
  a.Kout = K_out;
  a.kbar = kbar;
  a.vbar = vbar;
  a.kbar_lp = kbar_lp;
  a.vbar_lp = vbar_lp;
  a.BH = B * H;
  a.L = L;
  a.d = d;
  a.block = block_k;
  cudaError_t e = sol::launch_qknorm_rope_pool(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "QK-norm + RoPE + pooling launch");
  return SOL_OK;
}

size_t sol_attn_fwd_workspace_bytes(int B, int H, int L, int block_q) {
  if (B < 1 || H < 1 || L < 1 || block_q < 1) return 0;
  return ws_header_bytes(B, H) + ws_bits_bytes(B, H, L, block_q);
}

sol_status sol_attn_fwd(const void* Q, const void* K, const void* V, const float* kbar, const float* vbar,
                        const void* kbar_lp, const void* vbar_lp, const float* tau, sol_dtype dt, int B, int H, int L,
                        int d, int block_q, int block_k, int n_force, void* O, uint8_t* kept_mask, float* density,
                        void* workspace, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (dt != SOL_F32 && dt != SOL_BF16) return fail(SOL_EINVAL, "unknown dtype %d", static_cast<int>(dt));
  if (!size_ok(B, 1 << 16) || !size_ok(H, 1 << 16) || !size_ok(L, 1 << 28) || !size_ok(d, 1 << 16) ||
      !size_ok(block_q, 1 << 20) || !size_ok(block_k, 1 << 20))
    return fail(SOL_EINVAL, "sizes must be positive (B=%d H=%d L=%d d=%d block_q=%d block_k=%d)", B, H, L, d,
                block_q, block_k);
  if (Q == nullptr || K == nullptr || V == nullptr || kbar == nullptr || O == nullptr || tau == nullptr ||
      workspace == nullptr)
    return fail(SOL_EINVAL, "Q, K, V, kbar, O, tau and workspace must be non-null");
  const bool bf16 = dt == SOL_BF16;
  if (bf16 && (kbar_lp == nullptr || vbar_lp == nullptr))
    return fail(SOL_EINVAL, "kbar_lp and vbar_lp are required for bf16 inputs");
  if (!bf16 && vbar == nullptr) return fail(SOL_EINVAL, "vbar is required for fp32 inputs");
  const void* ptrs[] = {Q, K, V, kbar, O, workspace, vbar, bf16 ? kbar_lp : nullptr, bf16 ? vbar_lp : nullptr};
  for (const void* ptr : ptrs)
    if (ptr != nullptr && !aligned16(ptr)) return fail(SOL_EINVAL, "device pointers must be 16-byte aligned");
  if (H > sol::kMaxHeads) return fail(SOL_EUNSUPPORTED, "H=%d exceeds %d", H, sol::kMaxHeads);
  for (int h = 0; h < H; ++h)
    if (std::isnan(tau[h]) || tau[h] < 0.f) return fail(SOL_EINVAL, "tau[%d]=%g must be >= 0 and not NaN", h, tau[h]);
  if (block_q != block_k) return fail(SOL_EUNSUPPORTED, "block_q must equal block_k");
  if (bf16) {
    if (block_q != 128 || (d != 64 && d != 128))
      return fail(SOL_EUNSUPPORTED, "bf16 path needs block 128 and d in {64, 128} (block=%d d=%d)", block_q, d);
  } else {
    if ((block_q != 32 && block_q != 64 && block_q != 128) || (d != 32 && d != 64 && d != 128))
      return fail(SOL_EUNSUPPORTED, "fp32 path needs block in {32,64,128} and d in {32,64,128} (block=%d d=%d)",
                  block_q, d);
  }
  const long long nkb = (static_cast<long long>(L) + block_k - 1) / block_k;
  if (nkb > sol::kMaxKeyBlocks) return fail(SOL_EUNSUPPORTED, "N_kb=%lld exceeds %d", nkb, sol::kMaxKeyBlocks);
  if (n_force < 0 || n_force > nkb) return fail(SOL_EINVAL, "n_force=%d must be in [0, N_kb=%lld]", n_force, nkb);
  if (static_cast<long long>(B) * H * nkb >= (1ll << 31)) return fail(SOL_EUNSUPPORTED, "B*H*N_qb must be < 2^31");
  if (static_cast<long long>(B) * H > 65535) return fail(SOL_EUNSUPPORTED, "B*H must be <= 65535");
  const size_t need = ws_header_bytes(B, H);
  if (ws_bytes < need) return fail(SOL_EINVAL, "workspace too small (%zu < %zu bytes)", ws_bytes, need);
  // a workspace that also holds the keep bits gets the separate routing pass (bf16 path)
  const bool route_pass = bf16 && ws_bytes >= need + ws_bits_bytes(B, H, L, block_q);

  int sms = 0;
  sol_status st = current_device(&sms);
  if (st != SOL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  // zero the scheduler counter, the finished-CTA counter and the per-head counts; the sticky
  // error words (first 8 bytes) are left for sol_attn_check_device_error
  cudaError_t e = cudaMemsetAsync(static_cast<uint8_t*>(workspace) + 4 * sol::WS_COUNTER, 0,
                                  4 * (static_cast<size_t>(2) + static_cast<size_t>(B) * H), s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");

  sol::FwdArgs a;
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.kbar = kbar;
  a.vbar = vbar;
  a.kbar_lp = kbar_lp;
  a.vbar_lp = vbar_lp;
  a.tau = tau;
  a.bf16 = bf16;
  a.B = B;
  a.H = H;
  a.L = L;
  a.d = d;
  a.block = block_q;
  a.n_force = n_force;
  a.O = O;
  a.kept_mask = kept_mask;
  a.density = density;
  a.ws = static_cast<uint32_t*>(workspace);
  a.num_sms = sms;
  a.drop_one_load = 0;
  a.wait_limit_ns = 2000000000ull;
  a.route_bits = route_pass ? reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + need) : nullptr;

  if (bf16) {
    a.drop_one_load = g_drop_one_load;
    if (g_drop_one_load) a.wait_limit_ns = 200000000ull;
    g_drop_one_load = 0;
    CUtensorMap maps[5];
    const int nkb_i = static_cast<int>(nkb);
    if ((st = make_map(&maps[0], Q, d, L, B * H)) != SOL_OK) return st;
    if ((st = make_map(&maps[1], K, d, L, B * H)) != SOL_OK) return st;
    if ((st = make_map(&maps[2], V, d, L, B * H)) != SOL_OK) return st;
    if ((st = make_map(&maps[3], kbar_lp, d, nkb_i, B * H)) != SOL_OK) return st;
    if ((st = make_map(&maps[4], vbar_lp, d, nkb_i, B * H)) != SOL_OK) return st;
    if (route_pass) {
      e = sol::launch_route(a, s);
      if (e != cudaSuccess) return cuda_fail(e, "routing launch");
    }
    e = sol::launch_fwd_tc(a, maps, s);
    if (e != cudaSuccess) return cuda_fail(e, "tcgen05 forward launch");
  } else {
    e = sol::launch_fwd_simt(a, s);
    if (e != cudaSuccess) return cuda_fail(e, "fp32 forward launch");
  }
  return SOL_OK;
}

sol_status sol_attn_fwd_noalloc(const void* Q, const void* K, const void* V, const float* kbar, const float* vbar,
                                const void* kbar_lp, const void* vbar_lp, const float* tau, sol_dtype dt, int B, int H,
                                int L, int d, int block_q, int block_k, int n_force, void* O, uint8_t* kept_mask,
                                float* density, void* stream) {
  g_last_error.clear();
  if (B < 1 || H < 1) return fail(SOL_EINVAL, "B and H must be positive (B=%d H=%d)", B, H);
  if (static_cast<long long>(B) * H > kNoAllocMaxHeads)
    return fail(SOL_EUNSUPPORTED, "B*H=%lld exceeds the %d heads the static workspace holds; use sol_attn_fwd",
                static_cast<long long>(B) * H, kNoAllocMaxHeads);
  void* ws = nullptr;
  sol_status st = noalloc_workspace(&ws);
  if (st != SOL_OK) return st;
  // the array keeps the previous call's contents: clear all of it (counters and error word)
  const size_t bytes = sizeof(uint32_t) * kNoAllocWords;
  cudaError_t e = cudaMemsetAsync(ws, 0, bytes, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(static workspace)");
  return sol_attn_fwd(Q, K, V, kbar, vbar, kbar_lp, vbar_lp, tau, dt, B, H, L, d, block_q, block_k, n_force, O,
                      kept_mask, density, ws, bytes, stream);
}

sol_status sol_attn_check_device_error(void* workspace, void* stream) {
  g_last_error.clear();
  if (workspace == nullptr) return fail(SOL_EINVAL, "workspace must be non-null");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t words[2] = {0, 0};
  e = cudaMemcpy(words, workspace, sizeof(words), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(error word)");
  if (words[0] == 0) return SOL_OK;
  e = cudaMemset(workspace, 0, sizeof(words));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(error word)");
  static const char* roles[] = {"?", "producer", "mma", "softmax", "router"};
  return fail(SOL_ETIMEOUT, "device wait expired (first in the %s role)", roles[words[1] < 5 ? words[1] : 0]);
}

}  // extern "C"
