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
unsigned long long* g_cta_times = nullptr;  // measurement hook, consumed by the next bf16 launch
int g_cta_capacity = 0;

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

// 3-D view [BH][rows][d] with 128-byte-wide x 128 x 1 boxes (64 bf16 or 128 int8 values) and
// 128-byte swizzle. Rows past `rows` (a ragged last block) are zero-filled by the copy engine.
sol_status make_map(CUtensorMap* m, const void* base, int d, int rows, int BH, bool int8 = false) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(SOL_ECUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t es = int8 ? 1 : 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * es, static_cast<cuuint64_t>(rows) * d * es};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / es), 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, int8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estr,
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
// After the keep bits: the routing pass's query-block means, fp32 [B*H][N_qb][d], sized for the
// largest head dimension of the bf16 path (128) because the size function takes no d.
constexpr size_t kQbarMaxD = 128;
size_t ws_qbar_bytes(int B, int H, int L, int block) {
  const size_t nb = (static_cast<size_t>(L) + block - 1) / block;
  const size_t bytes = static_cast<size_t>(B) * H * nb * kQbarMaxD * 4;
  return (bytes + 255) / 256 * 256;
}
size_t ws_route_bytes(int B, int H, int L, int block) { return ws_bits_bytes(B, H, L, block) + ws_qbar_bytes(B, H, L, block); }

// ---- workspace in the library's own device memory, for sol_attn_fwd_noalloc -------------------
constexpr int kNoAllocMaxHeads = 4096;  // B * H
// the header of kNoAllocMaxHeads heads, rounded to 256 bytes as ws_header_bytes does (16,640 B)
constexpr size_t kNoAllocBytes = ((static_cast<size_t>(sol::WS_COUNTS) + kNoAllocMaxHeads) * 4 + 255) / 256 * 256;
constexpr size_t kNoAllocWords = kNoAllocBytes / 4;
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
void* g_noalloc_ctx[kMaxDevices] = {};  // the context the address was looked up in

// cuCtxGetCurrent through the runtime's driver entry point (no link-time libcuda).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static std::once_flag once;
  static CtxGetCurrentFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

}  // namespace

// One array per device that loads the library, alive until the process exits. In host code this
// name is only a host-side handle: its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint32_t g_noalloc_ws[kNoAllocWords];

namespace {

// Device address of g_noalloc_ws on the current device. It is looked up once per device and
// context: after a cudaDeviceReset the primary context, and with it the module that holds the
// array, is created anew, so a changed current context triggers a fresh lookup.
sol_status noalloc_workspace(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(SOL_EUNSUPPORTED, "device index %d beyond %d", dev, kMaxDevices);
  CtxGetCurrentFn get_ctx = ctx_get_current_fn();
  if (get_ctx == nullptr) return fail(SOL_ECUDA, "cuCtxGetCurrent is not available from the driver");
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  CUcontext ctx = nullptr;  // null while the runtime has not yet made a context current here
  if (get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
  if (ctx == nullptr || g_noalloc_ptr[dev] == nullptr || g_noalloc_ctx[dev] != static_cast<void*>(ctx)) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_ws);  // makes the device's primary context current if needed
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static workspace)");
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return fail(SOL_ECUDA, "no current CUDA context");
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = static_cast<void*>(ctx);
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

void sol_attn_debug_record_cta_times(unsigned long long* times, int capacity) {
  g_cta_times = capacity > 0 ? times : nullptr;
  g_cta_capacity = capacity > 0 ? capacity : 0;
}

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
  // a row is d / VEC 16-byte vectors (VEC = 8 bf16 or 4 fp32 values); the pool kernel needs that
  // count to be a power of two of at most 32, so the row groups of a warp reduce by shuffles
  const int vecs = d / (bf16 ? 8 : 4);
  if (d % (bf16 ? 8 : 4) != 0 || vecs > 32 || (vecs & (vecs - 1)) != 0)
    return fail(SOL_EUNSUPPORTED, "pool needs d / %d to be a power of two <= 32 (d=%d)", bf16 ? 8 : 4, d);
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

// The QK-norm + RoPE + pooling pass; qbar (optional) receives the query-block means.
static sol_status qknorm_rope_pool_impl(const void* Q, const void* K, const void* V, const float* gain_q,
                                        const float* gain_k, const float* rope_cos, const float* rope_sin, float eps,
                                        int B, int H, int L, int d, int block_k, void* Q_out, void* K_out,
                                        float* kbar, float* vbar, void* kbar_lp, void* vbar_lp, float* qbar,
                                        void* stream) {
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
  // the grid's second dimension runs over groups of 4 key blocks
  if ((static_cast<long long>(L) + block_k - 1) / block_k > 4ll * 65535)
    return fail(SOL_EUNSUPPORTED, "ceil(L / block_k) must be <= %d", 4 * 65535);
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
  a.qbar = qbar;
  a.BH = B * H;
  a.L = L;
  a.d = d;
  a.block = block_k;
  cudaError_t e = sol::launch_qknorm_rope_pool(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "QK-norm + RoPE + pooling launch");
  return SOL_OK;
}

sol_status sol_attn_qknorm_rope_pool(const void* Q, const void* K, const void* V, const float* gain_q,
                                     const float* gain_k, const float* rope_cos, const float* rope_sin, float eps,
                                     int B, int H, int L, int d, int block_k, void* Q_out, void* K_out, float* kbar,
                                     float* vbar, void* kbar_lp, void* vbar_lp, void* stream) {
  return qknorm_rope_pool_impl(Q, K, V, gain_q, gain_k, rope_cos, rope_sin, eps, B, H, L, d, block_k, Q_out, K_out,
                               kbar, vbar, kbar_lp, vbar_lp, nullptr, stream);
}

sol_status sol_attn_qknorm_rope_pool_qbar(const void* Q, const void* K, const void* V, const float* gain_q,
                                          const float* gain_k, const float* rope_cos, const float* rope_sin,
                                          float eps, int B, int H, int L, int d, int block_k, void* Q_out,
                                          void* K_out, float* kbar, float* vbar, void* kbar_lp, void* vbar_lp,
                                          float* qbar, void* stream) {
  if (qbar == nullptr || !aligned16(qbar)) {
    g_last_error.clear();
    return fail(SOL_EINVAL, "qbar must be a non-null, 16-byte aligned device pointer");
  }
  return qknorm_rope_pool_impl(Q, K, V, gain_q, gain_k, rope_cos, rope_sin, eps, B, H, L, d, block_k, Q_out, K_out,
                               kbar, vbar, kbar_lp, vbar_lp, qbar, stream);
}

sol_status sol_attn_quantize_qk8(const void* Q, const void* K, const float* kbar, int B, int H, int L, int d,
                                 int8_t* q8, int8_t* k8, int8_t* kbar8, float* q_scale, float* k_scale,
                                 float* kbar_scale, float* mu, void* stream) {
  g_last_error.clear();
  if (!size_ok(B, 1 << 16) || !size_ok(H, 1 << 16) || !size_ok(L, 1 << 28) || !size_ok(d, 1 << 16))
    return fail(SOL_EINVAL, "sizes must be positive (B=%d H=%d L=%d d=%d)", B, H, L, d);
  const void* ptrs[] = {Q, K, kbar, q8, k8, kbar8, q_scale, k_scale, kbar_scale, mu};
  for (const void* ptr : ptrs) {
    if (ptr == nullptr) return fail(SOL_EINVAL, "every pointer argument must be non-null");
    if (!aligned16(ptr)) return fail(SOL_EINVAL, "device pointers must be 16-byte aligned");
  }
  if (d != 64 && d != 128) return fail(SOL_EUNSUPPORTED, "8-bit operands need d in {64, 128} (d=%d)", d);
  if (static_cast<long long>(B) * H > 65535) return fail(SOL_EUNSUPPORTED, "B*H must be <= 65535");
  const long long nkb = (static_cast<long long>(L) + 127) / 128;
  if (nkb > sol::kMaxKeyBlocks) return fail(SOL_EUNSUPPORTED, "N_kb=%lld exceeds %d", nkb, sol::kMaxKeyBlocks);
  int sms = 0;
  sol_status st = current_device(&sms);
  if (st != SOL_OK) return st;
  sol::QuantArgs a;
  a.Q = Q;
  a.K = K;
  a.kbar = kbar;
  a.mu = mu;
  a.q8 = q8;
  a.k8 = k8;
  a.kb8 = kbar8;
  a.q_scale = q_scale;
  a.k_scale = k_scale;
  a.kb_scale = kbar_scale;
  a.BH = B * H;
  a.L = L;
  a.d = d;
  cudaError_t e = sol::launch_quant_qk8(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "8-bit quantization launch");
  return SOL_OK;
}

size_t sol_attn_fwd_workspace_bytes(int B, int H, int L, int block_q) {
  if (B < 1 || H < 1 || L < 1 || block_q < 1) return 0;
  return ws_header_bytes(B, H) + ws_route_bytes(B, H, L, block_q);
}

}  // extern "C"

namespace {

// The forward of sol_attn_fwd; k_keep > 0 selects fixed-sparsity routing in the routing pass.
sol_status fwd_impl(const void* Q, const void* K, const void* V, const float* kbar, const float* vbar,
                    const void* kbar_lp, const void* vbar_lp, const float* tau, sol_dtype dt, int B, int H, int L,
                    int d, int block_q, int block_k, int n_force, void* O, uint8_t* kept_mask, float* density,
                    void* workspace, size_t ws_bytes, void* stream, int k_keep,
                    const sol::Qk8Operands* qk8 = nullptr, const float* qbar_in = nullptr,
                    const sol::Pv8Operands* pv8 = nullptr) {
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
  // a workspace that also holds the keep bits and the query-block means gets the separate
  // routing pass (bf16 path)
  const bool route_pass = bf16 && ws_bytes >= need + ws_route_bytes(B, H, L, block_q);

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
  a.route_qbar = route_pass ? reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + need +
                                                       ws_bits_bytes(B, H, L, block_q))
                            : nullptr;
  a.k_keep = k_keep;

  if (bf16) {
    a.drop_one_load = g_drop_one_load;
    if (g_drop_one_load) a.wait_limit_ns = 200000000ull;
    g_drop_one_load = 0;
    a.cta_times = g_cta_times;
    a.cta_capacity = g_cta_capacity;
    g_cta_times = nullptr;
    g_cta_capacity = 0;
    CUtensorMap maps[5];
    const int nkb_i = static_cast<int>(nkb);
    const bool i8 = qk8 != nullptr;  // Q, K and the pooled keys as int8 codes
    if ((st = make_map(&maps[0], i8 ? qk8->q8 : Q, d, L, B * H, i8)) != SOL_OK) return st;
    if ((st = make_map(&maps[1], i8 ? qk8->k8 : K, d, L, B * H, i8)) != SOL_OK) return st;
    if (pv8 != nullptr) {
      // E4M3 codes stored transposed: rows are the d channels, the inner extent runs over keys
      // (N_kb * 128) or pooled blocks (128 * ceil(N_kb / 128))
      const int cp = (nkb_i + 127) / 128 * 128;
      if ((st = make_map(&maps[2], pv8->v8t, nkb_i * 128, d, B * H, true)) != SOL_OK) return st;
      if ((st = make_map(&maps[4], pv8->vb8t, cp, d, B * H, true)) != SOL_OK) return st;
    } else {
      if ((st = make_map(&maps[2], V, d, L, B * H)) != SOL_OK) return st;
      if ((st = make_map(&maps[4], vbar_lp, d, nkb_i, B * H)) != SOL_OK) return st;
    }
    if ((st = make_map(&maps[3], i8 ? qk8->kb8 : kbar_lp, d, nkb_i, B * H, i8)) != SOL_OK) return st;
    a.qk8 = qk8;
    a.pv8 = pv8;
    a.qbar_in = route_pass ? qbar_in : nullptr;
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

}  // namespace

extern "C" {

sol_status sol_attn_fwd(const void* Q, const void* K, const void* V, const float* kbar, const float* vbar,
                        const void* kbar_lp, const void* vbar_lp, const float* tau, sol_dtype dt, int B, int H, int L,
                        int d, int block_q, int block_k, int n_force, void* O, uint8_t* kept_mask, float* density,
                        void* workspace, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  return fwd_impl(Q, K, V, kbar, vbar, kbar_lp, vbar_lp, tau, dt, B, H, L, d, block_q, block_k, n_force, O, kept_mask,
                  density, workspace, ws_bytes, stream, 0);
}

sol_status sol_attn_fwd_topk(const void* Q, const void* K, const void* V, const float* kbar, const void* kbar_lp,
                             const void* vbar_lp, int k_keep, int B, int H, int L, int d, int n_force, void* O,
                             uint8_t* kept_mask, float* density, void* workspace, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (B < 1 || H < 1 || L < 1) return fail(SOL_EINVAL, "sizes must be positive (B=%d H=%d L=%d)", B, H, L);
  if (H > sol::kMaxHeads) return fail(SOL_EUNSUPPORTED, "H=%d exceeds %d", H, sol::kMaxHeads);
  const long long nkb = (static_cast<long long>(L) + 127) / 128;
  if (k_keep < 1 || k_keep > nkb) return fail(SOL_EINVAL, "k_keep=%d must be in [1, N_kb=%lld]", k_keep, nkb);
  if (workspace == nullptr || ws_bytes < sol_attn_fwd_workspace_bytes(B, H, L, 128))
    return fail(SOL_EINVAL, "fixed-sparsity routing needs the full workspace (keep bits)");
  float zeros[sol::kMaxHeads] = {};  // unused by the routing pass in this mode; valid thresholds
  return fwd_impl(Q, K, V, kbar, nullptr, kbar_lp, vbar_lp, zeros, SOL_BF16, B, H, L, d, 128, 128, n_force, O,
                  kept_mask, density, workspace, ws_bytes, stream, k_keep);
}

sol_status sol_attn_fwd_qbar(const void* Q, const void* K, const void* V, const float* kbar, const float* vbar,
                             const void* kbar_lp, const void* vbar_lp, const float* qbar, const float* tau, int B,
                             int H, int L, int d, int n_force, void* O, uint8_t* kept_mask, float* density,
                             void* workspace, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (B < 1 || H < 1 || L < 1) return fail(SOL_EINVAL, "sizes must be positive (B=%d H=%d L=%d)", B, H, L);
  if (qbar == nullptr || !aligned16(qbar)) return fail(SOL_EINVAL, "qbar must be a non-null, 16-byte aligned device pointer");
  if (workspace == nullptr || ws_bytes < sol_attn_fwd_workspace_bytes(B, H, L, 128))
    return fail(SOL_EINVAL, "the given query-block means feed the routing pass, which needs the full workspace");
  return fwd_impl(Q, K, V, kbar, vbar, kbar_lp, vbar_lp, tau, SOL_BF16, B, H, L, d, 128, 128, n_force, O, kept_mask,
                  density, workspace, ws_bytes, stream, 0, nullptr, qbar);
}

sol_status sol_attn_fwd_qk8(const void* Q, const int8_t* q8, const int8_t* k8, const int8_t* kbar8,
                            const float* q_scale, const float* k_scale, const float* kbar_scale, const void* V,
                            const float* kbar, const void* vbar_lp, const float* tau, int B, int H, int L, int d,
                            int n_force, void* O, uint8_t* kept_mask, float* density, void* workspace,
                            size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (B < 1 || H < 1 || L < 1) return fail(SOL_EINVAL, "sizes must be positive (B=%d H=%d L=%d)", B, H, L);
  const void* ptrs[] = {q8, k8, kbar8, q_scale, k_scale, kbar_scale};
  for (const void* ptr : ptrs) {
    if (ptr == nullptr) return fail(SOL_EINVAL, "every 8-bit operand and scale must be non-null");
    if (!aligned16(ptr)) return fail(SOL_EINVAL, "device pointers must be 16-byte aligned");
  }
  if (d != 128) return fail(SOL_EUNSUPPORTED, "8-bit QK^T needs d = 128 (d=%d)", d);
  if (workspace == nullptr || ws_bytes < sol_attn_fwd_workspace_bytes(B, H, L, 128))
    return fail(SOL_EINVAL, "8-bit QK^T needs the full workspace (its routing pass reads the bf16 Q)");
  sol::Qk8Operands ops{q8, k8, kbar8, q_scale, k_scale, kbar_scale};
  // K is not read on this path; k8 stands in for it in the argument checks
  return fwd_impl(Q, k8, V, kbar, nullptr, vbar_lp, vbar_lp, tau, SOL_BF16, B, H, L, d, 128, 128, n_force, O,
                  kept_mask, density, workspace, ws_bytes, stream, 0, &ops);
}

sol_status sol_attn_quantize_v8(const void* V, const float* vbar, int B, int H, int L, int d, uint8_t* v8t,
                                uint8_t* vbar8t, float* v_scale, void* stream) {
  g_last_error.clear();
  if (!size_ok(B, 1 << 16) || !size_ok(H, 1 << 16) || !size_ok(L, 1 << 28) || !size_ok(d, 1 << 16))
    return fail(SOL_EINVAL, "sizes must be positive (B=%d H=%d L=%d d=%d)", B, H, L, d);
  const void* ptrs[] = {V, vbar, v8t, vbar8t, v_scale};
  for (const void* ptr : ptrs) {
    if (ptr == nullptr) return fail(SOL_EINVAL, "every pointer argument must be non-null");
    if (!aligned16(ptr)) return fail(SOL_EINVAL, "device pointers must be 16-byte aligned");
  }
  if (d != 128) return fail(SOL_EUNSUPPORTED, "8-bit PV values need d = 128 (d=%d)", d);
  if (static_cast<long long>(B) * H > 65535) return fail(SOL_EUNSUPPORTED, "B*H must be <= 65535");
  const long long nkb = (static_cast<long long>(L) + 127) / 128;
  if (nkb > sol::kMaxKeyBlocks) return fail(SOL_EUNSUPPORTED, "N_kb=%lld exceeds %d", nkb, sol::kMaxKeyBlocks);
  int sms = 0;
  sol_status st = current_device(&sms);
  if (st != SOL_OK) return st;
  sol::QuantV8Args a;
  a.V = V;
  a.vbar = vbar;
  a.v8t = v8t;
  a.vb8t = vbar8t;
  a.v_scale = v_scale;
  a.BH = B * H;
  a.L = L;
  a.d = d;
  cudaError_t e = sol::launch_quant_v8(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "8-bit value quantization launch");
  return SOL_OK;
}

sol_status sol_attn_fwd_8bit(const void* Q, const int8_t* q8, const int8_t* k8, const int8_t* kbar8,
                             const float* q_scale, const float* k_scale, const float* kbar_scale, const uint8_t* v8t,
                             const uint8_t* vbar8t, const float* v_scale, const float* kbar, const float* tau, int B,
                             int H, int L, int d, int n_force, void* O, uint8_t* kept_mask, float* density,
                             void* workspace, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (B < 1 || H < 1 || L < 1) return fail(SOL_EINVAL, "sizes must be positive (B=%d H=%d L=%d)", B, H, L);
  const void* ptrs[] = {q8, k8, kbar8, q_scale, k_scale, kbar_scale, v8t, vbar8t, v_scale};
  for (const void* ptr : ptrs) {
    if (ptr == nullptr) return fail(SOL_EINVAL, "every 8-bit operand and scale must be non-null");
    if (!aligned16(ptr)) return fail(SOL_EINVAL, "device pointers must be 16-byte aligned");
  }
  if (d != 128) return fail(SOL_EUNSUPPORTED, "8-bit attention needs d = 128 (d=%d)", d);
  if (workspace == nullptr || ws_bytes < sol_attn_fwd_workspace_bytes(B, H, L, 128))
    return fail(SOL_EINVAL, "8-bit attention needs the full workspace (its routing pass reads the bf16 Q)");
  sol::Qk8Operands qk{q8, k8, kbar8, q_scale, k_scale, kbar_scale};
  sol::Pv8Operands pv{v8t, vbar8t, v_scale};
  // K, V and the bf16 pooled values are not read on this path; 8-bit operands stand in for them
  // in the argument checks
  return fwd_impl(Q, k8, v8t, kbar, nullptr, vbar8t, vbar8t, tau, SOL_BF16, B, H, L, d, 128, 128, n_force, O,
                  kept_mask, density, workspace, ws_bytes, stream, 0, &qk, nullptr, &pv);
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
  const size_t bytes = kNoAllocBytes;
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

// ---- host-buffer entry point: head chunks pipelined through caller-provided device scratch ------
namespace {

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// Where each buffer of sol_attn_fwd_host lives inside the scratch (byte offsets from its base).
// Two slots of Q, K, V and O chunks, so that a chunk's upload, the previous chunk's compute and
// the one before's download run at once. One set of pooled vectors and one workspace: the
// compute of consecutive chunks is ordered on one stream.
struct HostPlan {
  int c = 0;                 // heads per chunk
  size_t chunk_bytes = 0;    // one chunk of Q, K, V or O: c * L * d * element size
  size_t in[2][3] = {};      // Q, K, V of slot 0 and 1
  size_t out[2] = {};        // O of slot 0 and 1
  size_t kbar = 0, vbar = 0, kbar_lp = 0, vbar_lp = 0;
  size_t ws = 0, ws_bytes = 0;
  size_t dens = 0;           // float32 [B * H]
  size_t total = 0;
};

HostPlan host_plan(bool bf16, int B, int H, int L, int d, int block, int heads_per_chunk) {
  HostPlan p;
  p.c = heads_per_chunk < H ? heads_per_chunk : H;
  const size_t es = bf16 ? 2 : 4;
  const size_t nkb = (static_cast<size_t>(L) + block - 1) / block;
  p.chunk_bytes = static_cast<size_t>(p.c) * L * d * es;
  const size_t slot = round256(p.chunk_bytes);
  size_t off = 0;
  for (int s = 0; s < 2; ++s) {
    for (int t = 0; t < 3; ++t) {
      p.in[s][t] = off;
      off += slot;
    }
    p.out[s] = off;
    off += slot;
  }
  const size_t pooled_f32 = round256(static_cast<size_t>(p.c) * nkb * d * 4);
  const size_t pooled_lp = bf16 ? round256(static_cast<size_t>(p.c) * nkb * d * 2) : 0;
  p.kbar = off;
  off += pooled_f32;
  p.vbar = off;
  off += pooled_f32;
  p.kbar_lp = off;
  off += pooled_lp;
  p.vbar_lp = off;
  off += pooled_lp;
  p.ws = off;
  p.ws_bytes = round256(ws_header_bytes(1, p.c) + ws_route_bytes(1, p.c, L, block));
  off += p.ws_bytes;
  p.dens = off;
  off += round256(static_cast<size_t>(B) * H * 4);
  p.total = off;
  return p;
}

// The checks of sol_attn_fwd that depend only on sizes, made once for the whole call so that a
// bad argument is reported before any chunk is uploaded.
sol_status host_validate(const void* Q, const void* K, const void* V, void* O, const float* tau, sol_dtype dt, int B,
                         int H, int L, int d, int block, int n_force, int heads_per_chunk, const void* scratch) {
  if (dt != SOL_F32 && dt != SOL_BF16) return fail(SOL_EINVAL, "unknown dtype %d", static_cast<int>(dt));
  if (!size_ok(B, 1 << 16) || !size_ok(H, 1 << 16) || !size_ok(L, 1 << 28) || !size_ok(d, 1 << 16) ||
      !size_ok(block, 1 << 20))
    return fail(SOL_EINVAL, "sizes must be positive (B=%d H=%d L=%d d=%d block=%d)", B, H, L, d, block);
  if (heads_per_chunk < 1) return fail(SOL_EINVAL, "heads_per_chunk=%d must be >= 1", heads_per_chunk);
  if (Q == nullptr || K == nullptr || V == nullptr || O == nullptr || tau == nullptr || scratch == nullptr)
    return fail(SOL_EINVAL, "Q, K, V, O, tau and scratch must be non-null");
  if ((reinterpret_cast<uintptr_t>(scratch) & 255u) != 0) return fail(SOL_EINVAL, "scratch must be 256-byte aligned");
  for (int h = 0; h < H; ++h)
    if (std::isnan(tau[h]) || tau[h] < 0.f) return fail(SOL_EINVAL, "tau[%d]=%g must be >= 0 and not NaN", h, tau[h]);
  if (dt == SOL_BF16) {
    if (block != 128 || (d != 64 && d != 128))
      return fail(SOL_EUNSUPPORTED, "bf16 path needs block 128 and d in {64, 128} (block=%d d=%d)", block, d);
  } else {
    if ((block != 32 && block != 64 && block != 128) || (d != 32 && d != 64 && d != 128))
      return fail(SOL_EUNSUPPORTED, "fp32 path needs block in {32,64,128} and d in {32,64,128} (block=%d d=%d)",
                  block, d);
  }
  const long long nkb = (static_cast<long long>(L) + block - 1) / block;
  if (nkb > sol::kMaxKeyBlocks) return fail(SOL_EUNSUPPORTED, "N_kb=%lld exceeds %d", nkb, sol::kMaxKeyBlocks);
  if (n_force < 0 || n_force > nkb) return fail(SOL_EINVAL, "n_force=%d must be in [0, N_kb=%lld]", n_force, nkb);
  const int c = heads_per_chunk < H ? heads_per_chunk : H;
  if (c > sol::kMaxHeads) return fail(SOL_EUNSUPPORTED, "heads_per_chunk=%d exceeds %d", c, sol::kMaxHeads);
  if (static_cast<long long>(c) * nkb >= (1ll << 31)) return fail(SOL_EUNSUPPORTED, "chunk too large");
  return SOL_OK;
}

// Q, K, V, O must not be device memory; the scratch must be device memory of the current device.
sol_status host_check_memory(const void* const* host_ptrs, int n, const void* scratch) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  for (int i = 0; i < n; ++i) {
    cudaPointerAttributes at;
    e = cudaPointerGetAttributes(&at, host_ptrs[i]);
    if (e != cudaSuccess) return cuda_fail(e, "cudaPointerGetAttributes");
    if (at.type == cudaMemoryTypeDevice) return fail(SOL_EINVAL, "Q, K, V and O must be host memory");
  }
  cudaPointerAttributes at;
  e = cudaPointerGetAttributes(&at, scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaPointerGetAttributes");
  if (at.type != cudaMemoryTypeDevice || at.device != dev)
    return fail(SOL_EINVAL, "scratch must be device memory of the current device");
  return SOL_OK;
}

}  // namespace

extern "C" {

size_t sol_attn_fwd_host_scratch_bytes(sol_dtype dt, int B, int H, int L, int d, int block, int heads_per_chunk) {
  if ((dt != SOL_F32 && dt != SOL_BF16) || B < 1 || H < 1 || L < 1 || d < 1 || block < 1 || heads_per_chunk < 1)
    return 0;
  return host_plan(dt == SOL_BF16, B, H, L, d, block, heads_per_chunk).total;
}

sol_status sol_attn_fwd_host(const void* Q, const void* K, const void* V, void* O, const float* tau, sol_dtype dt,
                             int B, int H, int L, int d, int block, int n_force, int heads_per_chunk, float* density,
                             void* scratch, size_t scratch_bytes, void* stream) {
  g_last_error.clear();
  sol_status st = host_validate(Q, K, V, O, tau, dt, B, H, L, d, block, n_force, heads_per_chunk, scratch);
  if (st != SOL_OK) return st;
  const bool bf16 = dt == SOL_BF16;
  const HostPlan pl = host_plan(bf16, B, H, L, d, block, heads_per_chunk);
  if (scratch_bytes < pl.total) return fail(SOL_EINVAL, "scratch too small (%zu < %zu bytes)", scratch_bytes, pl.total);
  const void* host_ptrs[4] = {Q, K, V, O};
  if ((st = host_check_memory(host_ptrs, 4, scratch)) != SOL_OK) return st;
  int sms = 0;
  if ((st = current_device(&sms)) != SOL_OK) return st;

  uint8_t* base = static_cast<uint8_t*>(scratch);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t s_in = nullptr, s_out = nullptr;
  constexpr int kEvents = 7;  // start, uploaded[2], computed[2], downloaded[2]
  cudaEvent_t ev[kEvents] = {};
  cudaEvent_t& ev_start = ev[0];
  cudaEvent_t* ev_in = &ev[1];
  cudaEvent_t* ev_comp = &ev[3];
  cudaEvent_t* ev_out = &ev[5];
  cudaError_t e = cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking);
  for (int i = 0; i < kEvents && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming);
  if (e != cudaSuccess) st = cuda_fail(e, "stream / event creation");

  // a clean workspace (its sticky error word too), then both copy streams start after `stream`'s
  // earlier work, so a previous call on the same scratch has finished with it
  if (st == SOL_OK && (e = cudaMemsetAsync(base + pl.ws, 0, pl.ws_bytes, s)) != cudaSuccess)
    st = cuda_fail(e, "cudaMemsetAsync(workspace)");
  if (st == SOL_OK && ((e = cudaEventRecord(ev_start, s)) != cudaSuccess ||
                       (e = cudaStreamWaitEvent(s_in, ev_start, 0)) != cudaSuccess ||
                       (e = cudaStreamWaitEvent(s_out, ev_start, 0)) != cudaSuccess))
    st = cuda_fail(e, "stream ordering");

  const uint8_t* hq = static_cast<const uint8_t*>(Q);
  const uint8_t* hk = static_cast<const uint8_t*>(K);
  const uint8_t* hv = static_cast<const uint8_t*>(V);
  uint8_t* ho = static_cast<uint8_t*>(O);
  const size_t head_bytes = static_cast<size_t>(L) * d * (bf16 ? 2 : 4);
  float* dens_dev = reinterpret_cast<float*>(base + pl.dens);
  int chunk = 0;
  for (int b = 0; b < B && st == SOL_OK; ++b) {
    for (int h0 = 0; h0 < H && st == SOL_OK; h0 += pl.c, ++chunk) {
      const int ce = (H - h0) < pl.c ? (H - h0) : pl.c;
      const int sl = chunk & 1;
      const size_t host_off = (static_cast<size_t>(b) * H + h0) * head_bytes;
      const size_t bytes = static_cast<size_t>(ce) * head_bytes;  // <= pl.chunk_bytes
      uint8_t* dq = base + pl.in[sl][0];
      uint8_t* dk = base + pl.in[sl][1];
      uint8_t* dv = base + pl.in[sl][2];
      uint8_t* dout = base + pl.out[sl];
      // upload: the slot's inputs are free once the compute of chunk - 2 has finished
      if (chunk >= 2 && (e = cudaStreamWaitEvent(s_in, ev_comp[sl], 0)) != cudaSuccess) {
        st = cuda_fail(e, "stream ordering");
        break;
      }
      if ((e = cudaMemcpyAsync(dq, hq + host_off, bytes, cudaMemcpyHostToDevice, s_in)) != cudaSuccess ||
          (e = cudaMemcpyAsync(dk, hk + host_off, bytes, cudaMemcpyHostToDevice, s_in)) != cudaSuccess ||
          (e = cudaMemcpyAsync(dv, hv + host_off, bytes, cudaMemcpyHostToDevice, s_in)) != cudaSuccess ||
          (e = cudaEventRecord(ev_in[sl], s_in)) != cudaSuccess) {
        st = cuda_fail(e, "upload");
        break;
      }
      // compute: after this chunk's upload, and after the download of chunk - 2 freed the O slot
      if ((e = cudaStreamWaitEvent(s, ev_in[sl], 0)) != cudaSuccess ||
          (chunk >= 2 && (e = cudaStreamWaitEvent(s, ev_out[sl], 0)) != cudaSuccess)) {
        st = cuda_fail(e, "stream ordering");
        break;
      }
      float* kbar = reinterpret_cast<float*>(base + pl.kbar);
      float* vbar = reinterpret_cast<float*>(base + pl.vbar);
      void* klp = bf16 ? static_cast<void*>(base + pl.kbar_lp) : nullptr;
      void* vlp = bf16 ? static_cast<void*>(base + pl.vbar_lp) : nullptr;
      st = sol_attn_pool(dk, dv, dt, 1, ce, L, d, block, kbar, vbar, klp, vlp, stream);
      if (st != SOL_OK) break;
      st = sol_attn_fwd(dq, dk, dv, kbar, vbar, klp, vlp, tau + h0, dt, 1, ce, L, d, block, block, n_force, dout,
                        nullptr, density != nullptr ? dens_dev + static_cast<size_t>(b) * H + h0 : nullptr,
                        base + pl.ws, pl.ws_bytes, stream);
      if (st != SOL_OK) break;
      if ((e = cudaEventRecord(ev_comp[sl], s)) != cudaSuccess) {
        st = cuda_fail(e, "stream ordering");
        break;
      }
      // download
      if ((e = cudaStreamWaitEvent(s_out, ev_comp[sl], 0)) != cudaSuccess ||
          (e = cudaMemcpyAsync(ho + host_off, dout, bytes, cudaMemcpyDeviceToHost, s_out)) != cudaSuccess ||
          (e = cudaEventRecord(ev_out[sl], s_out)) != cudaSuccess) {
        st = cuda_fail(e, "download");
        break;
      }
    }
  }
  if (st == SOL_OK && density != nullptr &&
      (e = cudaMemcpyAsync(density, dens_dev, static_cast<size_t>(B) * H * 4, cudaMemcpyDeviceToHost, s)) !=
          cudaSuccess)
    st = cuda_fail(e, "density download");

  // whatever happened above, nothing may still be copying into the caller's buffers on return
  cudaError_t es = cudaSuccess;
  if (s_in != nullptr && (e = cudaStreamSynchronize(s_in)) != cudaSuccess) es = e;
  if (s_out != nullptr && (e = cudaStreamSynchronize(s_out)) != cudaSuccess) es = e;
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) es = e;
  for (int i = 0; i < kEvents; ++i)
    if (ev[i] != nullptr) cudaEventDestroy(ev[i]);
  if (s_in != nullptr) cudaStreamDestroy(s_in);
  if (s_out != nullptr) cudaStreamDestroy(s_out);
  if (st != SOL_OK) return st;  // its reason is already in the last-error string
  if (es != cudaSuccess) return cuda_fail(es, "cudaStreamSynchronize");
  uint32_t words[2] = {0, 0};
  if ((e = cudaMemcpy(words, base + pl.ws, sizeof(words), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return cuda_fail(e, "cudaMemcpy(error word)");
  if (words[0] != 0) {
    static const char* roles[] = {"?", "producer", "mma", "softmax", "router"};
    return fail(SOL_ETIMEOUT, "device wait expired (first in the %s role); the outputs are incomplete",
                roles[words[1] < 5 ? words[1] : 0]);
  }
  return SOL_OK;
}

}  // extern "C"
