/*
 * sol_attn.h -- C ABI of the Sol-Attn block-sparse attention forward for NVIDIA B200 (sm_100a).
 *
 * The operation: Sol-Attn project page ("Sol-Attn: Accelerating Video Generation Inference via
 * On-the-Fly Attention Sparsification"), Abstract. One online-softmax pass does three things:
 * it routes each query block to key blocks by a query-dependent threshold, selected on chip
 * from a proxy score that is never written to memory; it runs exact attention on the kept
 * blocks; and it adds an approximate correction for the skipped blocks. The Sol-Engine README,
 * section "Sol-Attention", says the same: only the most relevant key blocks are computed, and
 * a light compensating term covers the rest.
 *
 * Definition used (the pages give no formula; the CPU oracle follows the same one):
 *   k_bar_j, v_bar_j = mean of K, V over the n_j valid tokens of key block j
 *   q_bar_i          = mean of the valid query rows of query block i
 *   s_bar_ij         = q_bar_i . k_bar_j / sqrt(d); keep j iff s_bar_ij >= max_j s_bar_ij - tau[h]
 *                      or j < n_force
 *   kept block       : exact logits q . k_t / sqrt(d), values v_t
 *   skipped block    : one logit q . k_bar_j / sqrt(d) with multiplicity n_j, value v_bar_j
 *   all terms of one query row share one softmax; attention is bidirectional (no causal mask).
 *
 * Conventions shared by every call:
 *   - Tensors are dense, contiguous, row-major: [B, H, L, d] for Q, K, V, O (L = valid tokens, no
 *     padding; partial last blocks are masked inside the kernels), [B, H, N_kb, d] for pooled
 *     vectors, with N_kb = ceil(L / block_k) and N_qb = ceil(L / block_q).
 *   - Device pointers must be 16-byte aligned. All device memory and the stream belong to the
 *     caller; the library allocates nothing and keeps no global state (the one exception is the
 *     static device array of sol_attn_fwd_noalloc, described there).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). Every call
 *     that launches work is asynchronous on that stream, except sol_attn_fwd_host, whose host
 *     buffers make it synchronous (described there).
 *   - Arguments are validated on the host before any launch. Invalid ones return SOL_EINVAL,
 *     and shapes or dtypes the kernels do not implement return SOL_EUNSUPPORTED. In both cases
 *     nothing is launched. A failed CUDA runtime call returns SOL_ECUDA.
 *     sol_attn_last_error() gives the reason for the last failure on the calling thread.
 *   - NaN or Inf inside Q, K, V is not checked and gives undefined results.
 */
#ifndef SOL_ATTN_H
#define SOL_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SOL_OK = 0,
    SOL_EINVAL = 1,        /* invalid argument (null pointer, bad size, tau < 0 or NaN, misalignment) */
    SOL_EUNSUPPORTED = 2,  /* valid but not implemented (dtype / head dim / block size combination) */
    SOL_ECUDA = 3,         /* a CUDA runtime call failed (launch, attribute, memset, copy) */
    SOL_ETIMEOUT = 4       /* a bounded on-device wait expired; the kernel returned early (see check call) */
} sol_status;

typedef enum {
    SOL_F32 = 0,  /* float32 inputs and output; SIMT kernel, fp32 arithmetic throughout */
    SOL_BF16 = 1  /* bfloat16 inputs and output; tcgen05 tensor-core kernel, fp32 accumulation */
} sol_dtype;

/* Human-readable name of a status code. Never NULL. */
const char* sol_attn_status_string(sol_status s);

/* Detail of the most recent failing call on this thread ("" if none). Never NULL. */
const char* sol_attn_last_error(void);

/* Block pooling (definition of k_bar, v_bar above; Sol-Attn project page, Abstract: the routing
 * proxy and the skipped-block correction both read pooled block vectors).
 *
 *   K, V      device, [B, H, L, d] in dtype `dt`
 *   kbar,vbar device, float32 [B, H, N_kb, d]: mean over the n_j = min(block_k, L - j*block_k)
 *             valid tokens of block j, summed in fp32
 *   kbar_lp,  device, bfloat16 [B, H, N_kb, d]: the same means rounded to bf16 (nearest even),
 *   vbar_lp   the operands of the tensor-core correction tiles. Required when dt == SOL_BF16,
 *             must be NULL when dt == SOL_F32.
 * Supported: d / 8 (SOL_BF16) or d / 4 (SOL_F32) a power of two <= 32, i.e. d in {8, ..., 256} or
 * {4, ..., 128}; 1 <= block_k <= 4096.
 */
sol_status sol_attn_pool(const void* K, const void* V, sol_dtype dt, int B, int H, int L, int d,
                         int block_k, float* kbar, float* vbar, void* kbar_lp, void* vbar_lp,
                         void* stream);

/* QK RMS norm + rotary embedding + block pooling in one pass: the step before the attention,
 * which kernel fusion folds together (Sol-Engine README, "The five acceleration methods", kernel
 * fusion of QK-norm + RoPE). The pages print no formula; this is the textbook form. For each
 * (b, h) and token t, and for Q with gain_q and K with gain_k:
 *   y  = x / sqrt(mean_c x_c^2 + eps) * gain          (RMS norm over the d head channels)
 *   y' = each interleaved pair (y_2i, y_2i+1) turned by the angle with cosine rope_cos[t, i] and
 *        sine rope_sin[t, i]:  (y_2i c - y_2i+1 s,  y_2i s + y_2i+1 c)
 * y' goes to Q_out / K_out (bf16, nearest even). In the same pass, kbar/vbar (and their bf16
 * mirrors) receive the block means of the STORED keys (after rounding) and of V. These are the
 * same quantities sol_attn_pool computes from K_out and V, up to fp32 summation order. So K_out is
 * not read back by a separate pooling pass.
 *
 *   Q, K, V          device, bf16 [B, H, L, d]
 *   gain_q, gain_k   device, float32 [d]
 *   rope_cos/sin     device, float32 [L, d/2] (the same for every b, h)
 *   eps              > 0
 *   Q_out, K_out     device, bf16 [B, H, L, d]; may be Q and K themselves (in place)
 *   kbar, vbar       device, float32 [B, H, N_kb, d];  kbar_lp, vbar_lp: bf16 mirrors
 * Supported: d in {64, 128}, 1 <= block_k <= 4096, B*H <= 65535. All pointers non-null and
 * 16-byte aligned (else SOL_EINVAL). */
sol_status sol_attn_qknorm_rope_pool(const void* Q, const void* K, const void* V, const float* gain_q,
                                     const float* gain_k, const float* rope_cos, const float* rope_sin,
                                     float eps, int B, int H, int L, int d, int block_k, void* Q_out,
                                     void* K_out, float* kbar, float* vbar, void* kbar_lp, void* vbar_lp,
                                     void* stream);

/* The same pass, also writing the query-block means the routing proxy needs (NEXT-1: the pages'
 * "fused QK+RoPE" folds the pooling of Q into the pass that stores Q):
 *   qbar   device, out, float32 [B, H, N_kb, d]: for each block of block_k rows, the mean of the
 *          STORED (bf16-rounded) query rows Q_out, over the block's valid rows
 * Pass it to sol_attn_fwd_qbar with block_k = 128, and the routing pass does not read Q again.
 * Other arguments, limits and errors as for sol_attn_qknorm_rope_pool; qbar non-null and 16-byte
 * aligned, else SOL_EINVAL. */
sol_status sol_attn_qknorm_rope_pool_qbar(const void* Q, const void* K, const void* V,
                                          const float* gain_q, const float* gain_k,
                                          const float* rope_cos, const float* rope_sin, float eps, int B,
                                          int H, int L, int d, int block_k, void* Q_out, void* K_out,
                                          float* kbar, float* vbar, void* kbar_lp, void* vbar_lp,
                                          float* qbar, void* stream);

/* 8-bit operands of QK^T for sol_attn_fwd_qk8 (NEXT-2: the review page of the Sol Video Inference
 * Engine paper lists SageAttention's 8-bit attention with outlier smoothing; the Sol-Engine README
 * news reports fused 8-bit compute). From Q, K (bf16 [B, H, L, d]) and the fp32 pooled keys kbar
 * of sol_attn_pool, with blocks of 128:
 *   mu          device, out, float32 [B, H, d]: the head's mean key, sum_j n_j kbar_j / L
 *   q8          device, out, int8 [B, H, L, d]: Q, one scale per 128-row query block
 *   k8          device, out, int8 [B, H, L, d]: K - mu, one scale per key block
 *   kbar8       device, out, int8 [B, H, N_kb, d]: kbar - mu, one scale per chunk of 128 pooled keys
 *   q_scale     device, out, float32 [B, H, N_qb];  k_scale [B, H, N_kb];  kbar_scale
 *               [B, H, ceil(N_kb / 128)]: amax / 127 of each tile (1 for an all-zero tile)
 * A code is the fp32 round-to-nearest-even of x * 127 / amax, clamped to [-127, 127]. Subtracting
 * mu shifts every logit of a query row by the same amount, so in exact arithmetic it changes
 * nothing; it keeps a common key offset out of the 8-bit range (SageAttention's smoothing).
 * Errors, checked on the host before any launch: a non-positive size, a null or not 16-byte
 * aligned pointer -> SOL_EINVAL; d not in {64, 128}, B*H > 65535 or N_kb > 4096 ->
 * SOL_EUNSUPPORTED; a failed launch -> SOL_ECUDA. Asynchronous on `stream`. */
sol_status sol_attn_quantize_qk8(const void* Q, const void* K, const float* kbar, int B, int H, int L,
                                 int d, int8_t* q8, int8_t* k8, int8_t* kbar8, float* q_scale,
                                 float* k_scale, float* kbar_scale, float* mu, void* stream);

/* 8-bit values for PV (NEXT-2, the "e4m3_channel" reading of SageAttention's FP8 PV: V in E4M3
 * with one scale per channel). From V (bf16 [B, H, L, d]) and the fp32 pooled values vbar of
 * sol_attn_pool, with blocks of 128:
 *   v_scale   device, out, float32 [B, H, d]: amax_c / 448 of each channel over the head's L
 *             tokens (1 for an all-zero channel)
 *   v8t       device, out, uint8 (E4M3 codes) [B, H, d, N_kb * 128]: E4M3(V[t, c] / v_scale[c]),
 *             round to nearest even, saturating; transposed (tokens contiguous), 0 past L
 *   vbar8t    device, out, uint8 (E4M3 codes) [B, H, d, 128 * ceil(N_kb / 128)]: vbar with the same
 *             channel scales, transposed, 0 past N_kb
 * Errors, checked on the host before any launch: a non-positive size, a null or not 16-byte
 * aligned pointer -> SOL_EINVAL; d != 128, B*H > 65535 or N_kb > 4096 -> SOL_EUNSUPPORTED; a
 * failed launch -> SOL_ECUDA. Asynchronous on `stream`; v_scale doubles as the per-channel maximum
 * while the pass runs. */
sol_status sol_attn_quantize_v8(const void* V, const float* vbar, int B, int H, int L, int d,
                                uint8_t* v8t, uint8_t* vbar8t, float* v_scale, void* stream);

/* The forward with 8-bit kept tiles and correction (NEXT-2): QK^T from the int8 codes of
 * sol_attn_quantize_qk8 (kind::i8), PV from E4M3 weights and the E4M3 values of
 * sol_attn_quantize_v8 (tcgen05 kind::f8f6f4, fp32 accumulation). Each softmax group keeps an
 * integer running maximum m (a lazy rescale when a tile's max passes m + 2 moves it to the
 * ceiling of the new max and scales the accumulator by an exact power of two) and writes
 * P = E4M3(2^(l log2(e) + log2(n_j) - (m - 6))) <= 256, so every weight above 2^-12 of the
 * running max keeps E4M3's mantissa rounding with an exact exponent; the row sum adds those E4M3
 * values; the epilogue multiplies output column c by v_scale[c]. Routing is sol_attn_fwd's (bf16 Q, fp32
 * pooled keys kbar). SOL_BF16 semantics for O, d = 128, blocks of 128, the full workspace of
 * sol_attn_fwd_workspace_bytes. Other arguments, limits and errors as for sol_attn_fwd. */
sol_status sol_attn_fwd_8bit(const void* Q, const int8_t* q8, const int8_t* k8, const int8_t* kbar8,
                             const float* q_scale, const float* k_scale, const float* kbar_scale,
                             const uint8_t* v8t, const uint8_t* vbar8t, const float* v_scale,
                             const float* kbar, const float* tau, int B, int H, int L, int d,
                             int n_force, void* O, uint8_t* kept_mask, float* density, void* workspace,
                             size_t ws_bytes, void* stream);

/* Bytes of device workspace sol_attn_fwd needs for this problem. The workspace holds the
 * persistent scheduler's work counter, the per-(b,h) kept-block counters and the sticky device
 * error word (a header of 4 * (4 + B*H) bytes rounded up to 256), followed by the routing pass's
 * keep bits, B*H*N_qb*ceil(N_kb/32) 32-bit words, and its query-block means, B*H*N_qb*128 floats,
 * each rounded up to 256 bytes (1.8 MB + 12.1 MB for B=1, H=40, L=75600, block 128). Zero it once
 * after allocation; later calls keep it consistent. */
size_t sol_attn_fwd_workspace_bytes(int B, int H, int L, int block_q);

/* The forward: routing, exact attention on kept blocks, skipped-block correction and the epilogue
 * (Sol-Attn project page, Abstract). For SOL_BF16 with a workspace of the full size returned above,
 * routing runs as its own pass first. One kernel streams Q once and writes the query-block means
 * q_bar into the workspace; a second routes 4-16 query blocks of one head per CTA, so each head's
 * pooled keys are read once per group of query blocks instead of once per block, and writes only
 * the keep bits into the workspace. The fused kernel then turns them into its tile lists. With a workspace that holds only the header, the fused kernel routes each query block
 * itself, with the same fp32 arithmetic in the same order, so both paths keep the same blocks.
 *
 *   Q, K, V     device, [B, H, L, d] in dtype `dt`
 *   kbar        device, float32 [B, H, N_kb, d] from sol_attn_pool: the routing proxy
 *   vbar        device, float32 [B, H, N_kb, d]: correction values for SOL_F32; may be NULL for
 *               SOL_BF16
 *   kbar_lp,    device, bf16 [B, H, N_kb, d] from sol_attn_pool: correction operands for
 *   vbar_lp     SOL_BF16; ignored (may be NULL) for SOL_F32
 *   tau         HOST, float32 [H]: per-head threshold, >= 0. +INFINITY keeps every block
 *               (dense attention). Read during the call; the values travel in the launch.
 *   block_q,    query / key block sizes. SOL_BF16: both 128, d in {64, 128}.
 *   block_k     SOL_F32: equal, in {32, 64, 128}; d in {32, 64, 128}.
 *   n_force     leading key blocks always kept (e.g. text tokens), 0 <= n_force <= N_kb
 *   O           device, [B, H, L, d] in dtype `dt`: the output
 *   kept_mask   device, uint8 [B, H, N_qb, N_kb] or NULL: 1 where block j was kept for query
 *               block i
 *   density     device, float32 [B, H] or NULL: kept blocks / (N_qb * N_kb) per head
 *   workspace   device, zeroed once after allocation: sol_attn_fwd_workspace_bytes(...) bytes, or
 *               at least its header (4 * (4 + B*H) bytes rounded up to 256), which selects routing
 *               inside the fused kernel; smaller returns SOL_EINVAL
 * Limits: H <= 256, N_kb <= 4096, B*H*N_qb < 2^31.
 * The proxy scores s_bar stay in shared memory and are never written to global memory; only the
 * keep bits are.
 */
sol_status sol_attn_fwd(const void* Q, const void* K, const void* V, const float* kbar,
                        const float* vbar, const void* kbar_lp, const void* vbar_lp,
                        const float* tau, sol_dtype dt, int B, int H, int L, int d, int block_q,
                        int block_k, int n_force, void* O, uint8_t* kept_mask, float* density,
                        void* workspace, size_t ws_bytes, void* stream);

/* The forward with fixed-sparsity routing: each query block keeps the k_keep key blocks with the
 * highest proxy scores s_bar_ij (equal scores: the lower block index first), plus the first
 * n_force blocks. The review page of the Sol Video Inference Engine paper names this kind of
 * routing (PISA at sparsity 0.9) beside Sol-Attn's threshold. Exact tiles, correction and outputs
 * are those of sol_attn_fwd. Only SOL_BF16 with blocks of 128 and d in {64, 128} is supported, and
 * the workspace must have the full size of sol_attn_fwd_workspace_bytes (the routing pass writes
 * the keep bits). 1 <= k_keep <= N_kb, else SOL_EINVAL. */
sol_status sol_attn_fwd_topk(const void* Q, const void* K, const void* V, const float* kbar,
                             const void* kbar_lp, const void* vbar_lp, int k_keep, int B, int H, int L,
                             int d, int n_force, void* O, uint8_t* kept_mask, float* density,
                             void* workspace, size_t ws_bytes, void* stream);

/* sol_attn_fwd with the query-block means given by the caller (qbar, fp32 [B, H, N_qb, d], as
 * sol_attn_qknorm_rope_pool_qbar writes them for the Q it stores): the routing pass takes them
 * instead of reading Q to form q_bar (Sol-Attn project page, Abstract: the proxy score pools the
 * query block). The means may differ from the ones sol_attn_fwd forms in the last bits (another
 * fp32 summation order), which can move a block whose proxy score lies within that rounding of
 * the threshold. SOL_BF16 only, blocks of 128, d in {64, 128}; the workspace must have the full
 * size of sol_attn_fwd_workspace_bytes. qbar non-null and 16-byte aligned, else SOL_EINVAL. Other
 * arguments, limits and errors as for sol_attn_fwd. */
sol_status sol_attn_fwd_qbar(const void* Q, const void* K, const void* V, const float* kbar,
                             const float* vbar, const void* kbar_lp, const void* vbar_lp,
                             const float* qbar, const float* tau, int B, int H, int L, int d,
                             int n_force, void* O, uint8_t* kept_mask, float* density, void* workspace,
                             size_t ws_bytes, void* stream);

/* The forward with 8-bit QK^T (NEXT-2): the exact tiles' and the correction's scores come from the
 * int8 codes of sol_attn_quantize_qk8 (tcgen05 kind::i8, int32 accumulation), scaled by
 * q_scale * k_scale (or kbar_scale for a pooled tile) in the softmax; P and V stay bf16. Routing
 * is unchanged: the routing pass reads the bf16 Q and the fp32 pooled keys kbar, so the kept
 * blocks are those of sol_attn_fwd. vbar_lp is the bf16 pooled V of sol_attn_pool. SOL_BF16 only,
 * d = 128, blocks of 128, and the workspace must have the full size of
 * sol_attn_fwd_workspace_bytes. Other arguments, limits and errors as for sol_attn_fwd. */
sol_status sol_attn_fwd_qk8(const void* Q, const int8_t* q8, const int8_t* k8, const int8_t* kbar8,
                            const float* q_scale, const float* k_scale, const float* kbar_scale,
                            const void* V, const float* kbar, const void* vbar_lp, const float* tau,
                            int B, int H, int L, int d, int n_force, void* O, uint8_t* kept_mask,
                            float* density, void* workspace, size_t ws_bytes, void* stream);

/* Synchronises `stream`, then reads and clears the workspace's device error word. Returns
 * SOL_ETIMEOUT if any launch since the last check gave up on a bounded wait, after which that
 * launch's outputs are incomplete. Returns SOL_OK otherwise. */
sol_status sol_attn_check_device_error(void* workspace, void* stream);

/* The same fused forward for callers that cannot allocate device memory. There is no counterpart
 * on the Sol-Attn pages; this is a deployment convenience of this library.
 *
 * Some callers cannot call cudaMalloc. Examples: a host framework whose caching allocator has
 * already reserved the device memory and forbids foreign allocations; a plugin that must not
 * trigger the implicit device synchronisation cudaMalloc/cudaFree can cause on a latency-critical
 * path. Such callers cannot provide the workspace that sol_attn_fwd needs. This entry point takes
 * the same arguments minus the workspace. It uses a 16,640-byte array in the library's own device
 * memory instead: a file-scope static __device__ array, which every GPU that loads the library
 * holds until the process exits.
 *
 *   limit      B * H <= 4096 (the array holds the workspace header of at most 4096 heads); larger
 *              problems return SOL_EUNSUPPORTED without launching anything.
 *   routing    the array is passed to sol_attn_fwd as its workspace. When the routing pass's
 *              keep bits and query-block means fit in what the header leaves free (see
 *              sol_attn_fwd_workspace_bytes), the separate routing pass runs; otherwise the fused
 *              kernel routes each unit itself. Both give the same results bit for bit.
 *   set-up     the first call on a device (and the first after a cudaDeviceReset) looks up the
 *              array's device address (cudaGetSymbolAddress) with that device current, and
 *              caches it with the current context. Make that first call before any stream
 *              capture.
 *   sharing    every call on a device shares the one array. Each call clears it on `stream`
 *              before launching, so calls on one stream are safe, but calls that overlap on the
 *              GPU (different streams, no ordering) race on it.
 *   errors     host-side errors as for sol_attn_fwd. A bounded-wait expiry on the device is
 *              silent here: its error word lives in the shared array, is not readable through
 *              this ABI, and the next call's clear erases it. Use sol_attn_fwd with a workspace
 *              when that status is needed.
 * Calls no cudaMalloc, cudaFree or other allocating routine. */
sol_status sol_attn_fwd_noalloc(const void* Q, const void* K, const void* V, const float* kbar,
                                const float* vbar, const void* kbar_lp, const void* vbar_lp,
                                const float* tau, sol_dtype dt, int B, int H, int L, int d,
                                int block_q, int block_k, int n_force, void* O, uint8_t* kept_mask,
                                float* density, void* stream);

/* Bytes of device scratch sol_attn_fwd_host needs (0 for invalid sizes or dtype). The scratch holds
 * two slots of Q, K, V and O for `heads_per_chunk` heads, one set of pooled vectors for that many
 * heads, one workspace and B*H density words, each rounded up to 256 bytes. For bf16, H=40,
 * L=75600, d=128 with 2 heads per chunk that is 0.31 GB. */
size_t sol_attn_fwd_host_scratch_bytes(sol_dtype dt, int B, int H, int L, int d, int block,
                                       int heads_per_chunk);

/* The whole path (sol_attn_pool, then sol_attn_fwd) on inputs and output in HOST memory. This is
 * the same operation, with the same kernels and results, for callers whose tensors live on the
 * host. The pages describe no such call; it is a deployment convenience of this library.
 *
 * Heads are independent, so the call cuts each batch entry's H heads into chunks of
 * `heads_per_chunk` and pipelines them through two slots of the device scratch. Chunk c is
 * uploaded on one copy stream while chunk c-1 is pooled and attended on `stream`, and chunk c-2's
 * output is downloaded on a second copy stream. With pinned host memory the uploads, the compute
 * and the downloads overlap, so the call takes about as long as its slowest part (usually the
 * upload of Q, K and V over the host link) plus one chunk. Pageable host memory gives the same
 * results without that overlap. The copy streams and the events are created and destroyed inside
 * the call.
 *
 *   Q, K, V    HOST, [B, H, L, d] in dtype `dt` (pinned for overlap; must not be device memory)
 *   O          HOST, [B, H, L, d] in dtype `dt`: the output
 *   tau        HOST, float32 [H], as for sol_attn_fwd
 *   block      block_q = block_k; the sizes supported are those of sol_attn_fwd
 *   n_force    as for sol_attn_fwd
 *   heads_per_chunk  >= 1 (values above H mean H): smaller chunks start the pipeline sooner,
 *              larger ones give each launch more work units
 *   density    HOST, float32 [B, H] or NULL: kept blocks / (N_qb * N_kb) per head
 *   scratch    device memory of the current device, 256-byte aligned, at least
 *              sol_attn_fwd_host_scratch_bytes(...) bytes; no zeroing needed
 *   stream     the compute stream. Work enqueued on it earlier finishes before the call's first
 *              upload starts.
 * Synchronous: it returns once O and density are in host memory, or after a failure, once
 * nothing the call started is still running. All size checks run before the first copy. A
 * bounded-wait expiry in any chunk returns SOL_ETIMEOUT, and the outputs are then incomplete.
 * Not usable inside a CUDA graph capture. */
sol_status sol_attn_fwd_host(const void* Q, const void* K, const void* V, void* O, const float* tau,
                             sol_dtype dt, int B, int H, int L, int d, int block, int n_force,
                             int heads_per_chunk, float* density, void* scratch, size_t scratch_bytes,
                             void* stream);

/* Test hook for the failure-detection path. mode 0 (default) = normal operation. mode 1 makes
 * the next sol_attn_fwd launch (SOL_BF16 path) skip one K-tile load, so the consumer's bounded
 * wait expires: the launch returns early, sets the device error word, and
 * sol_attn_check_device_error then reports SOL_ETIMEOUT. The hook applies to one launch and
 * then resets to 0. The wait limit is about 0.2 s in that mode and about 2 s otherwise. */
void sol_attn_debug_drop_one_load(int mode);

/* Measurement hook for the persistent scheduler's load balance. The next sol_attn_fwd launch of
 * the SOL_BF16 fused kernel writes, for each CTA c < capacity, its start and finish time in
 * nanoseconds (the GPU's global timer) to times[2c] and times[2c + 1]. `times` is device memory
 * of 2 * capacity 64-bit words, owned by the caller. The hook applies to one launch and then
 * resets; capacity <= 0 disarms it. */
void sol_attn_debug_record_cta_times(unsigned long long* times, int capacity);

#ifdef __cplusplus
}
#endif

#endif /* SOL_ATTN_H */
