/*
 * arkattn.h -- C ABI of libarkattn: grouped-query attention over a static,
 * sequence-major KV cache, hand-written for NVIDIA B200 (sm_100a).
 *
 * The operation is the attention step of the ARK-ASR-3B decoder as the
 * "ARK-ASR-3B -- INT8 ONNX" model card describes it in its section Shapes:
 * 16 query heads share 2 KV heads (8 query heads per KV head), head dim 128,
 * and each layer keeps a static cache cache_{key,value}_i of shape
 * [1, max_total_len, 2, 128], sequence-major; each call produces
 * key_delta/value_delta rows for the positions it writes, and those rows go
 * into the cache at cache_position.  Here the batch dimension is B, so one
 * layer's cache is [B, T, Hkv, D] with T = max_total_len.  The decoder is a
 * Qwen2 language model (SGLang-Omni cookbook "ARK-ASR-3B", introduction), so
 * RoPE (rotate-half form) is applied to the new query and key rows.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers to contiguous, row-major memory
 *     in the layouts stated per call; bf16 tensors are `void*`.  Every tensor
 *     pointer must be 16-byte aligned.
 *   - The caller owns and allocates every buffer (tensors, workspace, RoPE
 *     table, status word).  The library allocates no device memory and keeps
 *     no per-call state, with two stated exceptions: ark_attn_decode_noalloc
 *     uses one fixed, file-scope device array (see there), and the host keeps
 *     a process-wide cache of the TMA tensor maps it encodes, keyed by buffer
 *     address and shape (a map describes only the address and shape, so a
 *     buffer freed and reallocated at the same address reuses a valid map).
 *   - Calls are asynchronous on `stream` and enqueue kernels only (except
 *     ark_attn_rope_table_init, which copies from the host and synchronises).
 *   - Arguments the host can see are checked before anything is launched; a
 *     failed check returns an error and launches nothing.
 *   - Values that live on the device (cache positions, lengths) cannot be
 *     checked by the host without a synchronisation.  Kernels check them,
 *     skip or clamp what is out of range and OR a bit into the caller's
 *     status word `*d_status` (device memory, uint32).  The caller reads the
 *     word after synchronising.  `d_status` may be NULL to skip reporting.
 *   - Only D = 128 and Hq/Hkv = 8 are instantiated (ARK_ERR_UNSUPPORTED
 *     otherwise); T <= ARK_MAX_T; decode takes B <= 4096.
 *   - A launch failure returns ARK_ERR_CUDA; the CUDA error is left to the
 *     caller (cudaGetLastError).
 */
#ifndef ARKATTN_H_
#define ARKATTN_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define ARK_API __attribute__((visibility("default")))
#else
#define ARK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ark_status {
    ARK_OK = 0,
    ARK_ERR_INVALID_ARG = 1,   /* null pointer, non-positive size, misalignment, Hq % Hkv != 0 */
    ARK_ERR_UNSUPPORTED = 2,   /* a shape this build does not instantiate (D != 128, Hq/Hkv != 8) */
    ARK_ERR_WORKSPACE = 3,     /* workspace missing or smaller than the *_workspace_size answer */
    ARK_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
    ARK_ERR_TIMEOUT = 5        /* reserved: a bounded device wait gave up (see ARK_DEV_TIMEOUT) */
} ark_status;

/* Decode modes.  Both give the same result (to fp32 rounding order).
 * LENGTH_AWARE reads only the kv_len[b] valid rows of each request.
 * MASKED_STATIC reads all T rows and gives the rows at or past kv_len[b] a
 * score of -inf, which is what a static cache graph does: the ONNX model card
 * ("ARK-ASR-3B -- INT8 ONNX", section Shapes) states that the decoder attends
 * over ALL max_total_len positions on every token however few are valid.
 * Precondition of MASKED_STATIC: the rows past kv_len hold finite values
 * (a masked row contributes 0 x its V row, which is NaN for a non-finite row). */
typedef enum ark_decode_mode {
    ARK_LENGTH_AWARE = 0,
    ARK_MASKED_STATIC = 1
} ark_decode_mode;

/* Bits OR-ed into the device status word. */
#define ARK_DEV_BAD_POS   1u  /* cache_position + t outside [0, T): that row was skipped */
#define ARK_DEV_BAD_KVLEN 2u  /* kv_len or n_new outside its range: clamped (kv_len 0 gives o = 0, lse = -inf) */
#define ARK_DEV_TIMEOUT   4u  /* a bounded wait on an asynchronous copy gave up; outputs of that block not written */

#define ARK_MAX_T 65536
#define ARK_MAX_LAYERS 64

/* Human-readable name of a status code (static string, never NULL). */
ARK_API const char* ark_attn_status_string(ark_status s);

/* ------------------------------------------------------------------ RoPE ----
 * Rotary table for positions 0..T-1: for pair i < D/2, inv_freq_i =
 * rope_theta^(-2i/D), angle = p * inv_freq_i computed in double, and the
 * table holds (float)cos(angle), (float)sin(angle).  The pages name the
 * decoder as Qwen2 (SGLang-Omni cookbook "ARK-ASR-3B", introduction) and give
 * no formula; this is the Qwen2 convention, with theta 1e6 for ARK-ASR-3B's
 * decoder as configured by the caller.
 * d_table: device, ark_attn_rope_table_bytes(T, D) bytes, layout [T][D/2] of
 *   float2 {cos, sin}.  Caller-owned.  Computed on the host, copied with
 *   cudaMemcpyAsync on `stream`, and the call synchronises `stream` before it
 *   returns (set-up only; not for stream capture).
 */
ARK_API size_t ark_attn_rope_table_bytes(int T, int D);
ARK_API ark_status ark_attn_rope_table_init(float* d_table, int T, int D, double rope_theta,
                                    cudaStream_t stream);

/* ---------------------------------------------------------- RoPE + write ----
 * For each request b < B and new row t < n_new[b] (t < S), at the absolute
 * position p = pos0[b] + t (pos0 is cache_position: the number of valid
 * cache rows before this call):
 *   q[b,t,h,:]       <- RoPE_p(q[b,t,h,:])     for h < Hq   (in place)
 *   cache_k[b,p,g,:] <- RoPE_p(k_new[b,t,g,:]) for g < Hkv  (the key delta)
 *   cache_v[b,p,g,:] <- v_new[b,t,g,:]                      (the value delta, bit copy)
 * ("ARK-ASR-3B -- INT8 ONNX", section Shapes: the delta rows land in the
 * cache at cache_position.)  RoPE_p pairs element i with i + D/2:
 *   x'[i] = x[i] c - x[i+D/2] s,  x'[i+D/2] = x[i+D/2] c + x[i] s,
 * c, s the fp32 table entries of (p, i); each output is formed in double and
 * rounded once to bf16 (nearest-even), so the result is bit-reproducible.
 * Layouts: q [B,S,Hq,D] bf16; k_new, v_new [B,S,Hkv,D] bf16; cache_k, cache_v
 * [B,T,Hkv,D] bf16; pos0, n_new int32[B] (device); d_table from
 * ark_attn_rope_table_init with at least T rows.
 * Rows t >= n_new[b] are not touched.  A row with p outside [0, T) is skipped
 * entirely (q not rotated, nothing written) and sets ARK_DEV_BAD_POS.
 */
ARK_API ark_status ark_attn_append_rope(void* q, const void* k_new, const void* v_new,
                                void* cache_k, void* cache_v,
                                const int32_t* pos0, const int32_t* n_new,
                                int B, int S, int T, int Hq, int Hkv, int D,
                                const float* d_table, uint32_t* d_status, cudaStream_t stream);

/* ---------------------------------------------------------------- decode ----
 * One query row per request (the new token, already rotated) attends to the
 * kv_len[b] valid cache rows of its KV head g = h / (Hq/Hkv):
 *   s_j = scale * <q[b,0,h,:], cache_k[b,j,g,:]>,  j < kv_len[b]
 *   o[b,0,h,:] = sum_j softmax(s)_j cache_v[b,j,g,:],   lse[b,h] = ln sum_j exp(s_j)
 * ("ARK-ASR-3B -- INT8 ONNX", section Shapes: 16 heads share 2 KV heads over
 * the static cache.)  All 8 query heads of a KV group are served from one read
 * of each K/V row.  The rows of all (request, KV head) pairs form one list of
 * 16-row tiles that the GPU's warps split into equal contiguous ranges, so a
 * request's rows may be cut into pieces processed in parallel; every warp
 * takes at least ceil(ceil(T/16) / max_splits) tiles, so one (request, KV
 * head) is cut into at most max_splits + 1 pieces.  Cut pieces leave fp32
 * partial results in `workspace`; a second kernel, enqueued by the same call
 * on the same stream (programmatic dependent launch, so it is resident as
 * the first kernel's CTAs retire), merges them by log-sum-exp.
 * Layouts: q [B,1,Hq,D] bf16; cache_k, cache_v [B,T,Hkv,D] bf16; kv_len
 * int32[B] (device; the new row is already appended, so the query attends to
 * itself); o [B,1,Hq,D] bf16; lse [B,Hq] fp32 (natural log).
 * kv_len outside [0, T] is clamped and sets ARK_DEV_BAD_KVLEN; kv_len = 0
 * gives o = 0, lse = -inf.  The decode kernel is launched with programmatic
 * dependent launch behind whatever kernel precedes it on `stream`; it waits
 * for that kernel's completion before it reads q, the caches or kv_len, so
 * the preceding kernel may write any of them (an append, or a kernel that
 * advances the lengths on the device).
 * Workspace: ark_attn_decode_workspace_size(...) bytes (about 16 MB: two
 * partial slots for each of up to 2048 warps), 16-byte aligned, caller-owned,
 * required.  It needs no initialisation and carries nothing from one call to
 * the next.  Calls that can run at the same time must not share a workspace.
 * Numerics: bf16 operands on the tensor cores with fp32 accumulation; the
 * softmax weights are rounded to bf16 before they multiply V, o is normalised
 * by the sum of those rounded weights and lse uses the fp32 weights.
 */
ARK_API size_t ark_attn_decode_workspace_size(int B, int Hq, int D, int T, int max_splits);
ARK_API ark_status ark_attn_decode(const void* q, const void* cache_k, const void* cache_v,
                                   const int32_t* kv_len, int B, int T, int Hq, int Hkv, int D,
                                   float scale, ark_decode_mode mode, int max_splits,
                                   void* workspace, size_t workspace_bytes,
                                   void* o, float* lse, uint32_t* d_status, cudaStream_t stream);

/* --------------------------------------------------------------- prefill ----
 * Causal prefill of a prompt ("ARK-ASR-3B -- INT8 ONNX", section Inference:
 * the audio+text prompt is prefilled, then decoded; section Shapes: the
 * call's rows are written into the static cache at cache_position).  Call it
 * after ark_attn_append_rope has rotated q and written this call's K/V rows.
 * For request b and new row t < n_new[b], at position p = pos0[b] + t, and
 * each query head h (KV head g = h / (Hq/Hkv)):
 *   o[b,t,h,:] = sum_{j <= p} softmax_j(scale * <q[b,t,h,:], cache_k[b,j,g,:]>) cache_v[b,j,g,:]
 *   lse[b,h,t] = ln sum_{j <= p} exp(scale * <q[b,t,h,:], cache_k[b,j,g,:]>)
 * Layouts: q [B,S,Hq,D] bf16 (rotated); cache_k, cache_v [B,T,Hkv,D] bf16;
 * pos0, n_new int32[B] (device); o [B,S,Hq,D] bf16; lse [B,Hq,S] fp32.
 * Rows t >= n_new[b] of o and lse are not written.  n_new outside [0, S] or
 * pos0 + n_new > T is clamped and sets ARK_DEV_BAD_POS.  The 5th-generation
 * tensor cores (tcgen05) compute Q K^T and P V with fp32 accumulation in
 * tensor memory; the softmax weights are rounded to bf16 before P V.
 */
ARK_API ark_status ark_attn_prefill(const void* q, const void* cache_k, const void* cache_v,
                                    const int32_t* pos0, const int32_t* n_new, int B, int S, int T,
                                    int Hq, int Hkv, int D, float scale, void* o, float* lse,
                                    uint32_t* d_status, cudaStream_t stream);

/* -------------------------------------------------- layer-batched variants ----
 * The same operations over L <= ARK_MAX_LAYERS independent layers in ONE
 * launch.  Every pointer argument that is per layer is a HOST array of L
 * device pointers (read during the call; the array itself may be freed when
 * the call returns).  All layers share B, S, T, the positions/lengths and the
 * rotary table.  Each layer's tensors follow the single-layer layouts above.
 * ark_attn_prefill_layers runs the work of up to 36 layers in one launch of
 * its persistent kernel (longer lists take several launches of near-equal
 * size, in order on `stream`), so that the GPU does not drain at every layer
 * boundary.
 * The decode workspace is ark_attn_decode_layers_workspace_size(L, ...) bytes
 * under the same rules.  Meant for callers that hold
 * several independent caches (the ARK-ASR-3B decoder has 36 layers), and for
 * measuring the kernels without per-launch overhead.
 */
ARK_API ark_status ark_attn_prefill_layers(int L, const void* const* q, const void* const* cache_k,
                                           const void* const* cache_v, const int32_t* pos0, const int32_t* n_new,
                                           int B, int S, int T, int Hq, int Hkv, int D, float scale,
                                           void* const* o, float* const* lse, uint32_t* d_status,
                                           cudaStream_t stream);
ARK_API ark_status ark_attn_append_rope_layers(int L, void* const* q, const void* const* k_new,
                                               const void* const* v_new, void* const* cache_k,
                                               void* const* cache_v, const int32_t* pos0,
                                               const int32_t* n_new, int B, int S, int T, int Hq,
                                               int Hkv, int D, const float* d_table,
                                               uint32_t* d_status, cudaStream_t stream);
ARK_API size_t ark_attn_decode_layers_workspace_size(int L, int B, int Hq, int D, int T, int max_splits);
ARK_API ark_status ark_attn_decode_layers(int L, const void* const* q, const void* const* cache_k,
                                          const void* const* cache_v, const int32_t* kv_len, int B,
                                          int T, int Hq, int Hkv, int D, float scale,
                                          ark_decode_mode mode, int max_splits, void* workspace,
                                          size_t workspace_bytes, void* const* o, float* const* lse,
                                          uint32_t* d_status, cudaStream_t stream);

/* --------------------------------------------------------------- combine ----
 * Log-sum-exp merge of nsplit partial results of the same query over
 * disjoint key ranges.  For each (b, h):
 *   M = max_c lse_part[b,h,c],  w_c = exp(lse_part[b,h,c] - M)
 *   o[b,h,:] = sum_c w_c o_part[b,h,c,:] / sum_c w_c,   lse[b,h] = M + ln sum_c w_c
 * A part with lse_part = -inf (no keys) has weight 0 and its o_part row is not
 * read; all parts empty gives o = 0, lse = -inf.  (The pages have no split;
 * this is the exact identity that lets a softmax be computed in pieces.)
 * Layouts: o_part [B,Hq,nsplit,D] fp32 (each part normalised by its own sum),
 * lse_part [B,Hq,nsplit] fp32; o [B,Hq,D] bf16 (the same memory as
 * [B,1,Hq,D]); lse [B,Hq] fp32.
 */
ARK_API ark_status ark_attn_combine(const float* o_part, const float* lse_part, int B, int Hq,
                            int nsplit, int D, void* o, float* lse, cudaStream_t stream);

/* ------------------------------------------------- decode, no allocation ----
 * The pages have no counterpart of this entry point; it exists for callers
 * that cannot call cudaMalloc (or any allocating routine) at the point where
 * they decode: code that runs while a CUDA graph is being captured, engines
 * that reserve all device memory up front and hand out none afterwards, and
 * plugins whose host framework owns the allocator.  Such a caller still
 * passes its inputs and outputs, but no workspace.
 * Same operation, arguments, layouts and results as ark_attn_decode, without
 * the workspace arguments.  The scratch (the partial results of cut pieces)
 * is a fixed array inside the library, ark_attn_decode_noalloc_scratch_bytes()
 * bytes (about 4.2 MB) on every GPU that loads the library, kept until the
 * process exits.  It holds the partials of at most 512 warps, so a call runs
 * on at most 512 warps and very large batches run slower than with
 * ark_attn_decode; the size limits are those of ark_attn_decode (B <= 4096,
 * ARK_ERR_UNSUPPORTED beyond).
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress); make that first call before any stream capture.
 * The address is cached per CUDA context: after a device reset the next call
 * looks it up again (make that call, too, before any capture).
 * Nothing in the scratch needs initialising and no call allocates.  All calls
 * share the one array, so calls that can overlap on the GPU (different
 * streams, or graphs replayed concurrently) race: serialise them.
 */
ARK_API size_t ark_attn_decode_noalloc_scratch_bytes(void);
ARK_API ark_status ark_attn_decode_noalloc(const void* q, const void* cache_k, const void* cache_v,
                                           const int32_t* kv_len, int B, int T, int Hq, int Hkv, int D,
                                           float scale, ark_decode_mode mode, int max_splits, void* o,
                                           float* lse, uint32_t* d_status, cudaStream_t stream);

/* ------------------------------------- prefill with RoPE on the q load ----
 * The same prefill for a caller that leaves q unrotated:
 * ark_attn_append_rope_kv(_layers) rotates and writes only the K rows and
 * copies the V rows into the cache (as ark_attn_append_rope does, q not
 * touched; the q argument is absent and Hq only sizes the checks), and
 * ark_attn_prefill_rope(_layers) rotates each q tile as it loads it, with the
 * append's arithmetic (products in double from the bf16 input and the fp32
 * table d_table of ark_attn_rope_table_init, one rounding to bf16), so its o
 * and lse equal those of ark_attn_append_rope + ark_attn_prefill bit for bit.
 * q is read only.  This saves the append's read and write of every prompt q
 * row.
 */
ARK_API ark_status ark_attn_append_rope_kv(const void* k_new, const void* v_new, void* cache_k, void* cache_v,
                                           const int32_t* pos0, const int32_t* n_new, int B, int S, int T, int Hq,
                                           int Hkv, int D, const float* d_table, uint32_t* d_status,
                                           cudaStream_t stream);
ARK_API ark_status ark_attn_append_rope_kv_layers(int L, const void* const* k_new, const void* const* v_new,
                                                  void* const* cache_k, void* const* cache_v, const int32_t* pos0,
                                                  const int32_t* n_new, int B, int S, int T, int Hq, int Hkv, int D,
                                                  const float* d_table, uint32_t* d_status, cudaStream_t stream);
ARK_API ark_status ark_attn_prefill_rope(const void* q, const void* cache_k, const void* cache_v,
                                         const int32_t* pos0, const int32_t* n_new, int B, int S, int T, int Hq,
                                         int Hkv, int D, float scale, const float* d_table, void* o, float* lse,
                                         uint32_t* d_status, cudaStream_t stream);
ARK_API ark_status ark_attn_prefill_rope_layers(int L, const void* const* q, const void* const* cache_k,
                                                const void* const* cache_v, const int32_t* pos0,
                                                const int32_t* n_new, int B, int S, int T, int Hq, int Hkv, int D,
                                                float scale, const float* d_table, void* const* o,
                                                float* const* lse, uint32_t* d_status, cudaStream_t stream);

/* ------------------------------------------------------- fp8 KV cache ----
 * A cache of 8-bit codes, half the bytes of the bf16 cache, for the same
 * attention.  The pages quantise weights only (the int8/int4 tiers of the
 * "ARK-ASR-3B -- INT8 ONNX" model card); the cache format here is this
 * library's own:
 *   - codes are OCP FP8 E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa
 *     bits; no infinities; S.1111.111 is NaN; largest finite value 448);
 *   - k_scale, v_scale: one fp32 scale per KV head for K and for V (device
 *     arrays [Hkv] per layer, caller-owned, 4-byte aligned); a stored code c
 *     stands for c * scale;
 *   - the append stores e4m3(fp32(x / scale)) for the rotated key x (formed
 *     in fp64 as for the bf16 cache, not rounded to bf16 first) and for the
 *     value row: the quotient in fp64, rounded to fp32, then to e4m3 with
 *     round-to-nearest-even, finite values beyond +-448 and infinities
 *     saturating to +-448, NaN kept.  q is rotated to bf16 in place as by
 *     ark_attn_append_rope.  Bit-reproducible.
 * Layouts: cache_k, cache_v head-major [B,Hkv,T,D] of uint8 codes (16-byte
 * aligned; unlike the bf16 cache's [B,T,Hkv,D], so that the positions of one
 * KV head are consecutive 128-byte rows); everything else, the arguments, the
 * status bits and the errors as for the bf16 entry points.  The decode computes Q K^T and P V on f16 tensor-core
 * operands (every e4m3 value is an f16 value; q is converted from bf16 to
 * f16, exact for |q| in [2^-14, 65504]; the softmax weights are rounded to
 * f16) with fp32 accumulation, and uses the workspace of ark_attn_decode.
 */
ARK_API ark_status ark_attn_append_rope_fp8(void* q, const void* k_new, const void* v_new, void* cache_k,
                                            void* cache_v, const float* k_scale, const float* v_scale,
                                            const int32_t* pos0, const int32_t* n_new, int B, int S, int T,
                                            int Hq, int Hkv, int D, const float* d_table, uint32_t* d_status,
                                            cudaStream_t stream);
ARK_API ark_status ark_attn_append_rope_fp8_layers(int L, void* const* q, const void* const* k_new,
                                                   const void* const* v_new, void* const* cache_k,
                                                   void* const* cache_v, const float* const* k_scale,
                                                   const float* const* v_scale, const int32_t* pos0,
                                                   const int32_t* n_new, int B, int S, int T, int Hq, int Hkv,
                                                   int D, const float* d_table, uint32_t* d_status,
                                                   cudaStream_t stream);
ARK_API ark_status ark_attn_decode_fp8(const void* q, const void* cache_k, const void* cache_v,
                                       const float* k_scale, const float* v_scale, const int32_t* kv_len, int B,
                                       int T, int Hq, int Hkv, int D, float scale, ark_decode_mode mode,
                                       int max_splits, void* workspace, size_t workspace_bytes, void* o,
                                       float* lse, uint32_t* d_status, cudaStream_t stream);
ARK_API ark_status ark_attn_decode_fp8_layers(int L, const void* const* q, const void* const* cache_k,
                                              const void* const* cache_v, const float* const* k_scale,
                                              const float* const* v_scale, const int32_t* kv_len, int B, int T,
                                              int Hq, int Hkv, int D, float scale, ark_decode_mode mode,
                                              int max_splits, void* workspace, size_t workspace_bytes,
                                              void* const* o, float* const* lse, uint32_t* d_status,
                                              cudaStream_t stream);

/* --------------------------------------------------- encoder attention ----
 * Bidirectional multi-head self-attention of the audio encoder.  The pages
 * describe a Whisper-style audio tower with rotary self-attention whose output
 * is 1280 wide ("ARK-ASR-3B -- INT8 ONNX", Inference step 1; "Inside
 * ARK-ASR-3B's Whisper and Qwen architecture", components) but give neither its
 * head count nor its rotary parameters; the reading taken is the Whisper-large
 * geometry of a 1280-wide model, H heads of D = 64 (H = 20), with q and k
 * already rotated.  For clip b, head h and frame i < len[b]:
 *   o[b,i,h,:] = sum_{j < len[b]} softmax_j(scale <q[b,i,h,:], k[b,j,h,:]>) v[b,j,h,:]
 *   lse[b,h,i] = ln sum_{j < len[b]} exp(scale <q[b,i,h,:], k[b,j,h,:]>)
 * Layouts: q, k, v [B,S,H,D] bf16 (16-byte aligned); len int32[B] (device);
 * o [B,S,H,D] bf16; lse [B,H,S] fp32.  Rows i >= len[b] are not written; len
 * outside [0, S] is clamped and sets ARK_DEV_BAD_KVLEN.  D != 64 or more than
 * 256 clips (B > 256) returns ARK_ERR_UNSUPPORTED.  tcgen05 MMAs (bf16 operands, fp32 accumulation in
 * tensor memory); the softmax weights are rounded to bf16 before P V.
 */
ARK_API ark_status ark_attn_encoder(const void* q, const void* k, const void* v, const int32_t* len, int B, int S,
                                    int H, int D, float scale, void* o, float* lse, uint32_t* d_status,
                                    cudaStream_t stream);

/* ------------------------------------------ Q/K/V projection (+ RoPE) ----
 * The step in front of the attention: the Q/K/V projections of a decoder
 * layer ("ARK-ASR-3B -- INT8 ONNX" model card: Qwen2 decoder, hidden 2048,
 * 16 query and 2 KV heads of 128 dims) as one Linear over the concatenated
 * weight W = [Wq; Wk; Wv], optionally with the RoPE + delta write of
 * ark_attn_append_rope fused into its epilogue (tcgen05 MMAs, fp32
 * accumulation).
 *
 * ark_attn_qkv_proj: out[m, n] = bf16(sum_k x[m, k] W[n, k] + bias[n]).
 *   x [M, K], W [N, K], out [M, N] bf16 row-major (16-byte aligned); bias [N]
 *   bf16 or NULL.  K % 64 == 0, N % 128 == 0, else ARK_ERR_INVALID_ARG.  The
 *   fp32 accumulator and the bias are added in double and rounded once to bf16.
 *
 * ark_attn_qkv_rope_append: x [B, S, K] token rows of B requests (row t of
 *   request b is live when t < n_new[b], at position pos0[b] + t); W [(Hq + 2
 *   Hkv) * 128, K] with the q heads first, then k, then v; bias as above.  For
 *   every live row: q[b, t] = RoPE(p_q) (q [B, S, Hq, 128]), cache_k[b, pos] =
 *   RoPE(p_k), cache_v[b, pos] = p_v (caches [B, T, Hkv, 128]), with p the
 *   bf16 projection above and RoPE exactly as in ark_attn_append_rope (table
 *   from ark_attn_rope_table_init).  Bit-identical to ark_attn_qkv_proj
 *   followed by ark_attn_append_rope.  Padded rows, and rows whose position
 *   falls outside [0, T) (ARK_DEV_BAD_POS), are not written; n_new outside
 *   [0, S] is clamped (ARK_DEV_BAD_KVLEN).  D != 128 returns ARK_ERR_UNSUPPORTED.
 *
 * Both are launched with programmatic stream serialisation: a launch may start
 * streaming W while the kernel before it in the stream finishes, and reads x
 * and writes its outputs only after that kernel has completed, so stream order
 * is kept.  Few tiles (a decode step) split K over a thread-block cluster.
 */
ARK_API ark_status ark_attn_qkv_proj(const void* x, const void* w, const void* bias, int M, int K, int N, void* out,
                                     uint32_t* d_status, cudaStream_t stream);

ARK_API ark_status ark_attn_qkv_rope_append(const void* x, const void* w, const void* bias, const int32_t* pos0,
                                            const int32_t* n_new, int B, int S, int T, int Hq, int Hkv, int D, int K,
                                            const float* d_table, void* q, void* cache_k, void* cache_v,
                                            uint32_t* d_status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* ARKATTN_H_ */
