/*
 * tq.h -- C ABI of libtq: on-the-fly int4 KV-cache quantization and decode
 * attention computed directly on the packed int4 cache (B200, sm_100a).
 *
 * The two operations follow the statement of the problem in
 * "Open-TQ-Metal: Fused Compressed-Domain Attention for Long-Context LLM
 * Inference on Apple Silicon" (arXiv 2604.16957v1), abstract: the KV cache is
 * quantized to int4 as it is generated, and attention (the fused "sdpa_int4"
 * kernel) runs on the compressed representation with no intermediate
 * dequantized K/V matrix.  The rotation is the Hadamard rotation of the AdapTQ
 * post (section "Fast Hadamard Rotation (HAR)") with random signs, which the
 * "SRFT + int4 KV-cache on Apple Silicon" post (core-method section) reports
 * as equivalent to its sign-randomized FFT; quantization is that post's
 * per-group abs-max symmetric int4 with nibble packing.  The call shape
 * mirrors AdapTQ's engine (section "native Python API": fixed capacity,
 * append(k, v), compute(q)), and, like that engine (section "zero heap
 * allocation"), no call allocates: the caller passes every buffer.
 *
 * Conventions for every call:
 *  - All pointers except `signs == NULL` markers are DEVICE pointers on the
 *    current CUDA device, owned by the caller; the library never allocates,
 *    frees or retains them.
 *  - Calls only enqueue work on `cuda_stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and return without synchronizing.
 *  - Arguments are validated on the host before any launch; an invalid call
 *    returns an error and enqueues nothing.  A failed launch returns
 *    TQ_ERR_CUDA.
 *  - Results are deterministic: the same inputs give bit-identical outputs.
 *
 * Data layout (row-major, dense):
 *  - head_dim d in {128, 256} (the SRFT calls below: any multiple of 32 up to
 *    256); group size g = 32; ng = d / 32 groups.
 *  - packed cache: uint8 [B][Hkv][capacity][d/2], one row per token.  Rotated
 *    coordinate i (group gi = i/32, in-group j = i%32) is stored as a 4-bit
 *    two's-complement code in byte (j/4)*(2*ng) + 2*gi + (j%4)/2 of its row,
 *    low nibble when j is even, high nibble when j is odd.  Codes are in
 *    [-7, 7].
 *  - scales: float [B][Hkv][capacity][ng]; scale = fl32(amax / 7) of the
 *    group's rotated values (0 for an all-zero group).
 *  - dequantized value of coordinate i = scale[i/32] * code[i], in the
 *    rotated basis R x, R = H_d diag(signs) / sqrt(d) (Sylvester H_d).
 *  - Alignment: packed rows, scale rows, q and out must be 16-byte aligned;
 *    with the layout above this holds when the base pointers are.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = -1,   /* bad pointer, size, shape or alignment */
  TQ_ERR_UNSUPPORTED = -2,   /* valid but not implemented (e.g. head_dim 64) */
  TQ_ERR_WORKSPACE = -3,     /* workspace NULL or smaller than required */
  TQ_ERR_CUDA = -4,          /* a CUDA launch or runtime call failed */
  TQ_ERR_SCRATCH_LIMIT = -5  /* sizes need more scratch than TQ_STATIC_SCRATCH_BYTES */
} tq_status;

/* Bytes of the built-in device scratch of tq_sdpa_int4_decode_static_scratch. */
#define TQ_STATIC_SCRATCH_BYTES (8u << 20)

typedef enum { TQ_F32 = 0, TQ_BF16 = 1 } tq_dtype;

/*
 * tq_quantize_append -- quantize n_new tokens of K and V per (sequence, kv
 * head) and write them into cache rows pos[b] .. pos[b]+n_new-1 of sequence
 * b.  ("On-the-fly quantization": Open-TQ-Metal abstract; rotation: AdapTQ
 * post, section "Fast Hadamard Rotation (HAR)"; abs-max int4 + nibble pack:
 * SRFT post, core-method section.)
 *
 *  k, v        [B][Hkv][n_new][d] inputs, dtype in_dtype (fp32 or bf16).
 *  group       must be 32.
 *  pos         device int32 [B]: first cache row to write for each sequence.
 *              Rows with pos[b]+n >= capacity (or pos[b] < 0) are skipped on
 *              the device (no write); the host cannot check device memory.
 *  signs       device int8 [d] of +1/-1, or NULL for no rotation.  Each
 *              vector x is rotated to y = H_d (signs * x) / sqrt(d) before
 *              quantization.
 *  k_packed, v_packed  uint8 [B][Hkv][capacity][d/2] (written rows only).
 *  k_scales, v_scales  float [B][Hkv][capacity][d/32] (written rows only).
 *
 * With signs == NULL the codes and scales are bit-identical to the plain
 * definition (fp32 IEEE division, round half to even).  With rotation the
 * rotated vector is computed in fp32, so a code may differ by 1 from one
 * computed with an exactly rounded rotation.
 * Returns TQ_ERR_INVALID_ARG for NULL pointers (other than signs), B, Hkv or
 * n_new < 1, capacity < n_new, batch * num_kv_heads * n_new > 2^31 - 1,
 * misaligned pointers; TQ_ERR_UNSUPPORTED for
 * head_dim not in {128, 256} or group != 32.
 */
TQ_API tq_status tq_quantize_append(const void* k, const void* v, tq_dtype in_dtype, int32_t batch,
                             int32_t num_kv_heads, int32_t n_new, int32_t head_dim,
                             int32_t group, const int32_t* pos, const int8_t* signs,
                             uint8_t* k_packed, float* k_scales, uint8_t* v_packed,
                             float* v_scales, int64_t capacity, void* cuda_stream);

/*
 * tq_decode_workspace_bytes -- bytes of device workspace tq_sdpa_int4_decode
 * needs for these sizes (split-K partials and per-sequence flags).  Host only.
 * Returns 0 for invalid sizes.
 */
TQ_API size_t tq_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t max_ctx);

/*
 * tq_decode_chunk_tokens -- context tokens per split-K chunk that
 * tq_sdpa_int4_decode uses for these sizes (host only; a deterministic
 * function of its arguments).  Returns 0 for invalid sizes.
 */
TQ_API int32_t tq_decode_chunk_tokens(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                               int32_t head_dim, int32_t max_ctx);

/*
 * tq_sdpa_int4_decode -- GQA decode attention of one query token per
 * sequence over the packed int4 cache ("fused sdpa_int4": Open-TQ-Metal
 * abstract; no dequantized K/V matrix is formed: forum summary, section
 * "eliminating intermediate matrices"; fp32 accumulation with a running
 * maximum: section "numerical stability").
 *
 *  q           [B][Hq][d], dtype q_dtype, in the unrotated basis.
 *  Hq % Hkv == 0; query head h attends kv head h / (Hq / Hkv).
 *  ctx_lens    device int32 [B]: sequence b attends cache rows
 *              0 .. ctx_lens[b]-1.  Must satisfy 1 <= ctx_lens[b] <= max_ctx.
 *              Values outside that range are clamped on the device; every
 *              call writes int32 flag[b] at the start of the workspace: 1 if
 *              ctx_lens[b] was out of range, else 0.
 *  max_ctx     host bound on ctx_lens (grid sizing); max_ctx <= capacity.
 *  signs       the same signs the cache was written with, or NULL.
 *              The query is rotated by them; the output is rotated back.
 *  attn_scale  softmax temperature: scores = attn_scale * q.k (1/sqrt(d)
 *              for Llama-style models, 1.0 for Gemma 4: Open-TQ-Metal
 *              abstract).  Any finite value > 0.
 *  out         float [B][Hq][d], in the unrotated basis.
 *  workspace   device scratch of at least
 *              tq_decode_workspace_bytes(B, Hq, Hkv, d, max_ctx) bytes,
 *              16-byte aligned; contents need no initialization.
 *
 * Returns TQ_ERR_INVALID_ARG for NULL pointers (other than signs), shapes
 * that do not divide, max_ctx < 1 or > capacity, non-finite or non-positive
 * attn_scale, misaligned pointers; TQ_ERR_UNSUPPORTED for head_dim not in
 * {128, 256}, group != 32 or Hq/Hkv > 16; TQ_ERR_WORKSPACE when the
 * workspace is NULL or too small.
 */
TQ_API tq_status tq_sdpa_int4_decode(const void* q, tq_dtype q_dtype, int32_t batch,
                              int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                              int32_t group, const uint8_t* k_packed, const float* k_scales,
                              const uint8_t* v_packed, const float* v_scales, int64_t capacity,
                              const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs,
                              float attn_scale, float* out, void* workspace,
                              size_t workspace_bytes, void* cuda_stream);

/*
 * tq_sdpa_int4_decode_append -- one decode step in one call: the new token's K
 * and V of every (sequence, kv head) are quantized into the cache (as
 * tq_quantize_append does, bit-identically) and the query then attends over
 * the cache including that token ("quantize the KV cache as it is generated,
 * then attend on the compressed cache": Open-TQ-Metal abstract; forum summary,
 * section "on-the-fly quantization").
 *
 *  k_new, v_new  [B][Hkv][1][d] of kv_dtype (fp32 or bf16), unrotated.
 *  ctx_lens      lengths INCLUDING the new token: with T_b = ctx_lens[b]
 *                clamped to [1, max_ctx] (flagged as in tq_sdpa_int4_decode),
 *                the new token is written to row T_b - 1 and rows 0 .. T_b - 1
 *                are attended.
 *  Every other argument is as in tq_sdpa_int4_decode; the cache buffers are
 *  written (row T_b - 1 of each sequence and kv head) as well as read.
 *
 * On the tensor-core decode (head_dim 128 with Hq/Hkv <= 8, head_dim 256 with
 * Hq/Hkv <= 4) the decode kernel quantizes the new tokens itself: the CTA that
 * attends a sequence's last chunk writes its row before copying it, so the
 * step is the decode's launches only.  Otherwise a small append launch runs
 * first.  Returns the errors of tq_sdpa_int4_decode, and TQ_ERR_INVALID_ARG
 * for NULL or misaligned k_new / v_new or an invalid kv_dtype.
 */
TQ_API tq_status tq_sdpa_int4_decode_append(
    const void* q, tq_dtype q_dtype, const void* k_new, const void* v_new, tq_dtype kv_dtype,
    int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t group,
    uint8_t* k_packed, float* k_scales, uint8_t* v_packed, float* v_scales, int64_t capacity,
    const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs, float attn_scale, float* out,
    void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * tq_sdpa_int4_decode_append_host -- tq_sdpa_int4_decode_append with the step's
 * inputs and output in HOST memory: it enqueues the host-to-device copies of
 * q, k_new and v_new into staging space at the end of the workspace, the
 * decode step, and the device-to-host copy of the output, all on cuda_stream,
 * and returns without synchronizing (the output is in out_host once the stream
 * reaches that point).  When all four host buffers are page-locked and mapped
 * into the device's address space (cudaHostAlloc / cudaMallocHost memory under
 * unified addressing, as cudaPointerGetAttributes reports) and 16-byte
 * aligned, no copies are enqueued: a small kernel reads q, k_new and v_new
 * over the bus into the staging space and the merge kernel writes the output
 * into out_host directly (the same bytes cross the bus).  Otherwise
 * the inputs and output are staged as above; pageable memory works, the
 * copies then staging through the driver.  Either way the host buffers must
 * not change (inputs) or be read (output) until the stream has passed the step.
 *
 *  q_host          [B][Hq][d] of q_dtype; k_new_host, v_new_host [B][Hkv][1][d] of
 *                  kv_dtype; out_host [B][Hq][d] fp32.
 *  workspace       device, workspace_bytes >= tq_decode_append_host_workspace_bytes().
 * The cache buffers, ctx_lens and signs are device pointers, as in
 * tq_sdpa_int4_decode_append, whose errors it returns (TQ_ERR_INVALID_ARG also
 * for a NULL host pointer).
 */
TQ_API size_t tq_decode_append_host_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                                    int32_t num_kv_heads, int32_t head_dim,
                                                    int32_t max_ctx, tq_dtype q_dtype,
                                                    tq_dtype kv_dtype);

TQ_API tq_status tq_sdpa_int4_decode_append_host(
    const void* q_host, tq_dtype q_dtype, const void* k_new_host, const void* v_new_host,
    tq_dtype kv_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t group, uint8_t* k_packed, float* k_scales, uint8_t* v_packed, float* v_scales,
    int64_t capacity, const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs,
    float attn_scale, float* out_host, void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * tq_sdpa_int4_decode_lse -- tq_sdpa_int4_decode that also returns each head's
 * softmax state, so that outputs over disjoint parts of a context (for
 * instance the token shards of several GPUs) can be combined exactly with
 * tq_merge_lse.  The pages do not describe this step: it is split-K
 * flash-decoding's log-sum-exp merge taken across calls.
 *
 *  lse   float [B][Hq][2], 8-byte aligned: (M, L) per head, M the maximum of
 *        attn_scale * q.k over the attended tokens in log2 units and
 *        L = sum_t 2^(attn_scale * q.k_t * log2(e) - M), so that the head's
 *        output is sum_t 2^(... - M) v_t / L.
 * Every other argument and error is that of tq_sdpa_int4_decode;
 * TQ_ERR_INVALID_ARG also for a NULL or misaligned lse.
 */
TQ_API tq_status tq_sdpa_int4_decode_lse(
    const void* q, tq_dtype q_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t group, const uint8_t* k_packed, const float* k_scales,
    const uint8_t* v_packed, const float* v_scales, int64_t capacity, const int32_t* ctx_lens,
    int32_t max_ctx, const int8_t* signs, float attn_scale, float* out, float* lse,
    void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * tq_merge_lse -- combine n_parts outputs of tq_sdpa_int4_decode_lse over
 * disjoint parts of the same sequences' contexts into the output over their
 * union: M = max_r M_r, w_r = 2^(M_r - M) L_r, out = sum_r w_r out_r / sum_r w_r.
 *
 *  outs  float [n_parts][B][Hq][d] (16-byte aligned), lses float
 *        [n_parts][B][Hq][2] (8-byte aligned), out float [B][Hq][d]
 *        (16-byte aligned; may not alias outs).
 * Returns TQ_ERR_INVALID_ARG for NULL or misaligned pointers or sizes < 1,
 * TQ_ERR_UNSUPPORTED for head_dim not a multiple of 32 in [32, 256].
 */
TQ_API tq_status tq_merge_lse(const float* outs, const float* lses, int32_t n_parts, int32_t batch,
                              int32_t num_q_heads, int32_t head_dim, float* out, void* cuda_stream);

/*
 * tq_sdpa_int4_decode_static_scratch -- tq_sdpa_int4_decode without a
 * caller-provided workspace.  The method's pages have no counterpart to this
 * call; it exists for callers that cannot allocate device memory: a plug-in
 * running inside a host framework that owns all device memory and hands out
 * no scratch, or a latency-critical caller that cannot accept cudaMalloc's
 * device-wide synchronization.
 *
 * Arguments, validation and results are those of tq_sdpa_int4_decode; the
 * workspace is a file-scope device array of TQ_STATIC_SCRATCH_BYTES (8 MiB)
 * inside libtq, which every GPU that loads the library holds until the
 * process exits.  The call allocates nothing: no cudaMalloc, cudaFree or
 * allocating library routine.
 *  - Sizes whose workspace (tq_decode_workspace_bytes) exceeds
 *    TQ_STATIC_SCRATCH_BYTES are rejected with TQ_ERR_SCRATCH_LIMIT before
 *    any launch.
 *  - The first call on a device looks up the array's device address on that
 *    device (the current one); make that first call before any stream
 *    capture.  A failed lookup returns TQ_ERR_CUDA.
 *  - All calls on a device share the one array, which keeps the last call's
 *    contents.  The decode writes every scratch byte it reads, so nothing
 *    needs clearing between calls, but calls whose kernels overlap on the GPU
 *    (different streams without ordering between them) race on the array and
 *    give wrong results: order them on one stream or with events.
 */
TQ_API tq_status tq_sdpa_int4_decode_static_scratch(
    const void* q, tq_dtype q_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t group, const uint8_t* k_packed, const float* k_scales,
    const uint8_t* v_packed, const float* v_scales, int64_t capacity, const int32_t* ctx_lens,
    int32_t max_ctx, const int8_t* signs, float attn_scale, float* out, void* cuda_stream);

/*
 * tq_dequantize -- materialize dequantized rows of a packed cache: value of
 * coordinate i = scale[i/32] * code[i], in the rotated basis the cache holds
 * (the layout above).  Not part of the decode path, which never forms these
 * values (Open-TQ-Metal abstract: attention on the compressed representation
 * with no intermediate dequantized K/V matrix); it serves callers that need
 * the plain values, and a dequantize-then-attend comparison.
 *
 *  packed      uint8 rows of d/2 bytes, scales float rows of d/32: n_seq
 *              sequences of `rows` rows each, sequence s starting at row
 *              s * row_stride (e.g. n_seq = B * Hkv, row_stride = capacity).
 *  out         [n_seq][rows][d] of out_dtype (fp32: exact products; bf16:
 *              the fp32 product rounded to nearest even).
 *
 * Returns TQ_ERR_INVALID_ARG for NULL pointers, n_seq or rows < 1,
 * row_stride < rows, misaligned pointers (16 bytes); TQ_ERR_UNSUPPORTED for
 * head_dim not a multiple of 32 in [32, 256] or group != 32.
 */
TQ_API tq_status tq_dequantize(const uint8_t* packed, const float* scales, int32_t n_seq,
                               int32_t rows, int64_t row_stride, int32_t head_dim, int32_t group,
                               void* out, tq_dtype out_dtype, void* cuda_stream);

/*
 * SRFT variant of the rotation ("SRFT + int4 KV-cache on Apple Silicon",
 * core method: a sign-randomized Fourier transform in place of the Hadamard
 * one, suited to widths that are not powers of two, then a per-coordinate
 * scale lambda before the group abs-max quantization).  The transform is the
 * orthonormal discrete Hartley transform
 *     F[k][j] = (cos(2 pi k j / d) + sin(2 pi k j / d)) / sqrt(d),
 * the real member of the Fourier family (F = F^T, F F = I).  A cache written
 * by tq_quantize_append_srft holds, for every token,
 *     K row: y = lambda_k (.) F (signs (.) k),   V row: lambda_v (.) F (signs (.) v)
 * in the packed layout above, and the SRFT decode calls use
 *     q_r = F (signs (.) q) / lambda_k,   out = signs (.) F (o_r / lambda_v),
 * so q_r . y = q . k and the output is in the unrotated basis.
 *
 *  head_dim      any multiple of 32 from 32 to 256 (e.g. 96, 160, 192).
 *  signs         int8 [d] of +1/-1 (device), or NULL for all +1.
 *  lambda_k/_v   float [d] (device, 4-byte aligned) of positive finite values,
 *                or NULL for all 1.  Values are not checked on the device.
 * The cache, q, k/v and out layouts, alignment, ownership and errors are those
 * of the Hadamard calls; head_dim outside the set above gives
 * TQ_ERR_UNSUPPORTED, a misaligned lambda TQ_ERR_INVALID_ARG.  A cache must be
 * read with the rotation (signs, lambdas) it was written with.
 */

/* Workspace bytes for tq_sdpa_int4_decode_srft(_append): the split-K partials
 * plus the rotated queries (4 * B * Hq * d bytes); 0 for invalid sizes. */
TQ_API size_t tq_decode_srft_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                             int32_t num_kv_heads, int32_t head_dim,
                                             int32_t max_ctx);

/* tq_quantize_append with the SRFT rotation (one complex FFT per token turns
 * its K and V rows together). */
TQ_API tq_status tq_quantize_append_srft(
    const void* k, const void* v, tq_dtype in_dtype, int32_t batch, int32_t num_kv_heads,
    int32_t n_new, int32_t head_dim, int32_t group, const int32_t* pos, const int8_t* signs,
    const float* lambda_k, const float* lambda_v, uint8_t* k_packed, float* k_scales,
    uint8_t* v_packed, float* v_scales, int64_t capacity, void* cuda_stream);

/* tq_sdpa_int4_decode over an SRFT cache.  Launches: one query-rotation
 * kernel, the split-K decode (tensor cores for head_dim 128 with Hq/Hkv <= 8
 * and head_dim 256 with Hq/Hkv <= 4, CUDA cores otherwise) and the merge with
 * the inverse transform.  workspace_bytes >= tq_decode_srft_workspace_bytes(). */
TQ_API tq_status tq_sdpa_int4_decode_srft(
    const void* q, tq_dtype q_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t group, const uint8_t* k_packed, const float* k_scales,
    const uint8_t* v_packed, const float* v_scales, int64_t capacity, const int32_t* ctx_lens,
    int32_t max_ctx, const int8_t* signs, const float* lambda_k, const float* lambda_v,
    float attn_scale, float* out, void* workspace, size_t workspace_bytes, void* cuda_stream);

/* tq_sdpa_int4_decode_srft that also returns each head's softmax state (as
 * tq_sdpa_int4_decode_lse), for tq_merge_lse across context parts. */
TQ_API tq_status tq_sdpa_int4_decode_srft_lse(
    const void* q, tq_dtype q_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t group, const uint8_t* k_packed, const float* k_scales,
    const uint8_t* v_packed, const float* v_scales, int64_t capacity, const int32_t* ctx_lens,
    int32_t max_ctx, const int8_t* signs, const float* lambda_k, const float* lambda_v,
    float attn_scale, float* out, float* lse, void* workspace, size_t workspace_bytes,
    void* cuda_stream);

/* tq_sdpa_int4_decode_append over an SRFT cache: one launch quantizes the new
 * tokens (as tq_quantize_append_srft, bit-identically) and rotates the
 * queries, then the query attends. */
TQ_API tq_status tq_sdpa_int4_decode_append_srft(
    const void* q, tq_dtype q_dtype, const void* k_new, const void* v_new, tq_dtype kv_dtype,
    int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t group,
    uint8_t* k_packed, float* k_scales, uint8_t* v_packed, float* v_scales, int64_t capacity,
    const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs, const float* lambda_k,
    const float* lambda_v, float attn_scale, float* out, void* workspace, size_t workspace_bytes,
    void* cuda_stream);

/* tq_sdpa_int4_decode_append_srft with q, k_new, v_new and out in HOST memory,
 * as tq_sdpa_int4_decode_append_host (the same mapped-buffer and staging
 * forms); workspace_bytes >= tq_decode_append_host_srft_workspace_bytes(). */
TQ_API size_t tq_decode_append_host_srft_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                                         int32_t num_kv_heads, int32_t head_dim,
                                                         int32_t max_ctx, tq_dtype q_dtype,
                                                         tq_dtype kv_dtype);
TQ_API tq_status tq_sdpa_int4_decode_append_srft_host(
    const void* q_host, tq_dtype q_dtype, const void* k_new_host, const void* v_new_host,
    tq_dtype kv_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t group, uint8_t* k_packed, float* k_scales, uint8_t* v_packed, float* v_scales,
    int64_t capacity, const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs,
    const float* lambda_k, const float* lambda_v, float attn_scale, float* out_host,
    void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * Codebook variant (the AdapTQ post, sections "unified SIMD pipeline",
 * "precomputed lookup tables", "performance and quality": 2-, 3- and 4-bit
 * indices into a Max-Lloyd codebook with +-3 sigma clipping; int2 is the
 * future work of Open-TQ-Metal).  After the Hadamard rotation of the int4
 * calls (signs, or none), each group of 32 coordinates y stores
 *     sigma = fl32(sqrt(S / 32)), S = sum of y^2 accumulated in fp64,
 *     index_j = #{ i : u_j > t_i },  u_j = clamp(fl32(y_j / sigma), -3, 3)
 *               (u_j = 0 when sigma = 0),  t_i = fl32(fl32(C_i + C_{i+1}) * 0.5),
 * and the value sigma * C[index].  Layout (row-major, dense):
 *  - packed cache: uint8 [B][Hkv][capacity][d * bits / 8]; a row holds its
 *    d/32 groups in order, 4 * bits bytes each; index j of a group occupies
 *    bits bits*j .. bits*j + bits - 1 of the group's little-endian bit string.
 *  - scales: float [B][Hkv][capacity][d/32] (sigma per group).
 *  - levels: float [2^bits] on the device, strictly increasing (not checked
 *    on the device; the host checks only the pointer, 4-byte aligned).
 * head_dim 128 or 256; bits 2, 3 or 4 (else TQ_ERR_UNSUPPORTED); every other
 * argument, alignment rule and error is that of the int4 calls.  The decode
 * runs on the tensor cores for head_dim 128 with 5..8 query heads per kv head
 * (levels as f16 hi + lo parts read from a table over index pairs), on CUDA
 * cores otherwise (with 2 bits its scores there read tables of 16 partial dot
 * products per pair of query coordinates: the post's lookup tables).  Levels
 * of any finite magnitude are accepted: the tensor-core decode scales them by
 * a power of two before splitting them.
 */

/* The Gaussian Max-Lloyd codebook of 2^bits levels (N(0,1) cell means at
 * midpoint thresholds), written to a HOST array of 2^bits floats. */
TQ_API tq_status tq_lloyd_max_gaussian(int32_t bits, float* levels);

/* Workspace bytes for tq_sdpa_cb_decode(_append); 0 for invalid sizes. */
TQ_API size_t tq_decode_cb_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                           int32_t num_kv_heads, int32_t head_dim,
                                           int32_t max_ctx);

/* tq_quantize_append for a codebook cache (one warp per vector). */
TQ_API tq_status tq_quantize_append_cb(
    const void* k, const void* v, tq_dtype in_dtype, int32_t batch, int32_t num_kv_heads,
    int32_t n_new, int32_t head_dim, int32_t group, int32_t bits, const float* levels,
    const int32_t* pos, const int8_t* signs, uint8_t* k_packed, float* k_scales,
    uint8_t* v_packed, float* v_scales, int64_t capacity, void* cuda_stream);

/* tq_sdpa_int4_decode over a codebook cache (split-K decode + merge). */
TQ_API tq_status tq_sdpa_cb_decode(
    const void* q, tq_dtype q_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t group, int32_t bits, const float* levels, const uint8_t* k_packed,
    const float* k_scales, const uint8_t* v_packed, const float* v_scales, int64_t capacity,
    const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs, float attn_scale, float* out,
    void* workspace, size_t workspace_bytes, void* cuda_stream);

/* tq_sdpa_cb_decode that also returns each head's softmax state (as
 * tq_sdpa_int4_decode_lse), for tq_merge_lse across context parts. */
TQ_API tq_status tq_sdpa_cb_decode_lse(
    const void* q, tq_dtype q_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t group, int32_t bits, const float* levels, const uint8_t* k_packed,
    const float* k_scales, const uint8_t* v_packed, const float* v_scales, int64_t capacity,
    const int32_t* ctx_lens, int32_t max_ctx, const int8_t* signs, float attn_scale, float* out,
    float* lse, void* workspace, size_t workspace_bytes, void* cuda_stream);

/* tq_sdpa_int4_decode_append over a codebook cache (append launch, then decode). */
TQ_API tq_status tq_sdpa_cb_decode_append(
    const void* q, tq_dtype q_dtype, const void* k_new, const void* v_new, tq_dtype kv_dtype,
    int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t group,
    int32_t bits, const float* levels, uint8_t* k_packed, float* k_scales, uint8_t* v_packed,
    float* v_scales, int64_t capacity, const int32_t* ctx_lens, int32_t max_ctx,
    const int8_t* signs, float attn_scale, float* out, void* workspace, size_t workspace_bytes,
    void* cuda_stream);

/* tq_sdpa_cb_decode_append with q, k_new, v_new and out in HOST memory, as
 * tq_sdpa_int4_decode_append_host (the same mapped-buffer and staging forms);
 * workspace_bytes >= tq_decode_append_host_cb_workspace_bytes(). */
TQ_API size_t tq_decode_append_host_cb_workspace_bytes(int32_t batch, int32_t num_q_heads,
                                                       int32_t num_kv_heads, int32_t head_dim,
                                                       int32_t max_ctx, tq_dtype q_dtype,
                                                       tq_dtype kv_dtype);
TQ_API tq_status tq_sdpa_cb_decode_append_host(
    const void* q_host, tq_dtype q_dtype, const void* k_new_host, const void* v_new_host,
    tq_dtype kv_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t group, int32_t bits, const float* levels, uint8_t* k_packed, float* k_scales,
    uint8_t* v_packed, float* v_scales, int64_t capacity, const int32_t* ctx_lens,
    int32_t max_ctx, const int8_t* signs, float attn_scale, float* out_host, void* workspace,
    size_t workspace_bytes, void* cuda_stream);

/*
 * Uniform low-bit variant (Open-TQ-Metal forum summary, future work: int2;
 * read as the int4 quantizer at fewer bits).  With m = 2^(bits-1) - 1 each
 * group of 32 rotated coordinates y stores
 *     s = fl32(amax / m) (IEEE fp32 division; s = amax at two bits),
 *     index_j = clamp(rne(fl32(y_j / s)), -m, m) + m   (0 codes when s = 0),
 * in the codebook layout above, scales = s.  The value is s * (index - m): a
 * uniform cache is a codebook cache whose levels are the integers u - m
 * (tq_uniform_levels), so tq_sdpa_cb_decode, tq_sdpa_cb_decode_lse and
 * tq_decode_cb_workspace_bytes serve it with those levels.  Only the calls
 * that quantize differ: tq_quantize_append_uniform, and the decode steps that
 * append the new token, whose levels argument must hold tq_uniform_levels(bits)
 * on the device.  bits 2, 3 or 4 (4 gives the int4 codes in this layout);
 * arguments, alignment and errors as the codebook calls.
 */

/* levels[u] = u - m for u < 2^bits, written to a HOST array of 2^bits floats. */
TQ_API tq_status tq_uniform_levels(int32_t bits, float* levels);

/* tq_quantize_append into a uniform low-bit cache (one warp per vector). */
TQ_API tq_status tq_quantize_append_uniform(
    const void* k, const void* v, tq_dtype in_dtype, int32_t batch, int32_t num_kv_heads,
    int32_t n_new, int32_t head_dim, int32_t group, int32_t bits, const int32_t* pos,
    const int8_t* signs, uint8_t* k_packed, float* k_scales, uint8_t* v_packed, float* v_scales,
    int64_t capacity, void* cuda_stream);

/* tq_sdpa_cb_decode_append for a uniform cache: the new token is quantized
 * with the uniform rule (inside the decode launch where the codebook decode
 * does that), then the decode runs with `levels` (= tq_uniform_levels). */
TQ_API tq_status tq_sdpa_uniform_decode_append(
    const void* q, tq_dtype q_dtype, const void* k_new, const void* v_new, tq_dtype kv_dtype,
    int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t group,
    int32_t bits, const float* levels, uint8_t* k_packed, float* k_scales, uint8_t* v_packed,
    float* v_scales, int64_t capacity, const int32_t* ctx_lens, int32_t max_ctx,
    const int8_t* signs, float attn_scale, float* out, void* workspace, size_t workspace_bytes,
    void* cuda_stream);

/* tq_sdpa_uniform_decode_append with q, k_new, v_new and out in HOST memory
 * (as tq_sdpa_cb_decode_append_host; its workspace size call serves). */
TQ_API tq_status tq_sdpa_uniform_decode_append_host(
    const void* q_host, tq_dtype q_dtype, const void* k_new_host, const void* v_new_host,
    tq_dtype kv_dtype, int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t group, int32_t bits, const float* levels, uint8_t* k_packed, float* k_scales,
    uint8_t* v_packed, float* v_scales, int64_t capacity, const int32_t* ctx_lens,
    int32_t max_ctx, const int8_t* signs, float attn_scale, float* out_host, void* workspace,
    size_t workspace_bytes, void* cuda_stream);

/*
 * tq_set_test_hooks -- testing only; leave at 0 (the default) in normal use.
 * Sets process-wide switches read once by every later decode or quantize
 * call:
 *  - TQ_TEST_HOOK_FAIL_LAUNCH: decode calls return TQ_ERR_CUDA after
 *    validation, before enqueueing anything (as a failed launch would).
 *  - TQ_TEST_HOOK_STARVE_PIPELINE: the tensor-core decode kernels and the
 *    tensor-core bulk quantize withhold each CTA's first copy, so their
 *    bounded waits run out (about 2 s); a decode's outputs are then NaN, a
 *    bulk quantize writes NaN scales into the rows it did not finish, and the
 *    context stays usable.
 *  - TQ_TEST_HOOK_TCGEN05_DECODE: the int4 decode at head_dim 128 with up to
 *    8 query heads per kv head runs on the tcgen05 / tensor-memory kernel
 *    instead of the default warp-level mma.sync kernel (for comparing the
 *    two; the default is the faster one on B200 for this decode).
 *  - TQ_TEST_HOOK_BUTTERFLY_QUANTIZE: bulk quantize-appends of bf16 vectors
 *    at head_dim 128 with rotation rotate with fp32 butterflies on the CUDA
 *    cores instead of the tensor-core product (for comparing the two).
 * No counterpart on the method's pages.
 */
#define TQ_TEST_HOOK_FAIL_LAUNCH 1u
#define TQ_TEST_HOOK_STARVE_PIPELINE 2u
#define TQ_TEST_HOOK_TCGEN05_DECODE 4u
#define TQ_TEST_HOOK_BUTTERFLY_QUANTIZE 8u
TQ_API void tq_set_test_hooks(uint32_t hooks);

/* tq_status_string -- static English text for a status code. */
TQ_API const char* tq_status_string(tq_status status);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
