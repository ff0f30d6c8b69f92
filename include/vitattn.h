/*
 * vitattn.h -- C ABI of libvitattn: the forward pass of non-causal multi-head
 * scaled-dot-product attention inside a vision-transformer encoder block, on
 * one NVIDIA B200 (sm_100a).
 *
 * The operation.  For every batch b < B and head h < H, with
 * Q_bh[i,:] = q[b,i,h,:] (likewise K_bh, V_bh):
 *
 *     O_bh = softmax(scale * Q_bh K_bh^T) V_bh        (row softmax, no mask)
 *
 * written to out[b,i,h,:].  Sources: hf2q "src/inference/vision/vit_gpu.rs",
 * doc of `vit_attention_gpu` (scores, softmax, P.V; inputs and output
 * seq-major [batch, num_heads, head_dim]; no mask because a ViT is
 * bidirectional) and of `vit_attention_scores_gpu` (the caller's scale is
 * applied as given, with no implicit 1/sqrt(head_dim)); inferencelayer
 * "src/vision_gpu.rs", doc of `vis_attn_coop_src` (Q.K^T and P.V as GEMMs
 * with an online softmax that rescales the running output); hanzo-ml
 * "src/vulkan_backend.rs", `flash_attn_gpu` (the (q, k, v, sizes, scale)
 * calling shape and argument checks before dispatch).
 *
 * Entry points (each documented below):
 *   vitattn_forward          the operation above (self-attention, Lq = Lk = N)
 *   vitattn_forward_varlen   a ragged batch of images packed along one axis
 *   vitattn_forward_gqa      grouped-query attention (fewer key/value heads)
 *   vitattn_forward_ext      Lq != Lk, aligned causal mask, log-sum-exp output
 *   vitattn_qkv_rope         the prologue: packed QKV split + rotary embedding
 *   vitattn_qkv_norm_rope    the same with a per-head q/k RMS norm before the rope
 *   vitattn_forward_strided  vitattn_forward on token-strided inputs (a packed projection)
 *   vitattn_qk_rope, vitattn_qk_norm_rope  the prologues without the v copy
 *   vitattn_forward_host     vitattn_forward from host buffers (copies overlapped)
 *   ..._checked, ..._check_args*, vitattn_strerror, vitattn_last_cuda_error,
 *   vitattn_version, vitattn_launches_per_call: synchronising variants for
 *   tests, argument checks alone, status text, versioning.
 *
 * Layout.  q, k, v and out are dense, token-major [B, N, H, D] tensors with D
 * contiguous: element (b, i, h, d) at ((b*N + i)*H + h)*D + d.  That is the
 * layout a QKV linear produces once its output is split into three.
 * Lq = Lk = N (self-attention) for vitattn_forward.  out has the dtype of the
 * inputs; products and sums accumulate in fp32.  The probabilities enter the P.V product as
 * f16 for both dtypes (f16 carries three more mantissa bits than bf16), and
 * for bf16 inputs V is converted to f16 for that product: exact for
 * |v| < 65536 outside f16's subnormal range (|v| < 2^-14, where the absolute
 * error stays below 2^-25).  A bf16 V value of magnitude >= 65536 (or an
 * infinite one) becomes inf in that product; vitattn_forward_checked reports
 * it as VITATTN_ERR_RANGE.
 *
 * Ownership.  The caller owns every buffer.  The library allocates no device
 * memory, keeps no reference to any buffer after a call returns, and never
 * frees caller memory.  out must not overlap q, k or v.
 *
 * Streams and errors.  Calls enqueue work on `stream` and return without
 * synchronising (except the ..._checked entries).  Every argument is checked
 * before anything is enqueued; a failed check returns a negative status and
 * enqueues nothing.  A CUDA error raised while enqueueing returns
 * VITATTN_ERR_CUDA (its cudaError_t value via vitattn_last_cuda_error()).
 * Errors that happen later on the device surface through the stream, as for
 * any CUDA kernel.  Every internal wait of the kernel is bounded in time; a
 * wait that runs out ends the kernel early and records VITATTN_ERR_TIMEOUT in
 * a device status word, which vitattn_forward_checked reports.
 *
 * Devices.  Every call runs on the current CUDA device.  Each device pointer
 * must be that device's memory (or managed / mapped pinned memory); a
 * pointer to plain host memory or to another GPU's memory is refused with
 * VITATTN_ERR_DEVICE before anything is enqueued.
 *
 * Thread safety.  Calls may come from several host threads; each call
 * launches on its own stream argument and keeps no state between calls.
 * One exception: the ..._checked entries (meant for tests) read two status
 * words that every call of the library on a device shares, so checked calls
 * that overlap in time on one device (several threads or streams) can see
 * each other's timeout or range report.
 */
#ifndef VITATTN_H
#define VITATTN_H

#include <stdint.h>

#if defined(__GNUC__)
#define VITATTN_API __attribute__((visibility("default")))
#else
#define VITATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream.  NULL means the legacy default stream. */
typedef struct CUstream_st* vitattn_stream_t;

/* Element type of q, k, v and out. */
enum vitattn_dtype {
    VITATTN_BF16 = 0, /* bfloat16 */
    VITATTN_F16 = 1   /* IEEE binary16 */
};

/* Return codes.  0 is success; every error is negative. */
enum vitattn_status {
    VITATTN_OK = 0,
    VITATTN_ERR_NULL = -1,    /* a required pointer is NULL */
    VITATTN_ERR_DIM = -2,     /* B, N or H < 1, or a size or offset would overflow */
    VITATTN_ERR_HEADDIM = -3, /* D unsupported: needs 16 <= D <= 128 and D % 8 == 0 */
    VITATTN_ERR_DTYPE = -4,   /* dtype is not a vitattn_dtype */
    VITATTN_ERR_ALIGN = -5,   /* a tensor pointer is not 16-byte aligned */
    VITATTN_ERR_ALIAS = -6,   /* out overlaps q, k or v */
    VITATTN_ERR_CUDA = -7,    /* the CUDA runtime or driver returned an error */
    VITATTN_ERR_TIMEOUT = -8, /* a bounded in-kernel wait ran out (checked entry only) */
    VITATTN_ERR_SCALE = -9,   /* scale is NaN or infinite (or eps negative / not finite) */
    VITATTN_ERR_DEVICE = -10, /* the current device is not an sm_100 GPU, or a pointer argument is plain
                                 host memory or another GPU's memory */
    VITATTN_ERR_RANGE = -11,  /* a bf16 V value has |v| >= 65536 (checked entry only) */
    VITATTN_ERR_SEQLENS = -12 /* cu_seqlens does not start at 0 or decreases somewhere */
};

/*
 * vitattn_forward -- out = softmax(scale * Q K^T) V per (batch, head).
 *   q, k, v  device pointers, [B, N, H, D] of `dtype`, 16-byte aligned.
 *   out      device pointer, [B, N, H, D] of `dtype`, 16-byte aligned,
 *            not overlapping q, k or v.  Every element is written.
 *   B, N, H  batch, tokens per sequence, heads (all >= 1).
 *   D        head dimension: 16 <= D <= 128, D % 8 == 0.
 *   scale    multiplies Q K^T as given (pass 1/sqrt(D) for a standard ViT).
 *   dtype    VITATTN_BF16 or VITATTN_F16.
 *   stream   stream to launch on.
 * Launches exactly one kernel on the current CUDA device and returns.
 */
VITATTN_API int vitattn_forward(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t N,
                    int64_t H, int64_t D, float scale, int dtype, vitattn_stream_t stream);

/*
 * vitattn_forward_checked -- vitattn_forward, then a stream synchronisation
 * and a read of the kernel's status words.  Returns VITATTN_ERR_TIMEOUT when a
 * bounded in-kernel wait ran out, VITATTN_ERR_RANGE when a bf16 V value was
 * outside the f16 range of the P.V product (out then holds inf or NaN in the
 * affected rows), VITATTN_ERR_CUDA when the stream reported an error.  Meant
 * for tests and debugging: it blocks the calling thread.  Checked calls that
 * overlap in time (several streams or threads) share the status words.
 */
VITATTN_API int vitattn_forward_checked(const void* q, const void* k, const void* v, void* out, int64_t B,
                            int64_t N, int64_t H, int64_t D, float scale, int dtype,
                            vitattn_stream_t stream);

/*
 * vitattn_forward_ext -- separate query and key lengths, an optional aligned
 * causal mask, and an optional log-sum-exp output.  Source: hanzo-ml
 * "src/vulkan_backend.rs", `flash_attn_gpu` (q [BH, Lq, D], k/v [BH, Lk, D];
 * `scale` multiplies Q K^T; `causal` applies aligned causal masking: query qi
 * attends to keys <= qi + (Lk - Lq)).
 *   q, out    [B, Lq, H, D];  k, v  [B, Lk, H, D] (token-major, as
 *             vitattn_forward); Lq, Lk >= 1.
 *   lse       NULL, or a 16-byte aligned device pointer to [B, H, Lq] float32
 *             receiving log(sum_j exp(scale * q_i . k_j)) over the keys row i
 *             sees (natural log), from the f32 sum of the probabilities
 *             (computed with the hardware exp2 approximation): within ~1e-3
 *             of the exact value.
 *   causal    nonzero: the aligned causal mask above.  A row that sees no key
 *             (only when Lq > Lk) is written as 0 with lse = -inf.
 * Lq = Lk with causal = 0 and lse = NULL is exactly vitattn_forward.
 */
VITATTN_API int vitattn_forward_ext(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B,
                                    int64_t Lq, int64_t Lk, int64_t H, int64_t D, float scale, int causal,
                                    int dtype, vitattn_stream_t stream);

/* vitattn_forward_ext, then a stream synchronisation and a read of the kernel's status words. */
VITATTN_API int vitattn_forward_ext_checked(const void* q, const void* k, const void* v, void* out, float* lse,
                                            int64_t B, int64_t Lq, int64_t Lk, int64_t H, int64_t D, float scale,
                                            int causal, int dtype, vitattn_stream_t stream);

/* The argument checks of vitattn_forward_ext alone (no CUDA call). */
VITATTN_API int vitattn_check_args_ext(const void* q, const void* k, const void* v, const void* out,
                                       const float* lse, int64_t B, int64_t Lq, int64_t Lk, int64_t H, int64_t D,
                                       float scale, int dtype);

/*
 * vitattn_forward_gqa -- grouped-query attention: H query heads share Hkv
 * key/value heads, query head h using key/value head h / (H / Hkv).
 * Source: hf2q "src/inference/vision/vit_gpu.rs", doc of `vit_repeat_kv_gpu`
 * (each kv head replicated num_kv_groups times; output row h reads kv head
 * h / num_kv_groups).  No replicated copy is made: each CTA reads its kv
 * head directly.
 *   q, out    [B, N, H, D];  k, v  [B, N, Hkv, D];  1 <= Hkv, H % Hkv == 0
 *             (VITATTN_ERR_DIM otherwise).  Everything else as for
 *             vitattn_forward (Hkv = H is exactly vitattn_forward).
 */
VITATTN_API int vitattn_forward_gqa(const void* q, const void* k, const void* v, void* out, int64_t B, int64_t N,
                                    int64_t H, int64_t Hkv, int64_t D, float scale, int dtype,
                                    vitattn_stream_t stream);

/* vitattn_forward_gqa, then a stream synchronisation and a read of the kernel's status words. */
VITATTN_API int vitattn_forward_gqa_checked(const void* q, const void* k, const void* v, void* out, int64_t B,
                                            int64_t N, int64_t H, int64_t Hkv, int64_t D, float scale, int dtype,
                                            vitattn_stream_t stream);

/* The argument checks of vitattn_forward_gqa alone (no CUDA call). */
VITATTN_API int vitattn_check_args_gqa(const void* q, const void* k, const void* v, const void* out, int64_t B,
                                       int64_t N, int64_t H, int64_t Hkv, int64_t D, float scale, int dtype);

/* Most segments one vitattn_forward_varlen call takes. */
#define VITATTN_MAX_SEQS 256

/*
 * vitattn_forward_varlen -- a ragged batch of images: the tokens of num_seqs
 * images packed along one axis, each attending only within its own image.
 * Source: inferencelayer "src/vision_gpu.rs", the vision tower's `forward`
 * (attention over an image is one ragged segment given by its start
 * offsets; several images are several segments).
 *   q, k, v   device pointers, [total, H, D] of `dtype` (token-major, D
 *             contiguous), total = cu_seqlens[num_seqs]; 16-byte aligned.
 *   out       device pointer, [total, H, D], not overlapping q, k or v.
 *             Every element of every token is written.
 *   cu_seqlens  HOST pointer to num_seqs + 1 int32 offsets, cu_seqlens[0] = 0,
 *             nondecreasing: segment s is tokens cu_seqlens[s] ..
 *             cu_seqlens[s+1] - 1 (empty segments are allowed).  Read before
 *             the call returns; not retained.
 *   num_seqs  1 .. VITATTN_MAX_SEQS.
 *   H, D, scale, dtype, stream: as for vitattn_forward.
 * For token i of segment s and head h:
 *     out[i,h,:] = softmax_j(scale * q[i,h,:] . k[j,h,:]) v[j,h,:], j in segment s.
 * total = 0 enqueues nothing and returns VITATTN_OK.  Returns
 * VITATTN_ERR_SEQLENS for malformed offsets, VITATTN_ERR_DIM for num_seqs out
 * of range; other errors as for vitattn_forward.  Launches one kernel.
 * A segment's key blocks may overlap the next segment's tokens in memory;
 * those keys get probability 0, so values there must be finite (a NaN or inf
 * in a neighbouring token's v can reach this segment's output as NaN).
 */
VITATTN_API int vitattn_forward_varlen(const void* q, const void* k, const void* v, void* out,
                                       const int32_t* cu_seqlens, int64_t num_seqs, int64_t H, int64_t D,
                                       float scale, int dtype, vitattn_stream_t stream);

/* vitattn_forward_varlen, then a stream synchronisation and a read of the
 * kernel's status words, as vitattn_forward_checked. */
VITATTN_API int vitattn_forward_varlen_checked(const void* q, const void* k, const void* v, void* out,
                                               const int32_t* cu_seqlens, int64_t num_seqs, int64_t H,
                                               int64_t D, float scale, int dtype, vitattn_stream_t stream);

/* The argument checks of vitattn_forward_varlen alone (no CUDA call). */
VITATTN_API int vitattn_check_args_varlen(const void* q, const void* k, const void* v, const void* out,
                                          const int32_t* cu_seqlens, int64_t num_seqs, int64_t H, int64_t D,
                                          float scale, int dtype);

/*
 * vitattn_qkv_rope -- the attention's prologue: split a packed QKV projection
 * into q, k, v and apply the rotary embedding to q and k, in one pass.
 * Source: inferencelayer "src/vision_gpu.rs", VIS_QKV_ROPE and its doc (the
 * projection output is q | k | v per token; the rope tables arrive
 * precomputed, so a 2-D rope is whatever row/column walk built them;
 * rotate_half pairs element d with d +- D/2, negated on the low half; v is
 * not rotated).
 *   qkv       device pointer, [T, 3, H, D] of `dtype` (token-major: each
 *             token's q heads, then its k heads, then its v heads).
 *   cos_table, sin_table  device pointers, [T, D] float32, one row per token
 *             (shared by every head).
 *   q, k, v   device pointers, [T, H, D] of `dtype`: the layout the
 *             attention entries read (T = B*N dense, or the ragged total).
 *             They must not overlap each other or the inputs.
 *   T, H      tokens and heads (>= 1); D as for vitattn_forward (16..128,
 *             D % 8 == 0).  All pointers 16-byte aligned.
 * Per token t, head h, and x = q or k:
 *     x'[d] = x[d] * cos[t,d] + r[d] * sin[t,d],
 *     r[d]  = -x[d + D/2] (d < D/2),  x[d - D/2] (d >= D/2),
 * computed in f32 and rounded once to `dtype`; v is copied bit for bit.
 * Enqueues one kernel on `stream`; errors as for vitattn_forward.
 */
VITATTN_API int vitattn_qkv_rope(const void* qkv, const float* cos_table, const float* sin_table, void* q,
                                 void* k, void* v, int64_t T, int64_t H, int64_t D, int dtype,
                                 vitattn_stream_t stream);

/* The argument checks of vitattn_qkv_rope alone (no CUDA call). */
VITATTN_API int vitattn_check_args_qkv_rope(const void* qkv, const float* cos_table, const float* sin_table,
                                            const void* q, const void* k, const void* v, int64_t T, int64_t H,
                                            int64_t D, int dtype);

/*
 * vitattn_qkv_norm_rope -- the prologue with a per-head RMS norm of q and k
 * ahead of the rotary embedding, in one pass.
 * Source: inferencelayer "src/vision_gpu.rs", GLM_QKV_QKNORM_ROPE and its doc
 * (GLM-OCR vision tower: split the packed qkv, normalise each head's q and k
 * row over its head_dim elements with a per-element weight, BEFORE the rope;
 * then the rope of vitattn_qkv_rope; v passes through).
 *   qkv, cos_table, sin_table, q, k, v, T, H, D, dtype  as for
 *             vitattn_qkv_rope.
 *   q_norm_w, k_norm_w  device pointers, [D] float32 each, 16-byte aligned:
 *             the weights of the q norm and of the k norm (one vector for
 *             all heads).  They must not overlap an output.
 *   eps       finite, >= 0 (else VITATTN_ERR_SCALE).  With eps = 0 a head
 *             row of zeros has no defined norm and its output is NaN.
 * Per token t, head h, x = q or k and its weight w:
 *     y[d]  = x[d] / sqrt(mean_e x[e]^2 + eps) * w[d],
 *     x'[d] = y[d] * cos[t,d] + r[d] * sin[t,d],
 *     r[d]  = -y[d + D/2] (d < D/2),  y[d - D/2] (d >= D/2),
 * computed in f32 (IEEE square root and divide) and rounded once to `dtype`;
 * v is copied bit for bit.  Enqueues one kernel on `stream`; errors as for
 * vitattn_forward.
 */
VITATTN_API int vitattn_qkv_norm_rope(const void* qkv, const float* cos_table, const float* sin_table,
                                      const float* q_norm_w, const float* k_norm_w, float eps, void* q, void* k,
                                      void* v, int64_t T, int64_t H, int64_t D, int dtype,
                                      vitattn_stream_t stream);

/* The argument checks of vitattn_qkv_norm_rope alone (no CUDA call). */
VITATTN_API int vitattn_check_args_qkv_norm_rope(const void* qkv, const float* cos_table, const float* sin_table,
                                                 const float* q_norm_w, const float* k_norm_w, float eps,
                                                 const void* q, const void* k, const void* v, int64_t T,
                                                 int64_t H, int64_t D, int dtype);

/*
 * vitattn_forward_strided -- vitattn_forward on inputs whose tokens are not
 * packed back to back: element (b, i, h, d) of q sits at
 * q[((b*N + i)*q_stride + h*D + d)], likewise k (k_stride) and v (v_stride).
 * The use: a QKV linear writes one packed [B, N, 3, H, D] projection; with
 * q = qkv, k = qkv + H*D, v = qkv + 2*H*D and all strides 3*H*D the attention
 * reads it in place, and after vitattn_qk_rope (which rotates q and k into
 * their own buffers) v still comes straight from the projection, so the
 * prologue never copies it.  Source: inferencelayer "src/vision_gpu.rs",
 * VIS_QKV_ROPE doc (the projection output is q | k | v per token; the
 * attention's q, k, v are three column ranges of it).
 *   q_stride, k_stride, v_stride  elements between consecutive tokens,
 *             each >= H*D and a multiple of 8 (token rows start on 16 bytes);
 *             H*D everywhere is exactly vitattn_forward.
 *   out       dense [B, N, H, D], not overlapping any input's span; the
 *             inputs may overlap one another (views of one projection).
 *   Everything else as for vitattn_forward (VITATTN_ERR_DIM for a bad stride).
 */
VITATTN_API int vitattn_forward_strided(const void* q, const void* k, const void* v, void* out, int64_t B,
                                        int64_t N, int64_t H, int64_t D, int64_t q_stride, int64_t k_stride,
                                        int64_t v_stride, float scale, int dtype, vitattn_stream_t stream);

/* vitattn_forward_strided, then a stream synchronisation and a read of the kernel's status words. */
VITATTN_API int vitattn_forward_strided_checked(const void* q, const void* k, const void* v, void* out, int64_t B,
                                                int64_t N, int64_t H, int64_t D, int64_t q_stride,
                                                int64_t k_stride, int64_t v_stride, float scale, int dtype,
                                                vitattn_stream_t stream);

/* The argument checks of vitattn_forward_strided alone (no CUDA call). */
VITATTN_API int vitattn_check_args_strided(const void* q, const void* k, const void* v, const void* out, int64_t B,
                                           int64_t N, int64_t H, int64_t D, int64_t q_stride, int64_t k_stride,
                                           int64_t v_stride, float scale, int dtype);

/*
 * vitattn_qk_rope -- vitattn_qkv_rope without the v output: q and k are
 * rotated into [T, H, D] buffers and v is neither read nor written (the
 * attention reads it from qkv through vitattn_forward_strided with
 * v_stride = 3*H*D).  Source: inferencelayer "src/vision_gpu.rs",
 * VIS_QKV_ROPE and its doc ("pure data movement plus one rotation": the
 * rotation applies to q and k only).  Arguments and errors as for
 * vitattn_qkv_rope without v.  Enqueues one kernel on `stream`.
 */
VITATTN_API int vitattn_qk_rope(const void* qkv, const float* cos_table, const float* sin_table, void* q, void* k,
                                int64_t T, int64_t H, int64_t D, int dtype, vitattn_stream_t stream);

/* The argument checks of vitattn_qk_rope alone (no CUDA call). */
VITATTN_API int vitattn_check_args_qk_rope(const void* qkv, const float* cos_table, const float* sin_table,
                                           const void* q, const void* k, int64_t T, int64_t H, int64_t D,
                                           int dtype);

/*
 * vitattn_qk_norm_rope -- vitattn_qkv_norm_rope without the v output (v
 * stays in qkv, as for vitattn_qk_rope).  Source: inferencelayer
 * "src/vision_gpu.rs", GLM_QKV_QKNORM_ROPE and its doc.
 */
VITATTN_API int vitattn_qk_norm_rope(const void* qkv, const float* cos_table, const float* sin_table,
                                     const float* q_norm_w, const float* k_norm_w, float eps, void* q, void* k,
                                     int64_t T, int64_t H, int64_t D, int dtype, vitattn_stream_t stream);

/* The argument checks of vitattn_qk_norm_rope alone (no CUDA call). */
VITATTN_API int vitattn_check_args_qk_norm_rope(const void* qkv, const float* cos_table, const float* sin_table,
                                                const float* q_norm_w, const float* k_norm_w, float eps,
                                                const void* q, const void* k, int64_t T, int64_t H, int64_t D,
                                                int dtype);

/*
 * vitattn_forward_host -- the same operation from HOST buffers: the copies
 * hq->dq, hk->dk, hv->dv, the attention, and dout->hout.  Source: hanzo-ml
 * "src/vulkan_backend.rs", `flash_attn` (the host-data convenience form of
 * `flash_attn_gpu`: upload the inputs, run the device entry, read the
 * output back).  Here the caller supplies the device staging buffers, so
 * the library still allocates no memory.
 *   The work is cut into groups: up to 8 runs of whole images when B >= 8,
 *   otherwise up to 16 groups of heads of one image each (rows of at least
 *   512 bytes of each token's heads, copied with 2-D copies; heads are
 *   independent).  Group
 *   c's inputs are copied in while the kernel of group c-1 runs and the
 *   output of group c-2 is copied out.  The copies run on two streams the
 *   library keeps per host thread and device (created on the first call);
 *   the kernels run on `stream`.  The copies start after the work already
 *   enqueued on `stream`, and work enqueued on `stream` after this call (or
 *   a synchronisation of `stream`) comes after the last output copy, so the
 *   caller synchronises `stream` before reading hout, as with one stream.
 *   Host buffers should be pinned (cudaHostAlloc / cudaHostRegister) for the
 *   copies to overlap; dq, dk, dv, dout are caller-owned device staging with
 *   the requirements of vitattn_forward.  All eight pointers are required.
 *   Launches one kernel per group.  A group of heads writes its part of the
 *   output rows; the other heads' columns of dout are left to their groups.
 */
VITATTN_API int vitattn_forward_host(const void* hq, const void* hk, const void* hv, void* hout, void* dq,
                         void* dk, void* dv, void* dout, int64_t B, int64_t N, int64_t H,
                         int64_t D, float scale, int dtype, vitattn_stream_t stream);

/*
 * vitattn_check_args -- the argument checks of vitattn_forward, alone: no
 * CUDA call is made, so it runs on a machine without a GPU.  Returns
 * VITATTN_OK or the status vitattn_forward would return for these arguments
 * before touching the device.
 */
VITATTN_API int vitattn_check_args(const void* q, const void* k, const void* v, const void* out, int64_t B,
                       int64_t N, int64_t H, int64_t D, float scale, int dtype);

/* Static text for a status code ("unknown status" for anything else). */
VITATTN_API const char* vitattn_strerror(int status);

/* The cudaError_t of the most recent VITATTN_ERR_CUDA on the calling thread (0 if none). */
VITATTN_API int vitattn_last_cuda_error(void);

/* Library version as major*10000 + minor*100 + patch. */
VITATTN_API int vitattn_version(void);

/* Kernel launches one vitattn_forward call makes (for launch accounting). */
VITATTN_API int vitattn_launches_per_call(void);

#ifdef __cplusplus
}
#endif

#endif /* VITATTN_H */
