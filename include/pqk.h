/*
 * pqk.h -- C ABI of libpqk, the B200 (sm_100a) hot path of one block of a
 * joint video + audio diffusion transformer: fused Q/K RMSNorm + RoPE,
 * packed variable-length self-attention, and fused adaLN modulation +
 * gated residual + SwiGLU.
 *
 * Source of the operations: "FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长"
 * (sections "长序列注意力与通信优化" and "融合 DiT 算子") and "MiniMax H3 FastH3
 * real-time serving with vLLM-Omni" (section "System-wide optimizations in
 * vLLM-Omni", bullets "Long-sequence attention & communication" and "Fused
 * DiT operators"). The pages describe what is fused and that packed
 * sequences carry no padding; the conventions they leave open are fixed
 * below and stated per call.
 *
 * General contract
 *   - Every pointer argument named *device* is CUDA device memory owned by the
 *     caller; the library allocates nothing and keeps no per-call state.
 *   - bf16 means IEEE bfloat16 (2 bytes). Tensors are row-major as stated.
 *   - Every device pointer must be 16-byte aligned; every row stride is in
 *     elements and must be a multiple of 8 (16 bytes).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Every call is asynchronous on it: it validates its arguments
 *     on the host, enqueues kernels and returns. Argument errors are
 *     reported before anything is enqueued.
 *   - Return value: PQK_OK (0) or a negative pqk_status. Conditions found by
 *     the GPU while running (invalid cu_seqlens contents, a pipeline wait
 *     that ran out) are written to a per-device status word; read it with
 *     pqk_get_device_status after the work completes.
 *   - All calls are deterministic: the same inputs give bit-identical
 *     outputs on every run (no floating-point atomics, fixed reduction
 *     order).
 *   - Input and output buffers must not partially overlap. Exact in-place
 *     use (output pointer == input pointer, same layout) is allowed where
 *     stated.
 *   - CUDA graphs: the compute calls enqueue only kernels and stream-ordered
 *     memory operations (tensor maps are encoded on the host and passed by
 *     value), so they can be captured and replayed. The first call of each
 *     compute entry point on a device queries and caches device attributes
 *     and kernel settings; make it before capturing. pqk_get_device_status
 *     synchronizes and must not be captured.
 *   - Per-device state (the status word's device address, cached device
 *     attributes) is looked up once per device and kept for the life of its
 *     CUDA context: do not use the library on a device after destroying and
 *     recreating its context (cudaDeviceReset).
 */
#ifndef PQK_H
#define PQK_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PQK_API __attribute__((visibility("default")))
#else
#define PQK_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PQK_OK = 0,
  PQK_ERR_INVALID_ARG = -1,  /* null pointer, bad size, bad enum value */
  PQK_ERR_UNSUPPORTED = -2,  /* head_dim or device not supported */
  PQK_ERR_MISALIGNED = -3,   /* pointer or stride not 16-byte aligned */
  PQK_ERR_CUDA = -4,         /* a CUDA runtime call failed */
  PQK_ERR_WORKSPACE = -5,    /* workspace missing or too small */
  PQK_ERR_TIMEOUT = -6,      /* device: a bounded pipeline wait ran out */
  PQK_ERR_BAD_SEQLENS = -7   /* device: cu_seqlens not 0 <= ... <= T, monotone */
} pqk_status;

/* RoPE pairing. INTERLEAVED rotates (x[2j], x[2j+1]); HALF rotates
 * (x[j], x[j + D/2]). */
typedef enum { PQK_ROPE_INTERLEAVED = 0, PQK_ROPE_HALF = 1 } pqk_rope_style;

/* Normalisation of modulate_swiglu. RMS: x / sqrt(mean(x^2) + eps).
 * LAYER: (x - mean) / sqrt(biased var + eps). NONE: x. No affine weight. */
typedef enum { PQK_NORM_RMS = 0, PQK_NORM_LAYER = 1, PQK_NORM_NONE = 2 } pqk_norm_type;

/*
 * pqk_qk_norm_rope -- fused Q/K RMSNorm + RoPE ("Q/K normalisation merged
 * with RoPE": first page, section "融合 DiT 算子"; second page, bullet "Fused
 * DiT operators").
 *
 * For every token t < T, head h < H and X in {Q, K}, on the D elements x of
 * row (t, h):
 *   y_d  = x_d / sqrt(mean_d(x_d^2) + eps) * w_X[d]        (norm per head)
 *   (a, b) <- (a cos phi - b sin phi, a sin phi + b cos phi) for every pair
 *   of pqk_rope_style j < D/2, phi = pos[t] * rope_base^(-2j/D).
 * Arithmetic in fp32 with the angle formed and reduced in fp64; outputs are
 * rounded to bf16 (nearest even).
 *
 * q_in, k_in    device bf16 [T, H, D], q_stride_t / k_stride_t elements
 *               between consecutive tokens (>= H*D; a fused QKV row works).
 * q_out, k_out  device bf16 [T, H, D] with their own token strides
 *               q_out_stride_t / k_out_stride_t (>= H*D, multiples of 8): a
 *               slot of a wider buffer works, such as the send buffer of a
 *               sequence-parallel exchange; equal to q_in / k_in with equal
 *               strides for in-place use (no other overlap allowed).
 * q_weight, k_weight  device bf16 [D], shared by all heads.
 * pos           device int32 [T], RoPE position id of every token.
 * D             64 or 128. T >= 0 (T == 0 enqueues nothing). eps > 0.
 */
PQK_API int pqk_qk_norm_rope(const void* q_in, const void* k_in, void* q_out, void* k_out,
                     int64_t q_stride_t, int64_t k_stride_t, int64_t q_out_stride_t,
                     int64_t k_out_stride_t, const void* q_weight, const void* k_weight,
                     const int32_t* pos, int64_t T, int H, int D, float eps, float rope_base,
                     int rope_style, void* stream);

/*
 * pqk_qk_norm_rope_e4m3 -- pqk_qk_norm_rope with its outputs as FP8 e4m3
 * codes, the SAGE FP8 quantisation of Q and K (first page, bullet on
 * TRTLLM_ATTN SAGE and Skip-Softmax) folded into the prologue, so that no
 * separate quantisation pass reads Q and K again. A reading: one scale per
 * tensor from a bound instead of the data. A normalised row has
 * sum_d (x_d / rms)^2 <= D, so every element of it, rotated or not, is at
 * most sqrt(D) * max_d |w_X[d]| in magnitude; with amax that bound (in
 * float), the codes are e4m3(y * 448 / amax) (nearest even) and the
 * dequantisation factor of every head of X is amax / 448 (1 if amax = 0).
 *
 * q_in, k_in, q_weight, k_weight, pos, T, H, D, eps, rope_base, rope_style:
 *               as pqk_qk_norm_rope.
 * q8, k8        device e4m3 codes [T, H, D] bytes, contiguous, 16-byte
 *               aligned (the layout pqk_varlen_attn_fwd_fp8qk / _fp8 read).
 * deq           device fp32 [2H]: Q's then K's per-head dequantisation
 *               factors (all heads of a tensor equal), as those entries take.
 */
PQK_API int pqk_qk_norm_rope_e4m3(const void* q_in, const void* k_in, void* q8, void* k8, int64_t q_stride_t,
                          int64_t k_stride_t, const void* q_weight, const void* k_weight,
                          const int32_t* pos, int64_t T, int H, int D, float eps, float rope_base,
                          int rope_style, float* deq, void* stream);

/*
 * pqk_qk_norm_rope_3axis -- pqk_qk_norm_rope with a (t, h, w) position per
 * token for video latents. The pages give no RoPE variant; the reading
 * taken: every pair j keeps theta_j = rope_base^(-2j/D) and takes its angle
 * from one axis, the D/2 pair indices being split into consecutive sections
 * of sec_t, sec_h, sec_w pairs (sec_t + sec_h + sec_w == D/2):
 *   phi_j = pos3[t][0] * theta_j for j < sec_t,
 *           pos3[t][1] * theta_j for sec_t <= j < sec_t + sec_h,
 *           pos3[t][2] * theta_j otherwise.
 * Tokens whose three ids are equal (text, audio) get exactly the one-axis
 * rotation of pqk_qk_norm_rope.
 *
 * pos3          device int32 [T, 3]. Other arguments and errors as in
 *               pqk_qk_norm_rope; sections that are negative or do not sum
 *               to D/2 return PQK_ERR_INVALID_ARG.
 */
PQK_API int pqk_qk_norm_rope_3axis(const void* q_in, const void* k_in, void* q_out, void* k_out,
                           int64_t q_stride_t, int64_t k_stride_t, const void* q_weight,
                           const void* k_weight, const int32_t* pos3, int sec_t, int sec_h,
                           int sec_w, int64_t T, int H, int D, float eps, float rope_base,
                           int rope_style, void* stream);

/*
 * pqk_qk_fullc_norm_rope -- pqk_qk_norm_rope with the RMS taken over all H*D
 * elements of a token's Q (and, separately, K) row instead of per head, and
 * one weight per element; then every head is rotated as in
 * pqk_qk_norm_rope. A reading of "Q/K normalisation merged with RoPE" (first
 * page, section "融合 DiT 算子") that the pages leave open, next to the
 * per-head default:
 *   y_{h,d} = x_{h,d} / sqrt(mean over the token's H*D elements of x^2 + eps)
 *             * w_X[h*D + d].
 *
 * q_weight, k_weight  device bf16 [H*D]. Other arguments, layouts and errors
 * as in pqk_qk_norm_rope.
 */
PQK_API int pqk_qk_fullc_norm_rope(const void* q_in, const void* k_in, void* q_out, void* k_out,
                           int64_t q_stride_t, int64_t k_stride_t, const void* q_weight,
                           const void* k_weight, const int32_t* pos, int64_t T, int H, int D,
                           float eps, float rope_base, int rope_style, void* stream);

/*
 * pqk_varlen_attn_workspace_size -- bytes of device workspace that
 * pqk_varlen_attn_fwd needs for B requests (its tile schedule).
 */
PQK_API size_t pqk_varlen_attn_workspace_size(int B);

/*
 * pqk_varlen_attn_fwd -- packed variable-length self-attention over one
 * unpadded sequence per request, valid tokens only (first page, section
 * "长序列注意力与通信优化"; second page, bullet "Long-sequence attention &
 * communication").
 *
 * Request i covers tokens [cu_seqlens[i], cu_seqlens[i+1]). For every token
 * t of request i and head h:
 *   O[t, h] = sum_j softmax_j(softmax_scale * <Q[t, h], K[j, h]>) V[j, h],
 *   j over request i only (bidirectional inside a request, nothing across),
 *   lse[h, t] = ln sum_j exp(softmax_scale * <Q[t, h], K[j, h]>).
 * bf16 tensor-core products with fp32 accumulation; probabilities are
 * rounded to bf16 before the second product; O rounded to bf16.
 *
 * q, k, v       device bf16 [T, H, D], q_stride_t / k_stride_t / v_stride_t
 *               elements between tokens (>= H*D).
 * o             device bf16 [T, H, D], o_stride_t elements between tokens;
 *               must not overlap q, k or v.
 * lse           device fp32 [H, T] or NULL.
 * cu_seqlens    device int32 [B+1], 0 = cu[0] <= cu[1] <= ... <= cu[B] = T;
 *               empty requests are allowed. Checked on the device: a
 *               violation sets PQK_ERR_BAD_SEQLENS in the status word and
 *               the call writes no output.
 * D             64 or 128. B >= 1, 0 <= T <= 2^31 - 513, and the work
 *               tiles of the schedule, (ceil(T/256) + B) * H, below
 *               2^31 - 2^20 (the other attention entry points alike).
 * workspace     device memory of at least pqk_varlen_attn_workspace_size(B)
 *               bytes, 16-byte aligned; it only holds this call's schedule
 *               and may be reused once the call has completed on `stream`.
 */
PQK_API int pqk_varlen_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                        int64_t q_stride_t, int64_t k_stride_t, int64_t v_stride_t,
                        int64_t o_stride_t, const int32_t* cu_seqlens, int B, int64_t T, int H,
                        int D, float softmax_scale, void* workspace, size_t workspace_bytes,
                        void* stream);

/*
 * pqk_varlen_attn_fwd_skip -- pqk_varlen_attn_fwd that leaves out the
 * softmax and the P x V product of key blocks whose scores are negligible
 * ("Skip-Softmax": first page, bullet on TRTLLM_ATTN SAGE and Skip-Softmax;
 * second page, bullet "Sparse & quantized attention"). The pages name the
 * idea only; the rule implemented:
 *   - blocks are 32 consecutive query rows x 128 consecutive keys of one
 *     request and head, counted from the request's first token;
 *   - key block j >= 1 is dropped for a query block when every one of its
 *     rows t has max_{k in block j} u(t,k) < M(t) - skip_threshold_log2,
 *     u = softmax_scale * <Q[t,h], K[k,h]> / ln 2 and M(t) the maximum of
 *     u(t, k) over the keys of blocks 0 .. j-1 (block 0 is always kept);
 *   - dropped keys contribute nothing to O or lse. Every dropped key has a
 *     weight below 2^-skip_threshold_log2 of the row's largest, so O moves
 *     by at most 2 * n_dropped * 2^-skip_threshold_log2 * max|V|.
 * The decision is taken in fp32 on the tensor-core scores, so rows whose
 * margin to the threshold is within fp32 rounding may decide either way.
 *
 * skip_threshold_log2  >= 0 (+inf keeps every block; NaN or negative is
 *               PQK_ERR_INVALID_ARG).
 * skip_counts   NULL, or device uint64 [2], 8-byte aligned, that the call
 *               adds to: [0] dropped (32-row block, head, key block)
 *               triples; [1] (128-row tile, head, key block) triples whose
 *               P x V product was left out because all four of the tile's
 *               32-row blocks inside the request dropped the key block.
 * Other arguments, layouts and errors are those of pqk_varlen_attn_fwd.
 */
PQK_API int pqk_varlen_attn_fwd_skip(const void* q, const void* k, const void* v, void* o, float* lse,
                             int64_t q_stride_t, int64_t k_stride_t, int64_t v_stride_t,
                             int64_t o_stride_t, const int32_t* cu_seqlens, int B, int64_t T, int H,
                             int D, float softmax_scale, float skip_threshold_log2,
                             unsigned long long* skip_counts, void* workspace, size_t workspace_bytes,
                             void* stream);

/*
 * pqk_quantize_qk_e4m3 -- Q and K to FP8 e4m3 for pqk_varlen_attn_fwd_fp8qk
 * (SAGE quantises the attention computation to FP8: first page, bullet on
 * TRTLLM_ATTN SAGE and Skip-Softmax; second page, bullet "Sparse & quantized
 * attention"). The pages give no scheme; the one implemented: per head h of
 * each tensor, amax = max |x| over all T tokens and D, code = e4m3(x * (448 /
 * amax)) rounded to nearest even, saturating at +-448 (e4m3 "fn": 4
 * exponent bits with bias 7, 3 mantissa bits, no infinities); the
 * dequantisation factor is amax / 448 (1 for an all-zero head).
 *
 * q, k      device bf16 [T, H, D], q_stride_t / k_stride_t elements between
 *           tokens (>= H*D, multiples of 8), 16-byte aligned.
 * q8, k8    device [T, H, D] bytes, contiguous, 16-byte aligned.
 * scales    device fp32 [4H], 16-byte aligned: [0, 2H) scratch, [2H, 3H) Q's
 *           and [3H, 4H) K's dequantisation factors (pass scales + 2H as
 *           `deq` to the attention). H <= 4096; D 64 or 128.
 */
PQK_API int pqk_quantize_qk_e4m3(const void* q, const void* k, int64_t q_stride_t, int64_t k_stride_t, int64_t T,
                         int H, int D, void* q8, void* k8, float* scales, void* stream);

/*
 * pqk_varlen_attn_fwd_fp8qk -- pqk_varlen_attn_fwd with S = Q K^T taken on
 * the FP8 tensor cores from e4m3 Q and K (pqk_quantize_qk_e4m3): for every
 * token t of request i and head h,
 *   s(t, j) = softmax_scale * deq[h] * deq[H + h] * <q8[t, h], k8[j, h]>,
 * then softmax and P V exactly as pqk_varlen_attn_fwd (P rounded to bf16, V
 * bf16, fp32 accumulation).
 *
 * q8, k8    device e4m3 [T, H, D] bytes, contiguous, 16-byte aligned.
 * deq       device fp32 [2H]: Q's then K's per-head dequantisation factors.
 * skip_threshold_log2, skip_counts: block skipping as pqk_varlen_attn_fwd_skip,
 *           decided on these FP8 scores; +inf skips nothing (and counts
 *           nothing).
 * v, o, lse, cu_seqlens, workspace: as pqk_varlen_attn_fwd. D must be 128
 * (PQK_ERR_UNSUPPORTED otherwise).
 */
PQK_API int pqk_varlen_attn_fwd_fp8qk(const void* q8, const void* k8, const void* v, const float* deq, void* o,
                              float* lse, int64_t v_stride_t, int64_t o_stride_t,
                              const int32_t* cu_seqlens, int B, int64_t T, int H, int D,
                              float softmax_scale, float skip_threshold_log2,
                              unsigned long long* skip_counts, void* workspace, size_t workspace_bytes,
                              void* stream);

/*
 * pqk_quantize_e4m3 -- one tensor to FP8 e4m3 with the per-head scheme of
 * pqk_quantize_qk_e4m3 (used for V by pqk_varlen_attn_fwd_fp8).
 *
 * x         device bf16 [T, H, D], x_stride_t elements between tokens.
 * x8        device [T, H, D] bytes, contiguous, 16-byte aligned.
 * scales    device fp32 [2H], 16-byte aligned: [0, H) scratch, [H, 2H) the
 *           dequantisation factors. H <= 4096; D 64 or 128.
 */
PQK_API int pqk_quantize_e4m3(const void* x, int64_t x_stride_t, int64_t T, int H, int D, void* x8,
                      float* scales, void* stream);

/*
 * pqk_varlen_attn_fwd_fp8 -- the whole attention computation in FP8 (SAGE
 * quantises the attention computation to FP8: first page, bullet on
 * TRTLLM_ATTN SAGE and Skip-Softmax), optionally with block skipping
 * (Skip-Softmax: the same bullet, and the second page's bullet "Sparse &
 * quantized attention", which credits the two together). Q, K, V are e4m3
 * per head (pqk_quantize_qk_e4m3, pqk_quantize_e4m3); S = Q K^T and
 * O += P V both run on the FP8 tensor cores. With u = s / ln 2 (s from the
 * dequantised Q, K), the probabilities are formed by an online softmax over
 * key blocks of 128 keys counted from the request's first token: the
 * running maximum m (log2 units) is set by the first block and moves only
 * when a block's maximum exceeds it by more than 8, the sums then scaling by
 * 2^(m_old - m_new); each key adds p = 2^(u - m) <= 256 to the denominator
 * and e4m3(p) * V~ to the numerator; O = numerator / denominator rounded to
 * bf16, lse = (m + log2 denominator) ln 2. Rounding p against the running
 * maximum rather than the row's final one changes each numerator term by
 * at most one e4m3 step (2^-3 of p, or 2^-9 below e4m3's normal range).
 *
 * q8, k8, v8  device e4m3 [T, H, D] bytes, contiguous, 16-byte aligned.
 * deq         device fp32 [3H]: Q's, K's, then V's dequantisation factors.
 * skip_threshold_log2, skip_counts: block skipping as pqk_varlen_attn_fwd_skip,
 *             decided on the FP8 scores; dropped keys take no part in the
 *             sums or the maximum; +inf skips nothing (and counts nothing).
 * o, lse, cu_seqlens, workspace: as pqk_varlen_attn_fwd. D must be 128.
 */
PQK_API int pqk_varlen_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* deq, void* o,
                            float* lse, int64_t o_stride_t, const int32_t* cu_seqlens, int B, int64_t T,
                            int H, int D, float softmax_scale, float skip_threshold_log2,
                            unsigned long long* skip_counts, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * pqk_varlen_attn_fwd_noalloc -- pqk_varlen_attn_fwd for callers that cannot
 * allocate device memory. The pages have no counterpart: this entry point
 * exists for callers such as plugins or embedded runtimes that are handed
 * only their input and output buffers by a host framework that owns the
 * whole device heap, and so have no way to obtain the schedule workspace.
 * The schedule lives instead in a fixed array inside the library's own
 * device memory (about 48 KB on every GPU that loads the library, held
 * until the process exits).
 *
 * Arguments and results are those of pqk_varlen_attn_fwd without the
 * workspace. B may be at most 4096; a larger B returns PQK_ERR_WORKSPACE.
 * The first call on a device looks up the array's device address (a CUDA
 * runtime query, no allocation); make that first call before capturing a
 * stream. The address is kept for the life of the device's CUDA context: a
 * caller that destroys and recreates the context (cudaDeviceReset) must not
 * call this entry point on that device afterwards. Every call uses the same
 * array, so calls whose work overlaps on the GPU (e.g. on different streams)
 * race and must be serialised by the caller; each call rewrites the whole
 * schedule it reads and resets the tile-claim counter in it, so nothing needs
 * to be cleared between calls.
 */
PQK_API int pqk_varlen_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                int64_t q_stride_t, int64_t k_stride_t, int64_t v_stride_t,
                                int64_t o_stride_t, const int32_t* cu_seqlens, int B, int64_t T,
                                int H, int D, float softmax_scale, void* stream);

/*
 * pqk_modulate_swiglu -- fused adaLN modulation + normalisation + gated
 * residual, and SwiGLU in one pass (first page, section "融合 DiT 算子": the
 * small DiT operators RMSNorm, SwiGLU and residual connections fused, SwiGLU
 * in place of separate SiLU and multiply; second page, bullet "Fused DiT
 * operators": modulation and normalization among them).
 *
 * For every token t of request s (cu_seqlens as in pqk_varlen_attn_fwd):
 *   x'  = x[t] + gate_res[s] * branch[t]       (branch == NULL: x' = x[t])
 *   h   = norm(x') * (1 + scale[s]) + shift[s] (pqk_norm_type over C)
 *   act = silu(gate[t]) * up[t],  silu(g) = g / (1 + exp(-g))
 * fp32 arithmetic on bf16 inputs, outputs rounded to bf16.
 *
 * x, branch     device bf16 [T, C] (branch may be NULL).
 * x_out         device bf16 [T, C] receiving x', or NULL; may equal x.
 * h             device bf16 [T, C]; may equal x.
 * shift, scale  device fp32 [B, C]; gate_res device fp32 [B, C], may be
 *               NULL when branch is NULL.
 * cu_seqlens    device int32 [B+1] (must be valid; not re-checked here).
 * gate, up      device bf16 [T, F] rows gu_stride_t elements apart (the two
 *               halves of one [T, 2F] buffer work); both NULL skips SwiGLU.
 * act           device bf16 [T, F] contiguous; may equal gate when
 *               gu_stride_t == F.
 * C, F          multiples of 8; C <= 16384. B >= 1, T >= 0, eps > 0.
 * A token's x' and h are written in the last pass over its row, each chunk
 * after that chunk's last read of x, and each act chunk after the read of
 * its gate chunk, so the aliases above are safe (x_out and h must not
 * alias each other).
 */
PQK_API int pqk_modulate_swiglu(const void* x, const void* branch, void* x_out, void* h,
                        const float* shift, const float* scale, const float* gate_res,
                        const int32_t* cu_seqlens, int B, int64_t T, int C, int norm_type,
                        float eps, const void* gate, const void* up, int64_t gu_stride_t,
                        void* act, int F, void* stream);

/*
 * pqk_linear_gated_residual -- a linear layer whose epilogue is the gated
 * residual: the output projection after attention (or W2 after SwiGLU)
 * with the residual add of the adaLN-gated branch done on the GEMM's fp32
 * accumulator, instead of writing the branch and re-reading it (first
 * page, section "融合 DiT 算子": residual connections among the fused DiT
 * operators; second page, bullet "Fused DiT operators"). For every token t
 * of request s:
 *   out[t, n] = x[t, n] + gate_res[s, n] * sum_k a[t, k] * w[n, k]
 * With x and gate_res both NULL: out = a w^T (the product alone; cu_seqlens
 * and B unused). tcgen05 tensor cores, fp32 accumulation, bf16 output
 * rounded to nearest even.
 *
 * a           device bf16 [T, K], rows a_stride_t elements apart.
 * w           device bf16 [N, K] contiguous (out x in features).
 * x           device bf16 [T, N], rows x_stride_t apart, or NULL.
 * gate_res    device fp32 [B, N] (one gate per request), or NULL with x.
 * cu_seqlens  device int32 [B+1] (must be valid; not re-checked here).
 * out         device bf16 [T, N], rows out_stride_t apart; may equal x
 *             (same stride); no other overlap with an input.
 * K, N        multiples of 8, >= 8; T <= 2^31 - 257, and the number of
 *             128 x 128 output tiles, ceil(T/128) * ceil(N/128), below
 *             2^31 - 2^20. Pointers 16-byte aligned, strides multiples of 8
 *             elements.
 * Errors: PQK_ERR_INVALID_ARG / PQK_ERR_MISALIGNED before anything is
 * enqueued; a pipeline wait that runs out records PQK_ERR_TIMEOUT in the
 * device status word (see pqk_get_device_status).
 */
PQK_API int pqk_linear_gated_residual(const void* a, int64_t a_stride_t, const void* w, const void* x,
                                      int64_t x_stride_t, const float* gate_res, const int32_t* cu_seqlens,
                                      int B, void* out, int64_t out_stride_t, int64_t T, int K, int N,
                                      void* stream);

/*
 * pqk_linear_swiglu -- W1 of the feed-forward with SwiGLU as its epilogue:
 * silu(gate) * up computed from the GEMM's fp32 accumulators, so that the
 * [T, 2F] product is never written (first page, section "融合 DiT 算子":
 * SwiGLU in place of separate SiLU and multiply; second page, bullet
 * "Fused DiT operators"). The first F rows of w1 give the SiLU operand, the
 * last F rows the linear one:
 *   act[t, f] = silu(sum_k a[t, k] w1[f, k]) * sum_k a[t, k] w1[F + f, k],
 *   silu(g) = g / (1 + exp(-g)).
 *
 * a           device bf16 [T, K], rows a_stride_t elements apart.
 * w1          device bf16 [2F, K] contiguous.
 * act         device bf16 [T, F], rows act_stride_t apart.
 * K, F        multiples of 8, >= 8. Size limits (with F for N), alignment
 *             and errors as pqk_linear_gated_residual.
 */
PQK_API int pqk_linear_swiglu(const void* a, int64_t a_stride_t, const void* w1, void* act, int64_t act_stride_t,
                              int64_t T, int K, int F, void* stream);

/*
 * pqk_get_device_status -- synchronises `stream`, then returns and clears
 * the current device's status word: PQK_OK, PQK_ERR_TIMEOUT or
 * PQK_ERR_BAD_SEQLENS (the first condition recorded since the last read),
 * or PQK_ERR_CUDA if the synchronisation itself failed.
 */
PQK_API int pqk_get_device_status(void* stream);

/*
 * pqk_set_wait_timeout_ns -- upper bound, in nanoseconds, on every pipeline
 * wait of the attention and linear-layer kernels (default 1e9). A wait that
 * runs out records PQK_ERR_TIMEOUT and its thread block stops issuing work;
 * once all of the block's roles have stopped it waits for the copies and
 * MMAs it still has in flight (a fixed bound of 2 s, independent of this
 * setting), frees its tensor memory and exits. Values <= 0 restore the
 * default; others are clamped to [1e3, 1e10] (1 us .. 10 s). Process-wide;
 * affects calls enqueued afterwards.
 */
PQK_API void pqk_set_wait_timeout_ns(int64_t ns);

/*
 * pqk_set_attn_cta_pairs -- nonzero: pqk_varlen_attn_fwd (and the
 * no-allocation entry) with bf16 operands and D = 128 runs on CTA pairs:
 * two SMs share each 512-row work tile, one thread issues the pair's
 * products with tcgen05 cta_group::2 (M = 256) and each SM streams half of
 * every K and V tile. The results are bit-identical to the default one-SM
 * kernel. On B200 it halves the L2-to-SM traffic and cuts the tensor cores'
 * shared-memory reads by a third, but the cross-CTA hand-offs lengthen each
 * tile's critical chain: in the 58,048-token step the two take the same
 * time, and a 16,384-token launch takes 5 % more cycles; hence off by
 * default. Process-wide; affects calls enqueued afterwards (and graphs
 * captured afterwards).
 */
PQK_API void pqk_set_attn_cta_pairs(int enable);

/*
 * pqk_selftest_wait_timeout -- diagnostic: enqueues one thread block that
 * waits, with the bounded wait used by the attention pipeline, on a
 * barrier that nothing completes. The wait runs out after timeout_ns and
 * records PQK_ERR_TIMEOUT in the status word; the context stays usable.
 */
PQK_API int pqk_selftest_wait_timeout(int64_t timeout_ns, void* stream);

/* Human-readable name of a pqk_status value. */
PQK_API const char* pqk_status_string(int status);

/* Library version, "major.minor.patch". */
PQK_API const char* pqk_version(void);

#ifdef __cplusplus
}
#endif
#endif /* PQK_H */
