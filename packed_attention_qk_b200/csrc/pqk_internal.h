// pqk_internal.h -- launchers shared between the C-ABI front end
// (pqk_api.cu) and the kernel translation units. Arguments are validated by
// the front end before any of these is called.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace pqk {

// Strides in elements between tokens, separately for the inputs and the
// outputs. sections == nullptr: one position per token; else pos is [T, 3] and
// sections[0..2] are the pairs per (t, h, w) axis. full_width: the norm runs
// over all H*D elements of a token with weights of H*D entries (one-axis
// positions only). e4m3_deq non-null: the outputs are e4m3 codes ([T, H, D]
// bytes, contiguous) at the per-tensor bound scale, whose [2H]
// dequantisation factors go to e4m3_deq (one-axis, per-head norm only).
int launch_qk_norm_rope(const void* q_in, const void* k_in, void* q_out, void* k_out, int64_t q_stride,
                        int64_t k_stride, int64_t q_out_stride, int64_t k_out_stride, const void* wq,
                        const void* wk, const int32_t* pos, const int* sections,
                        bool full_width, int64_t T, int H, int D, float eps, float rope_base, int style,
                        cudaStream_t stream, int num_sms, float* e4m3_deq = nullptr);

int launch_modulate_swiglu(const void* x, const void* branch, void* x_out, void* h, const float* shift,
                           const float* scale, const float* gate_res, const int32_t* cu_seqlens, int B, int64_t T,
                           int C, int norm_type, float eps, const void* gate, const void* up, int64_t gu_stride,
                           void* act, int F, cudaStream_t stream, int num_sms);

// Bytes of the attention tile schedule for B requests.
size_t attn_schedule_bytes(int B);

// Prepares and enqueues the attention kernel's TMA descriptors, the schedule
// builder and the persistent attention kernel. skip selects the block-
// skipping kernel (threshold skip_tau in log2 units; skip_counts nullable,
// two device counters the kernel adds to). deq non-null selects the kernel
// with Q, K given as e4m3 bytes ([T, H, D], strides in bytes) and deq their
// [2H] per-head dequantisation factors (D = 128; skipping may be combined
// with it). fp8_pv: V is e4m3 bytes too and P is rounded to e4m3 for P V
// (deq then [3H], V's last; skipping may be combined with it too). cta_pairs:
// the bf16, head_dim 128 attention without skipping runs on CTA pairs
// (tcgen05 cta_group::2). Returns 0, or -1 when a CUDA call failed, -2 when
// the tensor maps could not be encoded.
int launch_varlen_attn(const void* q, const void* k, const void* v, void* o, float* lse, int64_t q_stride,
                       int64_t k_stride, int64_t v_stride, int64_t o_stride, const int32_t* cu_seqlens, int B,
                       int64_t T, int H, int D, float softmax_scale, void* workspace, int* status,
                       long long timeout_ns, cudaStream_t stream, int num_sms, bool skip = false,
                       float skip_tau = 0.0f, unsigned long long* skip_counts = nullptr,
                       const float* deq = nullptr, bool fp8_pv = false, bool cta_pairs = false);

// Per-head absmax e4m3 quantisation of Q and K ([T, H, D] bf16, strides in
// elements) into q8, k8 ([T, H, D] bytes, contiguous). scales: [4H] floats,
// [0, 2H) scratch (absmax bits), [2H, 4H) the dequantisation factors (Q's
// heads, then K's). D is 64 or 128.
int launch_quantize_qk_e4m3(const void* q, const void* k, int64_t q_stride, int64_t k_stride, int64_t T, int H,
                            int D, void* q8, void* k8, float* scales, cudaStream_t stream, int num_sms);

// The same for one tensor x: scales [2H], [0, H) scratch, [H, 2H) its
// dequantisation factors.
int launch_quantize_e4m3(const void* x, int64_t x_stride, int64_t T, int H, int D, void* x8, float* scales,
                         cudaStream_t stream, int num_sms);

// Epilogues of the linear-layer GEMM (launch_linear).
constexpr int kEpiNone = 0;           // out = A W^T
constexpr int kEpiGatedResidual = 1;  // out = x + gate_res[request] * (A W^T)
constexpr int kEpiSwiglu = 2;         // out = silu(A W[:N]^T) * (A W[N:]^T), W [2N, K]

// Persistent tcgen05 GEMM out[T, N] = epilogue(A[T, K] W^T) with bf16 A, W
// (W row-major [N, K], or [2N, K] for SwiGLU) and bf16 out. x, gate_res, cu
// and B are used by the gated residual only. Returns 0, -1 when a CUDA call
// failed, -2 when the tensor maps could not be encoded.
int launch_linear(int epi, const void* a, int64_t a_stride, const void* w, const void* x, int64_t x_stride,
                  const float* gate_res, const int32_t* cu, int B, void* out, int64_t out_stride, int64_t T, int K,
                  int N, int* status, long long timeout_ns, cudaStream_t stream, int num_sms);

int launch_wait_selftest(int* status, long long timeout_ns, cudaStream_t stream);

// Status codes written by kernels into the device status word (same values
// as the public pqk_status).
constexpr int kStatusTimeout = -6;
constexpr int kStatusBadSeqlens = -7;

}  // namespace pqk
