// pqk_api.cu -- the C ABI declared in include/pqk.h: host-side argument
// validation (nothing is enqueued on an argument error), per-device cached
// properties, the device status word, and dispatch to the kernels.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "pqk.h"
#include "pqk_internal.h"

namespace {

// Per-device status word: first device-side condition (timeout, bad
// cu_seqlens) since it was last read.
__device__ int g_status = 0;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  std::atomic<int> ready{0};
  int num_sms = 0;
  int cc_major = 0;
  int cc_minor = 0;
  int* status = nullptr;
};
DeviceInfo g_dev[kMaxDevices];

std::atomic<long long> g_timeout_ns{1000000000LL};
std::atomic<int> g_attn_cta_pairs{0};

// Caches the properties of the current device; returns nullptr on failure.
DeviceInfo* current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  DeviceInfo& d = g_dev[dev];
  if (d.ready.load(std::memory_order_acquire)) return &d;
  int sms = 0, major = 0, minor = 0;
  void* status = nullptr;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return nullptr;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return nullptr;
  if (cudaGetSymbolAddress(&status, g_status) != cudaSuccess) return nullptr;
  d.num_sms = sms;
  d.cc_major = major;
  d.cc_minor = minor;
  d.status = static_cast<int*>(status);
  d.ready.store(1, std::memory_order_release);
  return &d;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// sm_100 (B200 class) is the only target the library is built for.
int check_device(DeviceInfo** out) {
  DeviceInfo* d = current_device();
  if (d == nullptr) return PQK_ERR_CUDA;
  if (d->cc_major != 10 || d->cc_minor != 0) return PQK_ERR_UNSUPPORTED;
  *out = d;
  return PQK_OK;
}

// The linear-layer kernel indexes its output tiles (128 tokens x 128
// columns at the finest) with 32-bit integers: keep their count, plus a grid
// stride of headroom, inside that range.
bool linear_tiles_fit(int64_t T, int N) {
  const int64_t tiles = ((T + 127) / 128) * ((static_cast<int64_t>(N) + 127) / 128);
  return tiles <= static_cast<int64_t>(INT32_MAX) - (1 << 20);
}

// The attention's tile schedule counts its work tiles (256 query rows x one
// head) in 32-bit integers; their number is at most (ceil(T/256) + B) * H.
bool attn_tiles_fit(int64_t T, int B, int H) {
  const int64_t tiles = ((T + 255) / 256 + B) * static_cast<int64_t>(H);
  return tiles <= static_cast<int64_t>(INT32_MAX) - (1 << 20);
}

}  // namespace

extern "C" {

const char* pqk_status_string(int status) {
  switch (status) {
    case PQK_OK: return "ok";
    case PQK_ERR_INVALID_ARG: return "invalid argument";
    case PQK_ERR_UNSUPPORTED: return "unsupported head_dim or device";
    case PQK_ERR_MISALIGNED: return "pointer or stride not 16-byte aligned";
    case PQK_ERR_CUDA: return "CUDA runtime error";
    case PQK_ERR_WORKSPACE: return "workspace missing or too small";
    case PQK_ERR_TIMEOUT: return "device: bounded pipeline wait ran out";
    case PQK_ERR_BAD_SEQLENS: return "device: cu_seqlens not monotone from 0 to T";
    default: return "unknown status";
  }
}

const char* pqk_version(void) { return "0.1.0"; }

void pqk_set_attn_cta_pairs(int enable) { g_attn_cta_pairs.store(enable != 0 ? 1 : 0); }

void pqk_set_wait_timeout_ns(int64_t ns) {
  constexpr int64_t kDefault = 1000000000LL, kMin = 1000LL, kMax = 10000000000LL;
  g_timeout_ns.store(ns <= 0 ? kDefault : (ns < kMin ? kMin : (ns > kMax ? kMax : ns)));
}

int pqk_qk_norm_rope(const void* q_in, const void* k_in, void* q_out, void* k_out, int64_t q_stride_t,
                     int64_t k_stride_t, int64_t q_out_stride_t, int64_t k_out_stride_t, const void* q_weight,
                     const void* k_weight, const int32_t* pos, int64_t T, int H, int D, float eps, float rope_base,
                     int rope_style, void* stream) {
  if (T < 0 || H <= 0 || !(eps > 0.f) || !(rope_base > 0.f)) return PQK_ERR_INVALID_ARG;
  if (rope_style != PQK_ROPE_INTERLEAVED && rope_style != PQK_ROPE_HALF) return PQK_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PQK_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(H) * D;
  if (q_stride_t < row || k_stride_t < row || q_out_stride_t < row || k_out_stride_t < row)
    return PQK_ERR_INVALID_ARG;
  if (T == 0) return PQK_OK;
  if (!q_in || !k_in || !q_out || !k_out || !q_weight || !k_weight || !pos) return PQK_ERR_INVALID_ARG;
  // in place needs the same layout on both sides
  if ((q_out == q_in && q_out_stride_t != q_stride_t) || (k_out == k_in && k_out_stride_t != k_stride_t))
    return PQK_ERR_INVALID_ARG;
  if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(q_out) || !aligned16(k_out) || !aligned16(q_weight) ||
      !aligned16(k_weight) || (q_stride_t % 8) || (k_stride_t % 8) || (q_out_stride_t % 8) ||
      (k_out_stride_t % 8))
    return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  return pqk::launch_qk_norm_rope(q_in, k_in, q_out, k_out, q_stride_t, k_stride_t, q_out_stride_t, k_out_stride_t,
                                  q_weight, k_weight, pos, nullptr, false, T, H, D, eps, rope_base, rope_style,
                                  static_cast<cudaStream_t>(stream), d->num_sms)
             ? PQK_ERR_CUDA
             : PQK_OK;
}

int pqk_qk_norm_rope_e4m3(const void* q_in, const void* k_in, void* q8, void* k8, int64_t q_stride_t,
                          int64_t k_stride_t, const void* q_weight, const void* k_weight, const int32_t* pos,
                          int64_t T, int H, int D, float eps, float rope_base, int rope_style, float* deq,
                          void* stream) {
  if (T < 0 || H <= 0 || !(eps > 0.f) || !(rope_base > 0.f)) return PQK_ERR_INVALID_ARG;
  if (rope_style != PQK_ROPE_INTERLEAVED && rope_style != PQK_ROPE_HALF) return PQK_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PQK_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(H) * D;
  if (q_stride_t < row || k_stride_t < row) return PQK_ERR_INVALID_ARG;
  if (T == 0) return PQK_OK;
  if (!q_in || !k_in || !q8 || !k8 || !q_weight || !k_weight || !pos || !deq) return PQK_ERR_INVALID_ARG;
  if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(q8) || !aligned16(k8) || !aligned16(q_weight) ||
      !aligned16(k_weight) || (reinterpret_cast<uintptr_t>(deq) % 4) || (q_stride_t % 8) || (k_stride_t % 8))
    return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  // the byte outputs are addressed as [T, H, D]; their "stride" is unused
  return pqk::launch_qk_norm_rope(q_in, k_in, q8, k8, q_stride_t, k_stride_t, row, row, q_weight, k_weight, pos,
                                  nullptr, false, T, H, D, eps, rope_base, rope_style,
                                  static_cast<cudaStream_t>(stream), d->num_sms, deq)
             ? PQK_ERR_CUDA
             : PQK_OK;
}

int pqk_qk_norm_rope_3axis(const void* q_in, const void* k_in, void* q_out, void* k_out, int64_t q_stride_t,
                           int64_t k_stride_t, const void* q_weight, const void* k_weight, const int32_t* pos3,
                           int sec_t, int sec_h, int sec_w, int64_t T, int H, int D, float eps, float rope_base,
                           int rope_style, void* stream) {
  if (T < 0 || H <= 0 || !(eps > 0.f) || !(rope_base > 0.f)) return PQK_ERR_INVALID_ARG;
  if (rope_style != PQK_ROPE_INTERLEAVED && rope_style != PQK_ROPE_HALF) return PQK_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PQK_ERR_UNSUPPORTED;
  if (sec_t < 0 || sec_h < 0 || sec_w < 0 || sec_t + sec_h + sec_w != D / 2) return PQK_ERR_INVALID_ARG;
  if (q_stride_t < static_cast<int64_t>(H) * D || k_stride_t < static_cast<int64_t>(H) * D)
    return PQK_ERR_INVALID_ARG;
  if (T == 0) return PQK_OK;
  if (!q_in || !k_in || !q_out || !k_out || !q_weight || !k_weight || !pos3) return PQK_ERR_INVALID_ARG;
  if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(q_out) || !aligned16(k_out) || !aligned16(q_weight) ||
      !aligned16(k_weight) || (q_stride_t % 8) || (k_stride_t % 8))
    return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  const int sections[3] = {sec_t, sec_h, sec_w};
  return pqk::launch_qk_norm_rope(q_in, k_in, q_out, k_out, q_stride_t, k_stride_t, q_stride_t, k_stride_t, q_weight,
                                  k_weight, pos3, sections, false, T, H, D, eps, rope_base, rope_style,
                                  static_cast<cudaStream_t>(stream), d->num_sms)
             ? PQK_ERR_CUDA
             : PQK_OK;
}

int pqk_qk_fullc_norm_rope(const void* q_in, const void* k_in, void* q_out, void* k_out, int64_t q_stride_t,
                           int64_t k_stride_t, const void* q_weight, const void* k_weight, const int32_t* pos,
                           int64_t T, int H, int D, float eps, float rope_base, int rope_style, void* stream) {
  if (T < 0 || H <= 0 || !(eps > 0.f) || !(rope_base > 0.f)) return PQK_ERR_INVALID_ARG;
  if (rope_style != PQK_ROPE_INTERLEAVED && rope_style != PQK_ROPE_HALF) return PQK_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PQK_ERR_UNSUPPORTED;
  if (q_stride_t < static_cast<int64_t>(H) * D || k_stride_t < static_cast<int64_t>(H) * D)
    return PQK_ERR_INVALID_ARG;
  if (T == 0) return PQK_OK;
  if (!q_in || !k_in || !q_out || !k_out || !q_weight || !k_weight || !pos) return PQK_ERR_INVALID_ARG;
  if (!aligned16(q_in) || !aligned16(k_in) || !aligned16(q_out) || !aligned16(k_out) || !aligned16(q_weight) ||
      !aligned16(k_weight) || (q_stride_t % 8) || (k_stride_t % 8))
    return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  return pqk::launch_qk_norm_rope(q_in, k_in, q_out, k_out, q_stride_t, k_stride_t, q_stride_t, k_stride_t, q_weight,
                                  k_weight, pos, nullptr, true, T, H, D, eps, rope_base, rope_style,
                                  static_cast<cudaStream_t>(stream), d->num_sms)
             ? PQK_ERR_CUDA
             : PQK_OK;
}

size_t pqk_varlen_attn_workspace_size(int B) { return B < 1 ? 0 : pqk::attn_schedule_bytes(B); }

int pqk_varlen_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t q_stride_t,
                        int64_t k_stride_t, int64_t v_stride_t, int64_t o_stride_t, const int32_t* cu_seqlens,
                        int B, int64_t T, int H, int D, float softmax_scale, void* workspace,
                        size_t workspace_bytes, void* stream) {
  if (B < 1 || T < 0 || H <= 0 || T > INT32_MAX - 512 || !(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return PQK_ERR_INVALID_ARG;
  if (!attn_tiles_fit(T, B, H)) return PQK_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PQK_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(H) * D;
  if (q_stride_t < row || k_stride_t < row || v_stride_t < row || o_stride_t < row) return PQK_ERR_INVALID_ARG;
  if (T == 0) return PQK_OK;
  if (!q || !k || !v || !o || !cu_seqlens) return PQK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (q_stride_t % 8) || (k_stride_t % 8) || (v_stride_t % 8) || (o_stride_t % 8))
    return PQK_ERR_MISALIGNED;
  if (workspace == nullptr || workspace_bytes < pqk_varlen_attn_workspace_size(B)) return PQK_ERR_WORKSPACE;
  if (!aligned16(workspace)) return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  const int rc = pqk::launch_varlen_attn(q, k, v, o, lse, q_stride_t, k_stride_t, v_stride_t, o_stride_t,
                                         cu_seqlens, B, T, H, D, softmax_scale, workspace, d->status,
                                         g_timeout_ns.load(), static_cast<cudaStream_t>(stream), d->num_sms, false,
                                         0.0f, nullptr, nullptr, false, g_attn_cta_pairs.load() != 0);
  return rc == 0 ? PQK_OK : (rc == -2 ? PQK_ERR_INVALID_ARG : PQK_ERR_CUDA);
}

int pqk_varlen_attn_fwd_skip(const void* q, const void* k, const void* v, void* o, float* lse, int64_t q_stride_t,
                             int64_t k_stride_t, int64_t v_stride_t, int64_t o_stride_t, const int32_t* cu_seqlens,
                             int B, int64_t T, int H, int D, float softmax_scale, float skip_threshold_log2,
                             unsigned long long* skip_counts, void* workspace, size_t workspace_bytes, void* stream) {
  if (B < 1 || T < 0 || H <= 0 || T > INT32_MAX - 512 || !(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return PQK_ERR_INVALID_ARG;
  if (!attn_tiles_fit(T, B, H)) return PQK_ERR_INVALID_ARG;
  if (!(skip_threshold_log2 >= 0.f)) return PQK_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PQK_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(H) * D;
  if (q_stride_t < row || k_stride_t < row || v_stride_t < row || o_stride_t < row) return PQK_ERR_INVALID_ARG;
  if (T == 0) return PQK_OK;
  if (!q || !k || !v || !o || !cu_seqlens) return PQK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (q_stride_t % 8) || (k_stride_t % 8) || (v_stride_t % 8) || (o_stride_t % 8) ||
      (reinterpret_cast<uintptr_t>(skip_counts) % 8))
    return PQK_ERR_MISALIGNED;
  if (workspace == nullptr || workspace_bytes < pqk_varlen_attn_workspace_size(B)) return PQK_ERR_WORKSPACE;
  if (!aligned16(workspace)) return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  const int rc = pqk::launch_varlen_attn(q, k, v, o, lse, q_stride_t, k_stride_t, v_stride_t, o_stride_t,
                                         cu_seqlens, B, T, H, D, softmax_scale, workspace, d->status,
                                         g_timeout_ns.load(), static_cast<cudaStream_t>(stream), d->num_sms,
                                         true, skip_threshold_log2, skip_counts);
  return rc == 0 ? PQK_OK : (rc == -2 ? PQK_ERR_INVALID_ARG : PQK_ERR_CUDA);
}

int pqk_quantize_qk_e4m3(const void* q, const void* k, int64_t q_stride_t, int64_t k_stride_t, int64_t T, int H,
                         int D, void* q8, void* k8, float* scales, void* stream) {
  if (T < 0 || H <= 0 || H > 4096) return PQK_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PQK_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(H) * D;
  if (q_stride_t < row || k_stride_t < row) return PQK_ERR_INVALID_ARG;
  if (!q || !k || !q8 || !k8 || !scales) return PQK_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q8) || !aligned16(k8) || !aligned16(scales) ||
      (q_stride_t % 8) || (k_stride_t % 8))
    return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  return pqk::launch_quantize_qk_e4m3(q, k, q_stride_t, k_stride_t, T, H, D, q8, k8, scales,
                                      static_cast<cudaStream_t>(stream), d->num_sms)
             ? PQK_ERR_CUDA
             : PQK_OK;
}

int pqk_varlen_attn_fwd_fp8qk(const void* q8, const void* k8, const void* v, const float* deq, void* o, float* lse,
                              int64_t v_stride_t, int64_t o_stride_t, const int32_t* cu_seqlens, int B, int64_t T,
                              int H, int D, float softmax_scale, float skip_threshold_log2,
                              unsigned long long* skip_counts, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (B < 1 || T < 0 || H <= 0 || T > INT32_MAX - 512 || !(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return PQK_ERR_INVALID_ARG;
  if (!attn_tiles_fit(T, B, H)) return PQK_ERR_INVALID_ARG;
  if (!(skip_threshold_log2 >= 0.f)) return PQK_ERR_INVALID_ARG;
  if (D != 128) return PQK_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(H) * D;
  if (v_stride_t < row || o_stride_t < row) return PQK_ERR_INVALID_ARG;
  if (T == 0) return PQK_OK;
  if (!q8 || !k8 || !v || !deq || !o || !cu_seqlens) return PQK_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(deq) % 4) || (v_stride_t % 8) || (o_stride_t % 8) ||
      (reinterpret_cast<uintptr_t>(skip_counts) % 8))
    return PQK_ERR_MISALIGNED;
  if (workspace == nullptr || workspace_bytes < pqk_varlen_attn_workspace_size(B)) return PQK_ERR_WORKSPACE;
  if (!aligned16(workspace)) return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  const int rc = pqk::launch_varlen_attn(q8, k8, v, o, lse, row, row, v_stride_t, o_stride_t, cu_seqlens, B, T, H, D,
                                         softmax_scale, workspace, d->status, g_timeout_ns.load(),
                                         static_cast<cudaStream_t>(stream), d->num_sms,
                                         std::isfinite(skip_threshold_log2), skip_threshold_log2, skip_counts, deq);
  return rc == 0 ? PQK_OK : (rc == -2 ? PQK_ERR_INVALID_ARG : PQK_ERR_CUDA);
}

int pqk_quantize_e4m3(const void* x, int64_t x_stride_t, int64_t T, int H, int D, void* x8, float* scales,
                      void* stream) {
  if (T < 0 || H <= 0 || H > 4096) return PQK_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return PQK_ERR_UNSUPPORTED;
  if (x_stride_t < static_cast<int64_t>(H) * D) return PQK_ERR_INVALID_ARG;
  if (!x || !x8 || !scales) return PQK_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x8) || !aligned16(scales) || (x_stride_t % 8)) return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  return pqk::launch_quantize_e4m3(x, x_stride_t, T, H, D, x8, scales, static_cast<cudaStream_t>(stream), d->num_sms)
             ? PQK_ERR_CUDA
             : PQK_OK;
}

int pqk_varlen_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* deq, void* o, float* lse,
                            int64_t o_stride_t, const int32_t* cu_seqlens, int B, int64_t T, int H, int D,
                            float softmax_scale, float skip_threshold_log2, unsigned long long* skip_counts,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (B < 1 || T < 0 || H <= 0 || T > INT32_MAX - 512 || !(softmax_scale > 0.f) || !std::isfinite(softmax_scale))
    return PQK_ERR_INVALID_ARG;
  if (!attn_tiles_fit(T, B, H)) return PQK_ERR_INVALID_ARG;
  if (!(skip_threshold_log2 >= 0.f)) return PQK_ERR_INVALID_ARG;
  if (D != 128) return PQK_ERR_UNSUPPORTED;
  const int64_t row = static_cast<int64_t>(H) * D;
  if (o_stride_t < row) return PQK_ERR_INVALID_ARG;
  if (T == 0) return PQK_OK;
  if (!q8 || !k8 || !v8 || !deq || !o || !cu_seqlens) return PQK_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) || !aligned16(lse) ||
      (reinterpret_cast<uintptr_t>(deq) % 4) || (o_stride_t % 8) || (reinterpret_cast<uintptr_t>(skip_counts) % 8))
    return PQK_ERR_MISALIGNED;
  if (workspace == nullptr || workspace_bytes < pqk_varlen_attn_workspace_size(B)) return PQK_ERR_WORKSPACE;
  if (!aligned16(workspace)) return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  const int rc = pqk::launch_varlen_attn(q8, k8, v8, o, lse, row, row, row, o_stride_t, cu_seqlens, B, T, H, D,
                                         softmax_scale, workspace, d->status, g_timeout_ns.load(),
                                         static_cast<cudaStream_t>(stream), d->num_sms,
                                         std::isfinite(skip_threshold_log2), skip_threshold_log2, skip_counts, deq,
                                         true);
  return rc == 0 ? PQK_OK : (rc == -2 ? PQK_ERR_INVALID_ARG : PQK_ERR_CUDA);
}

int pqk_modulate_swiglu(const void* x, const void* branch, void* x_out, void* h, const float* shift,
                        const float* scale, const float* gate_res, const int32_t* cu_seqlens, int B, int64_t T, int C,
                        int norm_type, float eps, const void* gate, const void* up, int64_t gu_stride_t, void* act,
                        int F, void* stream) {
  if (B < 1 || T < 0 || C <= 0 || C % 8 || C > 16384 || !(eps > 0.f)) return PQK_ERR_INVALID_ARG;
  if (norm_type != PQK_NORM_RMS && norm_type != PQK_NORM_LAYER && norm_type != PQK_NORM_NONE)
    return PQK_ERR_INVALID_ARG;
  const bool swiglu = gate != nullptr || up != nullptr;
  if (swiglu && (gate == nullptr || up == nullptr || act == nullptr || F <= 0 || F % 8 || gu_stride_t < F))
    return PQK_ERR_INVALID_ARG;
  if (T == 0) return PQK_OK;
  if (!x || !h || !shift || !scale || !cu_seqlens || (branch && !gate_res)) return PQK_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(branch) || !aligned16(x_out) || !aligned16(h) || !aligned16(shift) ||
      !aligned16(scale) || !aligned16(gate_res))
    return PQK_ERR_MISALIGNED;
  if (swiglu && (!aligned16(gate) || !aligned16(up) || !aligned16(act) || (gu_stride_t % 8)))
    return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  return pqk::launch_modulate_swiglu(x, branch, x_out, h, shift, scale, gate_res, cu_seqlens, B, T, C, norm_type, eps,
                                     swiglu ? gate : nullptr, swiglu ? up : nullptr, gu_stride_t, act, F,
                                     static_cast<cudaStream_t>(stream), d->num_sms)
             ? PQK_ERR_CUDA
             : PQK_OK;
}

int pqk_linear_gated_residual(const void* a, int64_t a_stride_t, const void* w, const void* x, int64_t x_stride_t,
                              const float* gate_res, const int32_t* cu_seqlens, int B, void* out,
                              int64_t out_stride_t, int64_t T, int K, int N, void* stream) {
  if (T < 0 || T > INT32_MAX - 256 || K < 8 || N < 8 || K % 8 || N % 8) return PQK_ERR_INVALID_ARG;
  if (!linear_tiles_fit(T, N)) return PQK_ERR_INVALID_ARG;
  const bool residual = x != nullptr || gate_res != nullptr;
  if (residual && (x == nullptr || gate_res == nullptr || cu_seqlens == nullptr || B < 1 || x_stride_t < N))
    return PQK_ERR_INVALID_ARG;
  if (a_stride_t < K || out_stride_t < N) return PQK_ERR_INVALID_ARG;
  if (T == 0) return PQK_OK;
  if (!a || !w || !out) return PQK_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(w) || !aligned16(out) || !aligned16(x) || !aligned16(gate_res) ||
      (a_stride_t % 8) || (out_stride_t % 8) || (residual && (x_stride_t % 8)))
    return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  const int rc = pqk::launch_linear(residual ? pqk::kEpiGatedResidual : pqk::kEpiNone, a, a_stride_t, w, x,
                                    x_stride_t, gate_res, cu_seqlens, B, out, out_stride_t, T, K, N, d->status,
                                    g_timeout_ns.load(), static_cast<cudaStream_t>(stream), d->num_sms);
  return rc == 0 ? PQK_OK : (rc == -2 ? PQK_ERR_INVALID_ARG : PQK_ERR_CUDA);
}

int pqk_linear_swiglu(const void* a, int64_t a_stride_t, const void* w1, void* act, int64_t act_stride_t, int64_t T,
                      int K, int F, void* stream) {
  if (T < 0 || T > INT32_MAX - 256 || K < 8 || F < 8 || K % 8 || F % 8) return PQK_ERR_INVALID_ARG;
  if (!linear_tiles_fit(T, F)) return PQK_ERR_INVALID_ARG;
  if (a_stride_t < K || act_stride_t < F) return PQK_ERR_INVALID_ARG;
  if (T == 0) return PQK_OK;
  if (!a || !w1 || !act) return PQK_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(w1) || !aligned16(act) || (a_stride_t % 8) || (act_stride_t % 8))
    return PQK_ERR_MISALIGNED;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  const int rc = pqk::launch_linear(pqk::kEpiSwiglu, a, a_stride_t, w1, nullptr, 0, nullptr, nullptr, 0, act,
                                    act_stride_t, T, K, F, d->status, g_timeout_ns.load(),
                                    static_cast<cudaStream_t>(stream), d->num_sms);
  return rc == 0 ? PQK_OK : (rc == -2 ? PQK_ERR_INVALID_ARG : PQK_ERR_CUDA);
}

int pqk_get_device_status(void* stream) {
  DeviceInfo* d = current_device();
  if (d == nullptr) return PQK_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int value = 0;
  if (cudaMemcpyAsync(&value, d->status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return PQK_ERR_CUDA;
  if (cudaMemsetAsync(d->status, 0, sizeof(int), s) != cudaSuccess) return PQK_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return PQK_ERR_CUDA;
  return value;
}

int pqk_selftest_wait_timeout(int64_t timeout_ns, void* stream) {
  if (timeout_ns <= 0 || timeout_ns > 10000000000LL) return PQK_ERR_INVALID_ARG;
  DeviceInfo* d = nullptr;
  if (int rc = check_device(&d)) return rc;
  return pqk::launch_wait_selftest(d->status, timeout_ns, static_cast<cudaStream_t>(stream)) ? PQK_ERR_CUDA
                                                                                             : PQK_OK;
}

}  // extern "C"
