// quant_fp8.cu -- per-head absmax quantisation of Q and K to FP8 e4m3 for
// the attention with Q K^T on the FP8 tensor cores (SAGE quantises the
// attention computation to FP8: "FastH3 在八卡 B300 上实现完整 MP4 生成快于播放
// 时长", bullet on TRTLLM_ATTN SAGE and Skip-Softmax).
//
// The reading: one scale per head and tensor. For head h, amax = max |x|
// over all tokens; code = e4m3(x * (448 / amax)) rounded to nearest even
// with saturation; the dequantisation factor is amax / 448 (both factors 1
// for an all-zero head). e4m3 is a floating-point format, so one scale per
// head costs precision only for values 2^15 below amax (the subnormal range).
//
// HBM-bound, two passes: absmax (read Q, K) and quantise (read Q, K again,
// write one byte per element). The same kernels quantise a single tensor
// (V for the attention with P V in FP8). Rows of D bf16 are spread over D/8
// lanes (16 bytes each), so a warp covers 32 / (D / 8) (token, head) rows
// per step.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pqk_internal.h"

namespace pqk {
namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float absmax8(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
  return m;
}

// Two floats to two e4m3 codes (nearest even, saturating): a -> low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(b), "f"(a));
  return r;
}

template <int D>
__global__ void __launch_bounds__(kThreads) absmax_kernel(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                                          int64_t qs, int64_t ks, int64_t T, int H,
                                                          unsigned* amax) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  extern __shared__ unsigned s_max[];  // [2H]: Q's heads, then K's (when K is given)
  const int nmax = (k != nullptr ? 2 : 1) * H;
  for (int i = threadIdx.x; i < nmax; i += blockDim.x) s_max[i] = 0u;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int part = lane % kLanesPerRow;
  const int64_t rows = T * H;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t base = warp0 * kRowsPerWarp; base < rows; base += nwarps * kRowsPerWarp) {
    const int64_t r = base + lane / kLanesPerRow;
    float mq = 0.f, mk = 0.f;
    int h = 0;
    if (r < rows) {
      const int64_t t = r / H;
      h = static_cast<int>(r % H);
      mq = absmax8(ld_nc16(q + t * qs + static_cast<int64_t>(h) * D + part * 8));
      if (k != nullptr) mk = absmax8(ld_nc16(k + t * ks + static_cast<int64_t>(h) * D + part * 8));
    }
#pragma unroll
    for (int off = kLanesPerRow / 2; off > 0; off >>= 1) {
      mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, off));
      mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, off));
    }
    if (part == 0 && r < rows) {
      atomicMax(&s_max[h], __float_as_uint(mq));  // non-negative floats order like their bits
      if (k != nullptr) atomicMax(&s_max[H + h], __float_as_uint(mk));
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nmax; i += blockDim.x)
    if (s_max[i] != 0u) atomicMax(&amax[i], s_max[i]);
}

__device__ __forceinline__ uint2 quant8(uint4 v, float inv) {
  uint2 o;
  o.x = e4m3x2(bf16_lo(v.x) * inv, bf16_hi(v.x) * inv) | (e4m3x2(bf16_lo(v.y) * inv, bf16_hi(v.y) * inv) << 16);
  o.y = e4m3x2(bf16_lo(v.z) * inv, bf16_hi(v.z) * inv) | (e4m3x2(bf16_lo(v.w) * inv, bf16_hi(v.w) * inv) << 16);
  return o;
}

__device__ __forceinline__ float inv_of(unsigned amax_bits) {
  const float a = __uint_as_float(amax_bits);
  return a > 0.f ? 448.0f / a : 1.0f;
}

template <int D>
__global__ void __launch_bounds__(kThreads) quantise_kernel(const __nv_bfloat16* q, const __nv_bfloat16* k,
                                                            int64_t qs, int64_t ks, int64_t T, int H,
                                                            const unsigned* amax, uint8_t* q8, uint8_t* k8,
                                                            float* deq) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i < (k != nullptr ? 2 : 1) * H; i += blockDim.x) {
      const float a = __uint_as_float(amax[i]);
      deq[i] = a > 0.f ? a / 448.0f : 1.0f;
    }
  }
  const int lane = threadIdx.x & 31;
  const int part = lane % kLanesPerRow;
  const int64_t rows = T * H;
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t base = warp0 * kRowsPerWarp; base < rows; base += nwarps * kRowsPerWarp) {
    const int64_t r = base + lane / kLanesPerRow;
    if (r >= rows) continue;
    const int64_t t = r / H;
    const int h = static_cast<int>(r % H);
    const int64_t o = r * D + part * 8;
    const uint4 vq = ld_nc16(q + t * qs + static_cast<int64_t>(h) * D + part * 8);
    *reinterpret_cast<uint2*>(q8 + o) = quant8(vq, inv_of(amax[h]));
    if (k != nullptr) {
      const uint4 vk = ld_nc16(k + t * ks + static_cast<int64_t>(h) * D + part * 8);
      *reinterpret_cast<uint2*>(k8 + o) = quant8(vk, inv_of(amax[H + h]));
    }
  }
}

// k == nullptr: one tensor; scales is then [2H] ([0, H) scratch, [H, 2H) its
// dequantisation factors), else [4H] as for Q and K.
template <int D>
int launch(const void* q, const void* k, int64_t qs, int64_t ks, int64_t T, int H, void* q8, void* k8,
           float* scales, cudaStream_t stream, int num_sms) {
  const int n = k != nullptr ? 2 : 1;
  unsigned* amax = reinterpret_cast<unsigned*>(scales);
  if (cudaMemsetAsync(amax, 0, sizeof(unsigned) * n * H, stream) != cudaSuccess) return -1;
  constexpr int kRowsPerBlock = (kThreads / 32) * (32 / (D / 8));
  const int64_t blocks_needed = (T * H + kRowsPerBlock - 1) / kRowsPerBlock;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const int grid = static_cast<int>(blocks_needed < cap ? (blocks_needed > 0 ? blocks_needed : 1) : cap);
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  absmax_kernel<D><<<grid, kThreads, sizeof(unsigned) * 2 * H, stream>>>(qb, kb, qs, ks, T, H, amax);
  if (cudaGetLastError() != cudaSuccess) return -1;
  quantise_kernel<D><<<grid, kThreads, 0, stream>>>(qb, kb, qs, ks, T, H, amax, static_cast<uint8_t*>(q8),
                                                     static_cast<uint8_t*>(k8), scales + n * H);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace

int launch_quantize_qk_e4m3(const void* q, const void* k, int64_t q_stride, int64_t k_stride, int64_t T, int H,
                            int D, void* q8, void* k8, float* scales, cudaStream_t stream, int num_sms) {
  if (D == 128) return launch<128>(q, k, q_stride, k_stride, T, H, q8, k8, scales, stream, num_sms);
  return launch<64>(q, k, q_stride, k_stride, T, H, q8, k8, scales, stream, num_sms);
}

int launch_quantize_e4m3(const void* x, int64_t x_stride, int64_t T, int H, int D, void* x8, float* scales,
                         cudaStream_t stream, int num_sms) {
  if (D == 128) return launch<128>(x, nullptr, x_stride, 0, T, H, x8, nullptr, scales, stream, num_sms);
  return launch<64>(x, nullptr, x_stride, 0, T, H, x8, nullptr, scales, stream, num_sms);
}

}  // namespace pqk
