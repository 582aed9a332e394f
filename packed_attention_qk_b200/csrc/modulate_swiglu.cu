// modulate_swiglu.cu -- fused adaLN modulation + normalisation + gated
// residual, and SwiGLU ("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长",
// section "融合 DiT 算子": RMSNorm, SwiGLU and residual connections fused,
// SwiGLU in place of a separate SiLU and multiply; "MiniMax H3 FastH3
// real-time serving with vLLM-Omni", bullet "Fused DiT operators":
// modulation and normalization among the fused operators).
//
// HBM-bound. A 256-thread block owns one token at a time (grid-stride over
// tokens). Part 1 keeps the token's C-wide row in registers (8 elements of
// 16 bytes per slot, up to kMaxSlots slots per thread), forms the gated
// residual, reduces sum / sum of squares across the block (warp shuffles,
// then one shared-memory exchange), and writes h = norm * (1 + scale) +
// shift with the request's modulation vectors (read through the read-only
// cache, shared by every token of the request). Part 2 streams the token's
// gate / up rows in 16-byte chunks, kUnroll chunks in flight per thread.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pqk_internal.h"

namespace pqk {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct ModParams {
  const __nv_bfloat16* x;
  const __nv_bfloat16* branch;
  __nv_bfloat16* x_out;
  __nv_bfloat16* h;
  const float* shift;
  const float* scale;
  const float* gate_res;
  const int32_t* cu;
  int B;
  int64_t T;
  int C;
  int norm_type;
  float eps;
  const __nv_bfloat16* gate;
  const __nv_bfloat16* up;
  int64_t gu_stride;
  __nv_bfloat16* act;
  int F;
};

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 v;
  v.x = pack_bf16x2(f[0], f[1]);
  v.y = pack_bf16x2(f[2], f[3]);
  v.z = pack_bf16x2(f[4], f[5]);
  v.w = pack_bf16x2(f[6], f[7]);
  return v;
}

__device__ __forceinline__ void load8f(const float* p, float (&f)[8]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p));
  const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// Request s with cu[s] <= t < cu[s+1] (the last such s when requests are empty).
__device__ __forceinline__ int find_segment(const int32_t* cu, int B, int64_t t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<int64_t>(__ldg(cu + mid)) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Block-wide sum of two values; every thread gets the result.
__device__ __forceinline__ float2 block_sum2(float a, float b, float2* scratch) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, off);
    b += __shfl_xor_sync(0xffffffffu, b, off);
  }
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) scratch[warp] = make_float2(a, b);
  __syncthreads();
  float2 r = make_float2(0.f, 0.f);
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) {
    r.x += scratch[w].x;
    r.y += scratch[w].y;
  }
  __syncthreads();
  return r;
}

__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

template <int kMaxSlots>
__global__ void __launch_bounds__(kThreads) modulate_swiglu_kernel(const ModParams p) {
  __shared__ float2 scratch[kThreads / 32];
  const int nchunks = p.C / 8;
  const int fchunks = p.F / 8;
  const float inv_c = 1.0f / static_cast<float>(p.C);
  for (int64_t t = blockIdx.x; t < p.T; t += gridDim.x) {
    const int seg = find_segment(p.cu, p.B, t);
    const int64_t mod_row = static_cast<int64_t>(seg) * p.C;
    // ---- part 1: gated residual, norm, modulation
    float xv[kMaxSlots][8];
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int k = 0; k < kMaxSlots; ++k) {
      const int c = threadIdx.x + k * kThreads;
      if (c < nchunks) {
        unpack8(*reinterpret_cast<const uint4*>(p.x + t * p.C + c * 8), xv[k]);
        if (p.branch != nullptr) {
          float br[8], g[8];
          unpack8(*reinterpret_cast<const uint4*>(p.branch + t * p.C + c * 8), br);
          load8f(p.gate_res + mod_row + c * 8, g);
#pragma unroll
          for (int i = 0; i < 8; ++i) xv[k][i] = fmaf(g[i], br[i], xv[k][i]);
        }
        if (p.x_out != nullptr) *reinterpret_cast<uint4*>(p.x_out + t * p.C + c * 8) = pack8(xv[k]);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          s1 += xv[k][i];
          s2 = fmaf(xv[k][i], xv[k][i], s2);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) xv[k][i] = 0.f;
      }
    }
    float mu = 0.f, inv = 1.f;
    if (p.norm_type == 0) {
      const float2 r = block_sum2(s1, s2, scratch);
      inv = rsqrtf(r.y * inv_c + p.eps);
    } else if (p.norm_type == 1) {
      // two passes over the registers: mean, then the centred second moment
      const float2 r = block_sum2(s1, 0.f, scratch);
      mu = r.x * inv_c;
      float d2 = 0.f;
#pragma unroll
      for (int k = 0; k < kMaxSlots; ++k) {
        const int c = threadIdx.x + k * kThreads;
        if (c < nchunks) {
#pragma unroll
          for (int i = 0; i < 8; ++i) d2 = fmaf(xv[k][i] - mu, xv[k][i] - mu, d2);
        }
      }
      const float2 r2 = block_sum2(d2, 0.f, scratch);
      inv = rsqrtf(r2.x * inv_c + p.eps);
    }
#pragma unroll
    for (int k = 0; k < kMaxSlots; ++k) {
      const int c = threadIdx.x + k * kThreads;
      if (c < nchunks) {
        float sc[8], sh[8], hv[8];
        load8f(p.scale + mod_row + c * 8, sc);
        load8f(p.shift + mod_row + c * 8, sh);
#pragma unroll
        for (int i = 0; i < 8; ++i) hv[i] = fmaf((xv[k][i] - mu) * inv, 1.0f + sc[i], sh[i]);
        *reinterpret_cast<uint4*>(p.h + t * p.C + c * 8) = pack8(hv);
      }
    }
    // ---- part 2: SwiGLU
    if (p.gate != nullptr) {
      const __nv_bfloat16* grow = p.gate + t * p.gu_stride;
      const __nv_bfloat16* urow = p.up + t * p.gu_stride;
      __nv_bfloat16* arow = p.act + t * static_cast<int64_t>(p.F);
      for (int c0 = threadIdx.x; c0 < fchunks; c0 += kThreads * kUnroll) {
        uint4 gr[kUnroll], ur[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int c = c0 + u * kThreads;
          if (c < fchunks) {
            gr[u] = *reinterpret_cast<const uint4*>(grow + c * 8);
            ur[u] = *reinterpret_cast<const uint4*>(urow + c * 8);
          }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int c = c0 + u * kThreads;
          if (c < fchunks) {
            float g[8], uu[8], a[8];
            unpack8(gr[u], g);
            unpack8(ur[u], uu);
#pragma unroll
            for (int i = 0; i < 8; ++i) a[i] = silu_mul(g[i], uu[i]);
            *reinterpret_cast<uint4*>(arow + c * 8) = pack8(a);
          }
        }
      }
    }
  }
}

}  // namespace

int launch_modulate_swiglu(const void* x, const void* branch, void* x_out, void* h, const float* shift,
                           const float* scale, const float* gate_res, const int32_t* cu_seqlens, int B, int64_t T,
                           int C, int norm_type, float eps, const void* gate, const void* up, int64_t gu_stride,
                           void* act, int F, cudaStream_t stream, int num_sms) {
  ModParams p;
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.branch = static_cast<const __nv_bfloat16*>(branch);
  p.x_out = static_cast<__nv_bfloat16*>(x_out);
  p.h = static_cast<__nv_bfloat16*>(h);
  p.shift = shift;
  p.scale = scale;
  p.gate_res = gate_res;
  p.cu = cu_seqlens;
  p.B = B;
  p.T = T;
  p.C = C;
  p.norm_type = norm_type;
  p.eps = eps;
  p.gate = static_cast<const __nv_bfloat16*>(gate);
  p.up = static_cast<const __nv_bfloat16*>(up);
  p.gu_stride = gu_stride;
  p.act = static_cast<__nv_bfloat16*>(act);
  p.F = gate != nullptr ? F : 0;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  const int grid = static_cast<int>(T < cap ? T : cap);
  const int slots = (C / 8 + kThreads - 1) / kThreads;
  if (slots <= 1)
    modulate_swiglu_kernel<1><<<grid, kThreads, 0, stream>>>(p);
  else if (slots <= 2)
    modulate_swiglu_kernel<2><<<grid, kThreads, 0, stream>>>(p);
  else if (slots <= 4)
    modulate_swiglu_kernel<4><<<grid, kThreads, 0, stream>>>(p);
  else
    modulate_swiglu_kernel<8><<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace pqk
