// modulate_swiglu.cu -- fused adaLN modulation + normalisation + gated
// residual, and SwiGLU ("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长",
// section "融合 DiT 算子": RMSNorm, SwiGLU and residual connections fused,
// SwiGLU in place of a separate SiLU and multiply; "MiniMax H3 FastH3
// real-time serving with vLLM-Omni", bullet "Fused DiT operators":
// modulation and normalization among the fused operators).
//
// HBM-bound. One warp owns one token at a time (grid-stride over tokens,
// eight warps per block, no block barriers): it streams the token's C-wide
// row in 16-byte chunks, forms the gated residual and its sum / sum of
// squares (shuffle reduction), reads the row again from cache to write x'
// and h = norm * (1 + scale) + shift with the request's modulation vectors
// (read-only cache, shared by every token of the request), then streams
// the token's gate / up rows, kUnroll chunks in flight per lane.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pqk_internal.h"

namespace pqk {
namespace {

constexpr int kThreads = 256;
// Two chunks of gate and up in flight per lane keep the kernel at 64
// registers, so four blocks (32 warps) fit on an SM: at 4,096 tokens every
// token has a resident warp from the start (with four chunks and 80
// registers only three blocks fit, and 15 % of the tokens waited for a
// second wave). Measured faster at every size from 4,096 to 186,489 tokens.
constexpr int kBlocksPerSm = 4;
constexpr int kUnroll = 2;

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

__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// x' chunk c of token t: x + gate_res[s] * branch (or x alone).
__device__ __forceinline__ void residual_chunk(const ModParams& p, int64_t t, int64_t mod_row, int c, float (&xv)[8]) {
  unpack8(*reinterpret_cast<const uint4*>(p.x + t * p.C + c * 8), xv);
  if (p.branch != nullptr) {
    float br[8], g[8];
    unpack8(*reinterpret_cast<const uint4*>(p.branch + t * p.C + c * 8), br);
    load8f(p.gate_res + mod_row + c * 8, g);
#pragma unroll
    for (int i = 0; i < 8; ++i) xv[i] = fmaf(g[i], br[i], xv[i]);
  }
}

// One warp per token (grid-stride over tokens). Pass 1 streams the token's
// C-wide row, forms x' and its sum and sum of squares; a shuffle reduction
// gives the statistics to every lane. Pass 2 reads the row again (now in
// L1/L2), re-forms x' bit-identically and writes x' (when requested) and h. Then the lanes stream the token's gate / up rows. No block
// barriers: each warp moves at its own pace.
__global__ void __launch_bounds__(kThreads, kBlocksPerSm) modulate_swiglu_kernel(const ModParams p) {
  const int lane = threadIdx.x & 31;
  const int nchunks = p.C / 8;
  const int fchunks = p.F / 8;
  const float inv_c = 1.0f / static_cast<float>(p.C);
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5); t < p.T;
       t += warps_total) {
    const int seg = find_segment(p.cu, p.B, t);
    const int64_t mod_row = static_cast<int64_t>(seg) * p.C;
    float s1 = 0.f, s2 = 0.f;
    for (int c = lane; c < nchunks; c += 32) {
      float xv[8];
      residual_chunk(p, t, mod_row, c, xv);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        s1 += xv[i];
        s2 = fmaf(xv[i], xv[i], s2);
      }
    }
    float mu = 0.f, inv = 1.f;
    if (p.norm_type == 0) {
      inv = rsqrtf(warp_sum(s2) * inv_c + p.eps);
    } else if (p.norm_type == 1) {
      mu = warp_sum(s1) * inv_c;
      // centred second moment from a second read of the row
      float d2 = 0.f;
      for (int c = lane; c < nchunks; c += 32) {
        float xv[8];
        residual_chunk(p, t, mod_row, c, xv);
#pragma unroll
        for (int i = 0; i < 8; ++i) d2 = fmaf(xv[i] - mu, xv[i] - mu, d2);
      }
      inv = rsqrtf(warp_sum(d2) * inv_c + p.eps);
    }
    for (int c = lane; c < nchunks; c += 32) {
      float xv[8], sc[8], sh[8], hv[8];
      residual_chunk(p, t, mod_row, c, xv);
      // x' goes out in this last pass over the row, after its statistics: x
      // is read for the last time here, so x_out (and h) may overwrite it
      if (p.x_out != nullptr) *reinterpret_cast<uint4*>(p.x_out + t * p.C + c * 8) = pack8(xv);
      load8f(p.scale + mod_row + c * 8, sc);
      load8f(p.shift + mod_row + c * 8, sh);
#pragma unroll
      for (int i = 0; i < 8; ++i) hv[i] = fmaf((xv[i] - mu) * inv, 1.0f + sc[i], sh[i]);
      *reinterpret_cast<uint4*>(p.h + t * p.C + c * 8) = pack8(hv);
    }
    if (p.gate != nullptr) {
      const __nv_bfloat16* grow = p.gate + t * p.gu_stride;
      const __nv_bfloat16* urow = p.up + t * p.gu_stride;
      __nv_bfloat16* arow = p.act + t * static_cast<int64_t>(p.F);
      for (int c0 = lane; c0 < fchunks; c0 += 32 * kUnroll) {
        uint4 gr[kUnroll], ur[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int c = c0 + u * 32;
          if (c < fchunks) {
            gr[u] = *reinterpret_cast<const uint4*>(grow + c * 8);
            ur[u] = *reinterpret_cast<const uint4*>(urow + c * 8);
          }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int c = c0 + u * 32;
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
  const int64_t warps_per_block = kThreads / 32;
  const int64_t want = (T + warps_per_block - 1) / warps_per_block;
  const int64_t cap = static_cast<int64_t>(num_sms) * kBlocksPerSm;
  const int grid = static_cast<int>(want < cap ? want : cap);
  modulate_swiglu_kernel<<<grid, kThreads, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace pqk
