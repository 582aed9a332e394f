// qk_norm_rope.cu -- fused Q/K RMSNorm + RoPE ("Q/K normalisation merged
// with RoPE": "FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长", section
// "融合 DiT 算子"; "MiniMax H3 FastH3 real-time serving with vLLM-Omni",
// bullet "Fused DiT operators").
//
// HBM-bound: every bf16 element is read once and written once. One warp owns
// one token at a time and walks its 2*H rows (Q heads, then K heads); each
// row of D elements is split over D/8 lanes holding 8 elements (16 bytes)
// apiece, so a warp step moves 2 (D=128) or 4 (D=64) full rows with fully
// coalesced 16-byte accesses. The RMS reduction is a shuffle butterfly over
// the row's lanes. A lane's RoPE angles only depend on the token and on its
// fixed column slice, so cos/sin are formed once per token and reused for
// all 2*H rows; the angle pos * base^(-2j/D) is formed and reduced modulo
// 2*pi in fp64 (positions reach ~1.9e5, where an fp32 angle is off by
// ~1e-2 rad) and only the reduced angle goes through the fp32 sine/cosine.
// The three-axis variant (video latents with (t, h, w) ids) keeps the same
// frequencies and takes each pair's position from the axis of its section.
// The full-width variant normalises over all H*D elements of a token's Q (or
// K) with one weight per element: a first pass of the warp over the token's
// rows sums the squares (full-warp reduction), the second pass re-reads the
// rows (now in cache), normalises, rotates and stores.
// The e4m3-output variant (SAGE FP8 folded into the prologue) writes codes
// [T, H, D] bytes at one scale per tensor, the bound sqrt(D) max|w| of a
// normalised row mapping to 448, and the [2H] dequantisation factors.
// Few tokens: with about one token per resident warp the slowest warps take
// two tokens while most take one, and the launch ends at the tail. The
// launcher then splits each token's 2*H rows into n_split tasks of
// rows_per_task rows (a warp task is a (token, row range) pair; every task
// forms its own cos/sin), chosen so that each warp gets several tasks; with
// enough tokens n_split is 1 and a task is a whole token.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pqk_internal.h"

namespace pqk {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;  // warp steps whose loads are in flight together

struct QkParams {
  const __nv_bfloat16* q_in;
  const __nv_bfloat16* k_in;
  __nv_bfloat16* q_out;
  __nv_bfloat16* k_out;
  int64_t q_stride;      // elements between tokens of q_in
  int64_t k_stride;
  int64_t q_out_stride;  // elements between tokens of q_out
  int64_t k_out_stride;
  const __nv_bfloat16* wq;
  const __nv_bfloat16* wk;
  const int32_t* pos;  // [T] ids, or [T, 3] (t, h, w) ids for the three-axis variant
  int sec0, sec1;      // three-axis: pairs j < sec0 use t, j < sec0 + sec1 use h, the rest w
  int64_t T;
  int H;
  float eps;
  double log2_base;
  int style;
  int n_split;        // tasks per token (1: the whole token)
  int rows_per_task;  // rows of the token's 2H a task covers (2H when n_split is 1)
  float* deq;         // e4m3 output: [2H] dequantisation factors (Q's heads, then K's)
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

// Angle phi = pos * theta reduced to [-pi, pi] in fp64, then the SFU sin/cos
// in fp32 (accurate on that range).
__device__ __forceinline__ void rope_sincos(int32_t pos, double theta, float& c, float& s) {
  const double kTwoPi = 6.283185307179586476925286766559;
  const double phi = static_cast<double>(pos) * theta;
  const double k = rint(phi * (1.0 / kTwoPi));
  const float r = static_cast<float>(fma(-k, kTwoPi, phi));
  __sincosf(r, &s, &c);  // |r| <= pi: absolute error ~4e-7
}

template <int D, bool kThreeAxis, bool kFullWidth, bool kSplit, bool kE4m3Out = false>
__global__ void __launch_bounds__(kThreads, 3) qk_norm_rope_kernel(const QkParams p) {
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerStep = 32 / kLanesPerRow;
  constexpr int kHalfLanes = kLanesPerRow / 2;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow;  // row within a warp step
  const int chunk = lane % kLanesPerRow;  // 8-element column slice of the row
  const bool interleaved = p.style == 0;

  // theta_j = base^(-2j/D) for the D/2 pair indices, shared by the block.
  // Interleaved: a lane's slice holds pairs j = 4*chunk .. 4*chunk+3. Half:
  // it holds first-half elements j = 8*(chunk mod D/16) .. +7 or their
  // second-half partners.
  __shared__ double theta[D / 2];
  for (int j = threadIdx.x; j < D / 2; j += kThreads)
    theta[j] = exp2(-2.0 * static_cast<double>(j) / static_cast<double>(D) * p.log2_base);
  __syncthreads();
  const int j0 = interleaved ? 4 * chunk : 8 * (chunk % kHalfLanes);
  // three-axis: which of (t, h, w) each of this lane's pair slots reads
  int axis[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int j = j0 + i;
    axis[i] = kThreeAxis ? (j < p.sec0 ? 0 : (j < p.sec0 + p.sec1 ? 1 : 2)) : 0;
  }
  // per-head weights ([D], shared by all heads) stay in registers
  const uint4 wq_raw = kFullWidth ? make_uint4(0, 0, 0, 0) : *reinterpret_cast<const uint4*>(p.wq + chunk * 8);
  const uint4 wk_raw = kFullWidth ? make_uint4(0, 0, 0, 0) : *reinterpret_cast<const uint4*>(p.wk + chunk * 8);
  // e4m3 output: a normalised row has sum (x/rms)^2 <= D, so every element of
  // it, rotated or not, is at most sqrt(D) max|w| in magnitude; that bound
  // maps to 448 (one scale per tensor, no pass over the data)
  float inv_q8 = 1.0f, inv_k8 = 1.0f;
  if constexpr (kE4m3Out) {
    float wv[8], mq = 0.f, mk = 0.f;
    unpack8(wq_raw, wv);
#pragma unroll
    for (int i = 0; i < 8; ++i) mq = fmaxf(mq, fabsf(wv[i]));
    unpack8(wk_raw, wv);
#pragma unroll
    for (int i = 0; i < 8; ++i) mk = fmaxf(mk, fabsf(wv[i]));
#pragma unroll
    for (int off = kHalfLanes; off >= 1; off >>= 1) {
      mq = fmaxf(mq, __shfl_xor_sync(0xffffffffu, mq, off));
      mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, off));
    }
    const float aq = sqrtf(static_cast<float>(D)) * mq, ak = sqrtf(static_cast<float>(D)) * mk;
    inv_q8 = aq > 0.0f ? 448.0f / aq : 1.0f;
    inv_k8 = ak > 0.0f ? 448.0f / ak : 1.0f;
    if (blockIdx.x == 0)
      for (int h = threadIdx.x; h < 2 * p.H; h += kThreads)
        p.deq[h] = h < p.H ? (aq > 0.0f ? aq / 448.0f : 1.0f) : (ak > 0.0f ? ak / 448.0f : 1.0f);
  }
  const int64_t warps_total = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  const int64_t n_tasks = kSplit ? p.T * p.n_split : p.T;
  for (int64_t task = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + threadIdx.x / 32; task < n_tasks;
       task += warps_total) {
    const int64_t t = kSplit ? task / p.n_split : task;
    // this task's rows [r_lo, rows) of the token's 2H (Q heads, then K heads)
    const int r_lo = kSplit ? static_cast<int>(task % p.n_split) * p.rows_per_task : 0;
    const int rows = kSplit ? min(2 * p.H, r_lo + p.rows_per_task) : 2 * p.H;
    int32_t pos3[3];
    if constexpr (kThreeAxis) {
      pos3[0] = p.pos[3 * t];
      pos3[1] = p.pos[3 * t + 1];
      pos3[2] = p.pos[3 * t + 2];
    } else {
      pos3[0] = p.pos[t];
    }
    // a slot's position by selection, not by indexing pos3 (which would
    // place pos3 in local memory)
    auto slot_pos = [&](int i) {
      if constexpr (kThreeAxis) return axis[i] == 0 ? pos3[0] : (axis[i] == 1 ? pos3[1] : pos3[2]);
      return pos3[0];
    };
    float cs[8], sn[8];
    if (interleaved) {
#pragma unroll
      for (int i = 0; i < 4; ++i) rope_sincos(slot_pos(i), theta[j0 + i], cs[i], sn[i]);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) rope_sincos(slot_pos(i), theta[j0 + i], cs[i], sn[i]);
    }
    // full width: the RMS of every Q (and K) element of the token, from a
    // first pass over its rows and a reduction over the whole warp
    float inv_q = 0.f, inv_k = 0.f;
    if constexpr (kFullWidth) {
      float ssq_q = 0.f, ssq_k = 0.f;
      for (int r0 = r_lo; r0 < rows; r0 += kRowsPerStep * kUnroll) {
        uint4 raw[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int r = r0 + u * kRowsPerStep + sub;
          raw[u] = make_uint4(0, 0, 0, 0);
          if (r < rows) {
            const bool is_q = r < p.H;
            const __nv_bfloat16* src = is_q ? p.q_in + t * p.q_stride : p.k_in + t * p.k_stride;
            raw[u] = *reinterpret_cast<const uint4*>(src + (is_q ? r : r - p.H) * D + chunk * 8);
          }
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
          const int r = r0 + u * kRowsPerStep + sub;
          float x[8];
          unpack8(raw[u], x);
          float ss = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
          if (r < p.H) ssq_q += ss; else ssq_k += ss;
        }
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        ssq_q += __shfl_xor_sync(0xffffffffu, ssq_q, off);
        ssq_k += __shfl_xor_sync(0xffffffffu, ssq_k, off);
      }
      const float inv_width = 1.0f / static_cast<float>(p.H * D);
      inv_q = rsqrtf(ssq_q * inv_width + p.eps);
      inv_k = rsqrtf(ssq_k * inv_width + p.eps);
    }
    for (int r0 = r_lo; r0 < rows; r0 += kRowsPerStep * kUnroll) {
      uint4 raw[kUnroll];
      bool live[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int r = r0 + u * kRowsPerStep + sub;
        live[u] = r < rows;
        raw[u] = make_uint4(0, 0, 0, 0);
        if (live[u]) {
          const bool is_q = r < p.H;
          const int h = is_q ? r : r - p.H;
          const __nv_bfloat16* src = is_q ? p.q_in + t * p.q_stride : p.k_in + t * p.k_stride;
          raw[u] = *reinterpret_cast<const uint4*>(src + h * D + chunk * 8);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int r = r0 + u * kRowsPerStep + sub;
        const bool is_q = r < p.H;
        float x[8];
        unpack8(raw[u], x);
        float inv;
        float wv[8], y[8];
        if constexpr (kFullWidth) {
          inv = is_q ? inv_q : inv_k;
          // one weight per element of the token's H*D row
          const int h = is_q ? r : r - p.H;
          uint4 wraw = make_uint4(0, 0, 0, 0);
          if (live[u]) wraw = __ldg(reinterpret_cast<const uint4*>((is_q ? p.wq : p.wk) + h * D + chunk * 8));
          unpack8(wraw, wv);
        } else {
          float ss = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) ss = fmaf(x[i], x[i], ss);
#pragma unroll
          for (int off = kHalfLanes; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
          inv = rsqrtf(ss * (1.0f / D) + p.eps);
          unpack8(is_q ? wq_raw : wk_raw, wv);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) y[i] = x[i] * inv * wv[i];
        float o[8];
        if (interleaved) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float a = y[2 * i], b = y[2 * i + 1];
            o[2 * i] = a * cs[i] - b * sn[i];
            o[2 * i + 1] = a * sn[i] + b * cs[i];
          }
        } else {
          const bool first_half = chunk < kHalfLanes;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float partner = __shfl_xor_sync(0xffffffffu, y[i], kHalfLanes);
            o[i] = first_half ? (y[i] * cs[i] - partner * sn[i]) : (partner * sn[i] + y[i] * cs[i]);
          }
        }
        if (live[u]) {
          const int h = is_q ? r : r - p.H;
          if constexpr (kE4m3Out) {
            // codes [T, H, D] bytes: 8 per lane
            const float inv = is_q ? inv_q8 : inv_k8;
            uint2 c;
            c.x = pack_e4m3x2(o[0] * inv, o[1] * inv) | (pack_e4m3x2(o[2] * inv, o[3] * inv) << 16);
            c.y = pack_e4m3x2(o[4] * inv, o[5] * inv) | (pack_e4m3x2(o[6] * inv, o[7] * inv) << 16);
            uint8_t* dst8 = reinterpret_cast<uint8_t*>(is_q ? p.q_out : p.k_out) + (t * p.H + h) * D + chunk * 8;
            *reinterpret_cast<uint2*>(dst8) = c;
          } else {
            __nv_bfloat16* dst = is_q ? p.q_out + t * p.q_out_stride : p.k_out + t * p.k_out_stride;
            *reinterpret_cast<uint4*>(dst + h * D + chunk * 8) = pack8(o);
          }
        }
      }
    }
  }
}

}  // namespace

int launch_qk_norm_rope(const void* q_in, const void* k_in, void* q_out, void* k_out, int64_t q_stride,
                        int64_t k_stride, int64_t q_out_stride, int64_t k_out_stride, const void* wq,
                        const void* wk, const int32_t* pos, const int* sections,
                        bool full_width, int64_t T, int H, int D, float eps, float rope_base, int style,
                        cudaStream_t stream, int num_sms, float* e4m3_deq) {
  QkParams p;
  p.q_in = static_cast<const __nv_bfloat16*>(q_in);
  p.k_in = static_cast<const __nv_bfloat16*>(k_in);
  p.q_out = static_cast<__nv_bfloat16*>(q_out);
  p.k_out = static_cast<__nv_bfloat16*>(k_out);
  p.q_stride = q_stride;
  p.k_stride = k_stride;
  p.q_out_stride = q_out_stride;
  p.k_out_stride = k_out_stride;
  p.deq = e4m3_deq;
  p.wq = static_cast<const __nv_bfloat16*>(wq);
  p.wk = static_cast<const __nv_bfloat16*>(wk);
  p.pos = pos;
  p.sec0 = sections ? sections[0] : 0;
  p.sec1 = sections ? sections[1] : 0;
  p.T = T;
  p.H = H;
  p.eps = eps;
  p.log2_base = log2(static_cast<double>(rope_base));
  p.style = style;
  const int64_t warps_per_block = kThreads / 32;
  const int64_t cap = static_cast<int64_t>(num_sms) * 3;
  // split tokens into row ranges when there are fewer than 2 * kTasksPerWarp
  // tokens per resident warp (not for the full-width norm, which needs all
  // of a token's rows in one warp): into enough ranges for kTasksPerWarp
  // tasks per warp, and at least two (measured at 40 heads: 0.83 -> 0.86 of
  // HBM at 16,384 tokens from the two-way split); ranges are whole warp steps
  // of rows
  constexpr int64_t kTasksPerWarp = 4;
  const int rows = 2 * H;
  const int step_rows = (32 / (D / 8)) * kUnroll;
  const int64_t resident_warps = cap * warps_per_block;
  int rows_per_task = rows;
  if (!full_width && T < 2 * kTasksPerWarp * resident_warps) {
    int64_t want_split = (kTasksPerWarp * resident_warps + T - 1) / (T > 0 ? T : 1);
    if (want_split < 2) want_split = 2;
    const int r = static_cast<int>(rows / want_split) / step_rows * step_rows;
    rows_per_task = r > step_rows ? r : step_rows;
    if (rows_per_task > rows) rows_per_task = rows;
  }
  p.rows_per_task = rows_per_task;
  p.n_split = (rows + rows_per_task - 1) / rows_per_task;
  const int64_t tasks = T * p.n_split;
  const int64_t want = (tasks + warps_per_block - 1) / warps_per_block;
  const int grid = static_cast<int>(want < cap ? want : cap);
  const bool three = sections != nullptr;
  const bool split = p.n_split > 1;
  if (e4m3_deq != nullptr) {
    // one-axis positions, per-head norm only
    if (three || full_width) return -1;
    if (D == 128)
      split ? qk_norm_rope_kernel<128, false, false, true, true><<<grid, kThreads, 0, stream>>>(p)
            : qk_norm_rope_kernel<128, false, false, false, true><<<grid, kThreads, 0, stream>>>(p);
    else
      split ? qk_norm_rope_kernel<64, false, false, true, true><<<grid, kThreads, 0, stream>>>(p)
            : qk_norm_rope_kernel<64, false, false, false, true><<<grid, kThreads, 0, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
  }
  if (D == 128) {
    if (full_width)
      qk_norm_rope_kernel<128, false, true, false><<<grid, kThreads, 0, stream>>>(p);
    else if (three)
      split ? qk_norm_rope_kernel<128, true, false, true><<<grid, kThreads, 0, stream>>>(p)
            : qk_norm_rope_kernel<128, true, false, false><<<grid, kThreads, 0, stream>>>(p);
    else
      split ? qk_norm_rope_kernel<128, false, false, true><<<grid, kThreads, 0, stream>>>(p)
            : qk_norm_rope_kernel<128, false, false, false><<<grid, kThreads, 0, stream>>>(p);
  } else {
    if (full_width)
      qk_norm_rope_kernel<64, false, true, false><<<grid, kThreads, 0, stream>>>(p);
    else if (three)
      split ? qk_norm_rope_kernel<64, true, false, true><<<grid, kThreads, 0, stream>>>(p)
            : qk_norm_rope_kernel<64, true, false, false><<<grid, kThreads, 0, stream>>>(p);
    else
      split ? qk_norm_rope_kernel<64, false, false, true><<<grid, kThreads, 0, stream>>>(p)
            : qk_norm_rope_kernel<64, false, false, false><<<grid, kThreads, 0, stream>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace pqk
