// linear_epilogue.cu -- persistent tcgen05 GEMM out = epilogue(A W^T) for
// the linear layers around the DiT block's fused operators, with the
// residual connection or SwiGLU done in the GEMM's epilogue instead of a
// separate pass over the GEMM's output (the pages fuse "residual
// connections" and SwiGLU into fewer launches: "FastH3 在八卡 B300 上实现完整
// MP4 生成快于播放时长", section "融合 DiT 算子"; "MiniMax H3 FastH3 real-time
// serving with vLLM-Omni", bullet "Fused DiT operators"):
//
//   kEpiGatedResidual  out[t, n] = x[t, n] + gate_res[s(t), n] * (A W^T)[t, n]
//                      (output projection after attention, W2 after SwiGLU)
//   kEpiSwiglu         out[t, f] = silu((A W_gate^T)[t, f]) * (A W_up^T)[t, f]
//                      (W1; W_gate = the first F rows of W1, W_up the last F)
//   kEpiNone           out = A W^T
//
// A: [T, K] bf16 (token stride a_stride), W: [N, K] bf16 (out x in). fp32
// accumulation in tensor memory, epilogue arithmetic in fp32, bf16 output
// rounded to nearest even.
//
// Structure (one CTA per SM, persistent over 128 x 256 accumulator tiles):
//   warp 0      TMA producer: per K block of 64, the A box (128 tokens x 64)
//               and two W boxes (2 x 128 rows x 64) into a 4-stage ring of
//               48 KB stages, 128-byte swizzled, K-major.
//   warp 1      allocates 512 tensor-memory columns (two 256-column fp32
//               accumulators) and issues tcgen05.mma M=128 N=256 K=16 (four
//               per stage) from one thread; commits free the stage, and the
//               last K block of a tile commits the accumulator to the
//               epilogue.
//   warps 2-5   epilogue: each thread owns one token row (tensor-memory lane)
//               of the tile, reads its accumulator columns 32 at a time, adds
//               the gated residual or applies SwiGLU and stores 16-byte
//               chunks; then releases the accumulator. The two accumulators
//               let the epilogue of one tile run under the main loop of the
//               next.
// The W boxes of a SwiGLU tile are the gate rows f0..f0+127 and the up rows
// F+f0..F+f0+127, so one N = 256 MMA computes both halves of 128 outputs.
// Rows past T or N read as zeros (TMA bounds) and are not stored. Tiles are
// rastered in groups of 16 M tiles so that concurrently running CTAs share
// A rows and W columns in L2.
//
// Every wait is bounded (the library's timeout); a wait that runs out raises
// the block's abort flag and the device status word and every role stops
// issuing work. Once all roles have stopped (a block barrier), the copies and
// MMAs still in flight are drained with waits bounded by kDrainTimeoutNs,
// not by the caller's timeout, and only then is the tensor memory freed.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "pqk_internal.h"

namespace pqk {
namespace {

constexpr int kBM = 128;         // tokens per tile (one tensor-memory lane each)
constexpr int kBK = 64;          // K per stage: one 128-byte swizzle row of bf16
constexpr int kBoxRows = 128;    // W rows per TMA box
constexpr int kAccCols = 256;    // fp32 accumulator columns per tile = MMA N
constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kGroupM = 16;      // tile raster: M tiles per group
constexpr uint32_t kABytes = kBM * kBK * 2;              // 16 KB
constexpr uint32_t kBBytes = 2 * kBoxRows * kBK * 2;     // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;

struct Layout {
  static constexpr int kAOff = 0;
  static constexpr int kBOff = kStages * kABytes;
  static constexpr int kBarOff = kBOff + kStages * kBBytes;
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemSlotOff + 4;
  static constexpr int kBytes = kAbortOff + 4;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
  static_assert(kAlloc <= 232448, "shared memory budget");
  static_assert(kBOff % 1024 == 0 && kBBytes % 1024 == 0 && kABytes % 1024 == 0, "swizzle atoms 1024-aligned");
};

struct LinearParams {
  __nv_bfloat16* out;
  int64_t out_stride;
  const __nv_bfloat16* x;   // gated residual input [T, N]
  int64_t x_stride;
  const float* gate_res;    // [B, N]
  const int32_t* cu;        // [B + 1]
  int B;
  int64_t T;
  int N;                    // output columns (F for SwiGLU)
  int n_kb;                 // K blocks of 64
  int m_tiles;
  int n_tiles;
  int* status;
  long long timeout_ns;
};

struct TileCoord {
  int m;
  int n;
};

// Tile i of the raster: groups of kGroupM M tiles, and inside a group the
// M tile varies fastest, so the CTAs that run together cover a few W column
// blocks of a 16-tile band of A.
__device__ __forceinline__ TileCoord tile_coord(int i, int m_tiles, int n_tiles) {
  const int group_tiles = kGroupM * n_tiles;
  const int g = i / group_tiles;
  const int first_m = g * kGroupM;
  const int gm = min(kGroupM, m_tiles - first_m);
  const int local = i - g * group_tiles;
  TileCoord c;
  c.m = first_m + local % gm;
  c.n = local / gm;
  return c;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int* status) {
  *abort_flag = 1;
  atomicCAS(status, 0, kStatusTimeout);
}

// Request s with cu[s] <= t < cu[s+1] (the last such s when requests are empty).
__device__ __forceinline__ int request_of(const int32_t* cu, int B, int64_t t) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (static_cast<int64_t>(__ldg(cu + mid)) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

template <int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
    linear_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                  const __grid_constant__ CUtensorMap tm_b1, const LinearParams p) {
  using L = Layout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t a_smem = base + L::kAOff;
  const uint32_t b_smem = base + L::kBOff;
  const uint32_t bar0 = base + L::kBarOff;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto acc_full = [&](int i) { return bar0 + 8u * (2 * kStages + i); };
  auto acc_empty = [&](int i) { return bar0 + 8u * (2 * kStages + 2 + i); };
  const uint32_t drain = bar0 + 8u * (2 * kStages + 4);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbortOff);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(base + L::kTmemSlotOff, 512);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensor_map(&tm_a);
    prefetch_tensor_map(&tm_b0);
    prefetch_tensor_map(&tm_b1);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int n_tiles_total = p.m_tiles * p.n_tiles;
  uint32_t loads = 0;  // stage copies issued by the producer thread, for the drain

  if (warp == kProducerWarp) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t& it = loads;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x) {
        const TileCoord tc = tile_coord(tile, p.m_tiles, p.n_tiles);
        // W rows of the tile's two boxes: 256 consecutive output columns, or
        // the same 128 rows of the gate and the up halves
        const int r0 = kEpi == kEpiSwiglu ? tc.n * kBoxRows : tc.n * kAccCols;
        const int r1 = kEpi == kEpiSwiglu ? tc.n * kBoxRows : tc.n * kAccCols + kBoxRows;
        const CUtensorMap* m1 = kEpi == kEpiSwiglu ? &tm_b1 : &tm_b0;
        for (int kb = 0; kb < p.n_kb; ++kb) {
          const int s = it % kStages;
          const uint32_t round = it / kStages;
          if (round > 0 && !(ok = mbar_wait(empty(s), (round - 1) & 1, abort_flag, p.timeout_ns))) break;
          mbar_arrive_expect_tx(full(s), kStageBytes);
          tma_load_2d(a_smem + s * kABytes, &tm_a, full(s), kb * kBK, tc.m * kBM);
          tma_load_2d(b_smem + s * kBBytes, &tm_b0, full(s), kb * kBK, r0);
          tma_load_2d(b_smem + s * kBBytes + kBBytes / 2, m1, full(s), kb * kBK, r1);
          ++it;
        }
      }
      if (!ok) raise_abort(abort_flag, p.status);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kAccCols, false);
      constexpr uint32_t kDescHi = smem_desc_hi_sw128(1024);
      const uint32_t a_lo = smem_desc_lo(a_smem, 16);
      const uint32_t b_lo = smem_desc_lo(b_smem, 16);
      uint32_t it = 0;
      int tcount = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x, ++tcount) {
        const int acc = tcount & 1;
        const uint32_t use = static_cast<uint32_t>(tcount >> 1);
        if (use > 0 && !(ok = mbar_wait(acc_empty(acc), (use - 1) & 1, abort_flag, p.timeout_ns))) break;
        tc_fence_after_sync();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * kAccCols);
        for (int kb = 0; kb < p.n_kb; ++kb) {
          const int s = it % kStages;
          if (!(ok = mbar_wait(full(s), (it / kStages) & 1, abort_flag, p.timeout_ns))) break;
          tc_fence_after_sync();
          // K steps of 16 (32 bytes inside the 128-byte swizzled row)
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            mma_bf16_ss_w(d, a_lo + s * (kABytes >> 4) + 2 * k, b_lo + s * (kBBytes >> 4) + 2 * k, kDescHi, kIdesc,
                          (kb > 0 || k > 0) ? 1u : 0u);
          tc_commit(empty(s));
          ++it;
        }
        if (!ok) break;
        tc_commit(acc_full(acc));
      }
      if (!ok) raise_abort(abort_flag, p.status);
    }
  } else {
    // ------------------------------------------------ epilogue warps 2-5
    const int quarter = warp & 3;  // tensor-memory lanes 32 * quarter .. + 31
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    int tcount = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles_total; tile += gridDim.x, ++tcount) {
      const TileCoord tc = tile_coord(tile, p.m_tiles, p.n_tiles);
      const int acc = tcount & 1;
      const uint32_t use = static_cast<uint32_t>(tcount >> 1);
      ok = __all_sync(0xffffffffu, mbar_wait(acc_full(acc), use & 1, abort_flag, p.timeout_ns));
      if (!ok) break;
      tc_fence_after_sync();
      const int64_t row = static_cast<int64_t>(tc.m) * kBM + quarter * 32 + lane;
      const bool row_ok = row < p.T;
      const uint32_t t_acc = tmem + lane_off + static_cast<uint32_t>(acc * kAccCols);
      __nv_bfloat16* dst = p.out + (row_ok ? row : 0) * p.out_stride;
      if constexpr (kEpi == kEpiSwiglu) {
        const int f0 = tc.n * kBoxRows;
#pragma unroll 1
        for (int c0 = 0; c0 < kBoxRows; c0 += 32) {
          uint32_t g[32], u[32];
          tmem_ld_x32(t_acc + c0, g);
          tmem_ld_x32(t_acc + kBoxRows + c0, u);
          if (row_ok) {
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              const int col = f0 + c0 + c;
              if (col < p.N) {
                uint4 v;
                v.x = pack_bf16x2(silu_mul(__uint_as_float(g[c]), __uint_as_float(u[c])),
                                  silu_mul(__uint_as_float(g[c + 1]), __uint_as_float(u[c + 1])));
                v.y = pack_bf16x2(silu_mul(__uint_as_float(g[c + 2]), __uint_as_float(u[c + 2])),
                                  silu_mul(__uint_as_float(g[c + 3]), __uint_as_float(u[c + 3])));
                v.z = pack_bf16x2(silu_mul(__uint_as_float(g[c + 4]), __uint_as_float(u[c + 4])),
                                  silu_mul(__uint_as_float(g[c + 5]), __uint_as_float(u[c + 5])));
                v.w = pack_bf16x2(silu_mul(__uint_as_float(g[c + 6]), __uint_as_float(u[c + 6])),
                                  silu_mul(__uint_as_float(g[c + 7]), __uint_as_float(u[c + 7])));
                *reinterpret_cast<uint4*>(dst + col) = v;
              }
            }
          }
        }
      } else {
        const int n0 = tc.n * kAccCols;
        const float* grow = nullptr;
        const __nv_bfloat16* xrow = nullptr;
        if (kEpi == kEpiGatedResidual && row_ok) {
          grow = p.gate_res + static_cast<int64_t>(request_of(p.cu, p.B, row)) * p.N;
          xrow = p.x + row * p.x_stride;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < kAccCols; c0 += 32) {
          uint32_t y[32];
          tmem_ld_x32(t_acc + c0, y);
          if (row_ok) {
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              const int col = n0 + c0 + c;
              if (col < p.N) {
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = __uint_as_float(y[c + e]);
                if constexpr (kEpi == kEpiGatedResidual) {
                  const uint4 xv = ld_nc16(xrow + col);
                  const float4 g0 = __ldg(reinterpret_cast<const float4*>(grow + col));
                  const float4 g1 = __ldg(reinterpret_cast<const float4*>(grow + col + 4));
                  o[0] = fmaf(g0.x, o[0], bf16_lo(xv.x));
                  o[1] = fmaf(g0.y, o[1], bf16_hi(xv.x));
                  o[2] = fmaf(g0.z, o[2], bf16_lo(xv.y));
                  o[3] = fmaf(g0.w, o[3], bf16_hi(xv.y));
                  o[4] = fmaf(g1.x, o[4], bf16_lo(xv.z));
                  o[5] = fmaf(g1.y, o[5], bf16_hi(xv.z));
                  o[6] = fmaf(g1.z, o[6], bf16_lo(xv.w));
                  o[7] = fmaf(g1.w, o[7], bf16_hi(xv.w));
                }
                uint4 v;
                v.x = pack_bf16x2(o[0], o[1]);
                v.y = pack_bf16x2(o[2], o[3]);
                v.z = pack_bf16x2(o[4], o[5]);
                v.w = pack_bf16x2(o[6], o[7]);
                *reinterpret_cast<uint4*>(dst + col) = v;
              }
            }
          }
        }
      }
      tc_fence_before_sync();
      mbar_arrive(acc_empty(acc));
    }
    if (!ok) raise_abort(abort_flag, p.status);
  }

  tc_fence_before_sync();
  __syncthreads();
  // Every role has stopped, so the abort flag is final. On an abort, wait for
  // the copies and MMAs still in flight before the memory is freed.
  if (*abort_flag) {
    if (warp == kProducerWarp && lane == 0) {
      // copy idx was issued only after copy idx - kStages had landed: the
      // last kStages copies are the ones that can be outstanding
      const uint32_t first = loads > static_cast<uint32_t>(kStages) ? loads - kStages : 0;
      for (uint32_t idx = first; idx < loads; ++idx) mbar_drain_wait(full(idx % kStages), (idx / kStages) & 1);
    } else if (warp == kMmaWarp && lane == 0) {
      // completes once every MMA this thread issued has
      tc_commit(drain);
      mbar_drain_wait(drain, 0);
    }
    __syncthreads();
  }
  tc_fence_after_sync();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// [rows, cols] bf16 with `stride` elements between rows, read as boxes of 64
// columns x box_rows rows, 128-byte swizzled; reads past the edges give 0.
bool make_rows_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int64_t stride, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(stride) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int kEpi>
bool set_smem_attr() {
  static int done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(linear_kernel<kEpi>, cudaFuncAttributeMaxDynamicSharedMemorySize, Layout::kAlloc) !=
        cudaSuccess)
      return false;
    done[dev] = 1;
  }
  return true;
}

template <int kEpi>
int launch(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1, const LinearParams& p,
           cudaStream_t stream, int num_sms) {
  if (!set_smem_attr<kEpi>()) return -1;
  const int tiles = p.m_tiles * p.n_tiles;
  const int grid = tiles < num_sms ? tiles : num_sms;
  linear_kernel<kEpi><<<grid, kThreads, Layout::kAlloc, stream>>>(ta, tb0, tb1, p);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace

int launch_linear(int epi, const void* a, int64_t a_stride, const void* w, const void* x, int64_t x_stride,
                  const float* gate_res, const int32_t* cu, int B, void* out, int64_t out_stride, int64_t T, int K,
                  int N, int* status, long long timeout_ns, cudaStream_t stream, int num_sms) {
  CUtensorMap ta, tb0, tb1;
  const bool swiglu = epi == kEpiSwiglu;
  bool ok = make_rows_map(&ta, a, T, K, a_stride, kBM);
  if (swiglu) {
    // W1 [2N, K]: gate rows [0, N), up rows [N, 2N), each its own map so that
    // the last tile's rows past N read as zeros rather than the other half
    ok = ok && make_rows_map(&tb0, w, N, K, K, kBoxRows) &&
         make_rows_map(&tb1, static_cast<const __nv_bfloat16*>(w) + static_cast<int64_t>(N) * K, N, K, K, kBoxRows);
  } else {
    ok = ok && make_rows_map(&tb0, w, N, K, K, kBoxRows);
    tb1 = tb0;
  }
  if (!ok) return -2;
  LinearParams p;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.out_stride = out_stride;
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.x_stride = x_stride;
  p.gate_res = gate_res;
  p.cu = cu;
  p.B = B;
  p.T = T;
  p.N = N;
  p.n_kb = (K + kBK - 1) / kBK;
  p.m_tiles = static_cast<int>((T + kBM - 1) / kBM);
  p.n_tiles = swiglu ? (N + kBoxRows - 1) / kBoxRows : (N + kAccCols - 1) / kAccCols;
  p.status = status;
  p.timeout_ns = timeout_ns;
  if (epi == kEpiGatedResidual) return launch<kEpiGatedResidual>(ta, tb0, tb1, p, stream, num_sms);
  if (swiglu) return launch<kEpiSwiglu>(ta, tb0, tb1, p, stream, num_sms);
  return launch<kEpiNone>(ta, tb0, tb1, p, stream, num_sms);
}

}  // namespace pqk
