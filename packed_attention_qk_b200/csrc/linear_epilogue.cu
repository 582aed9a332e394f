// linear_epilogue.cu -- persistent tcgen05 GEMM on CTA pairs,
// out = epilogue(A W^T), for the linear layers around the DiT block's fused
// operators, with the residual connection or SwiGLU done in the GEMM's
// epilogue instead of a separate pass over the GEMM's output (the pages fuse
// "residual connections" and SwiGLU into fewer launches: "FastH3 在八卡 B300 上
// 实现完整 MP4 生成快于播放时长", section "融合 DiT 算子"; "MiniMax H3 FastH3
// real-time serving with vLLM-Omni", bullet "Fused DiT operators"):
//
//   kEpiGatedResidual  out[t, n] = x[t, n] + gate_res[s(t), n] * (A W^T)[t, n]
//   kEpiSwiglu         out[t, f] = silu((A W_gate^T)[t, f]) * (A W_up^T)[t, f]
//   kEpiNone           out = A W^T
//
// A: [T, K] bf16 (token stride a_stride), W: [N, K] bf16 (out x in). fp32
// accumulation in tensor memory, epilogue arithmetic in fp32, bf16 output
// rounded to nearest even.
//
// Two CTAs of a cluster work on one 256-token x 256-column accumulator tile
// (tcgen05 cta_group::2, M = 256): each CTA loads its 128 A rows and 128 of
// the 256 W rows per K block of 64 into its own 6-stage ring (32 KB stages),
// the even CTA's single MMA thread drives both SMs' tensor cores, and each
// CTA's tensor memory holds its 128 rows of the tile in one of two
// 256-column accumulators.
//   warp 0      TMA producer in each CTA; copies complete on the even CTA's
//               stage barrier, where only the even CTA posts the stage's
//               bytes and then lets the odd CTA's producer load its halves.
//   warp 1      allocates the tensor memory of the pair; in the even CTA
//               issues the MMAs and commits stage releases and finished
//               accumulators to its own barriers.
//   warps 2-5   epilogue in each CTA: 32 token rows per warp, 32 columns of
//               the accumulator at a time, the gated residual or SwiGLU, 16-
//               byte stores; one release per warp to the even CTA's MMA
//               thread. The even CTA passes "accumulator ready" on to the odd
//               CTA.
// Hand-offs between the two CTAs are plain remote mbarrier arrives, one CTA
// signalling the other. A SwiGLU tile's W halves are 128 gate rows (even
// CTA) and the same 128 up rows (odd CTA). Rows past T or N and columns past
// K read as zeros and are not stored.
//
// Every wait is bounded (the library's timeout); a wait that runs out raises
// the abort flag of both CTAs and the device status word, and every role of
// the pair stops issuing work. After a cluster barrier (when both flags are
// final) the even CTA waits for the stages it posted that may still be
// loading (their barriers complete only once both CTAs' copies have landed:
// the odd CTA copies into a stage only after the even one posted it) and for
// every MMA it issued, with waits bounded by kDrainTimeoutNs rather than the
// caller's timeout; a second cluster barrier keeps the odd CTA, whose copies
// signal the even CTA's barriers, from exiting before that, and both free
// the pair's tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "pqk_internal.h"

namespace pqk {
namespace {

constexpr int kBM = 128;       // token rows per CTA (pair: 256)
constexpr int kBK = 64;        // K per stage: one 128-byte swizzle row of bf16
constexpr int kBoxRows = 128;  // W rows per CTA and stage
constexpr int kAccCols = 256;  // fp32 accumulator columns per tile = MMA N
constexpr int kStages = 6;
constexpr int kThreads = 192;
constexpr int kGroupM = 8;     // raster: pair M tiles per group
constexpr uint32_t kABytes = kBM * kBK * 2;        // 16 KB
constexpr uint32_t kBBytes = kBoxRows * kBK * 2;   // 16 KB
constexpr uint32_t kPairStageBytes = 2 * (kABytes + kBBytes);

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
};

struct Params {
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
  int m_pairs;              // 256-token tiles
  int n_tiles;
  int* status;
  long long timeout_ns;
};

struct TileCoord {
  int m;
  int n;
};
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
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

template <int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
    linear_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                       const __grid_constant__ CUtensorMap tm_b1, const Params p) {
  using L = Layout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = ctarank();
  const bool even = rank == 0;
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
  const uint32_t peer_abort = in_cta(base + L::kAbortOff, rank ^ 1u);
  auto raise_abort = [&]() {
    *abort_flag = 1;
    st_remote_u32(peer_abort, 1u);
    atomicCAS(p.status, 0, kStatusTimeout);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full(i), 1);
      mbar_init(acc_empty(i), 2 * 4);  // one arrive per epilogue warp of each CTA
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(base + L::kTmemSlotOff, 512);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensor_map(&tm_a);
    prefetch_tensor_map(&tm_b0);
    prefetch_tensor_map(&tm_b1);
  }
  tc_fence_before_sync();
  __syncwarp();
  cluster_sync_all();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int total = p.m_pairs * p.n_tiles;
  const int pair = static_cast<int>(cluster_x());
  const int npairs = static_cast<int>(nclusters_x());
  uint32_t loads = 0;  // stages this CTA's producer loaded into, for the drain

  if (warp == 0) {
    // ------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      uint32_t& it = loads;
      bool ok = true;
      const CUtensorMap* mb = (kEpi == kEpiSwiglu && !even) ? &tm_b1 : &tm_b0;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const TileCoord tc = tile_coord(tile, p.m_pairs, p.n_tiles);
        const int arow = tc.m * 2 * kBM + static_cast<int>(rank) * kBM;
        const int brow = kEpi == kEpiSwiglu ? tc.n * kBoxRows : tc.n * kAccCols + static_cast<int>(rank) * kBoxRows;
        for (int kb = 0; kb < p.n_kb; ++kb) {
          const int s = it % kStages;
          const uint32_t round = it / kStages;
          if (even) {
            // the MMAs that read this stage in both CTAs are complete; post the
            // stage's bytes, then let the odd CTA's producer load its halves
            // (so no copy of it completes before the count it belongs to)
            if (round > 0 && !(ok = mbar_wait(empty(s), (round - 1) & 1, abort_flag, p.timeout_ns))) break;
            mbar_arrive_expect_tx(full(s), kPairStageBytes);
            arrive_remote(in_cta(empty(s), 1));
          } else {
            if (!(ok = mbar_wait(empty(s), round & 1, abort_flag, p.timeout_ns))) break;
          }
          const uint32_t bar = in_cta(full(s), 0);
          tma_load_2d_pair(a_smem + s * kABytes, &tm_a, bar, kb * kBK, arow);
          tma_load_2d_pair(b_smem + s * kBBytes, mb, bar, kb * kBK, brow);
          ++it;
        }
      }
      if (!ok) raise_abort();
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && even) {
      constexpr uint32_t kIdesc = idesc_bf16_f32(2 * kBM, kAccCols, false);
      constexpr uint32_t kDescHi = smem_desc_hi_sw128(1024);
      const uint32_t a_lo = smem_desc_lo(a_smem, 16);
      const uint32_t b_lo = smem_desc_lo(b_smem, 16);
      uint32_t it = 0;
      int tcount = 0;
      bool ok = true;
      for (int tile = pair; tile < total && ok; tile += npairs, ++tcount) {
        const int acc = tcount & 1;
        const uint32_t use = static_cast<uint32_t>(tcount >> 1);
        if (use > 0 && !(ok = mbar_wait(acc_empty(acc), (use - 1) & 1, abort_flag, p.timeout_ns))) break;
        tc_fence_after_sync();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * kAccCols);
        for (int kb = 0; kb < p.n_kb; ++kb) {
          const int s = it % kStages;
          if (!(ok = mbar_wait(full(s), (it / kStages) & 1, abort_flag, p.timeout_ns))) break;
          tc_fence_after_sync();
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            mma_bf16_ss_pair(d, a_lo + s * (kABytes >> 4) + 2 * k, b_lo + s * (kBBytes >> 4) + 2 * k, kDescHi, kIdesc,
                             (kb > 0 || k > 0) ? 1u : 0u);
          tc_commit_pair(empty(s));
          ++it;
        }
        if (!ok) break;
        tc_commit_pair(acc_full(acc));
      }
      if (!ok) raise_abort();
    }
  } else {
    // ------------------------------------------------ epilogue warps 2-5 (both CTAs)
    const int quarter = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    int tcount = 0;
    bool ok = true;
    for (int tile = pair; tile < total; tile += npairs, ++tcount) {
      const TileCoord tc = tile_coord(tile, p.m_pairs, p.n_tiles);
      const int acc = tcount & 1;
      const uint32_t use = static_cast<uint32_t>(tcount >> 1);
      ok = __all_sync(0xffffffffu, mbar_wait(acc_full(acc), use & 1, abort_flag, p.timeout_ns));
      if (!ok) break;
      // the even CTA's MMAs wrote both CTAs' accumulators: tell the odd CTA
      if (even && warp == 2 && lane == 0) arrive_remote(in_cta(acc_full(acc), 1));
      tc_fence_after_sync();
      const int64_t row = static_cast<int64_t>(tc.m) * 2 * kBM + rank * kBM + quarter * 32 + lane;
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
      __syncwarp();
      // release the accumulator to the even CTA's MMA issuer (both CTAs' warps count)
      if (lane == 0) arrive_remote(in_cta(acc_empty(acc), 0));
    }
    if (!ok) raise_abort();
  }

  tc_fence_before_sync();
  __syncwarp();
  cluster_sync_all();  // no CTA frees its tensor memory or exits while its pair still works
  // Every role of both CTAs has stopped: the abort flags are final and the
  // same in both CTAs. On an abort, wait for what may still be in flight.
  if (*abort_flag) {
    if (even && warp == 0 && lane == 0) {
      // stage idx was posted only after stage idx - kStages had landed in
      // both CTAs: the last kStages posted stages are the ones outstanding
      const uint32_t first = loads > static_cast<uint32_t>(kStages) ? loads - kStages : 0;
      for (uint32_t idx = first; idx < loads; ++idx) mbar_drain_wait(full(idx % kStages), (idx / kStages) & 1);
    } else if (even && warp == 1 && lane == 0) {
      // completes once every MMA of the pair has
      tc_commit_pair(drain);
      mbar_drain_wait(drain, 0);
    }
    __syncwarp();
    cluster_sync_all();
  }
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc_pair(tmem, 512);
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

// Per device and epilogue: the shared-memory attribute is set and the number
// of CTA pairs that can be resident at once is queried on the first call
// (which must precede any stream capture), so that the persistent grid never
// leaves a pair waiting for a second wave.
template <int kEpi>
int resident_pairs(cudaLaunchConfig_t* cfg) {
  static int pairs[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  if (pairs[dev] == 0) {
    if (cudaFuncSetAttribute(linear_pair_kernel<kEpi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Layout::kAlloc) != cudaSuccess)
      return -1;
    int n = 0;
    cfg->gridDim = dim3(2, 1, 1);
    if (cudaOccupancyMaxActiveClusters(&n, linear_pair_kernel<kEpi>, cfg) != cudaSuccess || n < 1) return -1;
    pairs[dev] = n;
  }
  return pairs[dev];
}

template <int kEpi>
int launch(const CUtensorMap& ta, const CUtensorMap& tb0, const CUtensorMap& tb1, const Params& p,
           cudaStream_t stream) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Layout::kAlloc;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int max_pairs = resident_pairs<kEpi>(&cfg);
  if (max_pairs < 1) return -1;
  const int tiles = p.m_pairs * p.n_tiles;
  cfg.gridDim = dim3(2 * (tiles < max_pairs ? tiles : max_pairs), 1, 1);
  if (cudaLaunchKernelEx(&cfg, linear_pair_kernel<kEpi>, ta, tb0, tb1, p) != cudaSuccess) return -1;
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace

int launch_linear(int epi, const void* a, int64_t a_stride, const void* w, const void* x, int64_t x_stride,
                  const float* gate_res, const int32_t* cu, int B, void* out, int64_t out_stride, int64_t T, int K,
                  int N, int* status, long long timeout_ns, cudaStream_t stream, int num_sms) {
  (void)num_sms;
  CUtensorMap ta, tb0, tb1;
  const bool swiglu = epi == kEpiSwiglu;
  bool ok = make_rows_map(&ta, a, T, K, a_stride, kBM);
  if (swiglu) {
    // W1 [2N, K]: gate rows [0, N) for the even CTA, up rows [N, 2N) for the
    // odd one, each its own map so that rows past N read as zeros
    ok = ok && make_rows_map(&tb0, w, N, K, K, kBoxRows) &&
         make_rows_map(&tb1, static_cast<const __nv_bfloat16*>(w) + static_cast<int64_t>(N) * K, N, K, K, kBoxRows);
  } else {
    ok = ok && make_rows_map(&tb0, w, N, K, K, kBoxRows);
    tb1 = tb0;
  }
  if (!ok) return -2;
  Params p;
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
  p.m_pairs = static_cast<int>((T + 2 * kBM - 1) / (2 * kBM));
  p.n_tiles = swiglu ? (N + kBoxRows - 1) / kBoxRows : (N + kAccCols - 1) / kAccCols;
  p.status = status;
  p.timeout_ns = timeout_ns;
  if (epi == kEpiGatedResidual) return launch<kEpiGatedResidual>(ta, tb0, tb1, p, stream);
  if (swiglu) return launch<kEpiSwiglu>(ta, tb0, tb1, p, stream);
  return launch<kEpiNone>(ta, tb0, tb1, p, stream);
}

}  // namespace pqk
