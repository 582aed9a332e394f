// varlen_attn_fwd.cu -- packed variable-length bf16 self-attention on the
// fifth-generation tensor cores (tcgen05 + tensor memory + TMA).
//
// The operation: every request's tokens attend to all tokens of the same
// request and to nothing else; requests are packed back to back without
// padding and only valid tokens are processed ("FastH3 在八卡 B300 上实现完整
// MP4 生成快于播放时长", section "长序列注意力与通信优化"; "MiniMax H3 FastH3
// real-time serving with vLLM-Omni", bullet "Long-sequence attention &
// communication").
//
// Work unit ("work tile"): (request, head, block of 256 query rows) = two
// 128-row query tiles Q0, Q1 that share every K/V tile. A one-block
// schedule kernel turns cu_seqlens into a tile list (requests longest
// first, then head, then query block, so that the CTAs running at the same
// time read the same head's K/V from L2) and resets a claim counter; a
// persistent kernel with one CTA per SM claims tiles from that list in
// order with an atomic on the counter (each CTA's producer claims its next
// tile when it is ready to load it and hands the index to the block's other
// roles through shared memory), so a CTA that runs faster simply takes more
// tiles. Each tile has exactly one owner and writes only its own rows, so the
// result does not depend on which CTA computed what.
//
// CTA roles (320 threads):
//   warps 0-3  softmax for Q0; thread r owns query row r (tensor-memory lane r)
//   warps 4-7  softmax for Q1
//   warp  8    TMA producer: Q tiles, then K_j, V_j into a ring of stages
//   warp  9    tensor-memory allocator and single-thread MMA issuer
// Tensor memory (512 columns x 128 lanes x 32 bit):
//   [0,128) S0 = Q0 K^T (fp32), [128,256) S1; P_i (bf16 pairs) overwrites the
//   first 64 columns of S_i once the softmax has read S_i; [256,256+D) O0,
//   [256+D,256+2D) O1 (fp32 accumulators).
// MMA issue order per K/V tile j: O0 += P0 V_j, S0 = Q0 K_{j+1}^T,
// O1 += P1 V_j, S1 = Q1 K_{j+1}^T, so each softmax group works on its S
// while the tensor core runs the other group's two products. MMAs from one
// thread execute in issue order, which makes the S_i write after P_i's read
// safe; every other hand-off goes through an mbarrier:
//   kv_full/kv_empty (TMA <-> MMA, per stage), q_full/q_empty,
//   s_full[i] (MMA -> softmax i: S_i ready, and all earlier products of
//   this thread complete), p_full[i] (softmax i -> MMA: P_i in tensor
//   memory, O_i rescaled), o_done[i] (MMA -> softmax i: last product of
//   the work tile complete).
// Online softmax in the log2 domain with lazy rescaling: the running row
// maximum is only raised (and O, l rescaled) when the tile maximum exceeds
// it by more than 2^8, which keeps every probability <= 256 and makes
// rescales rare after the first tiles.
// Every wait is bounded (pqk::mbar_wait, the caller's timeout); a wait that
// runs out raises the block's abort flag and the device status word, and
// every role stops issuing work. Once all roles have stopped (a block
// barrier), the producer waits for every copy it issued that no one consumed
// and the MMA thread for every MMA it issued (a commit on a barrier used only
// for that), both bounded by kDrainTimeoutNs rather than the caller's
// timeout; only then is the tensor memory freed and the block exits.
//
// CTA pairs (kPair; bf16, head_dim 128, no block skipping): two CTAs of a
// cluster share one work tile of 512 query rows, 256 per CTA as above, and
// one thread of the first CTA (the leader) issues every MMA of the pair with
// tcgen05 cta_group::2, M = 256: S_i = Q_i K^T over both CTAs' 128-row Q_i
// with each CTA holding 64 of K_j's 128 keys, and O_i += P_i V_j with P_i in
// each CTA's tensor memory and each CTA holding 64 of V_j's columns. Each SM
// thus streams half of every K/V tile (16 KB stages, ten of them) and reads
// 96 instead of 128 bytes of operands from shared memory per cycle of a
// Q K^T product, whose one-CTA form is bound by that bandwidth. The leader
// claims the tiles, posts the bytes of both CTAs' copies on its own
// barriers before it hands each tile and stage to the second CTA's
// producer, and commits "S ready" and "O done" to both CTAs' barriers; the
// second CTA's softmax warps report "P ready" with one remote arrive per
// warp. On a timeout both CTAs' abort flags are raised; after a cluster
// barrier the leader drains the copies and MMAs of the pair and a second
// cluster barrier keeps the second CTA, whose copies signal the leader's
// barriers, resident until then.
//
// Two compile-time variants of the same pipeline:
//   kSkip  block skipping ("Skip-Softmax", first page, bullet on TRTLLM_ATTN
//          SAGE and Skip-Softmax): a softmax warp whose 32 rows all have the
//          tile maximum more than skip_tau below their earlier maximum writes
//          P = 0 and skips its exponentials; the MMA thread leaves out
//          O_i += P_i V_j when all four warps of the group voted so;
//   kFp8   Q and K as e4m3 bytes (SAGE FP8): S_i = Q_i K^T from 16 KB tiles
//          with kind::f8f6f4 MMAs, the heads' dequantisation factors folded
//          into the softmax scale;
//   kFp8Pv V as e4m3 bytes too and P rounded to e4m3 in tensor memory, so
//          that O_i += P_i V_j runs on the FP8 tensor cores as well; it
//          combines with kSkip (SAGE FP8 with Skip-Softmax).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "pqk_internal.h"

namespace pqk {
namespace {

constexpr int kBM = 128;          // query rows per Q tile
constexpr int kBN = 128;          // keys per K/V tile
constexpr int kRowsPerWork = 2 * kBM;      // one CTA: two 128-row query tiles
constexpr int kRowsPerPairWork = 4 * kBM;  // a CTA pair: two tiles in each CTA
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
// The running row maximum only moves when a tile's maximum exceeds it by
// more than this (log2 units), so probabilities stay <= 2^threshold.
#ifndef PQK_ATTN_RESCALE_LOG2
#define PQK_ATTN_RESCALE_LOG2 8.0f
#endif
constexpr float kRescaleThreshold = PQK_ATTN_RESCALE_LOG2;
// Softmax arithmetic on packed fp32 pairs (fma/add .f32x2) and three-input
// max, halving the non-SFU instructions per score.
#ifndef PQK_ATTN_PACKED
#define PQK_ATTN_PACKED 1
#endif
constexpr bool kPacked = PQK_ATTN_PACKED != 0;
constexpr int kSlabBytes = 128 * 128;      // 128 rows x 64 bf16 (one 128-byte swizzle width)
// Ring of claimed work-tile indices in shared memory. The producer claims
// tile wt + 1 only once the Q K^T products of tile wt are complete, and the
// MMA thread starts tile wt + 1 only after the softmax warps have handed over
// the last P of tile wt, so the producer is at most two tiles ahead of the
// softmax warps: at most three slots are live.
constexpr int kWorkSlots = 4;

template <int D, bool kPair = false>
struct Layout {
  static constexpr int kSlabs = D / 64;
  static constexpr int kTileBytes = kSlabs * kSlabBytes;  // a Q tile; a whole K or V tile
  // a K/V stage: a whole tile, or on a CTA pair this CTA's half (64 keys of
  // K; 64 of V's columns for all 128 keys)
  static constexpr int kStageBytes = kPair ? kTileBytes / 2 : kTileBytes;
  static constexpr int kStages = (kPair || D != 128) ? 10 : 5;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kStageBytes;
  // barriers: kv_full[S], kv_empty[S], q_full, q_empty, s_full[2], p_full[2], o_done[2], drain,
  // work_full[kWorkSlots]
  static constexpr int kNumBars = 2 * kStages + 9 + kWorkSlots;
  static constexpr int kTmemSlotOff = kBarOff + kNumBars * 8;
  static constexpr int kAbortOff = kTmemSlotOff + 4;
  // block-skip votes: one byte per softmax warp, [group][tile parity][warp]
  static constexpr int kVoteOff = kAbortOff + 4;
  // claimed work-tile indices, a ring of kWorkSlots (-1: no more work)
  static constexpr int kWorkOff = kVoteOff + 16;
  // the producer's copy counts (K/V stages, Q pairs), left for the drain
  static constexpr int kLoadsOff = kWorkOff + 4 * kWorkSlots;
  static constexpr int kBytes = kLoadsOff + 8;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
  static constexpr uint32_t kTmemS0 = 0, kTmemS1 = 128, kTmemO0 = 256, kTmemO1 = 256 + D;
  static_assert(kAlloc <= 232448, "shared memory budget");
};

// Schedule in the workspace (int32): [0] number of work tiles, [1] number of
// requests B, [2] the claim counter (reset to 0 by the schedule kernel on
// every call), [3] query rows per work tile, then for the requests in schedule order r =
// 0..B-1: tile_start[B+1] (prefix of tiles), seg_start[B], seg_len[B].
constexpr int kSchedHeader = 4;
__host__ __device__ constexpr size_t sched_words(int B) {
  return kSchedHeader + (B + 1) + 2 * static_cast<size_t>(B);
}

struct AttnParams {
  __nv_bfloat16* o;
  float* lse;
  int64_t o_stride;
  int64_t T;
  int H;
  float scale_log2;
  const int32_t* sched;
  int* status;
  long long timeout_ns;
  float skip_tau;                        // block-skip threshold (log2 units), kSkip only
  const float* deq;                      // kFp8: [2H] dequantisation factors of Q's, then K's heads
  unsigned long long* skip_counts;       // nullable: [0] skipped warp blocks, [1] skipped O += P V products
};

struct Work {
  int seg_start;
  int seg_len;
  int head;
  int q0;      // first query row of the work tile
  int n_kv;    // number of K/V tiles
};

__device__ __forceinline__ Work decode_work(const int32_t* sched, int H, int w) {
  const int B = sched[1];
  const int32_t* tile_start = sched + kSchedHeader;
  const int32_t* seg_start = tile_start + B + 1;
  const int32_t* seg_len = seg_start + B;
  int lo = 0, hi = B - 1;  // last r with tile_start[r] <= w
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= w) lo = mid; else hi = mid - 1;
  }
  Work wk;
  wk.seg_start = seg_start[lo];
  wk.seg_len = seg_len[lo];
  const int rows_per_work = sched[3];
  const int nqb = (wk.seg_len + rows_per_work - 1) / rows_per_work;
  const int local = w - tile_start[lo];
  wk.head = local / nqb;
  wk.q0 = wk.seg_start + (local % nqb) * rows_per_work;
  wk.n_kv = (wk.seg_len + kBN - 1) / kBN;
  (void)H;
  return wk;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int* status) {
  *abort_flag = 1;
  atomicCAS(status, 0, kStatusTimeout);
}

// Drain of an aborting block (after its final barrier). Kept out of line:
// inlined, the rarely run drain loops change the register allocation of the
// softmax loop.
// Producer: K/V copy idx was issued only after copy idx - n_stages had
// landed, so the last n_stages copies (and the last Q pair) are the ones
// that can be outstanding; each is the newest phase of its stage barrier
// (stage s at bar_kv_full + 8 s).
__device__ __noinline__ void drain_copies(uint32_t bar_kv_full, uint32_t bar_q_full, uint32_t n_stages,
                                          uint32_t load_idx, uint32_t q_loads) {
  const uint32_t first = load_idx > n_stages ? load_idx - n_stages : 0;
  for (uint32_t idx = first; idx < load_idx; ++idx)
    mbar_drain_wait(bar_kv_full + 8u * (idx % n_stages), (idx / n_stages) & 1);
  if (q_loads > 0) mbar_drain_wait(bar_q_full, (q_loads - 1) & 1);
}

// MMA thread: a commit on the (otherwise unused) drain barrier completes
// once every MMA this thread issued has, and with them the arrivals of their
// own commits.
__device__ __noinline__ void drain_mmas(uint32_t bar_drain) {
  tc_commit(bar_drain);
  mbar_drain_wait(bar_drain, 0);
}
__device__ __noinline__ void drain_mmas_pair(uint32_t bar_drain) {
  tc_commit_pair(bar_drain);
  mbar_drain_wait(bar_drain, 0);
}

// ------------------------------------------------------------ schedule

constexpr int kSchedThreads = 1024;
constexpr int kSortLimit = 8192;  // requests ordered longest first up to this B
// dynamic shared memory of the schedule kernel: one 64-bit sort key per request
constexpr int kSchedSmem = kSortLimit * 8;

__global__ void __launch_bounds__(kSchedThreads) build_schedule_kernel(const int32_t* cu, int B, int64_t T, int H,
                                                                        int rows_per_work, int32_t* sched,
                                                                        int* status) {
  extern __shared__ uint64_t sort_keys[];
  __shared__ int bad;
  __shared__ int32_t carry;
  if (threadIdx.x == 0) {
    bad = (cu[0] != 0 || static_cast<int64_t>(cu[B]) != T) ? 1 : 0;
    carry = 0;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < B; i += kSchedThreads)
    if (cu[i + 1] < cu[i]) bad = 1;
  __syncthreads();
  int32_t* tile_start = sched + kSchedHeader;
  int32_t* seg_start = tile_start + B + 1;
  int32_t* seg_len = seg_start + B;
  if (bad) {
    if (threadIdx.x == 0) {
      sched[0] = 0;
      sched[1] = B;
      sched[2] = 0;
      sched[3] = rows_per_work;
      atomicCAS(status, 0, kStatusBadSeqlens);
    }
    return;
  }
  if (B <= kSortLimit) {
    // requests longest first, ties by index: a bitonic sort of the keys
    // (INT32_MAX - length) << 32 | index over the next power of two, padded
    // with keys above every real one
    int n = 1;
    while (n < B) n <<= 1;
    for (int i = threadIdx.x; i < n; i += kSchedThreads)
      sort_keys[i] = i < B ? (static_cast<uint64_t>(static_cast<uint32_t>(INT32_MAX - (cu[i + 1] - cu[i]))) << 32) |
                                 static_cast<uint32_t>(i)
                           : ~0ull;
    __syncthreads();
    for (int k = 2; k <= n; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = threadIdx.x; i < n; i += kSchedThreads) {
          const int partner = i ^ j;
          if (partner > i) {
            const uint64_t a = sort_keys[i], b = sort_keys[partner];
            if ((a > b) == ((i & k) == 0)) {
              sort_keys[i] = b;
              sort_keys[partner] = a;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int r = threadIdx.x; r < B; r += kSchedThreads) {
      const int i = static_cast<int>(sort_keys[r] & 0xffffffffu);
      seg_start[r] = cu[i];
      seg_len[r] = cu[i + 1] - cu[i];
    }
  } else {
    // the given order
    for (int i = threadIdx.x; i < B; i += kSchedThreads) {
      seg_start[i] = cu[i];
      seg_len[i] = cu[i + 1] - cu[i];
    }
  }
  __syncthreads();
  // exclusive prefix of tiles per request in schedule order, one chunk of
  // kSchedThreads requests at a time (warp scans, then a scan of warp sums)
  __shared__ int32_t warp_sums[kSchedThreads / 32];
  for (int base = 0; base < B; base += kSchedThreads) {
    const int i = base + threadIdx.x;
    const int32_t n = i < B ? ((seg_len[i] + rows_per_work - 1) / rows_per_work) * H : 0;
    int32_t incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl, off);
      if ((threadIdx.x & 31) >= off) incl += y;
    }
    if ((threadIdx.x & 31) == 31) warp_sums[threadIdx.x >> 5] = incl;
    __syncthreads();
    int32_t before = carry;
    for (int w = 0; w < static_cast<int>(threadIdx.x >> 5); ++w) before += warp_sums[w];
    if (i < B) tile_start[i] = before + incl - n;
    __syncthreads();
    if (threadIdx.x == kSchedThreads - 1) carry = before + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    tile_start[B] = carry;
    sched[0] = carry;
    sched[1] = B;
    sched[2] = 0;  // claim counter
    sched[3] = rows_per_work;
  }
}

// ------------------------------------------------------------ attention

// The 128 fp32 scores of this thread's row from tensor memory; columns at
// or past `valid` become -inf.
__device__ __forceinline__ void load_scores(uint32_t taddr, int valid, float (&s)[128]) {
  uint32_t r[128];
  tmem_ld_x128(taddr, r);
#pragma unroll
  for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(r[c]);
  if (valid < kBN) {
#pragma unroll
    for (int c = 0; c < 128; ++c)
      if (c >= valid) s[c] = -INFINITY;
  }
}

__device__ __forceinline__ float row_max(const float (&s)[128]) {
  if constexpr (kPacked) {
    // eight independent chains of three-input maxima (two new columns each),
    // then a three-level tree
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = fmaxf(s[i], s[i + 8]);
#pragma unroll
    for (int c = 16; c < 128; c += 16) {
#pragma unroll
      for (int i = 0; i < 8; ++i) m[i] = max3(m[i], s[c + i], s[c + 8 + i]);
    }
    return fmaxf(max3(m[0], m[1], m[2]), max3(m[3], m[4], fmaxf(m[5], fmaxf(m[6], m[7]))));
  } else {
    float m0 = s[0], m1 = s[1], m2 = s[2], m3 = s[3];
#pragma unroll
    for (int c = 4; c < 128; c += 4) {
      m0 = fmaxf(m0, s[c]);
      m1 = fmaxf(m1, s[c + 1]);
      m2 = fmaxf(m2, s[c + 2]);
      m3 = fmaxf(m3, s[c + 3]);
    }
    return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
  }
}

// Exponentials of 4 consecutive columns starting at c (a multiple of 4).
__device__ __forceinline__ void exp4(const float (&s)[128], int c, float scale_log2, float neg_m, float (&e)[4]) {
  float x0, x1, x2, x3;
  if constexpr (kPacked) {
    fma2_bcast(s[c], s[c + 1], scale_log2, neg_m, x0, x1);
    fma2_bcast(s[c + 2], s[c + 3], scale_log2, neg_m, x2, x3);
  } else {
    x0 = fmaf(s[c], scale_log2, neg_m);
    x1 = fmaf(s[c + 1], scale_log2, neg_m);
    x2 = fmaf(s[c + 2], scale_log2, neg_m);
    x3 = fmaf(s[c + 3], scale_log2, neg_m);
  }
  e[0] = ex2_approx(x0);
  e[1] = ex2_approx(x1);
  e[2] = ex2_approx(x2);
  e[3] = ex2_approx(x3);
}

// p_c = 2^(s_c * scale_log2 - m) for the 128 columns, rounded to bf16 pairs
// and written over the first 64 columns of S at `t_p` (tensor memory), or,
// with kE4m3P, rounded to e4m3 (four per column) over the first 32; returns
// their unrounded fp32 sum. Waits for its tensor-memory stores before
// returning.
template <bool kE4m3P>
__device__ __forceinline__ float exp_tile_store(const float (&s)[128], float scale_log2, float neg_m, uint32_t t_p) {
  float l0 = 0.f, l1 = 0.f, l2 = 0.f, l3 = 0.f;
  if constexpr (kE4m3P) {
    uint32_t pk[32];
#pragma unroll
    for (int c = 0; c < 128; c += 4) {
      float e[4];
      exp4(s, c, scale_log2, neg_m, e);
      add2_acc(l0, l1, e[0], e[1]);
      add2_acc(l2, l3, e[2], e[3]);
      pk[c / 4] = pack_e4m3x2(e[0], e[1]) | (pack_e4m3x2(e[2], e[3]) << 16);
    }
    tmem_st_x32(t_p, pk);
    return (l0 + l1) + (l2 + l3);
  }
  uint32_t pk[64];
#pragma unroll
  for (int c = 0; c < 128; c += 4) {
    float e[4];
    exp4(s, c, scale_log2, neg_m, e);
    if constexpr (kPacked) {
      add2_acc(l0, l1, e[0], e[1]);
      add2_acc(l2, l3, e[2], e[3]);
    } else {
      l0 += e[0];
      l1 += e[1];
      l2 += e[2];
      l3 += e[3];
    }
    pk[c / 2] = pack_bf16x2(e[0], e[1]);
    pk[c / 2 + 1] = pack_bf16x2(e[2], e[3]);
  }
  tmem_st_x64(t_p, pk);
  return (l0 + l1) + (l2 + l3);
}

template <int D, bool kSkip, bool kFp8, bool kFp8Pv, bool kPair = false>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  using L = Layout<D, kPair>;
  static_assert(!kFp8 || D == 128, "FP8 Q K^T: one 128-byte swizzle row per token");
  static_assert(!kFp8Pv || kFp8, "FP8 P V comes with FP8 Q K^T");
  static_assert(!kPair || (D == 128 && !kSkip && !kFp8), "CTA pairs: bf16, head_dim 128, no block skipping");
  // FP8 Q K^T: the MMA thread waits for the next V stage (loaded long ago)
  // while it waits for P1 anyway, and probes the next K stage there without
  // blocking (its copy may still be in flight), instead of waiting for both
  // at the top of the next iteration, just before P0 (-3 % time with FP8;
  // +1 % with bf16 operands, where it is left out).
  constexpr bool kEarlyKv = kFp8;
  // bytes of one Q or K tile: bf16 slabs, or 128 rows x 128 e4m3 bytes
  constexpr uint32_t kQKBytes = kFp8 ? static_cast<uint32_t>(kBM) * 128u : static_cast<uint32_t>(L::kTileBytes);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_addr(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA pair: rank 0 (the leader) issues every MMA of the pair and owns the
  // barriers of the K/V and Q copies; each CTA keeps its own 256 query rows
  const uint32_t rank = kPair ? ctarank() : 0u;
  const bool leader = rank == 0;
  const uint32_t q_smem = base + L::kQOff;
  const uint32_t kv_smem = base + L::kKVOff;
  const uint32_t bar0 = base + L::kBarOff;
  auto kv_full = [&](int s) { return bar0 + 8u * s; };
  auto kv_empty = [&](int s) { return bar0 + 8u * (L::kStages + s); };
  const uint32_t q_full = bar0 + 8u * (2 * L::kStages);
  const uint32_t q_empty = q_full + 8;
  auto s_full = [&](int i) { return q_full + 16 + 8u * i; };
  auto p_full = [&](int i) { return q_full + 32 + 8u * i; };
  auto o_done = [&](int i) { return q_full + 48 + 8u * i; };
  const uint32_t drain = q_full + 64;
  auto work_full = [&](int i) { return q_full + 72 + 8u * i; };
  volatile int* work_slot = reinterpret_cast<volatile int*>(smem + L::kWorkOff);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + L::kTmemSlotOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kAbortOff);
  volatile uint8_t* votes = smem + L::kVoteOff;
  // a wait that ran out stops this CTA's roles and, on a pair, the other CTA's
  auto abort_all = [&]() {
    raise_abort(abort_flag, p.status);
    if constexpr (kPair) st_remote_u32(in_cta(base + L::kAbortOff, rank ^ 1u), 1u);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      // one arrival per softmax thread, or on a pair one per softmax warp of either CTA
      mbar_init(p_full(i), kPair ? 8 : kBM);
      mbar_init(o_done(i), 1);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < kWorkSlots; ++i) mbar_init(work_full(i), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    if constexpr (kPair) {
      tmem_alloc_pair(base + L::kTmemSlotOff, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(base + L::kTmemSlotOff, 512);
      tmem_relinquish();
    }
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensor_map(&tm_q);
    prefetch_tensor_map(&tm_k);
    prefetch_tensor_map(&tm_v);
  }
  tc_fence_before_sync();
  if constexpr (kPair) {
    __syncwarp();
    cluster_sync_all();  // both CTAs' barriers are initialised before any remote arrive
  } else {
    __syncthreads();
  }
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int n_work = p.sched[0];
  int* claim_counter = const_cast<int*>(p.sched + 2);
  // copies issued by the producer thread (K/V stages, Q tile pairs), kept in
  // shared memory for the drain so that no other thread holds them
  volatile uint32_t* loads_done = reinterpret_cast<volatile uint32_t*>(smem + L::kLoadsOff);
  // The index of this block's work tile wt, published by the producer in
  // slot wt % kWorkSlots (-1 once the list is exhausted); false when the
  // block aborts first.
  auto next_work = [&](int wt, int& w) {
    if (!mbar_wait(work_full(wt % kWorkSlots), (wt / kWorkSlots) & 1, abort_flag, p.timeout_ns)) return false;
    // on a pair's second CTA the slot was written by the leader's producer
    if (kPair && !leader) asm volatile("fence.acq_rel.cluster;" ::: "memory");
    w = work_slot[wt % kWorkSlots];
    return true;
  };

  if (warp == kProducerWarp) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t load_idx = 0;
      uint32_t q_loads = 0;
      bool ok = true;
      if constexpr (kPair) {
        // The leader claims each work tile, posts the bytes of both CTAs'
        // copies on its own barriers and only then hands the tile, and each
        // K/V stage, to the second CTA's producer (so that no copy completes
        // before the count it belongs to). Both CTAs copy their own two Q
        // tiles, their 64 of each K tile's keys and their 64 of each V
        // tile's columns; every copy completes on the leader's barrier.
        const uint32_t q_bar = in_cta(q_full, 0);
        for (int wt = 0; ok; ++wt) {
          int w;
          if (leader) {
            if (wt > 0 && !(ok = mbar_wait(q_empty, (wt - 1) & 1, abort_flag, p.timeout_ns))) break;
            const int claimed = atomicAdd(claim_counter, 1);
            w = claimed < n_work ? claimed : -1;
            if (w >= 0) {
              mbar_arrive_expect_tx(q_full, 4 * kQKBytes);
              ++q_loads;
            }
            work_slot[wt % kWorkSlots] = w;
            mbar_arrive(work_full(wt % kWorkSlots));
            st_remote_u32(in_cta(base + L::kWorkOff + 4u * (wt % kWorkSlots), 1), static_cast<uint32_t>(w));
            arrive_remote_release(in_cta(work_full(wt % kWorkSlots), 1));
          } else if (!(ok = next_work(wt, w))) {
            break;
          }
          if (w < 0) break;
          const Work wk = decode_work(p.sched, p.H, w);
          const int qrow = wk.q0 + static_cast<int>(rank) * kRowsPerWork;
          for (int i = 0; i < 2; ++i)
            for (int sl = 0; sl < L::kSlabs; ++sl)
              tma_load_3d_pair(q_smem + i * L::kTileBytes + sl * kSlabBytes, &tm_q, q_bar, sl * 64, wk.head,
                               qrow + i * kBM);
          for (int j = 0; j < wk.n_kv && ok; ++j) {
            const int key0 = wk.seg_start + j * kBN;
            for (int kv = 0; kv < 2; ++kv) {
              const int s = load_idx % L::kStages;
              const uint32_t round = load_idx / L::kStages;
              if (leader) {
                if (round > 0 && !(ok = mbar_wait(kv_empty(s), (round - 1) & 1, abort_flag, p.timeout_ns))) break;
                mbar_arrive_expect_tx(kv_full(s), 2 * L::kStageBytes);
                arrive_remote(in_cta(kv_empty(s), 1));
              } else if (!(ok = mbar_wait(kv_empty(s), round & 1, abort_flag, p.timeout_ns))) {
                break;
              }
              const uint32_t dst = kv_smem + s * L::kStageBytes;
              const uint32_t bar = in_cta(kv_full(s), 0);
              if (kv == 0) {
                for (int sl = 0; sl < L::kSlabs; ++sl)
                  tma_load_3d_pair(dst + sl * (kSlabBytes / 2), &tm_k, bar, sl * 64, wk.head,
                                   key0 + static_cast<int>(rank) * (kBN / 2));
              } else {
                tma_load_3d_pair(dst, &tm_v, bar, static_cast<int>(rank) * 64, wk.head, key0);
              }
              ++load_idx;
            }
          }
        }
      } else {
      for (int wt = 0; ok; ++wt) {
        // the Q tiles of the previous work tile are no longer needed: claim the next one
        if (wt > 0 && !(ok = mbar_wait(q_empty, (wt - 1) & 1, abort_flag, p.timeout_ns))) break;
        const int claimed = atomicAdd(claim_counter, 1);
        const int w = claimed < n_work ? claimed : -1;
        work_slot[wt % kWorkSlots] = w;
        mbar_arrive(work_full(wt % kWorkSlots));
        if (w < 0) break;
        const Work wk = decode_work(p.sched, p.H, w);
        mbar_arrive_expect_tx(q_full, 2 * kQKBytes);
        ++q_loads;
        for (int i = 0; i < 2; ++i) {
          if constexpr (kFp8) {
            tma_load_3d(q_smem + i * L::kTileBytes, &tm_q, q_full, 0, wk.head, wk.q0 + i * kBM);
          } else {
            for (int sl = 0; sl < L::kSlabs; ++sl)
              tma_load_3d(q_smem + i * L::kTileBytes + sl * kSlabBytes, &tm_q, q_full, sl * 64, wk.head,
                          wk.q0 + i * kBM);
          }
        }
        for (int j = 0; j < wk.n_kv && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv) {
            const int s = load_idx % L::kStages;
            const uint32_t round = load_idx / L::kStages;
            if (round > 0 && !(ok = mbar_wait(kv_empty(s), (round - 1) & 1, abort_flag, p.timeout_ns))) break;
            if ((kFp8 && kv == 0) || (kFp8Pv && kv == 1)) {
              // one 128-byte e4m3 row per token: a single 16 KB box
              mbar_arrive_expect_tx(kv_full(s), kQKBytes);
              tma_load_3d(kv_smem + s * L::kStageBytes, kv == 0 ? &tm_k : &tm_v, kv_full(s), 0, wk.head,
                          wk.seg_start + j * kBN);
            } else {
              mbar_arrive_expect_tx(kv_full(s), L::kTileBytes);
              const CUtensorMap* tm = kv == 0 ? &tm_k : &tm_v;
              for (int sl = 0; sl < L::kSlabs; ++sl)
                tma_load_3d(kv_smem + s * L::kStageBytes + sl * kSlabBytes, tm, kv_full(s), sl * 64, wk.head,
                            wk.seg_start + j * kBN);
            }
            ++load_idx;
          }
        }
      }
      }
      if (!ok) abort_all();
      loads_done[0] = load_idx;
      loads_done[1] = q_loads;
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer (the leader's, on a pair)
    if (lane == 0 && leader) {
      // a pair's products have M = 256: each CTA's 128 rows of Q_i, S_i, P_i, O_i
      constexpr int kM = kPair ? 2 * kBM : kBM;
      constexpr uint32_t kIdescQK = kFp8 ? idesc_e4m3_f32(kBM, kBN) : idesc_bf16_f32(kM, kBN, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(kM, D, true);
      // completions: of this CTA's copies' consumers (stages, Q), or seen by
      // both CTAs' softmax warps (S ready, O done)
      auto commit_own = [&](uint32_t bar) {
        if constexpr (kPair) tc_commit_pair(bar); else tc_commit(bar);
      };
      auto commit_all = [&](uint32_t bar) {
        if constexpr (kPair) tc_commit_pair_both(bar); else tc_commit(bar);
      };
      constexpr uint32_t kIdescPV8 = idesc_e4m3_f32(kBM, D, true);
      uint32_t cons_idx = 0;
      uint32_t p_phase = 0;
      unsigned long long pv_skips = 0;
      // every softmax warp of group i voted to skip K/V tile j
      auto group_skips = [&](int i, int j) {
        return *reinterpret_cast<volatile uint32_t*>(votes + (i * 2 + (j & 1)) * 4) == 0x01010101u;
      };
      int wt = 0;
      bool ok = true;
      // Descriptor low words of Q0 and of stage 0 (K: K-major, V: MN-major
      // with 64-wide column slabs kSlabBytes apart); one high word for all.
      constexpr uint32_t kDescHi = smem_desc_hi_sw128(1024);
      constexpr uint32_t kTileWords = L::kTileBytes >> 4;
      constexpr uint32_t kStageWords = L::kStageBytes >> 4;
      // a K stage's two 64-column slabs (on a pair 64 keys each)
      constexpr uint32_t kKSlabBytes = kPair ? kSlabBytes / 2 : kSlabBytes;
      const uint32_t q_lo = smem_desc_lo(q_smem, 16);
      const uint32_t k_lo = smem_desc_lo(kv_smem, 16);
      const uint32_t v_lo = smem_desc_lo(kv_smem, kSlabBytes);
      // S_i = Q_i K^T over D/16 K-steps of 16 (32 bytes inside the 128-byte row)
      auto issue_qk = [&](int i, int stage) {
        const uint32_t a0 = q_lo + i * kTileWords;
        const uint32_t b0 = k_lo + stage * kStageWords;
        if constexpr (kFp8) {
          // e4m3: K = 32 per instruction, 32 bytes inside the one 128-byte row
#pragma unroll
          for (int k = 0; k < D / 32; ++k)
            mma_f8_ss_w(tmem + (i == 0 ? L::kTmemS0 : L::kTmemS1), a0 + 2 * k, b0 + 2 * k, kDescHi, kIdescQK,
                        k > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t off_a = ((k / 4) * kSlabBytes + (k % 4) * 32) >> 4;
            const uint32_t off_b = ((k / 4) * kKSlabBytes + (k % 4) * 32) >> 4;
            if constexpr (kPair)
              mma_bf16_ss_pair(tmem + (i == 0 ? L::kTmemS0 : L::kTmemS1), a0 + off_a, b0 + off_b, kDescHi, kIdescQK,
                               k > 0 ? 1u : 0u);
            else
              mma_bf16_ss_w(tmem + (i == 0 ? L::kTmemS0 : L::kTmemS1), a0 + off_a, b0 + off_b, kDescHi, kIdescQK,
                            k > 0 ? 1u : 0u);
          }
        }
      };
      // O_i (+)= P_i V over kBN/16 K-steps; V is MN-major: 64-wide column
      // slabs kSlabBytes apart, 8-row groups 1024 bytes apart
      auto issue_pv = [&](int i, int stage, bool accumulate) {
        const uint32_t b0 = v_lo + stage * kStageWords;
        const uint32_t p_col = tmem + (i == 0 ? L::kTmemS0 : L::kTmemS1);
        if constexpr (kFp8Pv) {
          // e4m3 P (four keys per column, 8 columns per K = 32 step) and V as
          // 128-byte rows: MN-major, one swizzle atom wide, 32 keys = 4096 bytes
#pragma unroll
          for (int k = 0; k < kBN / 32; ++k)
            mma_f8_ts_w(tmem + (i == 0 ? L::kTmemO0 : L::kTmemO1), p_col + 8 * k, b0 + ((k * 4096) >> 4), kDescHi,
                        kIdescPV8, (accumulate || k > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int k = 0; k < kBN / 16; ++k) {
            if constexpr (kPair)
              mma_bf16_ts_pair(tmem + (i == 0 ? L::kTmemO0 : L::kTmemO1), p_col + 8 * k, b0 + ((k * 2048) >> 4),
                               kDescHi, kIdescPV, (accumulate || k > 0) ? 1u : 0u);
            else
              mma_bf16_ts_w(tmem + (i == 0 ? L::kTmemO0 : L::kTmemO1), p_col + 8 * k, b0 + ((k * 2048) >> 4),
                            kDescHi, kIdescPV, (accumulate || k > 0) ? 1u : 0u);
          }
        }
      };
      auto wait_stage = [&](uint32_t idx) {
        return mbar_wait(kv_full(idx % L::kStages), (idx / L::kStages) & 1, abort_flag, p.timeout_ns);
      };
      for (;; ++wt) {
        int w;
        if (!(ok = next_work(wt, w)) || w < 0) break;
        const Work wk = decode_work(p.sched, p.H, w);
        const bool q1_in_request = wk.q0 + kBM < wk.seg_start + wk.seg_len;
        if (!(ok = mbar_wait(q_full, wt & 1, abort_flag, p.timeout_ns))) break;
        uint32_t k_stage_idx = cons_idx;
        if (!(ok = wait_stage(k_stage_idx))) break;
        tc_fence_after_sync();
        issue_qk(0, k_stage_idx % L::kStages);
        commit_all(s_full(0));
        issue_qk(1, k_stage_idx % L::kStages);
        commit_all(s_full(1));
        commit_own(kv_empty(k_stage_idx % L::kStages));
        if (wk.n_kv == 1) commit_own(q_empty);
        ++cons_idx;
        // stages of iteration j: V_j and K_{j+1}
        uint32_t v_idx = cons_idx++;
        uint32_t nk_idx = wk.n_kv > 1 ? cons_idx++ : 0;
        bool v_ready = false, k_ready = false;
        for (int j = 0; j < wk.n_kv; ++j) {
          const bool more = j + 1 < wk.n_kv;
          // V_j and K_{j+1} are complete before P0 is waited for, so no copy
          // wait sits between O0 += P0 V_j and S0 = Q0 K_{j+1}^T
          if (!v_ready && !(ok = wait_stage(v_idx))) break;
          if (more && !k_ready && !(ok = wait_stage(nk_idx))) break;
          if (!(ok = mbar_wait(p_full(0), p_phase, abort_flag, p.timeout_ns))) break;
          tc_fence_after_sync();
          if (kSkip && j > 0 && group_skips(0, j)) {
            ++pv_skips;
          } else {
            issue_pv(0, v_idx % L::kStages, j > 0);
          }
          if (!more) commit_all(o_done(0));
          if (more) {
            issue_qk(0, nk_idx % L::kStages);
            commit_all(s_full(0));
          }
          uint32_t next_v = 0, next_nk = 0;
          if (more) {
            next_v = cons_idx++;
            next_nk = j + 2 < wk.n_kv ? cons_idx++ : 0;
          }
          v_ready = k_ready = false;
          if (kEarlyKv && more) {
            if (!(ok = wait_stage(next_v))) break;
            v_ready = true;
            k_ready = j + 2 < wk.n_kv &&
                      mbar_test_wait(kv_full(next_nk % L::kStages), (next_nk / L::kStages) & 1);
          }
          if (!(ok = mbar_wait(p_full(1), p_phase, abort_flag, p.timeout_ns))) break;
          tc_fence_after_sync();
          if (kSkip && j > 0 && group_skips(1, j)) {
            if (q1_in_request) ++pv_skips;
          } else {
            issue_pv(1, v_idx % L::kStages, j > 0);
          }
          if (!more) commit_all(o_done(1));
          commit_own(kv_empty(v_idx % L::kStages));
          if (more) {
            issue_qk(1, nk_idx % L::kStages);
            commit_all(s_full(1));
            commit_own(kv_empty(nk_idx % L::kStages));
            if (j + 2 == wk.n_kv) commit_own(q_empty);
          }
          p_phase ^= 1u;
          v_idx = next_v;
          nk_idx = next_nk;
        }
      }
      if (kSkip && p.skip_counts != nullptr && pv_skips != 0) atomicAdd(&p.skip_counts[1], pv_skips);
      if (!ok) abort_all();
    }
  } else {
    // ------------------------------------------------ softmax groups
    const int grp = warp >> 2;  // 0 -> Q0, 1 -> Q1
    const int r = threadIdx.x & 127;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_off + (grp == 0 ? L::kTmemS0 : L::kTmemS1);
    const uint32_t t_o = tmem + lane_off + (grp == 0 ? L::kTmemO0 : L::kTmemO1);
    uint32_t s_phase = 0;
    int wt = 0;
    bool ok = true;
    unsigned long long warp_skips = 0;
    for (;; ++wt) {
      int w;
      ok = __all_sync(0xffffffffu, next_work(wt, w));
      if (!ok || w < 0) break;
      const Work wk = decode_work(p.sched, p.H, w);
      const int row = wk.q0 + static_cast<int>(rank) * kRowsPerWork + grp * kBM + r;
      // log2-domain score factor; FP8 scores carry the two heads' dequantisation factors
      const float sl2 = kFp8 ? p.scale_log2 * p.deq[wk.head] * p.deq[p.H + wk.head] : p.scale_log2;
      float m = -INFINITY, l = 0.f;
      float m_seen = -INFINITY;  // block skipping: running maximum over all earlier tiles
      for (int j = 0; j < wk.n_kv; ++j) {
        ok = __all_sync(0xffffffffu, mbar_wait(s_full(grp), s_phase, abort_flag, p.timeout_ns));
        if (!ok) break;
        s_phase ^= 1u;
        tc_fence_after_sync();
        // keys at or past the request end (last tile only) are masked
        const int valid = j == wk.n_kv - 1 ? wk.seg_len - j * kBN : kBN;
        float s[128];
        load_scores(t_s, valid, s);
        const float mx = row_max(s) * sl2;
        if constexpr (kSkip) {
          // Skip-Softmax: this warp's 32 rows drop K/V tile j when every row
          // of the request has its tile maximum more than skip_tau below its
          // maximum over tiles 0..j-1. The vote goes to the MMA thread, which
          // leaves out O_i += P_i V_j when all four warps of the group drop it.
          const bool in_request = row < wk.seg_start + wk.seg_len;
          const bool skip = __all_sync(0xffffffffu, !in_request || (j > 0 && mx < m_seen - p.skip_tau));
          m_seen = fmaxf(m_seen, mx);
          if (lane == 0) votes[(grp * 2 + (j & 1)) * 4 + (warp & 3)] = skip ? 1 : 0;
          if (skip) {
            if (__any_sync(0xffffffffu, in_request) && lane == 0) ++warp_skips;
            // P = 0 for these rows (the product still runs if another warp
            // keeps the tile): 64 columns of bf16 pairs, or 32 of e4m3 quads
            if constexpr (kFp8Pv) {
              uint32_t zero[32];
#pragma unroll
              for (int c = 0; c < 32; ++c) zero[c] = 0u;
              tmem_st_x32(t_s, zero);
            } else {
              uint32_t zero[64];
#pragma unroll
              for (int c = 0; c < 64; ++c) zero[c] = 0u;
              tmem_st_x64(t_s, zero);
            }
            tc_fence_before_sync();
            mbar_arrive(p_full(grp));
            continue;
          }
        }
        const bool need_rescale = j > 0 && mx > m + kRescaleThreshold;
        float alpha = 1.0f;
        if (j == 0) {
          m = mx;
        } else if (need_rescale) {
          alpha = ex2_approx(m - mx);
          l *= alpha;
          m = mx;
        }
        // O_i holds the products of tiles 0..j-1, all complete (s_full for
        // tile j completed after them): rescale it before P_j V_j. Tensor-
        // memory loads and stores are warp-collective (.sync.aligned), so
        // the whole warp takes this path when any of its rows needs it, the
        // other rows with alpha = 1. Eight columns at a time in a rolled
        // loop: the 128 scores are live here, and wider chunks push the
        // kernel past its register budget (spills in every variant).
        if (__any_sync(0xffffffffu, need_rescale)) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 8) {
            uint32_t ov[8];
            tmem_ld_x8(t_o + c0, ov);
#pragma unroll
            for (int c = 0; c < 8; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * alpha);
            tmem_st_x8(t_o + c0, ov);
          }
        }
        l += exp_tile_store<kFp8Pv>(s, sl2, -m, t_s);
        tc_fence_before_sync();
        if constexpr (kPair) {
          // one arrival per warp at the leader's barrier. P and the rescaled
          // O are in this CTA's tensor memory, their stores complete
          // (tcgen05.wait::st) and fenced before this point, so a plain
          // remote arrive hands them over; a cluster-scope release here,
          // on every tile's critical path, cost 15 % of the kernel's time
          __syncwarp();
          if (lane == 0) {
            if (leader) mbar_arrive(p_full(grp));
            else arrive_remote(in_cta(p_full(grp), 0));
          }
        } else {
          mbar_arrive(p_full(grp));
        }
      }
      if (!ok) break;
      // epilogue: normalise O_i and write the valid rows
      ok = __all_sync(0xffffffffu, mbar_wait(o_done(grp), wt & 1, abort_flag, p.timeout_ns));
      if (!ok) break;
      tc_fence_after_sync();
      // FP8 P V accumulates V's codes: its dequantisation factor comes in here
      const float inv_l = (kFp8Pv ? p.deq[2 * p.H + wk.head] : 1.0f) / l;
      const bool valid_row = row < wk.seg_start + wk.seg_len;
      __nv_bfloat16* dst = p.o + static_cast<int64_t>(row) * p.o_stride + wk.head * D;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t ov[32];
        tmem_ld_x32(t_o + c0, ov);
        if (valid_row) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(ov[c]) * inv_l, __uint_as_float(ov[c + 1]) * inv_l);
            v.y = pack_bf16x2(__uint_as_float(ov[c + 2]) * inv_l, __uint_as_float(ov[c + 3]) * inv_l);
            v.z = pack_bf16x2(__uint_as_float(ov[c + 4]) * inv_l, __uint_as_float(ov[c + 5]) * inv_l);
            v.w = pack_bf16x2(__uint_as_float(ov[c + 6]) * inv_l, __uint_as_float(ov[c + 7]) * inv_l);
            *reinterpret_cast<uint4*>(dst + c0 + c) = v;
          }
        }
      }
      if (valid_row && p.lse != nullptr)
        p.lse[static_cast<int64_t>(wk.head) * p.T + row] = (m + __log2f(l)) * 0.69314718055994530942f;
      tc_fence_before_sync();
    }
    if (kSkip && p.skip_counts != nullptr && lane == 0 && warp_skips != 0) atomicAdd(&p.skip_counts[0], warp_skips);
    if (!ok) abort_all();
  }

  tc_fence_before_sync();
  auto block_sync = [&]() {
    if constexpr (kPair) {
      __syncwarp();
      cluster_sync_all();
    } else {
      __syncthreads();
    }
  };
  block_sync();
  // Every role (of both CTAs, on a pair) has stopped, so the abort flag is
  // final. On an abort, copies and MMAs may still be in flight into the
  // block's shared and tensor memory: wait for all of them before the memory
  // is freed. On a pair every copy completes on a leader's barrier, which
  // completes only once both CTAs' halves have landed; the second CTA waits
  // at the cluster barrier meanwhile.
  if (*abort_flag) {
    if (leader && warp == kProducerWarp && lane == 0)
      drain_copies(kv_full(0), q_full, L::kStages, loads_done[0], loads_done[1]);
    else if (leader && warp == kMmaWarp && lane == 0)
      kPair ? drain_mmas_pair(drain) : drain_mmas(drain);
    block_sync();
  }
  tc_fence_after_sync();
  if (warp == kMmaWarp) {
    if constexpr (kPair) tmem_dealloc_pair(tmem, 512); else tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------ self-test

__global__ void wait_selftest_kernel(int* status, long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t b = smem_addr(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // nothing ever arrives on `bar`: the bounded wait must give up
    if (!mbar_wait(b, 0, &abort_flag, timeout_ns)) atomicCAS(status, 0, kStatusTimeout);
  }
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

// [T, H, D] bf16 with `stride` elements between tokens, read as boxes of
// 64 columns x 1 head x box_rows tokens, 128-byte swizzled; rows past T read as 0.
bool make_qkv_map(CUtensorMap* map, const void* ptr, int64_t T, int H, int D, int64_t stride, int box_rows = kBM) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(stride) * 2};
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [T, H, D] e4m3 bytes with `stride` elements (bytes) between tokens, read
// as boxes of 128 bytes x 1 head x 128 tokens, 128-byte swizzled.
bool make_e4m3_map(CUtensorMap* map, const void* ptr, int64_t T, int H, int D, int64_t stride) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr || D != 128) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(stride)};
  const cuuint32_t box[3] = {128, 1, static_cast<cuuint32_t>(kBM)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool set_schedule_smem_attr() {
  static int done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(build_schedule_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSchedSmem) !=
        cudaSuccess)
      return false;
    done[dev] = 1;
  }
  return true;
}

// Per device: the shared-memory attribute of the pair kernel is set and the
// number of CTA pairs that can be resident at once is queried on the first
// call (which must precede any stream capture), so that the persistent grid
// never leaves a pair waiting for a second wave.
int resident_attn_pairs(cudaLaunchConfig_t* cfg) {
  static int pairs[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
  if (pairs[dev] == 0) {
    if (cudaFuncSetAttribute(attn_fwd_kernel<128, false, false, false, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, Layout<128, true>::kAlloc) != cudaSuccess)
      return -1;
    int n = 0;
    cfg->gridDim = dim3(2, 1, 1);
    if (cudaOccupancyMaxActiveClusters(&n, attn_fwd_kernel<128, false, false, false, true>, cfg) != cudaSuccess ||
        n < 1)
      return -1;
    pairs[dev] = n;
  }
  return pairs[dev];
}

int launch_attn_pair(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const AttnParams& p,
                     int64_t max_work, cudaStream_t stream) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Layout<128, true>::kAlloc;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int max_pairs = resident_attn_pairs(&cfg);
  if (max_pairs < 1) return -1;
  cfg.gridDim = dim3(2 * static_cast<unsigned>(max_work < max_pairs ? max_work : max_pairs), 1, 1);
  if (cudaLaunchKernelEx(&cfg, attn_fwd_kernel<128, false, false, false, true>, tq, tk, tv, p) != cudaSuccess)
    return -1;
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <int D, bool kSkip, bool kFp8, bool kFp8Pv>
bool set_smem_attr() {
  static int done[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  if (!done[dev]) {
    if (cudaFuncSetAttribute(attn_fwd_kernel<D, kSkip, kFp8, kFp8Pv>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Layout<D>::kAlloc) != cudaSuccess)
      return false;
    done[dev] = 1;
  }
  return true;
}

}  // namespace

size_t attn_schedule_bytes(int B) { return ((sched_words(B) * sizeof(int32_t)) + 255) & ~static_cast<size_t>(255); }

int launch_varlen_attn(const void* q, const void* k, const void* v, void* o, float* lse, int64_t q_stride,
                       int64_t k_stride, int64_t v_stride, int64_t o_stride, const int32_t* cu_seqlens, int B,
                       int64_t T, int H, int D, float softmax_scale, void* workspace, int* status,
                       long long timeout_ns, cudaStream_t stream, int num_sms, bool skip, float skip_tau,
                       unsigned long long* skip_counts, const float* deq, bool fp8_pv, bool cta_pairs) {
  CUtensorMap tq, tk, tv;
  const bool maps_ok = deq != nullptr
                           ? make_e4m3_map(&tq, q, T, H, D, q_stride) && make_e4m3_map(&tk, k, T, H, D, k_stride)
                           : make_qkv_map(&tq, q, T, H, D, q_stride) && make_qkv_map(&tk, k, T, H, D, k_stride);
  const bool v_ok = fp8_pv ? make_e4m3_map(&tv, v, T, H, D, v_stride) : make_qkv_map(&tv, v, T, H, D, v_stride);
  if (!maps_ok || !v_ok) return -2;
  // bf16, head_dim 128, no block skipping: on CTA pairs when asked, whose K
  // copies are 64-key halves
  const bool pair = cta_pairs && deq == nullptr && !skip && D == 128;
  if (pair && !make_qkv_map(&tk, k, T, H, D, k_stride, kBN / 2)) return -2;
  const int rows_per_work = pair ? kRowsPerPairWork : kRowsPerWork;
  int32_t* sched = static_cast<int32_t*>(workspace);
  int sort_n = 1;
  while (sort_n < B) sort_n <<= 1;
  const size_t sched_smem = B <= kSortLimit ? static_cast<size_t>(sort_n) * 8 : 0;
  if (sched_smem > 48 * 1024 && !set_schedule_smem_attr()) return -1;
  build_schedule_kernel<<<1, kSchedThreads, sched_smem, stream>>>(cu_seqlens, B, T, H, rows_per_work, sched,
                                                                  status);
  if (cudaGetLastError() != cudaSuccess) return -1;
  AttnParams p;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.o_stride = o_stride;
  p.T = T;
  p.H = H;
  p.scale_log2 = softmax_scale * 1.4426950408889634f;
  p.sched = sched;
  p.status = status;
  p.timeout_ns = timeout_ns;
  p.skip_tau = skip_tau;
  p.skip_counts = skip_counts;
  p.deq = deq;
  // upper bound of work tiles: every request adds at most one partial block
  const int64_t max_work = static_cast<int64_t>(H) * ((T + rows_per_work - 1) / rows_per_work + B);
  const int grid = static_cast<int>(max_work < num_sms ? max_work : num_sms);
  if (pair) return launch_attn_pair(tq, tk, tv, p, max_work, stream);
  if (fp8_pv && !skip) {
    if (D != 128 || deq == nullptr) return -1;
    if (!set_smem_attr<128, false, true, true>()) return -1;
    attn_fwd_kernel<128, false, true, true><<<grid, kThreads, Layout<128>::kAlloc, stream>>>(tq, tk, tv, p);
  } else if (fp8_pv) {
    if (D != 128 || deq == nullptr) return -1;
    if (!set_smem_attr<128, true, true, true>()) return -1;
    attn_fwd_kernel<128, true, true, true><<<grid, kThreads, Layout<128>::kAlloc, stream>>>(tq, tk, tv, p);
  } else if (deq != nullptr && !skip) {
    if (D != 128) return -1;
    if (!set_smem_attr<128, false, true, false>()) return -1;
    attn_fwd_kernel<128, false, true, false><<<grid, kThreads, Layout<128>::kAlloc, stream>>>(tq, tk, tv, p);
  } else if (deq != nullptr) {
    if (D != 128) return -1;
    if (!set_smem_attr<128, true, true, false>()) return -1;
    attn_fwd_kernel<128, true, true, false><<<grid, kThreads, Layout<128>::kAlloc, stream>>>(tq, tk, tv, p);
  } else if (D == 128 && !skip) {
    if (!set_smem_attr<128, false, false, false>()) return -1;
    attn_fwd_kernel<128, false, false, false><<<grid, kThreads, Layout<128>::kAlloc, stream>>>(tq, tk, tv, p);
  } else if (D == 128) {
    if (!set_smem_attr<128, true, false, false>()) return -1;
    attn_fwd_kernel<128, true, false, false><<<grid, kThreads, Layout<128>::kAlloc, stream>>>(tq, tk, tv, p);
  } else if (!skip) {
    if (!set_smem_attr<64, false, false, false>()) return -1;
    attn_fwd_kernel<64, false, false, false><<<grid, kThreads, Layout<64>::kAlloc, stream>>>(tq, tk, tv, p);
  } else {
    if (!set_smem_attr<64, true, false, false>()) return -1;
    attn_fwd_kernel<64, true, false, false><<<grid, kThreads, Layout<64>::kAlloc, stream>>>(tq, tk, tv, p);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int launch_wait_selftest(int* status, long long timeout_ns, cudaStream_t stream) {
  wait_selftest_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace pqk
