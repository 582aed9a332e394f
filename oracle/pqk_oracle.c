/*
 * pqk_oracle.c -- plain float64 CPU oracle for the DiT-block hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's
 * CPU-baseline leg load this library. The CUDA library never links, includes
 * or calls it, and it shares no code, header, table or constant with it.
 *
 * What it computes, and where the pages say so:
 *   oracle_qk_norm_rope    -- Q/K normalisation merged with RoPE
 *                             ("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长",
 *                             section "融合 DiT 算子"; "MiniMax H3 FastH3 real-time
 *                             serving with vLLM-Omni", section "System-wide
 *                             optimizations in vLLM-Omni", bullet "Fused DiT
 *                             operators").
 *   oracle_qk_norm_rope_3axis -- the same with a (t, h, w) position per
 *                             token for video latents (a reading: the pages
 *                             give no RoPE variant; see the function).
 *   oracle_qk_norm_rope_e4m3 -- the same followed by e4m3 codes with a
 *                             per-tensor scale from the normalised rows'
 *                             bound (SAGE FP8 folded into the prologue; a
 *                             reading).
 *   oracle_qk_fullc_norm_rope -- the same with the norm over all heads of
 *                             a token (weight of H*D entries), a reading of
 *                             "Q/K normalisation" the pages leave open.
 *   oracle_varlen_attn     -- softmax attention over one packed sequence per
 *                             request, valid tokens only (first page, section
 *                             "长序列注意力与通信优化"; second page, bullet
 *                             "Long-sequence attention & communication").
 *   oracle_varlen_attn_fp8qk -- the same attention with Q and K quantised to
 *                             FP8 e4m3 per head (SAGE FP8, a reading).
 *   oracle_varlen_attn_fp8  -- the attention with Q, K, V and P in FP8 e4m3
 *                             (the whole SAGE reading), P rounded against
 *                             each row's exact maximum.
 *   oracle_varlen_attn_fp8_online -- the same quantities in the rounding
 *                             order of an online softmax with a lazily moved
 *                             maximum (a streaming implementation's schedule,
 *                             block size and threshold given by the caller).
 *   oracle_varlen_attn_skip -- the same attention with key blocks skipped
 *                             where their scores are negligible ("Skip-Softmax";
 *                             a reading, see the function; the block geometry
 *                             is the caller's).
 *   oracle_modulate_swiglu -- modulation + normalisation + gated residual and
 *                             SwiGLU in place of separate SiLU and multiply
 *                             (first page "融合 DiT 算子"; second page bullet
 *                             "Fused DiT operators").
 *   oracle_linear_gated_residual, oracle_linear_swiglu -- the linear
 *                             layers around them with the gated residual or
 *                             SwiGLU as their epilogue (same passages; the
 *                             fusion into the GEMM is a reading).
 *
 * The pages state the operations, not their conventions; the readings taken
 * where they are silent (norm per head over head_dim, norm before RoPE,
 * theta_j = base^(-2j/D), pairing, adaLN as h = n*(1+scale)+shift with one
 * vector set per request, x' = x + g*branch, SwiGLU = silu(gate)*up, the
 * softmax scale passed by the caller, LSE in natural log) are listed with
 * the pins that check each function in the repository's design notes. Every
 * function is pinned by closed forms, brute force and invariants in the CPU
 * test suite.
 *
 * Every function is the plain definition: no blocking, fusion or
 * reordering. Inputs are either bfloat16 bit patterns (widened exactly) or
 * float64 values, selected per call.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_IN_BF16 0
#define ORACLE_IN_F64 1

#define ORACLE_ROPE_INTERLEAVED 0 /* pairs (2j, 2j+1) */
#define ORACLE_ROPE_HALF 1        /* pairs (j, j + D/2) */

#define ORACLE_NORM_RMS 0
#define ORACLE_NORM_LAYER 1
#define ORACLE_NORM_NONE 2

/* Exact widening of a bfloat16 bit pattern: its bits are the top half of an
 * IEEE binary32. */
static double bf16_bits_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Element i of a buffer given as bf16 bits or as float64. */
static double load(const void* p, int kind, int64_t i) {
  if (kind == ORACLE_IN_BF16) return bf16_bits_to_double(((const uint16_t*)p)[i]);
  return ((const double*)p)[i];
}

/* Segment s with cu[s] <= t < cu[s+1]; -1 if none. Linear scan: the plain
 * definition of "the request that token t belongs to". */
static int segment_of(const int32_t* cu, int B, int64_t t) {
  for (int s = 0; s < B; ++s)
    if (cu[s] <= t && t < cu[s + 1]) return s;
  return -1;
}

static int check_cu(const int32_t* cu, int B, int64_t T) {
  if (B < 0 || cu == NULL) return -1;
  if (cu[0] != 0 || cu[B] != T) return -1;
  for (int s = 0; s < B; ++s)
    if (cu[s + 1] < cu[s]) return -1;
  return 0;
}

/* RMSNorm of the D elements of one (token, head) row, times the weight:
 * n_d = x_d / sqrt(mean(x^2) + eps) * w_d. */
static void rms_times_weight(const void* x, int x_kind, int64_t row, const void* w, int w_kind, int D,
                             double eps, double* n) {
  double ms = 0.0;
  for (int d = 0; d < D; ++d) {
    double v = load(x, x_kind, row + d);
    ms += v * v;
  }
  ms /= (double)D;
  const double inv = 1.0 / sqrt(ms + eps);
  for (int d = 0; d < D; ++d) n[d] = load(x, x_kind, row + d) * inv * load(w, w_kind, d);
}

/* Element indices of RoPE pair j. */
static void pair_of(int style, int j, int D, int* ia, int* ib) {
  if (style == ORACLE_ROPE_INTERLEAVED) { *ia = 2 * j; *ib = 2 * j + 1; }
  else { *ia = j; *ib = j + D / 2; }
}

/* theta_j = base^(-2j/D). */
static double rope_theta(double base, int j, int D) { return pow(base, -2.0 * (double)j / (double)D); }

/* (a, b) <- (a cos phi - b sin phi, a sin phi + b cos phi). */
static void rotate_pair(const double* n, double* out, int ia, int ib, double phi) {
  const double a = n[ia], b = n[ib];
  out[ia] = a * cos(phi) - b * sin(phi);
  out[ib] = a * sin(phi) + b * cos(phi);
}

/*
 * RMSNorm over the D elements of one (token, head) row, weight w (shared by
 * all heads), then RoPE with angle phi_j = pos[t] * base^(-2j/D), j < D/2:
 *   (a, b) <- (a cos phi - b sin phi, a sin phi + b cos phi).
 * x: [T, H, D] with stride_t elements between tokens (a fused QKV buffer
 * has stride_t > H*D). rows: token indices to evaluate (NULL = all T).
 * y: [nrows, H, D] float64 contiguous.
 */
int oracle_qk_norm_rope(const void* x, int x_kind, int64_t stride_t, const void* w, int w_kind,
                        const int32_t* pos, int64_t T, int H, int D, double eps, double base,
                        int style, const int32_t* rows, int64_t nrows, double* y) {
  if (D <= 0 || D % 2 || H <= 0 || T < 0 || !(eps >= 0.0) || !(base > 0.0)) return -1;
  if (style != ORACLE_ROPE_INTERLEAVED && style != ORACLE_ROPE_HALF) return -1;
  if (rows == NULL) nrows = T;
  int64_t bad = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t t = rows ? rows[r] : r;
    if (t < 0 || t >= T) { ++bad; continue; }
    double* n = (double*)malloc(sizeof(double) * (size_t)D);
    for (int h = 0; h < H; ++h) {
      rms_times_weight(x, x_kind, t * stride_t + (int64_t)h * D, w, w_kind, D, eps, n);
      double* out = y + (r * H + h) * (int64_t)D;
      for (int j = 0; j < D / 2; ++j) {
        int ia, ib;
        pair_of(style, j, D, &ia, &ib);
        rotate_pair(n, out, ia, ib, (double)pos[t] * rope_theta(base, j, D));
      }
    }
    free(n);
  }
  return bad ? -1 : 0;
}

/*
 * RMSNorm as in oracle_qk_norm_rope, then RoPE with three position axes:
 * pair j < D/2 keeps the frequency theta_j = base^(-2j/D) but takes its
 * position from axis a(j) of pos3[t] = (t-id, h-id, w-id), where the pair
 * indices are split into consecutive sections of sec[0], sec[1], sec[2]
 * pairs (sec[0] + sec[1] + sec[2] = D/2): a(j) = 0 for j < sec[0], 1 for
 * j < sec[0] + sec[1], else 2. pos3: [T, 3] int32.
 */
int oracle_qk_norm_rope_3axis(const void* x, int x_kind, int64_t stride_t, const void* w, int w_kind,
                              const int32_t* pos3, const int32_t* sec, int64_t T, int H, int D, double eps,
                              double base, int style, const int32_t* rows, int64_t nrows, double* y) {
  if (D <= 0 || D % 2 || H <= 0 || T < 0 || !(eps >= 0.0) || !(base > 0.0)) return -1;
  if (style != ORACLE_ROPE_INTERLEAVED && style != ORACLE_ROPE_HALF) return -1;
  if (sec[0] < 0 || sec[1] < 0 || sec[2] < 0 || sec[0] + sec[1] + sec[2] != D / 2) return -1;
  if (rows == NULL) nrows = T;
  int64_t bad = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t t = rows ? rows[r] : r;
    if (t < 0 || t >= T) { ++bad; continue; }
    double* n = (double*)malloc(sizeof(double) * (size_t)D);
    for (int h = 0; h < H; ++h) {
      rms_times_weight(x, x_kind, t * stride_t + (int64_t)h * D, w, w_kind, D, eps, n);
      double* out = y + (r * H + h) * (int64_t)D;
      for (int j = 0; j < D / 2; ++j) {
        const int axis = j < sec[0] ? 0 : (j < sec[0] + sec[1] ? 1 : 2);
        int ia, ib;
        pair_of(style, j, D, &ia, &ib);
        rotate_pair(n, out, ia, ib, (double)pos3[t * 3 + axis] * rope_theta(base, j, D));
      }
    }
    free(n);
  }
  return bad ? -1 : 0;
}

/*
 * Full-width variant: the RMS is taken over all H*D elements of the token's
 * row of X (every head together), the weight w has H*D entries, then every
 * head is rotated as in oracle_qk_norm_rope:
 *   y_{h,d} = x_{h,d} / sqrt(mean_{h',d'}(x^2) + eps) * w[h*D + d].
 */
int oracle_qk_fullc_norm_rope(const void* x, int x_kind, int64_t stride_t, const void* w, int w_kind,
                              const int32_t* pos, int64_t T, int H, int D, double eps, double base, int style,
                              const int32_t* rows, int64_t nrows, double* y) {
  if (D <= 0 || D % 2 || H <= 0 || T < 0 || !(eps >= 0.0) || !(base > 0.0)) return -1;
  if (style != ORACLE_ROPE_INTERLEAVED && style != ORACLE_ROPE_HALF) return -1;
  if (rows == NULL) nrows = T;
  int64_t bad = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t t = rows ? rows[r] : r;
    if (t < 0 || t >= T) { ++bad; continue; }
    const int64_t width = (int64_t)H * D;
    double ms = 0.0;
    for (int64_t e = 0; e < width; ++e) {
      const double v = load(x, x_kind, t * stride_t + e);
      ms += v * v;
    }
    ms /= (double)width;
    const double inv = 1.0 / sqrt(ms + eps);
    double* n = (double*)malloc(sizeof(double) * (size_t)D);
    for (int h = 0; h < H; ++h) {
      for (int d = 0; d < D; ++d)
        n[d] = load(x, x_kind, t * stride_t + (int64_t)h * D + d) * inv * load(w, w_kind, (int64_t)h * D + d);
      double* out = y + (r * H + h) * (int64_t)D;
      for (int j = 0; j < D / 2; ++j) {
        int ia, ib;
        pair_of(style, j, D, &ia, &ib);
        rotate_pair(n, out, ia, ib, (double)pos[t] * rope_theta(base, j, D));
      }
    }
    free(n);
  }
  return bad ? -1 : 0;
}

/*
 * Packed variable-length attention, bidirectional within each request and
 * nothing across requests. For token t in request i = [cu[i], cu[i+1]) and
 * head h:
 *   s_j = scale * <q_t, k_j>, j in request i
 *   m = max_j s_j, p_j = exp(s_j - m), l = sum_j p_j
 *   o_t = sum_j p_j v_j / l,  lse_t = m + ln l.
 * q, k, v: [T, H, D], stride_t elements between tokens. o: [nrows, H, D];
 * lse: [nrows, H] or NULL.
 */
int oracle_varlen_attn(const void* q, const void* k, const void* v, int in_kind, int64_t stride_t,
                       const int32_t* cu, int B, int64_t T, int H, int D, double scale,
                       const int32_t* rows, int64_t nrows, double* o, double* lse) {
  if (check_cu(cu, B, T) || H <= 0 || D <= 0) return -1;
  if (rows == NULL) nrows = T;
  int64_t bad = 0;
#pragma omp parallel for schedule(dynamic, 1) collapse(2) reduction(+ : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    for (int h = 0; h < H; ++h) {
      const int64_t t = rows ? rows[r] : r;
      const int seg = (t >= 0 && t < T) ? segment_of(cu, B, t) : -1;
      if (seg < 0) { ++bad; continue; }
      const int64_t lo = cu[seg], L = (int64_t)cu[seg + 1] - cu[seg];
      double* s = (double*)malloc(sizeof(double) * (size_t)L);
      double* qt = (double*)malloc(sizeof(double) * (size_t)D);
      for (int d = 0; d < D; ++d) qt[d] = load(q, in_kind, t * stride_t + (int64_t)h * D + d);
      double m = -INFINITY;
      for (int64_t j = 0; j < L; ++j) {
        double acc = 0.0;
        const int64_t kb = (lo + j) * stride_t + (int64_t)h * D;
        for (int d = 0; d < D; ++d) acc += qt[d] * load(k, in_kind, kb + d);
        s[j] = scale * acc;
        if (s[j] > m) m = s[j];
      }
      double l = 0.0;
      for (int64_t j = 0; j < L; ++j) { s[j] = exp(s[j] - m); l += s[j]; }
      double* ot = o + (r * H + h) * (int64_t)D;
      for (int d = 0; d < D; ++d) ot[d] = 0.0;
      for (int64_t j = 0; j < L; ++j) {
        const int64_t vb = (lo + j) * stride_t + (int64_t)h * D;
        for (int d = 0; d < D; ++d) ot[d] += s[j] * load(v, in_kind, vb + d);
      }
      for (int d = 0; d < D; ++d) ot[d] /= l;
      if (lse) lse[r * H + h] = m + log(l);
      free(s);
      free(qt);
    }
  }
  return bad ? -1 : 0;
}

/*
 * FP8 e4m3 ("fn": 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
 * no infinities, largest finite 448, subnormal spacing 2^-9): the value of a
 * code, and the code nearest to a float (ties to even), values beyond 448 in
 * magnitude saturating to 448.
 */
static double e4m3_value(uint8_t c) {
  const int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
  const double mag = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return sgn ? -mag : mag;
}

static uint8_t e4m3_code(float x) {
  const uint8_t sgn = (x < 0.0f || (x == 0.0f && signbit(x))) ? 0x80 : 0;
  double a = fabs((double)x);
  if (a >= 448.0) return (uint8_t)(sgn | 0x7E);
  int E;
  frexp(a, &E);                 /* a in [2^(E-1), 2^E) */
  int e = a > 0.0 ? E - 1 : -6;
  if (e < -6) e = -6;           /* subnormal spacing below 2^-6 */
  const double quantum = ldexp(1.0, e - 3);
  const double r = rint(a / quantum) * quantum; /* ties to even: a / quantum is exact */
  if (r == 0.0) return sgn;
  if (r >= 448.0) return (uint8_t)(sgn | 0x7E);
  frexp(r, &E);
  e = E - 1;
  if (e < -6) return (uint8_t)(sgn | (uint8_t)(r / ldexp(1.0, -9)));
  const int mant = (int)((r / ldexp(1.0, e) - 1.0) * 8.0);
  return (uint8_t)(sgn | (uint8_t)((e + 7) << 3) | (uint8_t)mant);
}

/*
 * Per-head absmax quantisation of a [T, H, D] tensor to e4m3 (a reading of
 * the SAGE FP8 attention named on the first page, bullet on TRTLLM_ATTN SAGE
 * and Skip-Softmax: "quantise the attention computation to FP8"): for head
 * h, amax = max |x| over all tokens and D; in float arithmetic
 * inv = 448 / amax and code = e4m3(x * inv); the dequantisation factor is
 * deq = amax / 448 (both 1 when amax = 0). codes: [T, H, D]; deq: [H].
 */
int oracle_quantize_e4m3(const void* x, int x_kind, int64_t stride_t, int64_t T, int H, int D, uint8_t* codes,
                         float* deq) {
  if (T < 0 || H <= 0 || D <= 0 || stride_t < (int64_t)H * D) return -1;
  for (int h = 0; h < H; ++h) {
    float amax = 0.0f;
    for (int64_t t = 0; t < T; ++t)
      for (int d = 0; d < D; ++d) {
        const float v = (float)fabs(load(x, x_kind, t * stride_t + (int64_t)h * D + d));
        if (v > amax) amax = v;
      }
    const float inv = amax > 0.0f ? 448.0f / amax : 1.0f;
    deq[h] = amax > 0.0f ? amax / 448.0f : 1.0f;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
      for (int d = 0; d < D; ++d) {
        const float v = (float)load(x, x_kind, t * stride_t + (int64_t)h * D + d);
        codes[(t * H + h) * (int64_t)D + d] = e4m3_code(v * inv);
      }
  }
  return 0;
}

int oracle_varlen_attn_skip(const void* q, const void* k, const void* v, int in_kind, int64_t stride_t,
                            const int32_t* cu, int B, int64_t T, int H, int D, double scale, double tau,
                            int qrows, int kblock, int tile_rows, const int32_t* rows, int64_t nrows, double* o,
                            double* lse, int64_t* counts);
static void skip_block_flags(const void* q, const void* k, int in_kind, int64_t stride_t, int64_t lo, int64_t n_keys,
                             int64_t r0, int64_t r1, int h, int D, double scale, double tau, int kblock,
                             unsigned char* keep);
static int64_t skip_tile_count(const unsigned char* keep, int H, int64_t nqb, int64_t nkb, int64_t per_tile);

/*
 * RMSNorm + RoPE as oracle_qk_norm_rope, then e4m3 codes with one scale per
 * tensor taken from a bound rather than from the data (a reading of SAGE's
 * FP8 quantisation folded into the Q/K prologue, first page, bullet on
 * TRTLLM_ATTN SAGE and Skip-Softmax): a normalised row has
 * sum_d (x_d / rms)^2 <= D, so every element of it, and of its rotation
 * (which preserves each pair's norm), is at most sqrt(D) * max_d |w_d| in
 * magnitude. In float arithmetic, amax = sqrtf(D) * max_d |w_d|,
 * inv = 448 / amax and deq = amax / 448 (both 1 when amax = 0); every element
 * y (the float64 result) gets code e4m3((float)(y * inv)). codes:
 * [nrows, H, D]; deq_out: that one factor.
 */
int oracle_qk_norm_rope_e4m3(const void* x, int x_kind, int64_t stride_t, const void* w, int w_kind,
                             const int32_t* pos, int64_t T, int H, int D, double eps, double base, int style,
                             const int32_t* rows, int64_t nrows, uint8_t* codes, float* deq_out) {
  if (D <= 0 || H <= 0 || T < 0) return -1;
  const int64_t nr = rows ? nrows : T;
  const int64_t n = nr * (int64_t)H * D;
  double* y = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  int rc = oracle_qk_norm_rope(x, x_kind, stride_t, w, w_kind, pos, T, H, D, eps, base, style, rows, nrows, y);
  if (!rc) {
    float maxw = 0.0f;
    for (int d = 0; d < D; ++d) {
      const float a = (float)fabs(load(w, w_kind, d));
      if (a > maxw) maxw = a;
    }
    const float amax = sqrtf((float)D) * maxw;
    const float inv = amax > 0.0f ? 448.0f / amax : 1.0f;
    *deq_out = amax > 0.0f ? amax / 448.0f : 1.0f;
    for (int64_t e = 0; e < n; ++e) codes[e] = e4m3_code((float)(y[e] * (double)inv));
  }
  free(y);
  return rc;
}

/*
 * Attention with Q and K quantised to e4m3 per head (oracle_quantize_e4m3)
 * and V, P kept at their precision: the plain attention of
 * oracle_varlen_attn on Q~ = code(Q) * deq_Q and K~ = code(K) * deq_K, or,
 * for a finite tau, the block-skipping attention of oracle_varlen_attn_skip
 * on them with the block geometry (qrows, kblock, tile_rows) given (counts as
 * there; the geometry is unused for an infinite tau). q8_out, k8_out
 * ([T, H, D]) and deq_out ([2H]: Q's, then K's) are optional.
 */
int oracle_varlen_attn_fp8qk(const void* q, const void* k, const void* v, int in_kind, int64_t stride_t,
                             const int32_t* cu, int B, int64_t T, int H, int D, double scale, double tau,
                             int qrows, int kblock, int tile_rows, const int32_t* rows, int64_t nrows, double* o,
                             double* lse, int64_t* counts, uint8_t* q8_out, uint8_t* k8_out, float* deq_out) {
  if (check_cu(cu, B, T) || H <= 0 || D <= 0) return -1;
  const int64_t n = T * (int64_t)H * D;
  uint8_t* qc = q8_out ? q8_out : (uint8_t*)malloc((size_t)(n > 0 ? n : 1));
  uint8_t* kc = k8_out ? k8_out : (uint8_t*)malloc((size_t)(n > 0 ? n : 1));
  float* dq = (float*)malloc(sizeof(float) * (size_t)H * 2);
  double* qd = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double* kd = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  double* vd = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  int rc = oracle_quantize_e4m3(q, in_kind, stride_t, T, H, D, qc, dq);
  if (!rc) rc = oracle_quantize_e4m3(k, in_kind, stride_t, T, H, D, kc, dq + H);
  if (!rc) {
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
      for (int h = 0; h < H; ++h)
        for (int d = 0; d < D; ++d) {
          const int64_t i = (t * H + h) * (int64_t)D + d;
          qd[i] = e4m3_value(qc[i]) * (double)dq[h];
          kd[i] = e4m3_value(kc[i]) * (double)dq[H + h];
          vd[i] = load(v, in_kind, t * stride_t + (int64_t)h * D + d);
        }
    if (isinf(tau) && tau > 0)
      rc = oracle_varlen_attn(qd, kd, vd, ORACLE_IN_F64, (int64_t)H * D, cu, B, T, H, D, scale, rows, nrows, o, lse);
    else
      rc = oracle_varlen_attn_skip(qd, kd, vd, ORACLE_IN_F64, (int64_t)H * D, cu, B, T, H, D, scale, tau, qrows,
                                   kblock, tile_rows, rows, nrows, o, lse, counts);
  }
  if (deq_out) memcpy(deq_out, dq, sizeof(float) * (size_t)H * 2);
  if (!q8_out) free(qc);
  if (!k8_out) free(kc);
  free(dq);
  free(qd);
  free(kd);
  free(vd);
  return rc;
}

/*
 * Attention with Q, K and V quantised to e4m3 per head and the
 * probabilities P quantised to e4m3: the whole attention computation in FP8
 * (SAGE, first page, bullet on TRTLLM_ATTN SAGE and Skip-Softmax; a
 * reading). With Q~, K~, V~ the dequantised tensors (code * deq per head),
 * for query row t of request i and head h:
 *   s_j  = scale * <q~_t, k~_j>,  j in request i
 *   m    = max_j s_j,  p_j = exp(s_j - m)          (so 0 < p_j <= 1)
 *   o_t  = sum_j e4m3(p_j) v~_j / sum_j p_j         (P rounded in the numerator only)
 *   lse_t = m + ln sum_j p_j.
 * e4m3(p) is the code nearest to p taken as a float (oracle_e4m3_codes),
 * read back as its value. deq_out: [3H] (Q's, K's, V's dequantisation
 * factors), optional.
 * With a finite tau the key blocks that the block-skipping rule of
 * oracle_varlen_attn_skip drops (decided on the scores of Q~, K~ with the
 * caller's geometry) are left out of every sum and of the maximum, and
 * counts (nullable) receives that rule's two counts for all T rows.
 */
static void fp8_row(const double* qd, const double* kd, const double* vd, int64_t lo, int64_t n_keys, int64_t t,
                    int H, int h, int D, double scale, const unsigned char* keep, int kblock, double* ot,
                    double* lse_out) {
  const double* qr = qd + (t * H + h) * (int64_t)D;
  double* s = (double*)malloc(sizeof(double) * (size_t)(n_keys > 0 ? n_keys : 1));
  double m = -INFINITY;
  for (int64_t j = 0; j < n_keys; ++j) {
    if (keep && !keep[j / kblock]) continue;
    const double* kr = kd + ((lo + j) * H + h) * (int64_t)D;
    double dot = 0.0;
    for (int d = 0; d < D; ++d) dot += qr[d] * kr[d];
    s[j] = scale * dot;
    if (s[j] > m) m = s[j];
  }
  double den = 0.0;
  for (int d = 0; d < D; ++d) ot[d] = 0.0;
  for (int64_t j = 0; j < n_keys; ++j) {
    if (keep && !keep[j / kblock]) continue;
    const double pj = exp(s[j] - m);
    const double pq = e4m3_value(e4m3_code((float)pj));
    den += pj;
    const double* vr = vd + ((lo + j) * H + h) * (int64_t)D;
    for (int d = 0; d < D; ++d) ot[d] += pq * vr[d];
  }
  for (int d = 0; d < D; ++d) ot[d] /= den;
  if (lse_out) *lse_out = m + log(den);
  free(s);
}

/*
 * The same FP8 attention accumulated the way a streaming (online-softmax)
 * implementation does it: NOT the definition above but the rounding schedule
 * of such an implementation, kept as a second, tighter check on one. Per
 * row, over key blocks of kblock keys counted from the request's first token,
 * in order, with u = s / ln 2 (log2 units):
 *   - the running maximum m is set by the first block and afterwards moves
 *     only when a block's maximum exceeds it by more than threshold; the sums
 *     are then scaled by 2^(m_old - m_new);
 *   - each key adds p = 2^(u - m) to the denominator l and e4m3(p) * v~ to
 *     the numerator (p <= 2^threshold);
 *   - o = numerator / l and lse = (m + log2 l) ln 2.
 * With threshold = 0 and one block per request this is the definition; any
 * other schedule rounds each p against a smaller maximum, which changes each
 * numerator term by at most one e4m3 step. With block skipping (a finite
 * tau) dropped keys take no part: a block's maximum is over its kept keys.
 */
static void fp8_row_online(const double* qd, const double* kd, const double* vd, int64_t lo, int64_t n_keys,
                           int64_t t, int H, int h, int D, double scale, int kblock, double threshold,
                           const unsigned char* keep, int skip_kblock, double* ot, double* lse_out) {
  const double* qr = qd + (t * H + h) * (int64_t)D;
  double* num = (double*)calloc((size_t)D, sizeof(double));
  double* ublock = (double*)malloc(sizeof(double) * (size_t)kblock);
  double mrun = -INFINITY, den = 0.0;
  for (int64_t b0 = 0; b0 < n_keys; b0 += kblock) {
    const int64_t b1 = b0 + kblock < n_keys ? b0 + kblock : n_keys;
    double bmax = -INFINITY;  /* over the block's kept keys */
    for (int64_t j = b0; j < b1; ++j) {
      const double* kr = kd + ((lo + j) * H + h) * (int64_t)D;
      double dot = 0.0;
      for (int d = 0; d < D; ++d) dot += qr[d] * kr[d];
      ublock[j - b0] = scale * dot / log(2.0);
      if ((!keep || keep[j / skip_kblock]) && ublock[j - b0] > bmax) bmax = ublock[j - b0];
    }
    if (b0 == 0) {
      mrun = bmax;
    } else if (bmax > mrun + threshold) {
      const double alpha = exp2(mrun - bmax);
      den *= alpha;
      for (int d = 0; d < D; ++d) num[d] *= alpha;
      mrun = bmax;
    }
    for (int64_t j = b0; j < b1; ++j) {
      if (keep && !keep[j / skip_kblock]) continue;
      const double pj = exp2(ublock[j - b0] - mrun);
      const double pq = e4m3_value(e4m3_code((float)pj));
      den += pj;
      const double* vr = vd + ((lo + j) * H + h) * (int64_t)D;
      for (int d = 0; d < D; ++d) num[d] += pq * vr[d];
    }
  }
  for (int d = 0; d < D; ++d) ot[d] = num[d] / den;
  if (lse_out) *lse_out = (mrun + log2(den)) * log(2.0);
  free(ublock);
  free(num);
}

/* Both FP8 attentions: online == 0 the definition, else the online schedule
 * with (kblock, threshold); a finite tau adds block skipping with the
 * geometry (skip_qrows, skip_kblock, skip_tile_rows). */
static int fp8_attention(const void* q, const void* k, const void* v, int in_kind, int64_t stride_t,
                         const int32_t* cu, int B, int64_t T, int H, int D, double scale, int online, int kblock,
                         double threshold, double tau, int skip_qrows, int skip_kblock, int skip_tile_rows,
                         const int32_t* rows, int64_t nrows, double* o, double* lse, int64_t* counts,
                         float* deq_out) {
  if (check_cu(cu, B, T) || H <= 0 || D <= 0 || isnan(tau)) return -1;
  if (online && (kblock <= 0 || !(threshold >= 0.0))) return -1;
  const int skipping = !(isinf(tau) && tau > 0);
  if (skipping && (skip_qrows <= 0 || skip_kblock <= 0 || skip_tile_rows <= 0 || skip_tile_rows % skip_qrows))
    return -1;
  const int64_t n = T * (int64_t)H * D;
  uint8_t* c8 = (uint8_t*)malloc((size_t)(n > 0 ? n : 1));
  float* dq = (float*)malloc(sizeof(float) * (size_t)H * 3);
  double* xd[3];
  const void* src[3] = {q, k, v};
  int rc = 0;
  for (int i = 0; i < 3; ++i) {
    xd[i] = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    if (!rc) rc = oracle_quantize_e4m3(src[i], in_kind, stride_t, T, H, D, c8, dq + (int64_t)i * H);
    if (!rc) {
#pragma omp parallel for schedule(static)
      for (int64_t e = 0; e < n; ++e) xd[i][e] = e4m3_value(c8[e]) * (double)dq[(int64_t)i * H + (e / D) % H];
    }
  }
  /* skip decisions per (request, head, query block), on the dequantised Q, K */
  unsigned char** keep = NULL;
  if (!rc && skipping) {
    keep = (unsigned char**)calloc((size_t)(B > 0 ? B : 1), sizeof(unsigned char*));
    int64_t n_block = 0, n_tile = 0;
    for (int seg = 0; seg < B; ++seg) {
      const int64_t lo = cu[seg], n_keys = (int64_t)cu[seg + 1] - cu[seg];
      if (n_keys == 0) continue;
      const int64_t nqb = (n_keys + skip_qrows - 1) / skip_qrows, nkb = (n_keys + skip_kblock - 1) / skip_kblock;
      keep[seg] = (unsigned char*)malloc((size_t)(H * nqb * nkb));
#pragma omp parallel for schedule(dynamic, 1) collapse(2) reduction(+ : n_block)
      for (int64_t b = 0; b < nqb; ++b) {
        for (int h = 0; h < H; ++h) {
          const int64_t r0 = lo + b * skip_qrows;
          const int64_t r1 = r0 + skip_qrows < lo + n_keys ? r0 + skip_qrows : lo + n_keys;
          unsigned char* kp = keep[seg] + ((int64_t)h * nqb + b) * nkb;
          skip_block_flags(xd[0], xd[1], ORACLE_IN_F64, (int64_t)H * D, lo, n_keys, r0, r1, h, D, scale, tau,
                           skip_kblock, kp);
          for (int64_t jb = 0; jb < nkb; ++jb) n_block += !kp[jb];
        }
      }
      n_tile += skip_tile_count(keep[seg], H, nqb, nkb, skip_tile_rows / skip_qrows);
    }
    if (counts) {
      counts[0] = n_block;
      counts[1] = n_tile;
    }
  }
  if (!rc) {
    const int64_t nr = rows ? nrows : T;
    int64_t bad = 0;
#pragma omp parallel for schedule(dynamic, 1) collapse(2) reduction(+ : bad)
    for (int64_t r = 0; r < nr; ++r) {
      for (int h = 0; h < H; ++h) {
        const int64_t t = rows ? rows[r] : r;
        const int seg = (t >= 0 && t < T) ? segment_of(cu, B, t) : -1;
        if (seg < 0) { ++bad; continue; }
        const int64_t lo = cu[seg], n_keys = (int64_t)cu[seg + 1] - cu[seg];
        const unsigned char* kp = NULL;
        if (keep) {
          const int64_t nqb = (n_keys + skip_qrows - 1) / skip_qrows, nkb = (n_keys + skip_kblock - 1) / skip_kblock;
          kp = keep[seg] + ((int64_t)h * nqb + (t - lo) / skip_qrows) * nkb;
        }
        double* ot = o + (r * H + h) * (int64_t)D;
        double* lt = lse ? &lse[r * H + h] : NULL;
        if (online)
          fp8_row_online(xd[0], xd[1], xd[2], lo, n_keys, t, H, h, D, scale, kblock, threshold, kp, skip_kblock, ot,
                         lt);
        else
          fp8_row(xd[0], xd[1], xd[2], lo, n_keys, t, H, h, D, scale, kp, skip_kblock, ot, lt);
      }
    }
    if (bad) rc = -1;
  }
  if (keep) {
    for (int seg = 0; seg < B; ++seg) free(keep[seg]);
    free(keep);
  }
  if (deq_out) memcpy(deq_out, dq, sizeof(float) * (size_t)H * 3);
  for (int i = 0; i < 3; ++i) free(xd[i]);
  free(c8);
  free(dq);
  return rc;
}

int oracle_varlen_attn_fp8(const void* q, const void* k, const void* v, int in_kind, int64_t stride_t,
                           const int32_t* cu, int B, int64_t T, int H, int D, double scale, double tau, int qrows,
                           int kblock, int tile_rows, const int32_t* rows, int64_t nrows, double* o, double* lse,
                           int64_t* counts, float* deq_out) {
  return fp8_attention(q, k, v, in_kind, stride_t, cu, B, T, H, D, scale, 0, 0, 0.0, tau, qrows, kblock, tile_rows,
                       rows, nrows, o, lse, counts, deq_out);
}

int oracle_varlen_attn_fp8_online(const void* q, const void* k, const void* v, int in_kind, int64_t stride_t,
                                  const int32_t* cu, int B, int64_t T, int H, int D, double scale, int kblock,
                                  double threshold, double tau, int qrows, int skip_kblock, int tile_rows,
                                  const int32_t* rows, int64_t nrows, double* o, double* lse, int64_t* counts,
                                  float* deq_out) {
  return fp8_attention(q, k, v, in_kind, stride_t, cu, B, T, H, D, scale, 1, kblock, threshold, tau, qrows,
                       skip_kblock, tile_rows, rows, nrows, o, lse, counts, deq_out);
}

/* e4m3 codes of a float32 array (the conversion alone, for its pins). */
void oracle_e4m3_codes(const float* x, int64_t n, uint8_t* codes) {
  for (int64_t i = 0; i < n; ++i) codes[i] = e4m3_code(x[i]);
}

/*
 * Attention with block skipping: "Skip-Softmax" skips the softmax and the
 * P x V work of unimportant blocks (first page, bullet on TRTLLM_ATTN SAGE and
 * Skip-Softmax; second page, section "System-wide optimizations in
 * vLLM-Omni", bullet "Sparse & quantized attention"). The pages name the idea
 * only, not a block size. The reading taken, for a block geometry given by
 * the caller:
 *   - a block is qrows consecutive query rows x kblock consecutive keys of
 *     one request and head, both counted from the request's first token; key
 *     blocks are visited in increasing order;
 *   - with u(r,k) = s(r,k) / ln 2 (the score s includes the softmax scale),
 *     key block j >= 1 is skipped for query block b when every row r of b
 *     inside the request has max_{k in j} u(r,k) < M(r) - tau, where M(r) is
 *     the maximum of u(r,k) over the keys of blocks 0 .. j-1 (key block 0 is
 *     never skipped);
 *   - a skipped block contributes nothing: o_r = sum_kept e^(s-m) v /
 *     sum_kept e^(s-m) with m the maximum over kept keys, lse_r = m + ln(sum).
 * A very large tau skips nothing and gives oracle_varlen_attn's result.
 * rows: tokens to output (NULL = all T); each row's whole query block is
 * evaluated to take that block's decisions. counts (nullable, filled only
 * when rows == NULL): counts[0] = skipped (query block, head, key block)
 * triples; counts[1] = skipped (tile, head, key block) triples, a tile being
 * tile_rows consecutive query rows (a multiple of qrows, also counted from the
 * request's first token) that skips a key block when all of its query blocks
 * inside the request do.
 */

/* Number of (tile, head, key block) triples in which every query block of
 * the tile (per_tile consecutive query blocks of one request) drops the key
 * block. keep: [H][nqb][nkb] flags of one request. */
static int64_t skip_tile_count(const unsigned char* keep, int H, int64_t nqb, int64_t nkb, int64_t per_tile) {
  int64_t n_tile = 0;
  for (int h = 0; h < H; ++h)
    for (int64_t tb = 0; tb * per_tile < nqb; ++tb)
      for (int64_t jb = 0; jb < nkb; ++jb) {
        int all = 1;
        for (int64_t b = tb * per_tile; b < (tb + 1) * per_tile && b < nqb; ++b)
          if (keep[((int64_t)h * nqb + b) * nkb + jb]) all = 0;
        n_tile += all;
      }
  return n_tile;
}

/* Keep flags of the key blocks of query block [r0, r1) (rows of one request
 * starting at lo, n_keys keys), head h. keep: [ceil(n_keys / kblock)]. */
static void skip_block_flags(const void* q, const void* k, int in_kind, int64_t stride_t, int64_t lo, int64_t n_keys,
                             int64_t r0, int64_t r1, int h, int D, double scale, double tau, int kblock,
                             unsigned char* keep) {
  const int64_t nkb = (n_keys + kblock - 1) / kblock;
  const int64_t nr = r1 - r0;
  double* tmax = (double*)malloc(sizeof(double) * (size_t)(nr * nkb));
  double* qt = (double*)malloc(sizeof(double) * (size_t)D);
  for (int64_t i = 0; i < nr; ++i) {
    const int64_t t = r0 + i;
    for (int d = 0; d < D; ++d) qt[d] = load(q, in_kind, t * stride_t + (int64_t)h * D + d);
    for (int64_t jb = 0; jb < nkb; ++jb) tmax[i * nkb + jb] = -INFINITY;
    for (int64_t j = 0; j < n_keys; ++j) {
      double dot = 0.0;
      const int64_t key_at = (lo + j) * stride_t + (int64_t)h * D;
      for (int d = 0; d < D; ++d) dot += qt[d] * load(k, in_kind, key_at + d);
      const double u = scale * dot / log(2.0);
      double* tm = &tmax[i * nkb + j / kblock];
      if (u > *tm) *tm = u;
    }
  }
  for (int64_t jb = 0; jb < nkb; ++jb) {
    int skip = jb >= 1;
    for (int64_t i = 0; i < nr && skip; ++i) {
      double M = -INFINITY;
      for (int64_t pb = 0; pb < jb; ++pb)
        if (tmax[i * nkb + pb] > M) M = tmax[i * nkb + pb];
      if (!(tmax[i * nkb + jb] < M - tau)) skip = 0;
    }
    keep[jb] = (unsigned char)!skip;
  }
  free(qt);
  free(tmax);
}

/* Output row t (of request lo, n_keys), head h, over the kept key blocks. */
static void skip_row_output(const void* q, const void* k, const void* v, int in_kind, int64_t stride_t, int64_t lo,
                            int64_t n_keys, int64_t t, int h, int D, double scale, int kblock, const unsigned char* keep,
                            double* ot, double* lse_out) {
  double* sc = (double*)malloc(sizeof(double) * (size_t)n_keys);
  double* qt = (double*)malloc(sizeof(double) * (size_t)D);
  for (int d = 0; d < D; ++d) qt[d] = load(q, in_kind, t * stride_t + (int64_t)h * D + d);
  double m = -INFINITY;
  for (int64_t j = 0; j < n_keys; ++j) {
    if (!keep[j / kblock]) continue;
    double dot = 0.0;
    const int64_t key_at = (lo + j) * stride_t + (int64_t)h * D;
    for (int d = 0; d < D; ++d) dot += qt[d] * load(k, in_kind, key_at + d);
    sc[j] = scale * dot;
    if (sc[j] > m) m = sc[j];
  }
  double mass = 0.0;
  for (int d = 0; d < D; ++d) ot[d] = 0.0;
  for (int64_t j = 0; j < n_keys; ++j) {
    if (!keep[j / kblock]) continue;
    const double pj = exp(sc[j] - m);
    mass += pj;
    const int64_t val_at = (lo + j) * stride_t + (int64_t)h * D;
    for (int d = 0; d < D; ++d) ot[d] += pj * load(v, in_kind, val_at + d);
  }
  for (int d = 0; d < D; ++d) ot[d] /= mass;
  if (lse_out) *lse_out = m + log(mass);
  free(sc);
  free(qt);
}

int oracle_varlen_attn_skip(const void* q, const void* k, const void* v, int in_kind, int64_t stride_t,
                            const int32_t* cu, int B, int64_t T, int H, int D, double scale, double tau,
                            int qrows, int kblock, int tile_rows, const int32_t* rows, int64_t nrows, double* o,
                            double* lse, int64_t* counts) {
  if (check_cu(cu, B, T) || H <= 0 || D <= 0 || isnan(tau)) return -1;
  if (qrows <= 0 || kblock <= 0 || tile_rows <= 0 || tile_rows % qrows) return -1;
  if (rows != NULL) {
    int64_t bad = 0;
#pragma omp parallel for schedule(dynamic, 1) collapse(2) reduction(+ : bad)
    for (int64_t r = 0; r < nrows; ++r) {
      for (int h = 0; h < H; ++h) {
        const int64_t t = rows[r];
        const int seg = (t >= 0 && t < T) ? segment_of(cu, B, t) : -1;
        if (seg < 0) { ++bad; continue; }
        const int64_t lo = cu[seg], n_keys = (int64_t)cu[seg + 1] - (int64_t)cu[seg];
        const int64_t r0 = lo + ((t - lo) / qrows) * qrows;
        const int64_t r1 = r0 + qrows < lo + n_keys ? r0 + qrows : lo + n_keys;
        unsigned char* keep = (unsigned char*)malloc((size_t)((n_keys + kblock - 1) / kblock));
        skip_block_flags(q, k, in_kind, stride_t, lo, n_keys, r0, r1, h, D, scale, tau, kblock, keep);
        skip_row_output(q, k, v, in_kind, stride_t, lo, n_keys, t, h, D, scale, kblock, keep,
                        o + (r * H + h) * (int64_t)D, lse ? &lse[r * H + h] : NULL);
        free(keep);
      }
    }
    return bad ? -1 : 0;
  }
  int64_t n_block = 0, n_tile = 0;
  for (int seg = 0; seg < B; ++seg) {
    const int64_t lo = cu[seg], n_keys = (int64_t)cu[seg + 1] - (int64_t)cu[seg];
    if (n_keys == 0) continue;
    const int64_t nqb = (n_keys + qrows - 1) / qrows;
    const int64_t nkb = (n_keys + kblock - 1) / kblock;
    unsigned char* keep = (unsigned char*)malloc((size_t)(H * nqb * nkb));
#pragma omp parallel for schedule(dynamic, 1) collapse(2) reduction(+ : n_block)
    for (int64_t b = 0; b < nqb; ++b) {
      for (int h = 0; h < H; ++h) {
        const int64_t r0 = lo + b * qrows;
        const int64_t r1 = r0 + qrows < lo + n_keys ? r0 + qrows : lo + n_keys;
        unsigned char* kp = keep + ((int64_t)h * nqb + b) * nkb;
        skip_block_flags(q, k, in_kind, stride_t, lo, n_keys, r0, r1, h, D, scale, tau, kblock, kp);
        for (int64_t t = r0; t < r1; ++t)
          skip_row_output(q, k, v, in_kind, stride_t, lo, n_keys, t, h, D, scale, kblock, kp,
                          o + (t * H + h) * (int64_t)D, lse ? &lse[t * H + h] : NULL);
        for (int64_t jb = 0; jb < nkb; ++jb) n_block += !kp[jb];
      }
    }
    /* a tile skips key block jb when each of its query blocks inside the request does */
    n_tile += skip_tile_count(keep, H, nqb, nkb, tile_rows / qrows);
    free(keep);
  }
  if (counts) {
    counts[0] = n_block;
    counts[1] = n_tile;
  }
  return 0;
}

/*
 * Per token t of request s:
 *   x'  = x + gate_res[s] * branch            (branch == NULL: x' = x)
 *   n   = x' / sqrt(mean(x'^2) + eps)         (RMS, no affine)
 *       = (x' - mu) / sqrt(var + eps)         (LAYER, biased variance)
 *       = x'                                  (NONE)
 *   h   = n * (1 + scale[s]) + shift[s]
 *   act = gate / (1 + exp(-gate)) * up        (gate == NULL: skipped)
 * x, branch: [T, C]; shift, scale, gate_res: [B, C] float32; gate, up:
 * [T, F] with gu_stride elements between tokens. Outputs float64 with rows
 * [nrows, C] / [nrows, F]; x_out may be NULL.
 */
int oracle_modulate_swiglu(const void* x, const void* branch, int in_kind, const float* shift,
                           const float* scale, const float* gate_res, const int32_t* cu, int B,
                           int64_t T, int C, int norm_type, double eps, const void* gate,
                           const void* up, int64_t gu_stride, int F, const int32_t* rows,
                           int64_t nrows, double* x_out, double* h_out, double* act_out) {
  if (check_cu(cu, B, T) || C <= 0 || F < 0 || !(eps >= 0.0)) return -1;
  if (norm_type != ORACLE_NORM_RMS && norm_type != ORACLE_NORM_LAYER && norm_type != ORACLE_NORM_NONE)
    return -1;
  if (rows == NULL) nrows = T;
  int64_t bad = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t t = rows ? rows[r] : r;
    const int seg = (t >= 0 && t < T) ? segment_of(cu, B, t) : -1;
    if (seg < 0) { ++bad; continue; }
    double* xp = (double*)malloc(sizeof(double) * (size_t)C);
    for (int c = 0; c < C; ++c) {
      double xv = load(x, in_kind, t * C + c);
      if (branch) xv += (double)gate_res[(int64_t)seg * C + c] * load(branch, in_kind, t * C + c);
      xp[c] = xv;
      if (x_out) x_out[r * C + c] = xv;
    }
    double mu = 0.0, ms = 0.0, var = 0.0;
    for (int c = 0; c < C; ++c) { mu += xp[c]; ms += xp[c] * xp[c]; }
    mu /= (double)C;
    ms /= (double)C;
    for (int c = 0; c < C; ++c) var += (xp[c] - mu) * (xp[c] - mu);
    var /= (double)C;
    for (int c = 0; c < C; ++c) {
      double n;
      if (norm_type == ORACLE_NORM_RMS) n = xp[c] / sqrt(ms + eps);
      else if (norm_type == ORACLE_NORM_LAYER) n = (xp[c] - mu) / sqrt(var + eps);
      else n = xp[c];
      h_out[r * C + c] = n * (1.0 + (double)scale[(int64_t)seg * C + c]) + (double)shift[(int64_t)seg * C + c];
    }
    if (gate && up && act_out) {
      for (int f = 0; f < F; ++f) {
        const double g = load(gate, in_kind, t * gu_stride + f);
        const double u = load(up, in_kind, t * gu_stride + f);
        act_out[r * (int64_t)F + f] = g / (1.0 + exp(-g)) * u;
      }
    }
    free(xp);
  }
  return bad ? -1 : 0;
}

/*
 * A linear layer whose epilogue is the gated residual: the output
 * projection after attention (or W2 after SwiGLU) followed by the residual
 * add with the adaLN gate, the fusion of residual connections into fewer
 * launches ("FastH3 在八卡 B300 上实现完整 MP4 生成快于播放时长", section
 * "融合 DiT 算子"; "MiniMax H3 FastH3 real-time serving with vLLM-Omni",
 * bullet "Fused DiT operators"). Per token t of request s and feature n:
 *   y[t, n]  = sum_k a[t, k] * w[n, k]         (w: [N, K], out x in features)
 *   x'[t, n] = x[t, n] + gate_res[s, n] * y[t, n]
 * x == NULL: the product alone (x' = y; gate_res and cu unused).
 * a: [T, K] with a_stride elements between tokens; x: [T, N]; gate_res:
 * [B, N] float32. Output float64 rows [nrows, N] for the tokens in rows
 * (all T when rows is NULL).
 */
int oracle_linear_gated_residual(const void* a, int64_t a_stride, const void* w, const void* x, int in_kind,
                                 const float* gate_res, const int32_t* cu, int B, int64_t T, int K, int N,
                                 const int32_t* rows, int64_t nrows, double* out) {
  if (T < 0 || K <= 0 || N <= 0 || a_stride < K) return -1;
  if (x && (gate_res == NULL || check_cu(cu, B, T))) return -1;
  if (rows == NULL) nrows = T;
  int64_t bad = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t t = rows ? rows[r] : r;
    if (t < 0 || t >= T) { ++bad; continue; }
    const int seg = x ? segment_of(cu, B, t) : 0;
    for (int n = 0; n < N; ++n) {
      double y = 0.0;
      for (int k = 0; k < K; ++k) y += load(a, in_kind, t * a_stride + k) * load(w, in_kind, (int64_t)n * K + k);
      out[r * N + n] = x ? load(x, in_kind, t * N + n) + (double)gate_res[(int64_t)seg * N + n] * y : y;
    }
  }
  return bad ? -1 : 0;
}

/*
 * A linear layer whose epilogue is SwiGLU: W1 of the feed-forward with
 * silu(gate) * up applied to its two halves in place of separate SiLU and
 * multiply passes (same passages). The first F rows of w1 give the SiLU
 * operand, the last F rows the linear one. Per token t and feature f:
 *   g = sum_k a[t, k] * w1[f, k]
 *   u = sum_k a[t, k] * w1[F + f, k]
 *   act[t, f] = g / (1 + exp(-g)) * u     (gv, uv below)
 * a: [T, K] with a_stride elements between tokens; w1: [2F, K]. Output
 * float64 rows [nrows, F].
 */
int oracle_linear_swiglu(const void* a, int64_t a_stride, const void* w1, int in_kind, int64_t T, int K, int F,
                         const int32_t* rows, int64_t nrows, double* act) {
  if (T < 0 || K <= 0 || F <= 0 || a_stride < K) return -1;
  if (rows == NULL) nrows = T;
  int64_t bad = 0;
#pragma omp parallel for schedule(static) reduction(+ : bad)
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t t = rows ? rows[r] : r;
    if (t < 0 || t >= T) { ++bad; continue; }
    for (int f = 0; f < F; ++f) {
      double gv = 0.0, uv = 0.0;
      for (int k = 0; k < K; ++k) {
        const double av = load(a, in_kind, t * a_stride + k);
        gv += av * load(w1, in_kind, (int64_t)f * K + k);
        uv += av * load(w1, in_kind, ((int64_t)F + f) * K + k);
      }
      act[r * (int64_t)F + f] = gv / (1.0 + exp(-gv)) * uv;
    }
  }
  return bad ? -1 : 0;
}

/* Sets the number of OpenMP threads later parallel regions use (n >= 1);
 * for timing the oracle on one core beside its all-core figure. */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n >= 1) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

/* Number of OpenMP threads a parallel region of this library uses. */
int oracle_num_threads(void) {
  int n = 1;
#ifdef _OPENMP
#pragma omp parallel
  {
#pragma omp single
    n = omp_get_num_threads();
  }
#endif
  return n;
}
