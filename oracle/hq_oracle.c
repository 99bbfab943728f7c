/*
 * hq_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, single-threaded CPU restatement of the hybrid BF16/Int4 compression of
 * tensor-parallel partial sums described on the page "Revolutionizing LLM Inference: The
 * Power of Efficient Low-Bit Communication" (blog summary of "Towards Efficient Low-Bit
 * Communication for Tensor Parallel LLM Inference"), section "The Hybrid Quantization
 * Algorithm": Calibration -> Selection of High Precision Features -> Inference.
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg may load this
 * library.  It shares no code with the CUDA path: every helper below is written here.
 *
 * The page gives prose only (no formula, no bit layout), so each step follows a stated
 * reading, labelled R1..R14 in comments and listed in the design notes:
 *   R1  moving average = EMA with decay beta: ema = beta*ema + (1-beta)*b, 1-beta in fp32;
 *       the first batch sets ema = b; no bias correction.
 *   R2  each rank keeps its own statistics and parameters.
 *   R3  asymmetric 4-bit grid with zero inside the range: lo = min(ema_min, 0),
 *       hi = max(ema_max, 0), scale = (hi-lo)/15, inv_scale = 1/scale (correctly rounded),
 *       zero = clamp(rint(-lo*inv_scale), 0, 15); a scale that is zero, subnormal,
 *       infinite or NaN is degenerate: scale = inv_scale = 1, zero = 0.
 *   R4  a feature's rank score is the sum over ranks (in rank order, fp32) of its ranges.
 *   R5  top-k by score descending, equal scores -> lower column first (NaN ranks as +inf);
 *       keep_idx and rest_idx are each stored ascending.
 *   R6  q = clamp(rint(x*inv_scale) + zero, 0, 15), round-half-even, the product in fp32;
 *       +-inf saturate; NaN -> q = zero (dequantizes to exactly 0).
 *   R7  wire layout: only the H-k non-kept columns, in rest_idx order, 8 codes per uint32,
 *       code c in bits 4*(c%8)..4*(c%8)+3 of word c/8; k % 8 == 0 and H % 8 == 0.  The kept
 *       features' bf16 bits travel feature-major, side[r][j][t] (kept feature j in keep_idx
 *       order, all rows of one feature contiguous).
 *   R9  dequant-reduce of a non-kept column: acc = +0; for r = 0..P-1:
 *       acc = fma(float(q_r - zero_r), scale_r, acc)  (one rounding per rank).
 *   R10 kept column: acc = +0; for r = 0..P-1: acc = acc + float(side_r).
 *   R11 output: fp32, or bf16 by round-to-nearest-even; a NaN result is written as the
 *       canonical quiet NaN in both types (0x7FC00000 / 0x7FC0).
 *   R12 the fused compress-reduce equals quantize-pack followed by dequant-reduce.
 *   R14 parameters are computed for every column, kept ones included (unused there).
 *   R19 the literal variant of the receiving side (every received tensor made BF16 before the
 *       devices' tensors are combined): each
 *       rank's dequantized value v_r = float(q_r - zero_r) * scale_r (one fp32 product) is
 *       rounded to bf16 (nearest, ties to even) before the rank-ordered fp32 sum:
 *       acc = +0; for r = 0..P-1: acc = acc + bf16(v_r).  Kept columns and the output
 *       rounding are as in R10 and R11.
 *   R20 partial-channel synchronisation: only the block of features [c0, c0 + Hs) goes through
 *       the hybrid wire and the rank-ordered sum; every rank keeps its own partial sum in the
 *       other features.
 * Calibration detail: batch min/max ignore NaN (no comparison with NaN is true); a batch
 * minimum or maximum of -0 is stored as +0 (adding +0.0f), so that results do not depend
 * on which zero a comparison happened to keep.
 *
 * Compile with -ffp-contract=off and without fast-math, so that every float operation
 * written below is one IEEE-754 single-precision operation.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 bits -> float: the bf16 value is the high half of the float. */
static float ref_bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* A NaN result as the canonical quiet NaN 0x7FC00000 (R11); other values unchanged. */
static float ref_canonical(float f) {
  if (!isnan(f)) return f;
  const uint32_t q = 0x7FC00000u;
  float c;
  memcpy(&c, &q, sizeof c);
  return c;
}

/* float -> bf16 bits, round to nearest, ties to even; NaN -> 0x7FC0 (R11). */
static uint16_t ref_bf16_round(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if (isnan(f)) return 0x7FC0u;
  uint32_t keep = u >> 16;
  uint32_t dropped = u & 0xFFFFu;
  if (dropped > 0x8000u || (dropped == 0x8000u && (keep & 1u))) keep += 1u;
  return (uint16_t)keep;
}

/*
 * Calibration (section "The Hybrid Quantization Algorithm", bullet "Calibration"):
 * per rank r and feature h, the min and max of this batch's T rows, folded into the
 * moving averages ema_min/ema_max [P][H] (R1, R2).
 */
void hq_ref_calibrate(const uint16_t* x, int P, int T, int H, float beta, int first_batch,
                      float* ema_min, float* ema_max) {
  const float one_minus_beta = 1.0f - beta;
  for (int r = 0; r < P; ++r) {
    for (int h = 0; h < H; ++h) {
      float bmin = INFINITY, bmax = -INFINITY;
      for (int t = 0; t < T; ++t) {
        float v = ref_bf16_value(x[((size_t)r * T + t) * H + h]);
        if (v < bmin) bmin = v;
        if (v > bmax) bmax = v;
      }
      bmin = bmin + 0.0f; /* -0 -> +0 */
      bmax = bmax + 0.0f;
      size_t i = (size_t)r * H + h;
      if (first_batch) {
        ema_min[i] = bmin;
        ema_max[i] = bmax;
      } else {
        float a = beta * ema_min[i];
        float b = one_minus_beta * bmin;
        ema_min[i] = a + b;
        a = beta * ema_max[i];
        b = one_minus_beta * bmax;
        ema_max[i] = a + b;
      }
    }
  }
}

/*
 * Per-(rank, feature) 4-bit parameters from the calibrated statistics (R3, R14), and the
 * feature's quantization range on each rank, range[r][h] = hi - lo.
 */
void hq_ref_params(const float* ema_min, const float* ema_max, int P, int H, float* scale,
                   float* inv_scale, uint8_t* zero, float* range) {
  for (int r = 0; r < P; ++r) {
    for (int h = 0; h < H; ++h) {
      size_t i = (size_t)r * H + h;
      float lo = (ema_min[i] < 0.0f) ? ema_min[i] : 0.0f;
      float hi = (ema_max[i] > 0.0f) ? ema_max[i] : 0.0f;
      float rg = hi - lo;
      float s = rg / 15.0f;
      range[i] = rg;
      if (!(s >= FLT_MIN) || !(s <= FLT_MAX)) {
        scale[i] = 1.0f;
        inv_scale[i] = 1.0f;
        zero[i] = 0;
        continue;
      }
      float inv = 1.0f / s;
      float zf = rintf((-lo) * inv);
      if (zf < 0.0f) zf = 0.0f;
      if (zf > 15.0f) zf = 15.0f;
      scale[i] = s;
      inv_scale[i] = inv;
      zero[i] = (uint8_t)zf;
    }
  }
}

typedef struct {
  float score;
  int32_t col;
} ref_ranked;

/* Order for "Selection of High Precision Features": larger score first (NaN as +inf),
 * then lower column index (R5). */
static int ref_rank_order(const void* pa, const void* pb) {
  const ref_ranked* a = (const ref_ranked*)pa;
  const ref_ranked* b = (const ref_ranked*)pb;
  float sa = isnan(a->score) ? INFINITY : a->score;
  float sb = isnan(b->score) ? INFINITY : b->score;
  if (sa > sb) return -1;
  if (sa < sb) return 1;
  return (a->col < b->col) ? -1 : (a->col > b->col) ? 1 : 0;
}

static int ref_ascending(const void* pa, const void* pb) {
  int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
  return (a < b) ? -1 : (a > b) ? 1 : 0;
}

/*
 * Selection of High Precision Features: score[h] = sum_r range[r][h] (R4), the k best
 * features by score are kept in BF16 (R5).  Plain full sort.  Writes the score too.
 * Returns 0, or 1 on bad arguments / allocation failure.
 */
int hq_ref_select(const float* range, int P, int H, int k, float* score, int32_t* keep_idx,
                  int32_t* rest_idx) {
  if (k < 0 || k > H) return 1;
  ref_ranked* order = (ref_ranked*)malloc(sizeof(ref_ranked) * (size_t)H);
  unsigned char* kept = (unsigned char*)calloc((size_t)H, 1);
  if (!order || !kept) {
    free(order);
    free(kept);
    return 1;
  }
  for (int h = 0; h < H; ++h) {
    float acc = 0.0f;
    for (int r = 0; r < P; ++r) acc = acc + range[(size_t)r * H + h];
    score[h] = acc;
    order[h].score = acc;
    order[h].col = h;
  }
  qsort(order, (size_t)H, sizeof(ref_ranked), ref_rank_order);
  for (int j = 0; j < k; ++j) {
    keep_idx[j] = order[j].col;
    kept[order[j].col] = 1;
  }
  qsort(keep_idx, (size_t)k, sizeof(int32_t), ref_ascending);
  int c = 0;
  for (int h = 0; h < H; ++h)
    if (!kept[h]) rest_idx[c++] = h;
  free(order);
  free(kept);
  return 0;
}

/* Calibrated statistics -> parameters + selection in one call (the boundary's select step). */
int hq_ref_select_topk(const float* ema_min, const float* ema_max, int P, int H, int k,
                       int32_t* keep_idx, int32_t* rest_idx, float* scale, float* inv_scale,
                       uint8_t* zero, float* score) {
  float* range = (float*)malloc(sizeof(float) * (size_t)P * H);
  if (!range) return 1;
  hq_ref_params(ema_min, ema_max, P, H, scale, inv_scale, zero, range);
  int rc = hq_ref_select(range, P, H, k, score, keep_idx, rest_idx);
  free(range);
  return rc;
}

/* One 4-bit code (R6). */
static unsigned ref_quantize(float v, float inv_scale, unsigned zero) {
  float a = v * inv_scale;
  if (isnan(a)) return zero;
  float n = rintf(a); /* round half to even (default rounding mode) */
  if (n <= -(float)zero) return 0u;
  if (n >= 15.0f - (float)zero) return 15u;
  return (unsigned)((int)n + (int)zero);
}

/*
 * Inference, sending side: the kept features' bf16 bits go to side[r][j][t] in keep_idx
 * order; every other feature is quantized to 4 bits and packed in rest_idx order into
 * codes[r][t][(H-k)/8] (R6, R7).
 */
void hq_ref_quantize_pack(const uint16_t* x, int P, int T, int H, int k, const int32_t* keep_idx,
                          const int32_t* rest_idx, const float* inv_scale, const uint8_t* zero,
                          uint32_t* codes, uint16_t* side) {
  const int Hr = H - k, W = Hr / 8;
  for (int r = 0; r < P; ++r) {
    for (int t = 0; t < T; ++t) {
      const uint16_t* row = x + ((size_t)r * T + t) * H;
      uint32_t* crow = codes + ((size_t)r * T + t) * W;
      for (int j = 0; j < k; ++j) side[((size_t)r * k + j) * T + t] = row[keep_idx[j]];
      for (int w = 0; w < W; ++w) crow[w] = 0u;
      for (int c = 0; c < Hr; ++c) {
        int h = rest_idx[c];
        size_t p = (size_t)r * H + h;
        unsigned q = ref_quantize(ref_bf16_value(row[h]), inv_scale[p], zero[p]);
        crow[c / 8] |= (uint32_t)q << (4 * (c % 8));
      }
    }
  }
}

/*
 * Inference, receiving side (section "The Hybrid Quantization Algorithm", bullet "Inference"):
 * every rank's shard is converted back and the ranks are summed in rank order; out is [T][H],
 * fp32 (out_f32 != 0) or bf16 bits (R11).  shard_bf16 == 0: a non-kept value enters the sum
 * through one fused multiply-add per rank (R9).  shard_bf16 != 0: the literal reading, each
 * rank's dequantized value is first rounded to bf16 (R19).  Kept columns: R10 in both.
 */
static void ref_dequant_reduce(const uint32_t* codes, const uint16_t* side, int P, int T, int H, int k,
                               const int32_t* keep_idx, const int32_t* rest_idx, const float* scale,
                               const uint8_t* zero, void* out, int out_f32, int shard_bf16) {
  const int Hr = H - k, W = Hr / 8;
  for (int t = 0; t < T; ++t) {
    for (int j = 0; j < k; ++j) {
      float acc = 0.0f;
      for (int r = 0; r < P; ++r) acc = acc + ref_bf16_value(side[((size_t)r * k + j) * T + t]);
      size_t o = (size_t)t * H + keep_idx[j];
      if (out_f32) ((float*)out)[o] = ref_canonical(acc);
      else ((uint16_t*)out)[o] = ref_bf16_round(acc);
    }
    for (int c = 0; c < Hr; ++c) {
      int h = rest_idx[c];
      float acc = 0.0f;
      for (int r = 0; r < P; ++r) {
        uint32_t word = codes[((size_t)r * T + t) * W + c / 8];
        int q = (int)((word >> (4 * (c % 8))) & 0xFu);
        size_t p = (size_t)r * H + h;
        if (shard_bf16) {
          float v = (float)(q - (int)zero[p]) * scale[p];
          acc = acc + ref_bf16_value(ref_bf16_round(v));
        } else {
          acc = fmaf((float)(q - (int)zero[p]), scale[p], acc);
        }
      }
      size_t o = (size_t)t * H + h;
      if (out_f32) ((float*)out)[o] = ref_canonical(acc);
      else ((uint16_t*)out)[o] = ref_bf16_round(acc);
    }
  }
}

void hq_ref_dequant_reduce(const uint32_t* codes, const uint16_t* side, int P, int T, int H, int k,
                           const int32_t* keep_idx, const int32_t* rest_idx, const float* scale,
                           const uint8_t* zero, void* out, int out_f32) {
  ref_dequant_reduce(codes, side, P, T, H, k, keep_idx, rest_idx, scale, zero, out, out_f32, 0);
}

void hq_ref_dequant_reduce_bf16_shards(const uint32_t* codes, const uint16_t* side, int P, int T, int H,
                                       int k, const int32_t* keep_idx, const int32_t* rest_idx,
                                       const float* scale, const uint8_t* zero, void* out, int out_f32) {
  ref_dequant_reduce(codes, side, P, T, H, k, keep_idx, rest_idx, scale, zero, out, out_f32, 1);
}

/* The fused call: quantize-pack then dequant-reduce, literally (R12).  codes/side may be
 * NULL, in which case temporary buffers are used.  Returns 0, or 1 on allocation failure. */
int hq_ref_compress_reduce(const uint16_t* x, int P, int T, int H, int k, const int32_t* keep_idx,
                           const int32_t* rest_idx, const float* scale, const float* inv_scale,
                           const uint8_t* zero, void* out, int out_f32, uint32_t* codes,
                           uint16_t* side) {
  uint32_t* c = codes;
  uint16_t* s = side;
  if (!c) c = (uint32_t*)malloc(sizeof(uint32_t) * ((size_t)P * T * (H - k) / 8 + 1));
  if (!s) s = (uint16_t*)malloc(sizeof(uint16_t) * ((size_t)P * T * k + 1));
  int rc = 0;
  if (!c || !s) {
    rc = 1;
  } else {
    hq_ref_quantize_pack(x, P, T, H, k, keep_idx, rest_idx, inv_scale, zero, c, s);
    hq_ref_dequant_reduce(c, s, P, T, H, k, keep_idx, rest_idx, scale, zero, out, out_f32);
  }
  if (c != codes) free(c);
  if (s != side) free(s);
  return rc;
}

/*
 * Partial-channel synchronisation (the abstract of "Communication-Aware Architecture for
 * Tensor-parallelism" (CAAT-Net) on the first page: tensor-parallel ranks can do without
 * synchronising every activation channel), with the synchronised channels sent through the hybrid
 * wire.  Reading R20: the synchronised features are the block [c0, c0 + Hs) of consecutive
 * features; the block alone is quantize-packed (R6, R7) and reduced (R9-R11, bf16 output), and
 * every rank keeps its own partial sum in the other features:
 *   y[r][t][h] = reduced block value at h - c0   for c0 <= h < c0 + Hs
 *   y[r][t][h] = x[r][t][h]                      otherwise
 * keep_idx / rest_idx index the block (0 .. Hs-1); scale, inv_scale, zero are [P][Hs].
 * Returns 0, or 1 on bad arguments / allocation failure.
 */
int hq_ref_partial_sync(const uint16_t* x, int P, int T, int H, int c0, int Hs, int k, const int32_t* keep_idx,
                        const int32_t* rest_idx, const float* scale, const float* inv_scale, const uint8_t* zero,
                        uint16_t* y) {
  if (c0 < 0 || Hs < 0 || c0 + Hs > H || k < 0 || k > Hs) return 1;
  const size_t rows = (size_t)P * T;
  for (size_t i = 0; i < rows * (size_t)H; ++i) y[i] = x[i];
  if (Hs == 0 || T == 0) return 0;
  uint16_t* xb = (uint16_t*)malloc(sizeof(uint16_t) * rows * (size_t)Hs);
  uint32_t* codes = (uint32_t*)malloc(sizeof(uint32_t) * (rows * (size_t)(Hs - k) / 8 + 1));
  uint16_t* side = (uint16_t*)malloc(sizeof(uint16_t) * (rows * (size_t)k + 1));
  uint16_t* red = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)T * Hs);
  int rc = 0;
  if (!xb || !codes || !side || !red) {
    rc = 1;
  } else {
    for (size_t i = 0; i < rows; ++i)
      for (int h = 0; h < Hs; ++h) xb[i * Hs + h] = x[i * H + c0 + h];
    hq_ref_quantize_pack(xb, P, T, Hs, k, keep_idx, rest_idx, inv_scale, zero, codes, side);
    hq_ref_dequant_reduce(codes, side, P, T, Hs, k, keep_idx, rest_idx, scale, zero, red, 0);
    for (int r = 0; r < P; ++r)
      for (int t = 0; t < T; ++t)
        for (int h = 0; h < Hs; ++h) y[((size_t)r * T + t) * H + c0 + h] = red[(size_t)t * Hs + h];
  }
  free(xb);
  free(codes);
  free(side);
  free(red);
  return rc;
}

/* Exposed for the pins: the oracle's own bf16 rounding and 4-bit quantizer. */
uint16_t hq_ref_bf16_round(float f) { return ref_bf16_round(f); }
unsigned hq_ref_quantize_one(float v, float inv_scale, unsigned zero) {
  return ref_quantize(v, inv_scale, zero);
}
