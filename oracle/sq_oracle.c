/*
 * sq_oracle.c -- CPU oracle for the quantized gated delta-rule decode step.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the bench's CPU-baseline leg load
 * or call this file. The product (the CUDA library, its header and its Python binding) shares
 * no code, table or constant generator with it, and never calls it.
 *
 * It is deliberately plain: loops in natural index order, no SIMD, no blocking, no fusion.
 * Floating point follows one rule, written out here once:
 *   - the state itself is FP32 (the STEPQuant explainer's experimental-setup paragraph uses
 *     the FP32 state as the baseline); every decision that turns a float into an integer
 *     (a scale, a code, an outlier choice) is taken in fp32, as the GPU takes it;
 *   - the recurrence between two quantized states (gate, delta correction, output) is
 *     evaluated in fp64 from the fp32 dequantized state, and its result is rounded once to
 *     fp32 before it is requantized. Outputs o are returned in fp64.
 * Compile with -ffp-contract=off (no fused multiply-adds) and without -ffast-math.
 *
 * Sources (the pages give prose only, no formulas; where they leave a step open, the reading
 * taken is stated at the function):
 *   [SQ-E] STEPQuant explainer (blog.ontle.kr/blog/302)
 *   [SQ-N] STEPQuant news, "STEPQuant、推論メモリを最大68.7%削減" (news.affectosphere.group),
 *          section 研究の概要
 *   [LQ-N] LeapQuant news, "LeapQuant、線形注意の推論を1.47倍高速化" (news.affectosphere.group),
 *          section 研究の概要
 *
 * Parity pins (tests/test_oracle_pins.py) cover every exported function: closed forms of the
 * delta rule, Proposition 1, quantize/dequantize idempotence, the half-step error bound, the
 * textbook special cases, brute force on 4x4 tiles, and a format-size check against the
 * compression ratios [SQ-E] prints. The row-impact weighting of orc_fit (omega != NULL),
 * whose formula the pages do not print, is pinned by its stated purpose (a lower
 * impact-weighted reconstruction error than the plain fit on seeded heads) and its special
 * cases (a hand-worked 2 x 2 example, equal impacts giving the plain fit, codes within [-Q, Q]
 * and the half-step bound, monotone first alternation).
 */
#include "sq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORC_SCALE_FLOOR 0x1p-14f /* smallest normal fp16: scales never go below it */

/* ------------------------------------------------------------------------------------------
 * fp16 helpers. fp16 is the pivot and scale format of [SQ-E] (paragraph on lifetime-aware
 * bit allocation: high-risk units stay in FP16). Conversion is IEEE round-to-nearest-even,
 * done by the compiler's _Float16 type.
 * ---------------------------------------------------------------------------------------- */
uint16_t orc_f32_to_f16_bits(float x) {
  _Float16 h = (_Float16)x;
  uint16_t b;
  memcpy(&b, &h, 2);
  return b;
}

float orc_f16_bits_to_f32(uint16_t b) {
  _Float16 h;
  memcpy(&h, &b, 2);
  return (float)h;
}

static uint16_t rd16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }
static void wr16(uint8_t* p, uint16_t v) {
  p[0] = (uint8_t)(v & 0xff);
  p[1] = (uint8_t)(v >> 8);
}

/* ------------------------------------------------------------------------------------------
 * Format. [SQ-E] ("limitations" paragraph) says the compressed values are packed densely in
 * memory, and (efficiency paragraph) that the compression ratio follows from the storage
 * format; it does not print the format. Reading taken:
 *   - unit widths b in {2,4,6,8}; 16 marks an FP16 pivot unit. A unit is a whole head or one
 *     key row ([SQ-E], lifetime-aware bit allocation paragraph);
 *   - symmetric codes in [-Q, Q], Q = 2^(b-1) - 1, stored offset-binary u = code + 2^(b-1);
 *   - a row is a little-endian bit stream: element j occupies bits [j*b, (j+1)*b);
 *     a pivot row is the same stream with b = 16 holding fp16 bit patterns;
 *   - quantized head block: r16[d_k] | c16[d_v] | row 0 .. row d_k-1 | outliers, where the
 *     outliers (windowed variant only) are n_outliers pairs (u16 flat index, fp16 value);
 *   - pivot head block (head unit only): the d_k x d_v fp16 matrix, row-major;
 *   - every head block is padded to a multiple of 16 bytes; a slot is the heads in order.
 * ---------------------------------------------------------------------------------------- */
static int width_of(const orc_layout* L, const uint8_t* bits, int h, int i) {
  return L->unit == ORC_UNIT_HEAD ? bits[h] : bits[(size_t)h * L->d_k + i];
}

static int head_is_pivot(const orc_layout* L, const uint8_t* bits, int h) {
  return L->unit == ORC_UNIT_HEAD && bits[h] == 16;
}

static int width_ok(int b) { return b == 2 || b == 4 || b == 6 || b == 8 || b == 16; }

int orc_validate(const orc_layout* L, const uint8_t* bits) {
  if (!L || !bits) return ORC_ERR_ARG;
  if (L->n_heads < 1 || L->d_k < 1 || L->d_v < 1) return ORC_ERR_ARG;
  if (L->d_k * L->d_v > 65536) return ORC_ERR_ARG; /* outlier index is a u16 */
  if (L->unit != ORC_UNIT_HEAD && L->unit != ORC_UNIT_ROW) return ORC_ERR_ARG;
  if (L->gate != ORC_GATE_SCALAR && L->gate != ORC_GATE_DIAG) return ORC_ERR_ARG;
  if (L->fit_iters < 1 || L->window < 1 || L->n_outliers < 0) return ORC_ERR_ARG;
  int n_units = L->unit == ORC_UNIT_HEAD ? L->n_heads : L->n_heads * L->d_k;
  for (int u = 0; u < n_units; ++u)
    if (!width_ok(bits[u])) return ORC_ERR_ARG;
  for (int h = 0; h < L->n_heads; ++h) {
    if (head_is_pivot(L, bits, h)) continue;
    int eligible = 0;
    for (int i = 0; i < L->d_k; ++i)
      if (width_of(L, bits, h, i) != 16) eligible += L->d_v;
    if (L->n_outliers > eligible) return ORC_ERR_ARG;
  }
  return ORC_OK;
}

size_t orc_row_bytes(int b, int d_v) { return ((size_t)d_v * (size_t)b + 7) / 8; }

size_t orc_head_bytes(const orc_layout* L, const uint8_t* bits, int h) {
  size_t n;
  if (head_is_pivot(L, bits, h)) {
    n = 2u * (size_t)L->d_k * (size_t)L->d_v;
  } else {
    n = 2u * (size_t)(L->d_k + L->d_v);
    for (int i = 0; i < L->d_k; ++i) n += orc_row_bytes(width_of(L, bits, h, i), L->d_v);
    n += 4u * (size_t)L->n_outliers;
  }
  return (n + 15) / 16 * 16;
}

int orc_slot_layout(const orc_layout* L, const uint8_t* bits, size_t* head_off,
                    size_t* slot_bytes) {
  int st = orc_validate(L, bits);
  if (st) return st;
  size_t off = 0;
  for (int h = 0; h < L->n_heads; ++h) {
    if (head_off) head_off[h] = off;
    off += orc_head_bytes(L, bits, h);
  }
  if (slot_bytes) *slot_bytes = off;
  return ORC_OK;
}

/* Write the b low bits of each u[j] at bit offset j*b of a zeroed little-endian stream. */
void orc_pack_row(int b, int n, const int32_t* u, uint8_t* out) {
  memset(out, 0, orc_row_bytes(b, n));
  for (int j = 0; j < n; ++j)
    for (int t = 0; t < b; ++t)
      if ((u[j] >> t) & 1) {
        size_t bit = (size_t)j * b + t;
        out[bit >> 3] |= (uint8_t)(1u << (bit & 7));
      }
}

void orc_unpack_row(int b, int n, const uint8_t* in, int32_t* u) {
  for (int j = 0; j < n; ++j) {
    int32_t v = 0;
    for (int t = 0; t < b; ++t) {
      size_t bit = (size_t)j * b + t;
      v |= (int32_t)((in[bit >> 3] >> (bit & 7)) & 1) << t;
    }
    u[j] = v;
  }
}

/* ------------------------------------------------------------------------------------------
 * Dual-axis scale fit. [SQ-E], "Key-Row-Aware Dual-Axis Fitting" paragraph: outliers sit on
 * rows and columns at once, so key rows and value columns each get their own scale;
 * [SQ-N] 研究の概要: the key-row and value-column scales are optimized together; [SQ-E]
 * experimental-setup paragraph: the two scales are recomputed at every decode step on the
 * updated state. The impact-weighted form is not printed; the plain form taken is an
 * alternating max-abs fit, all in fp32 with correctly rounded operations:
 *   c_j = 1 (cold start); repeat fit_iters times:
 *     r_i = max( max_j fl(|S_ij| * fl(1/c_j)) / Q_i , 2^-14 )
 *     w_i = fl(1 / fl(r_i * Q_i));  c_j = max( max_i fl(|S_ij| * w_i) , 2^-14 )
 * Rows with qmax[i] == 0 (fp16 pivot rows) and elements with excluded[] set (outliers) take
 * no part. The caller rounds r and c to fp16 once, at the end.
 *
 * Impact weighting (omega != NULL; the pages print no formula). [SQ-E] experimental-setup
 * paragraph: the row scale weighs the row's current size together with its impact score, and
 * the column scale penalizes reconstruction error more in high-impact rows (wide range for
 * large rows, finer resolution for important rows). Reading taken: every row pass stays as
 * above (each row's scale follows its own size), and the column pass counts row i with a
 * weight omega_i in (0, 1], w_i = fl(omega_i * fl(1 / fl(r_i * Q_i))) (omega_i = 1: the plain
 * w_i), so the column scales follow the high-impact rows; after the last alternation every
 * row with omega_i < 1 is fit once more against the final column scales,
 *     r_i = max( r_i , fl( max_j fl(|S_ij| * fl(1/c_j)) / Q_i ) ),
 * so no element of it leaves [-Q, Q]. The weights come from orc_impact_weights. omega = 1
 * everywhere is the plain fit bit for bit.
 * ---------------------------------------------------------------------------------------- */
int orc_fit(int d_k, int d_v, int fit_iters, const float* S, const int32_t* qmax,
            const uint8_t* excluded, const float* omega, float* r, float* c) {
  float* inv_c = (float*)malloc(sizeof(float) * (size_t)d_v);
  float* w = (float*)malloc(sizeof(float) * (size_t)d_k);
  if (!inv_c || !w) {
    free(inv_c);
    free(w);
    return ORC_ERR_ARG;
  }
  for (int j = 0; j < d_v; ++j) {
    c[j] = 1.0f;
    inv_c[j] = 1.0f;
  }
  for (int it = 0; it < fit_iters; ++it) {
    for (int i = 0; i < d_k; ++i) { /* row pass */
      if (qmax[i] == 0) {
        r[i] = 0.0f;
        continue;
      }
      float m = 0.0f;
      for (int j = 0; j < d_v; ++j) {
        if (excluded && excluded[(size_t)i * d_v + j]) continue;
        float a = fabsf(S[(size_t)i * d_v + j]) * inv_c[j];
        if (a > m) m = a;
      }
      float ri = m / (float)qmax[i];
      r[i] = ri > ORC_SCALE_FLOOR ? ri : ORC_SCALE_FLOOR;
    }
    for (int i = 0; i < d_k; ++i) {
      w[i] = qmax[i] ? 1.0f / (r[i] * (float)qmax[i]) : 0.0f;
      if (omega && omega[i] < 1.0f) w[i] = omega[i] * w[i];
    }
    for (int j = 0; j < d_v; ++j) { /* column pass */
      float m = 0.0f;
      for (int i = 0; i < d_k; ++i) {
        if (qmax[i] == 0) continue;
        if (excluded && excluded[(size_t)i * d_v + j]) continue;
        float a = fabsf(S[(size_t)i * d_v + j]) * w[i];
        if (a > m) m = a;
      }
      c[j] = m > ORC_SCALE_FLOOR ? m : ORC_SCALE_FLOOR;
      inv_c[j] = 1.0f / c[j];
    }
  }
  if (omega) { /* rows counted with omega < 1: fit once more against the final column scales */
    for (int i = 0; i < d_k; ++i) {
      if (qmax[i] == 0 || !(omega[i] < 1.0f)) continue;
      float m = 0.0f;
      for (int j = 0; j < d_v; ++j) {
        if (excluded && excluded[(size_t)i * d_v + j]) continue;
        float a = fabsf(S[(size_t)i * d_v + j]) * inv_c[j];
        if (a > m) m = a;
      }
      float ri = m / (float)qmax[i];
      if (ri > r[i]) r[i] = ri;
    }
  }
  free(inv_c);
  free(w);
  return ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * Column-pass weights of the impact-weighted fit (reading of [SQ-E] experimental-setup
 * paragraph; see orc_fit). A quantization step of r_i c_j costs row i an error that grows with
 * (r_i c_j)^2, weighted by its impact. Lowering a column scale c_j refines that column in every
 * row, but the row that sets it (its "anchor") must widen its own scale r_i by the same factor
 * f to keep its codes in range. With d_v columns of similar scale, the gain is about
 * (1 - 1/f^2) times the head's mean weighted row error and the cost f^2 - 1 times the anchor's,
 * so the lowering pays while f^2 < mean impact / impact_i. The column pass therefore counts
 * row i with weight 1 / f = min(1, sqrt(impact_i / mean impact of its head)), in fp64, rounded
 * to fp32 once. impact: [n_heads][d_k], every entry > 0 and finite. Equal impacts give 1.
 * ---------------------------------------------------------------------------------------- */
int orc_impact_weights(int n_heads, int d_k, const float* impact, float* omega) {
  for (int h = 0; h < n_heads; ++h) {
    const float* im = impact + (size_t)h * d_k;
    double sum = 0.0;
    for (int i = 0; i < d_k; ++i) {
      if (!(im[i] > 0.0f) || !isfinite(im[i])) return ORC_ERR_ARG;
      sum += (double)im[i];
    }
    const double mean = sum / (double)d_k;
    for (int i = 0; i < d_k; ++i) {
      double x = sqrt((double)im[i] / mean);
      omega[(size_t)h * d_k + i] = (float)(x < 1.0 ? x : 1.0);
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------------------------
 * Compensation entries. [LQ-N] 研究の概要: large outliers of the state are kept as a few
 * high-precision elements and ride the same update path as everything else. Reading taken:
 * at each requantization the n entries of largest |S| (fp32) among the quantized rows are
 * kept in fp16; ties go to the lower flat index i*d_v + j. Returned in ascending index order.
 * ---------------------------------------------------------------------------------------- */
int orc_select_outliers(int d_k, int d_v, const float* S, const int32_t* qmax, int n,
                        int32_t* idx_out) {
  size_t total = (size_t)d_k * d_v;
  uint8_t* taken = (uint8_t*)calloc(total, 1);
  if (!taken) return ORC_ERR_ARG;
  for (int t = 0; t < n; ++t) { /* n passes of a plain arg-max: slow and obviously right */
    long best = -1;
    float best_a = -1.0f;
    for (size_t e = 0; e < total; ++e) {
      if (taken[e] || qmax[e / d_v] == 0) continue;
      float a = fabsf(S[e]);
      if (a > best_a) { /* strict: an equal later element never displaces an earlier one */
        best_a = a;
        best = (long)e;
      }
    }
    if (best < 0) {
      free(taken);
      return ORC_ERR_ARG;
    }
    taken[best] = 1;
  }
  int k = 0;
  for (size_t e = 0; e < total; ++e)
    if (taken[e]) idx_out[k++] = (int32_t)e;
  free(taken);
  return ORC_OK;
}

static int all_finite_f(const float* x, size_t n) {
  for (size_t e = 0; e < n; ++e)
    if (!isfinite(x[e])) return 0;
  return 1;
}

/* ------------------------------------------------------------------------------------------
 * Quantize one head's fp32 state into its block. [SQ-E]: codes per unit width (lifetime-
 * aware allocation paragraph), fp16 pivots (same paragraph), dual-axis scales (fitting
 * paragraph). Quantization arithmetic, all fp32 except the last product:
 *   ir_i = fl(1/r16_i), ic_j = fl(1/c16_j), x1 = fl(S_ij * ir_i),
 *   code = clamp(nearest-even integer to (x1 * ic_j) taken exactly, -Q_i, Q_i).
 * Pivot units and outliers are stored as fp16 (round to nearest even); outlier positions
 * carry code 0. Returns ORC_ERR_RANGE if a scale or an fp16 value overflows fp16.
 * ---------------------------------------------------------------------------------------- */
int orc_quantize_head(const orc_layout* L, const uint8_t* bits, int h, const float* S,
                      uint8_t* block) {
  const int dk = L->d_k, dv = L->d_v;
  const size_t total = (size_t)dk * dv;
  if (!all_finite_f(S, total)) return ORC_ERR_NONFINITE;
  memset(block, 0, orc_head_bytes(L, bits, h));
  int32_t* u = (int32_t*)malloc(sizeof(int32_t) * (size_t)dv);
  if (!u) return ORC_ERR_ARG;
  int st = ORC_OK;

  if (head_is_pivot(L, bits, h)) {
    for (int i = 0; i < dk && st == ORC_OK; ++i) {
      for (int j = 0; j < dv; ++j) {
        uint16_t hb = orc_f32_to_f16_bits(S[(size_t)i * dv + j]);
        if ((hb & 0x7c00) == 0x7c00) st = ORC_ERR_RANGE;
        u[j] = hb;
      }
      orc_pack_row(16, dv, u, block + (size_t)i * orc_row_bytes(16, dv));
    }
    free(u);
    return st;
  }

  int32_t* qmax = (int32_t*)malloc(sizeof(int32_t) * (size_t)dk);
  float* r = (float*)malloc(sizeof(float) * (size_t)dk);
  float* c = (float*)malloc(sizeof(float) * (size_t)dv);
  uint8_t* excl = (uint8_t*)calloc(total, 1);
  int32_t* oidx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(L->n_outliers + 1));
  if (!qmax || !r || !c || !excl || !oidx) {
    st = ORC_ERR_ARG;
    goto done;
  }
  for (int i = 0; i < dk; ++i) {
    int b = width_of(L, bits, h, i);
    qmax[i] = b == 16 ? 0 : (1 << (b - 1)) - 1;
  }
  if (L->n_outliers > 0) {
    st = orc_select_outliers(dk, dv, S, qmax, L->n_outliers, oidx);
    if (st) goto done;
    for (int t = 0; t < L->n_outliers; ++t) excl[oidx[t]] = 1;
  }
  orc_fit(dk, dv, L->fit_iters, S, qmax, excl, L->omega ? L->omega + (size_t)h * dk : NULL, r, c);

  uint8_t* r16p = block;
  uint8_t* c16p = block + 2 * (size_t)dk;
  float* c16f = c; /* reuse: c16 as float from here on */
  for (int j = 0; j < dv; ++j) {
    uint16_t hb = orc_f32_to_f16_bits(c[j]);
    if ((hb & 0x7c00) == 0x7c00) st = ORC_ERR_RANGE;
    wr16(c16p + 2 * (size_t)j, hb);
    c16f[j] = orc_f16_bits_to_f32(hb);
  }
  uint8_t* row = block + 2 * (size_t)(dk + dv);
  for (int i = 0; i < dk; ++i) {
    int b = width_of(L, bits, h, i);
    if (b == 16) { /* pivot row: fp16 values, row scale unused (stored as 0) */
      wr16(r16p + 2 * (size_t)i, 0);
      for (int j = 0; j < dv; ++j) {
        uint16_t hb = orc_f32_to_f16_bits(S[(size_t)i * dv + j]);
        if ((hb & 0x7c00) == 0x7c00) st = ORC_ERR_RANGE;
        u[j] = hb;
      }
    } else {
      uint16_t rb = orc_f32_to_f16_bits(r[i]);
      if ((rb & 0x7c00) == 0x7c00) st = ORC_ERR_RANGE;
      wr16(r16p + 2 * (size_t)i, rb);
      const float ir = 1.0f / orc_f16_bits_to_f32(rb);
      const int Q = qmax[i];
      for (int j = 0; j < dv; ++j) {
        int32_t code = 0;
        if (!excl[(size_t)i * dv + j]) {
          const float ic = 1.0f / c16f[j];
          const float x1 = S[(size_t)i * dv + j] * ir;
          double x = (double)x1 * (double)ic; /* exact: two 24-bit significands */
          if (x > Q) x = Q;
          if (x < -Q) x = -Q;
          code = (int32_t)nearbyint(x); /* default rounding mode: nearest, ties to even */
        }
        u[j] = code + (1 << (b - 1));
      }
    }
    orc_pack_row(b, dv, u, row);
    row += orc_row_bytes(b, dv);
  }
  for (int t = 0; t < L->n_outliers; ++t) {
    uint16_t hb = orc_f32_to_f16_bits(S[oidx[t]]);
    if ((hb & 0x7c00) == 0x7c00) st = ORC_ERR_RANGE;
    wr16(row + 4 * (size_t)t, (uint16_t)oidx[t]);
    wr16(row + 4 * (size_t)t + 2, hb);
  }
done:
  free(u);
  free(qmax);
  free(r);
  free(c);
  free(excl);
  free(oidx);
  return st;
}

/* ------------------------------------------------------------------------------------------
 * Dequantize one head's block to fp32: S_ij = fl32(code_ij * r16_i * c16_j) (the exact
 * product rounded once), pivots and outliers as their fp16 values.
 * ---------------------------------------------------------------------------------------- */
int orc_dequantize_head(const orc_layout* L, const uint8_t* bits, int h, const uint8_t* block,
                        float* S) {
  const int dk = L->d_k, dv = L->d_v;
  int32_t* u = (int32_t*)malloc(sizeof(int32_t) * (size_t)dv);
  if (!u) return ORC_ERR_ARG;
  if (head_is_pivot(L, bits, h)) {
    for (int i = 0; i < dk; ++i) {
      orc_unpack_row(16, dv, block + (size_t)i * orc_row_bytes(16, dv), u);
      for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] = orc_f16_bits_to_f32((uint16_t)u[j]);
    }
    free(u);
    return ORC_OK;
  }
  const uint8_t* r16p = block;
  const uint8_t* c16p = block + 2 * (size_t)dk;
  const uint8_t* row = block + 2 * (size_t)(dk + dv);
  for (int i = 0; i < dk; ++i) {
    int b = width_of(L, bits, h, i);
    orc_unpack_row(b, dv, row, u);
    row += orc_row_bytes(b, dv);
    if (b == 16) {
      for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] = orc_f16_bits_to_f32((uint16_t)u[j]);
      continue;
    }
    const double ri = orc_f16_bits_to_f32(rd16(r16p + 2 * (size_t)i));
    for (int j = 0; j < dv; ++j) {
      const double cj = orc_f16_bits_to_f32(rd16(c16p + 2 * (size_t)j));
      const int32_t code = u[j] - (1 << (b - 1));
      S[(size_t)i * dv + j] = (float)((double)code * ri * cj);
    }
  }
  int st = ORC_OK;
  for (int t = 0; t < L->n_outliers; ++t) {
    const uint32_t idx = rd16(row + 4 * (size_t)t);
    if (idx >= (uint32_t)(dk * dv) || width_of(L, bits, h, (int)(idx / dv)) == 16) {
      st = ORC_ERR_ARG;
      continue;
    }
    S[idx] = orc_f16_bits_to_f32(rd16(row + 4 * (size_t)t + 2));
  }
  free(u);
  return st;
}

/* ------------------------------------------------------------------------------------------
 * The gated delta rule, one token, in fp64. [SQ-E], paragraph introducing linear attention:
 * a fixed-size recurrent state that is partly erased and overwritten at every step (the gated
 * Delta rule; GDN with a per-head gate, KDA with a per-key-channel gate); [LQ-N] 研究の概要
 * names the same two forms. The state is M[i][j] with i the key channel (row) and j the
 * value channel (column). Reading taken for the order of operations:
 *   S' = D M             (D = alpha I for the scalar gate, diag(alpha_i) for the diagonal one)
 *   u  = S'^T k          b = beta (v - u)          M <- S' + k b^T
 *   o  = M^T q           (the updated state, before any requantization; no 1/sqrt(d) factor)
 * which is M <- (I - beta k k^T) D M + beta k v^T.
 * ---------------------------------------------------------------------------------------- */
void orc_delta_update(int d_k, int d_v, int gate, double* M, const double* q, const double* k,
                      const double* v, const double* alpha, double beta, double* o) {
  for (int i = 0; i < d_k; ++i) {
    const double a = gate == ORC_GATE_SCALAR ? alpha[0] : alpha[i];
    for (int j = 0; j < d_v; ++j) M[(size_t)i * d_v + j] *= a;
  }
  for (int j = 0; j < d_v; ++j) {
    double u = 0.0;
    for (int i = 0; i < d_k; ++i) u += M[(size_t)i * d_v + j] * k[i];
    const double b = beta * (v[j] - u);
    for (int i = 0; i < d_k; ++i) M[(size_t)i * d_v + j] += k[i] * b;
  }
  for (int j = 0; j < d_v; ++j) {
    double acc = 0.0;
    for (int i = 0; i < d_k; ++i) acc += M[(size_t)i * d_v + j] * q[i];
    o[j] = acc;
  }
}

/* ------------------------------------------------------------------------------------------
 * Batched entry points over a pool of slots. [SQ-E], paragraph on the state pool: one state
 * per concurrent request, held in a pool with spare slots; slot_idx[b] names request b's slot.
 * Input layouts: q, k, v [batch][H][d] (float, upcast by the caller from the I/O dtype);
 * alpha [batch][H] (scalar gate) or [batch][H][d_k] (diagonal gate); beta [batch][H];
 * o [batch][H][d_v] (double); s_new [batch][H][d_k][d_v] (float, optional).
 * ---------------------------------------------------------------------------------------- */
static void load_vec(double* dst, const float* src, int n) {
  for (int e = 0; e < n; ++e) dst[e] = (double)src[e];
}

/* One request-head of the per-step path: [SQ-E] experimental-setup paragraph (unpack, update,
 * write out at every decode step, scales refit on the updated state) and the paragraph on
 * per-step requantization (the state is requantized after every update). */
static int decode_one(const orc_layout* L, const uint8_t* bits, int h, uint8_t* block,
                      const float* q, const float* k, const float* v, const float* alpha,
                      float beta, double* o, float* s_new) {
  const int dk = L->d_k, dv = L->d_v;
  const size_t total = (size_t)dk * dv;
  float* S = (float*)malloc(sizeof(float) * total);
  double* M = (double*)malloc(sizeof(double) * total);
  double* vec = (double*)malloc(sizeof(double) * (size_t)(3 * (dk > dv ? dk : dv) + dk));
  int st = ORC_ERR_ARG;
  if (!S || !M || !vec) goto out;
  st = orc_dequantize_head(L, bits, h, block, S);
  if (st) goto out;
  for (size_t e = 0; e < total; ++e) M[e] = (double)S[e];
  const int n = dk > dv ? dk : dv;
  double *dq = vec, *dkk = vec + n, *dvv = vec + 2 * n, *da = vec + 3 * n;
  load_vec(dq, q, dk);
  load_vec(dkk, k, dk);
  load_vec(dvv, v, dv);
  load_vec(da, alpha, L->gate == ORC_GATE_SCALAR ? 1 : dk);
  orc_delta_update(dk, dv, L->gate, M, dq, dkk, dvv, da, (double)beta, o);
  for (size_t e = 0; e < total; ++e) S[e] = (float)M[e];
  if (s_new) memcpy(s_new, S, sizeof(float) * total);
  st = orc_quantize_head(L, bits, h, S, block);
out:
  free(S);
  free(M);
  free(vec);
  return st;
}

static int slot_ok(int32_t s) { return s >= 0; }

int orc_quantize(const orc_layout* L, const uint8_t* bits, uint8_t* pool, const int32_t* slot_idx,
                 int n, const float* S, int n_threads) {
  size_t slot_bytes;
  size_t* off = (size_t*)malloc(sizeof(size_t) * (size_t)L->n_heads);
  if (!off) return ORC_ERR_ARG;
  int st = orc_slot_layout(L, bits, off, &slot_bytes);
  if (st) {
    free(off);
    return st;
  }
  const int H = L->n_heads;
  const size_t hs = (size_t)L->d_k * L->d_v;
  int err = 0;
#pragma omp parallel for num_threads(n_threads > 0 ? n_threads : 1) schedule(dynamic, 1) reduction(max : err)
  for (long it = 0; it < (long)n * H; ++it) {
    const int b = (int)(it / H), h = (int)(it % H);
    if (!slot_ok(slot_idx[b])) {
      err = err > ORC_ERR_ARG ? err : ORC_ERR_ARG;
      continue;
    }
    uint8_t* blk = pool + (size_t)slot_idx[b] * slot_bytes + off[h];
    int e = orc_quantize_head(L, bits, h, S + (size_t)it * hs, blk);
    if (e > err) err = e;
  }
  free(off);
  return err;
}

int orc_dequantize(const orc_layout* L, const uint8_t* bits, const uint8_t* pool,
                   const int32_t* slot_idx, int n, float* S, int n_threads) {
  size_t slot_bytes;
  size_t* off = (size_t*)malloc(sizeof(size_t) * (size_t)L->n_heads);
  if (!off) return ORC_ERR_ARG;
  int st = orc_slot_layout(L, bits, off, &slot_bytes);
  if (st) {
    free(off);
    return st;
  }
  const int H = L->n_heads;
  const size_t hs = (size_t)L->d_k * L->d_v;
  int err = 0;
#pragma omp parallel for num_threads(n_threads > 0 ? n_threads : 1) schedule(dynamic, 1) reduction(max : err)
  for (long it = 0; it < (long)n * H; ++it) {
    const int b = (int)(it / H), h = (int)(it % H);
    if (!slot_ok(slot_idx[b])) {
      err = err > ORC_ERR_ARG ? err : ORC_ERR_ARG;
      continue;
    }
    const uint8_t* blk = pool + (size_t)slot_idx[b] * slot_bytes + off[h];
    int e = orc_dequantize_head(L, bits, h, blk, S + (size_t)it * hs);
    if (e > err) err = e;
  }
  free(off);
  return err;
}

int orc_decode_step(const orc_layout* L, const uint8_t* bits, uint8_t* pool,
                    const int32_t* slot_idx, int batch, const float* q, const float* k,
                    const float* v, const float* alpha, const float* beta, double* o,
                    float* s_new, int n_threads) {
  size_t slot_bytes;
  size_t* off = (size_t*)malloc(sizeof(size_t) * (size_t)L->n_heads);
  if (!off) return ORC_ERR_ARG;
  int st = orc_slot_layout(L, bits, off, &slot_bytes);
  if (st) {
    free(off);
    return st;
  }
  const int H = L->n_heads, dk = L->d_k, dv = L->d_v;
  const size_t hs = (size_t)dk * dv;
  const int na = L->gate == ORC_GATE_SCALAR ? 1 : dk;
  int err = 0;
#pragma omp parallel for num_threads(n_threads > 0 ? n_threads : 1) schedule(dynamic, 1) reduction(max : err)
  for (long it = 0; it < (long)batch * H; ++it) {
    const int b = (int)(it / H), h = (int)(it % H);
    if (!slot_ok(slot_idx[b])) {
      err = err > ORC_ERR_ARG ? err : ORC_ERR_ARG;
      continue;
    }
    uint8_t* blk = pool + (size_t)slot_idx[b] * slot_bytes + off[h];
    int e = decode_one(L, bits, h, blk, q + (size_t)it * dk, k + (size_t)it * dk,
                       v + (size_t)it * dv, alpha + (size_t)it * na, beta[it],
                       o + (size_t)it * dv, s_new ? s_new + (size_t)it * hs : NULL);
    if (e > err) err = e;
  }
  free(off);
  return err;
}

/* ------------------------------------------------------------------------------------------
 * Windowed variant. [LQ-N] 研究の概要: quantize only at the end of a window of tokens; inside
 * the window the output comes from the frozen low-bit state plus the update kept in high
 * precision. Reading taken: per slot, count = tokens folded in since the last quantization.
 * While count > 0 the exact state S_t = frozen + delta lives in wstate[slot][h] (fp64; the
 * delta is S_t minus the frozen state); at count == 0 it is the dequantized frozen block.
 * After the step that makes count reach W, the state is rounded to fp32 and requantized
 * (outliers re-selected), and count returns to 0. o is taken from S_t after the update.
 * wstate is [n_slots][H][d_k][d_v] doubles, count is [n_slots], both indexed by slot.
 * ---------------------------------------------------------------------------------------- */
static int window_one(const orc_layout* L, const uint8_t* bits, int h, uint8_t* block,
                      double* W, int count, int flush_after, const float* q, const float* k,
                      const float* v, const float* alpha, float beta, double* o) {
  const int dk = L->d_k, dv = L->d_v;
  const size_t total = (size_t)dk * dv;
  float* S = (float*)malloc(sizeof(float) * total);
  const int n = dk > dv ? dk : dv;
  double* vec = (double*)malloc(sizeof(double) * (size_t)(3 * n + dk));
  int st = ORC_ERR_ARG;
  if (!S || !vec) goto out;
  if (count == 0) {
    st = orc_dequantize_head(L, bits, h, block, S);
    if (st) goto out;
    for (size_t e = 0; e < total; ++e) W[e] = (double)S[e];
  }
  double *dq = vec, *dkk = vec + n, *dvv = vec + 2 * n, *da = vec + 3 * n;
  load_vec(dq, q, dk);
  load_vec(dkk, k, dk);
  load_vec(dvv, v, dv);
  load_vec(da, alpha, L->gate == ORC_GATE_SCALAR ? 1 : dk);
  orc_delta_update(dk, dv, L->gate, W, dq, dkk, dvv, da, (double)beta, o);
  st = ORC_OK;
  if (flush_after) {
    for (size_t e = 0; e < total; ++e) S[e] = (float)W[e];
    st = orc_quantize_head(L, bits, h, S, block);
  }
out:
  free(S);
  free(vec);
  return st;
}

int orc_window_step(const orc_layout* L, const uint8_t* bits, uint8_t* pool,
                    const int32_t* slot_idx, int batch, const float* q, const float* k,
                    const float* v, const float* alpha, const float* beta, double* o,
                    double* wstate, int32_t* count, int n_threads) {
  size_t slot_bytes;
  size_t* off = (size_t*)malloc(sizeof(size_t) * (size_t)L->n_heads);
  if (!off) return ORC_ERR_ARG;
  int st = orc_slot_layout(L, bits, off, &slot_bytes);
  if (st) {
    free(off);
    return st;
  }
  const int H = L->n_heads, dk = L->d_k, dv = L->d_v;
  const size_t hs = (size_t)dk * dv;
  const int na = L->gate == ORC_GATE_SCALAR ? 1 : dk;
  for (int b = 0; b < batch; ++b)
    if (!slot_ok(slot_idx[b])) {
      free(off);
      return ORC_ERR_ARG;
    }
  int err = 0;
#pragma omp parallel for num_threads(n_threads > 0 ? n_threads : 1) schedule(dynamic, 1) reduction(max : err)
  for (long it = 0; it < (long)batch * H; ++it) {
    const int b = (int)(it / H), h = (int)(it % H);
    const int32_t s = slot_idx[b];
    uint8_t* blk = pool + (size_t)s * slot_bytes + off[h];
    const int flush = count[s] + 1 >= L->window;
    int e = window_one(L, bits, h, blk, wstate + ((size_t)s * H + h) * hs, count[s], flush,
                       q + (size_t)it * dk, k + (size_t)it * dk, v + (size_t)it * dv,
                       alpha + (size_t)it * na, beta[it], o + (size_t)it * dv);
    if (e > err) err = e;
  }
  for (int b = 0; b < batch; ++b) {
    const int32_t s = slot_idx[b];
    count[s] = count[s] + 1 >= L->window ? 0 : count[s] + 1;
  }
  free(off);
  return err;
}

/* Fold the open window of each listed slot into its quantized block now (no-op at count 0). */
int orc_window_flush(const orc_layout* L, const uint8_t* bits, uint8_t* pool,
                     const int32_t* slot_idx, int n, double* wstate, int32_t* count,
                     int n_threads) {
  size_t slot_bytes;
  size_t* off = (size_t*)malloc(sizeof(size_t) * (size_t)L->n_heads);
  if (!off) return ORC_ERR_ARG;
  int st = orc_slot_layout(L, bits, off, &slot_bytes);
  if (st) {
    free(off);
    return st;
  }
  const int H = L->n_heads;
  const size_t hs = (size_t)L->d_k * L->d_v;
  for (int b = 0; b < n; ++b)
    if (!slot_ok(slot_idx[b])) {
      free(off);
      return ORC_ERR_ARG;
    }
  int err = 0;
#pragma omp parallel for num_threads(n_threads > 0 ? n_threads : 1) schedule(dynamic, 1) reduction(max : err)
  for (long it = 0; it < (long)n * H; ++it) {
    const int b = (int)(it / H), h = (int)(it % H);
    const int32_t s = slot_idx[b];
    if (count[s] == 0) continue;
    float* S = (float*)malloc(sizeof(float) * hs);
    if (!S) {
      err = err > ORC_ERR_ARG ? err : ORC_ERR_ARG;
      continue;
    }
    const double* W = wstate + ((size_t)s * H + h) * hs;
    for (size_t e = 0; e < hs; ++e) S[e] = (float)W[e];
    int e2 = orc_quantize_head(L, bits, h, S, pool + (size_t)s * slot_bytes + off[h]);
    if (e2 > err) err = e2;
    free(S);
  }
  for (int b = 0; b < n; ++b) count[slot_idx[b]] = 0;
  free(off);
  return err;
}

/* ----------------------------------------------------------------------------------------
 * Offline width allocation. [SQ-E] lifetime-aware allocation paragraph: under a fixed average
 * bit budget, units whose error is large and long-lived get more bits, from a score that
 * combines the unit's reconstruction distortion with the mean lifetime of its memory; a few
 * high-risk units stay FP16 (pivots).
 *
 * Reading (the pages give no formula): unit u has risk R_u = lifetime_u * variance_u and, at b
 * bits, score R_u 2^(-2b) (a uniform b-bit quantizer's distortion scales as variance 2^(-2b)).
 * The n_pivots largest risks (ties: lower index) are pivots (width 16). The other n' units take
 * widths in {2, 4, 6, 8} with exactly K = floor((avg_bits - 2) n' / 2) steps of 2 bits above 2,
 * chosen to MINIMIZE sum_u R_u 2^(-2 b_u). This function solves that problem exactly by dynamic
 * programming over (unit, steps used) -- the plain definition of the optimum, independent of
 * any greedy rule. Returns the minimum in *objective (sum over non-pivot units).
 * ---------------------------------------------------------------------------------------- */
int orc_allocate_bits(int n, const double* variance, const double* lifetime, double avg_bits,
                      int n_pivots, uint8_t* bits_out, double* objective) {
  if (n < 1 || n_pivots < 0 || n_pivots >= n || !(avg_bits >= 2.0 && avg_bits <= 8.0))
    return ORC_ERR_ARG;
  double* R = (double*)malloc(sizeof(double) * n);
  int* is_piv = (int*)calloc((size_t)n, sizeof(int));
  if (!R || !is_piv) {
    free(R);
    free(is_piv);
    return ORC_ERR_ARG;
  }
  for (int u = 0; u < n; ++u) R[u] = variance[u] * lifetime[u];
  for (int p = 0; p < n_pivots; ++p) {  // the largest remaining risk, lowest index on ties
    int best = -1;
    for (int u = 0; u < n; ++u)
      if (!is_piv[u] && (best < 0 || R[u] > R[best])) best = u;
    is_piv[best] = 1;
  }
  const int nq = n - n_pivots;
  long K = (long)floor((avg_bits - 2.0) * nq / 2.0 + 1e-9);
  if (K < 0) K = 0;
  if (K > 3L * nq) K = 3L * nq;
  /* f[k] = least score of the units seen so far using exactly k steps; choice[u][k] = steps
   * given to unit u in that optimum */
  double* f = (double*)malloc(sizeof(double) * (K + 1));
  double* g = (double*)malloc(sizeof(double) * (K + 1));
  uint8_t* choice = (uint8_t*)malloc((size_t)n * (K + 1));
  if (!f || !g || !choice) {
    free(R);
    free(is_piv);
    free(f);
    free(g);
    free(choice);
    return ORC_ERR_ARG;
  }
  for (long k = 0; k <= K; ++k) f[k] = k == 0 ? 0.0 : INFINITY;
  for (int u = 0; u < n; ++u) {
    if (is_piv[u]) continue;
    for (long k = 0; k <= K; ++k) {
      double best = INFINITY;
      int bl = 0;
      for (int l = 0; l <= 3 && l <= k; ++l) {
        const double v = f[k - l] + R[u] * pow(2.0, -2.0 * (2 + 2 * l));
        if (v < best) {
          best = v;
          bl = l;
        }
      }
      g[k] = best;
      choice[(size_t)u * (K + 1) + k] = (uint8_t)bl;
    }
    double* t = f;
    f = g;
    g = t;
  }
  if (objective) *objective = f[K];
  long k = K;
  for (int u = n - 1; u >= 0; --u) {
    if (is_piv[u]) {
      bits_out[u] = 16;
      continue;
    }
    const int l = choice[(size_t)u * (K + 1) + k];
    bits_out[u] = (uint8_t)(2 + 2 * l);
    k -= l;
  }
  free(R);
  free(is_piv);
  free(f);
  free(g);
  free(choice);
  return ORC_OK;
}
