/*
 * sq_oracle.h -- CPU oracle for the quantized gated delta-rule decode step.
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the bench's CPU-baseline leg may
 * load, link or call this code. The product (the CUDA library and its Python binding) never
 * does, and shares no source with it.
 *
 * What it computes is described in sq_oracle.c, function by function, with the passage of
 * the pages each step follows:
 *   STEPQuant explainer   = "STEPQuant" article, blog.ontle.kr/blog/302
 *   STEPQuant news        = "STEPQuant、推論メモリを最大68.7%削減", news.affectosphere.group
 *   LeapQuant news        = "LeapQuant、線形注意の推論を1.47倍高速化", news.affectosphere.group
 *
 * Parity status of each function is listed at the top of sq_oracle.c: the row-impact
 * weighting of orc_fit (orc_layout.omega) is pinned by its stated purpose and special cases.
 */
#ifndef SQ_ORACLE_H
#define SQ_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_OK = 0, ORC_ERR_ARG = 1, ORC_ERR_NONFINITE = 2, ORC_ERR_RANGE = 3 };
enum { ORC_UNIT_HEAD = 0, ORC_UNIT_ROW = 1 };
enum { ORC_GATE_SCALAR = 0, ORC_GATE_DIAG = 1 };

typedef struct {
  int32_t n_heads, d_k, d_v;
  int32_t unit;       /* ORC_UNIT_HEAD: one width per head; ORC_UNIT_ROW: one per key row */
  int32_t gate;       /* ORC_GATE_SCALAR: alpha per head; ORC_GATE_DIAG: alpha per key channel */
  int32_t fit_iters;  /* alternations of the row/column max-abs fit (>= 1) */
  int32_t window;     /* 1: requantize after every step; W > 1: after every W steps */
  int32_t n_outliers; /* entries per head kept in fp16 at each requantization */
  const float* omega; /* NULL, or per key row of each head [n_heads][d_k]: the row's weight
                         in the column pass of the fit (orc_impact_weights, orc_fit) */
} orc_layout;

/* ---- format ---- */
int orc_validate(const orc_layout* L, const uint8_t* bits);
size_t orc_row_bytes(int b, int d_v);
size_t orc_head_bytes(const orc_layout* L, const uint8_t* bits, int h);
int orc_slot_layout(const orc_layout* L, const uint8_t* bits, size_t* head_off, size_t* slot_bytes);
void orc_pack_row(int b, int n, const int32_t* u, uint8_t* out);
void orc_unpack_row(int b, int n, const uint8_t* in, int32_t* u);
uint16_t orc_f32_to_f16_bits(float x);
float orc_f16_bits_to_f32(uint16_t h);

/* ---- one head ---- */
int orc_fit(int d_k, int d_v, int fit_iters, const float* S, const int32_t* qmax,
            const uint8_t* excluded, const float* omega, float* r, float* c);
int orc_impact_weights(int n_heads, int d_k, const float* impact, float* omega);
int orc_select_outliers(int d_k, int d_v, const float* S, const int32_t* qmax, int n,
                        int32_t* idx_out);
int orc_quantize_head(const orc_layout* L, const uint8_t* bits, int h, const float* S,
                      uint8_t* block);
int orc_dequantize_head(const orc_layout* L, const uint8_t* bits, int h, const uint8_t* block,
                        float* S);
void orc_delta_update(int d_k, int d_v, int gate, double* M, const double* q, const double* k,
                      const double* v, const double* alpha, double beta, double* o);

/* ---- a batch of slots in a pool (pool = n_slots * slot_bytes bytes) ---- */
int orc_quantize(const orc_layout* L, const uint8_t* bits, uint8_t* pool, const int32_t* slot_idx,
                 int n, const float* S, int n_threads);
int orc_dequantize(const orc_layout* L, const uint8_t* bits, const uint8_t* pool,
                   const int32_t* slot_idx, int n, float* S, int n_threads);
int orc_decode_step(const orc_layout* L, const uint8_t* bits, uint8_t* pool,
                    const int32_t* slot_idx, int batch, const float* q, const float* k,
                    const float* v, const float* alpha, const float* beta, double* o,
                    float* s_new, int n_threads);
int orc_window_step(const orc_layout* L, const uint8_t* bits, uint8_t* pool,
                    const int32_t* slot_idx, int batch, const float* q, const float* k,
                    const float* v, const float* alpha, const float* beta, double* o,
                    double* wstate, int32_t* count, int n_threads);
int orc_window_flush(const orc_layout* L, const uint8_t* bits, uint8_t* pool,
                     const int32_t* slot_idx, int n, double* wstate, int32_t* count,
                     int n_threads);

/* ---- offline width allocation (exact optimum by dynamic programming) ---- */
int orc_allocate_bits(int n, const double* variance, const double* lifetime, double avg_bits,
                      int n_pivots, uint8_t* bits_out, double* objective);

#ifdef __cplusplus
}
#endif
#endif
