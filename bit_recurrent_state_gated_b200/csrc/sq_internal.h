// sq_internal.h -- structures shared by the host API and the kernels of libsq.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

struct sq_pool;

namespace sq {

constexpr int kThreads = 256;  // 8 warps; warp w owns key rows [16w, 16w+16)
constexpr int kMaxD = 128;     // d_k, d_v <= 128, multiples of 16
constexpr int kSlack = 16;     // bytes after a staged head block (6-bit unpack reads ahead)

// Device status word bits (the same values as SQ_FLAG_* in include/sq.h).
constexpr int32_t SQ_FLAG_BAD_SLOT_BIT = 1, SQ_FLAG_NONFINITE_BIT = 2, SQ_FLAG_RANGE_BIT = 4,
                  SQ_FLAG_TIMEOUT_BIT = 8;

// Per head, shared by all slots (the widths are fixed offline).
struct HeadDesc {
  uint32_t off;         // byte offset of the head block within a slot
  uint32_t bytes;       // block bytes, a multiple of 16
  uint32_t pivot_head;  // 1: the head is one fp16 matrix (no scales)
  uint32_t width;       // head units: the width; key-row units: 0 (see the row table)
};

// Row table: rows[h * d_k + i] = (byte offset of row i within the head block) << 8 | width,
// width 16 for an fp16 pivot row.
__host__ __device__ inline uint32_t row_off(uint32_t d) { return d >> 8; }
__host__ __device__ inline int row_width(uint32_t d) { return (int)(d & 0xff); }
// Key-row units' processing-order descriptors carry this bit when their four-row chunk has one
// width.
constexpr uint32_t kChunkUniform = 0x80u;

// Windowed variant: the side block of one (slot, head) holds a 16-byte header (int32 token
// count; for the scalar gate the cumulative gate g, fp32, at byte 4), for the diagonal gate the
// cumulative gates g [d_k] fp32, then up to `window` low-rank terms. A term is a k part, then a
// b part [d_v] fp32. Scalar gate: the token's own k in the I/O type and b / g_s, since
// b (k_hat . y) = (b / g_s)(k . y) with k_hat = k / g_s; diagonal gate: k_hat in fp32 and b.
struct SideFmt {
  uint32_t head;    // bytes before the first term
  uint32_t kbytes;  // k part of a term, a multiple of 16
  uint32_t stride;  // bytes of a term
  bool k16;         // k part in bf16
  __host__ __device__ SideFmt(int dk, int dv, int gate, int io) {
    k16 = gate == 0 && io == 1;
    head = gate == 1 ? 16u + 4u * (uint32_t)dk : 16u;
    kbytes = gate == 1 ? 4u * (uint32_t)dk : ((uint32_t)dk * (io == 1 ? 2u : 4u) + 15u) / 16u * 16u;
    stride = kbytes + 4u * (uint32_t)dv;
  }
};

struct StepArgs {
  uint8_t* pool;
  int64_t slot_bytes;
  int32_t n_slots;
  const int32_t* slot_idx;
  int32_t batch;
  const void* q;
  const void* k;
  const void* v;
  const float* alpha;
  const float* beta;
  float* out;
  float* s_new;  // optional fp32 state after the update (tests)
  const HeadDesc* heads;
  const uint32_t* rows;
  const uint32_t* srows;  // key-row units: [H][d_k] row descriptors in processing order
                          // (original row << 24 | byte offset << 8 | width), rows grouped by width
  const int32_t* order;  // heads sorted by width: items run head-major in this order
  int32_t H, dk, dv, fit_iters;
  int32_t per_row;       // 1: key-row units (the row table is staged with each head block)
  uint32_t stage_bytes;  // smem bytes reserved for one staged head block
  int32_t n_stages;      // staged items in flight (set by the decode launcher)
  int32_t* flag;
  // windowed variant
  uint8_t* side;          // side region base (n_slots * side_slot_bytes)
  int64_t side_slot_bytes, side_head_bytes;
  int32_t window, n_outliers;
  int32_t n_tok;  // tokens of a chunk (sq_decode_chunk)
  const float* omega;  // null, or [H][d_k] column-pass weights of the impact-weighted fit
                       // (sq_pool_set_row_impact)
  int32_t update_only;  // with s_new: write the updated fp32 state and stop (no refit, no
                        // requantization); a skipped item gets a NaN in its s_new block
  uint64_t wait_ns;     // limit of every wait on a bulk copy (global-timer nanoseconds)
  uint32_t extra_tx;    // test hook: bytes the staging barrier of the decode, window and chunk
                        // kernels expects beyond what its copies bring (0 in normal use; > 0
                        // makes the wait run out)
  int32_t full_fit;     // test hook: 1 = never skip the last column pass of the fit
};

struct QuantArgs {
  uint8_t* pool;
  int64_t slot_bytes;
  int32_t n_slots;
  const int32_t* slot_idx;
  int32_t n;
  const float* S;  // quantize: input; dequantize: output (cast away const)
  const float* omega;  // null, or [H][d_k] column-pass weights (as StepArgs::omega)
  float* S_out;
  const HeadDesc* heads;
  const uint32_t* rows;
  int32_t H, dk, dv, fit_iters, n_outliers;
  uint32_t stage_bytes;
  int32_t* flag;
  uint8_t* side;
  int64_t side_slot_bytes, side_head_bytes;
};

// Launchers (sq_decode.cu, sq_quant.cu, sq_window_step.cu, sq_window.cu, sq_chunk.cu). Return
// cudaSuccess or the launch error.
cudaError_t launch_decode(const StepArgs& a, int gate, int io, bool want_state, int num_sms,
                          cudaStream_t st);
cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t st);
cudaError_t launch_dequantize(const QuantArgs& a, cudaStream_t st);
cudaError_t launch_window_step(const StepArgs& a, int gate, int io, int num_sms,
                               cudaStream_t st);
cudaError_t launch_window_flush(const StepArgs& a, int gate, int io, cudaStream_t st);
cudaError_t launch_chunk(const StepArgs& a, int gate, int io, int num_sms, cudaStream_t st);
// Heads and tile shape of a pool (for entry points outside the pool's own file).
void pool_dims(const sq_pool* p, int* n_heads, int* d_k, int* d_v);
constexpr int kMaxChunkTokens = 16;

}  // namespace sq
