// sq_kernels.cu -- the CUDA kernels of libsq (sm_100a).
//
// One CTA of 256 threads handles one (request, head) state tile at a time: warp w owns key
// rows [16w, 16w+16), lane l owns value columns [4l, 4l+4), so every thread keeps 16 x 4
// fp32 state values in registers and each packed row is read and written by one warp
// (a row's width is warp-uniform even when widths vary per key row).
//
// Decode step (STEPQuant explainer, experimental-setup paragraph: unpack, update and write
// back in one fused kernel; the dual-axis scales are refit on the updated state every step):
//   bulk-copy the packed head block and q, k, v (alpha) into shared memory, one tile ahead;
//   unpack the codes; u = S'^T k and S'^T q as code dot-products (S' = D M); b = beta (v - u);
//   M_new = S' + k b^T; o = S'^T q + b (k.q); refit row and column scales by alternating
//   max-abs passes; requantize and store the packed rows in place.
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {
namespace {

constexpr int kWarps = kThreads / 32;
constexpr int kRows = 16;  // rows per warp
enum { MODE_ROWS = 0, MODE_W2 = 2, MODE_W4 = 4, MODE_W6 = 6, MODE_W8 = 8, MODE_PIVOT = 16 };
template <int M>
using ModeT = std::integral_constant<int, M>;

__host__ __device__ constexpr uint32_t round16(uint32_t x) { return (x + 15u) & ~15u; }

// Column arrays in shared memory (kMaxD floats each).
enum { COL_C = 0, COL_IC, COL_B, COL_P, COL_X, COL_INV, COL_IC16, COL_V, N_COL };
// misc words: [0] bad slot, [1] bad input, [2] k.q (float bits), [3] range overflow
enum { MISC_SLOT = 0, MISC_INPUT, MISC_KQ, MISC_RANGE };

struct StageHdr {
  int32_t valid;
  float beta;
  float alpha;
  int32_t slot;
};

// Shared-memory plan of the decode kernel, identical on host (sizing) and device (carving).
struct Plan {
  uint32_t esz, kqv, k_off, q_off, v_off, al_off, stage, total;
  uint32_t off_bar, off_red, off_rowA, off_rowW, off_rowR, off_rowIR, off_rowtmp, off_col,
      off_misc;
  __host__ __device__ Plan(int dk, int dv, int io, int gate, uint32_t stage_bytes) {
    esz = io == 1 ? 2u : 4u;
    k_off = 0;
    q_off = dk * esz;
    v_off = 2u * dk * esz;
    al_off = v_off + dv * esz;
    kqv = al_off + (gate == 1 ? 4u * dk : 0u);  // every piece a multiple of 16 bytes
    stage = 16u + kqv + round16(stage_bytes + kSlack);
    uint32_t o = 2 * stage;
    off_bar = o;
    o += 16;
    off_red = o;
    o += kWarps * 2 * kMaxD * 4;
    off_rowA = o;
    o += kMaxD * 16;
    off_rowW = o;
    o += kMaxD * 4;
    off_rowR = o;
    o += kMaxD * 4;
    off_rowIR = o;
    o += kMaxD * 4;
    off_rowtmp = o;
    o += kWarps * kRows * 4;
    off_col = o;
    o += N_COL * kMaxD * 4;
    off_misc = o;
    o += 16;
    total = o;
  }
};

__device__ __forceinline__ float ld_io(const void* base, int io, int idx) {
  if (io == 1) {
    const uint16_t h = reinterpret_cast<const uint16_t*>(base)[idx];
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
  }
  return reinterpret_cast<const float*>(base)[idx];
}

__device__ __forceinline__ int q_of_width(int b) { return b == 16 ? 0 : (1 << (b - 1)) - 1; }

// Row and column scales of the tile held in S by alternating max-abs passes, the same rule as
// the oracle: cold start c = 1; r_i = max(max_j fl(|S_ij| fl(1/c_j)) / Q_i, 2^-14);
// w_i = fl(1 / fl(r_i Q_i)); c_j = max(max_i fl(|S_ij| w_i), 2^-14). Rows with Q = 0 (fp16
// pivot rows) get w = 0 and drop out of the column maxima; zeroed elements (outliers, idle
// lanes) contribute nothing. On return rowR[i] = r_i and col[COL_X][j] = c_j.
__device__ __forceinline__ void fit_scales(const float (&S)[kRows][4], int fit_iters, int warp,
                                           int lane, int dk, int dv, const uint32_t* rows,
                                           float* rowW, float* rowR, float* rowtmp, float* red,
                                           float* col) {
  float inv_c[4] = {1.f, 1.f, 1.f, 1.f};
  float* tmp = rowtmp + warp * kRows;
  for (int it = 0; it < fit_iters; ++it) {
    float rm[kRows];
#pragma unroll
    for (int s = 0; s < kRows; ++s) {
      float m;
      if (it == 0)
        m = fmaxf(fmaxf(fabsf(S[s][0]), fabsf(S[s][1])), fmaxf(fabsf(S[s][2]), fabsf(S[s][3])));
      else
        m = fmaxf(fmaxf(fabsf(S[s][0]) * inv_c[0], fabsf(S[s][1]) * inv_c[1]),
                  fmaxf(fabsf(S[s][2]) * inv_c[2], fabsf(S[s][3]) * inv_c[3]));
      rm[s] = warp_max_nonneg(m);
    }
    if (lane == 0) {
#pragma unroll
      for (int s = 0; s < kRows; s += 4)
        *reinterpret_cast<float4*>(tmp + s) = make_float4(rm[s], rm[s + 1], rm[s + 2], rm[s + 3]);
    }
    __syncwarp();
    if (lane < kRows) {
      const int i = warp * kRows + lane;
      if (i < dk) {
        const int Q = q_of_width(row_width(rows[i]));
        float r = 0.f, w = 0.f;
        if (Q > 0) {
          r = fmaxf(__fdiv_rn(tmp[lane], (float)Q), kScaleFloor);
          w = __frcp_rn(__fmul_rn(r, (float)Q));
        }
        rowR[i] = r;
        rowW[i] = w;
      } else {
        rowW[i] = 0.f;
      }
    }
    __syncwarp();
    float cm[4] = {0.f, 0.f, 0.f, 0.f};
    const float* wrow = rowW + warp * kRows;
#pragma unroll
    for (int s = 0; s < kRows; s += 4) {
      const float4 w4 = *reinterpret_cast<const float4*>(wrow + s);
      const float ws[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) cm[e] = fmaxf(cm[e], fabsf(S[s + t][e]) * ws[t]);
    }
    *reinterpret_cast<float4*>(red + warp * 2 * kMaxD + 4 * lane) =
        make_float4(cm[0], cm[1], cm[2], cm[3]);
    __syncthreads();
    const int t = threadIdx.x;
    if (t < dv) {
      float c = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) c = fmaxf(c, red[w * 2 * kMaxD + t]);
      c = fmaxf(c, kScaleFloor);
      col[COL_X * kMaxD + t] = c;
      col[COL_INV * kMaxD + t] = __frcp_rn(c);
    } else if (t < kMaxD) {  // columns past d_v: neutral values for the idle lanes
      col[COL_X * kMaxD + t] = kScaleFloor;
      col[COL_INV * kMaxD + t] = 1.f;
    }
    __syncthreads();
    if (it + 1 < fit_iters) {
      const float4 iv = *reinterpret_cast<const float4*>(col + COL_INV * kMaxD + 4 * lane);
      inv_c[0] = iv.x;
      inv_c[1] = iv.y;
      inv_c[2] = iv.z;
      inv_c[3] = iv.w;
    }
  }
}

// Round the fitted scales to fp16, check the fp16 range, quantize the tile and store scales
// and packed rows to the head block `dst` (global memory). Codes: nearest-even integer to
// fl(S_ij fl(1/r16_i)) * fl(1/c16_j) (the last product exact, inside one fma), clamped to
// [-Q, Q]. Returns false (and stores nothing) if a scale or a pivot value overflows fp16.
// Contains __syncthreads; *bad must be 0 on entry.
template <int MODE>
__device__ __forceinline__ bool requant_store(const float (&S)[kRows][4], uint8_t* dst,
                                              const uint32_t* rows, int warp, int lane, int dk,
                                              int dv, const float* rowR, float* rowIR,
                                              float* col, int* bad) {
  const bool active = 4 * lane < dv;
  const int t = threadIdx.x;
  if (lane < kRows) {
    const int i = warp * kRows + lane;
    if (i < dk) {
      float ir = 0.f;
      if (q_of_width(row_width(rows[i])) > 0) {
        const __half r16 = __float2half_rn(rowR[i]);
        if (__hisinf(r16)) atomicOr(bad, 1);
        ir = __frcp_rn(__half2float(r16));
      }
      rowIR[i] = ir;
    }
  }
  if (t < dv) {
    const __half c16 = __float2half_rn(col[COL_X * kMaxD + t]);
    if (__hisinf(c16)) atomicOr(bad, 1);
    col[COL_IC16 * kMaxD + t] = __frcp_rn(__half2float(c16));
  } else if (t < kMaxD) {
    col[COL_IC16 * kMaxD + t] = 0.f;
  }
#pragma unroll
  for (int s = 0; s < kRows; ++s) {
    const int i = warp * kRows + s;
    if (i < dk && row_width(rows[i]) == 16 && active && f16_overflows(S[s])) atomicOr(bad, 1);
  }
  __syncthreads();
  if (*bad) return false;
  if (lane < kRows) {
    const int i = warp * kRows + lane;
    if (i < dk)
      reinterpret_cast<__half*>(dst)[i] = q_of_width(row_width(rows[i])) > 0
                                             ? __float2half_rn(rowR[i])
                                             : __float2half_rn(0.f);
  }
  if (t < dv) reinterpret_cast<__half*>(dst)[dk + t] = __float2half_rn(col[COL_X * kMaxD + t]);
  const float4 ic4 = *reinterpret_cast<const float4*>(col + COL_IC16 * kMaxD + 4 * lane);
  const float ic[4] = {ic4.x, ic4.y, ic4.z, ic4.w};
#pragma unroll
  for (int s = 0; s < kRows; ++s) {
    const int i = warp * kRows + s;
    if (i < dk) {
      const uint32_t d = rows[i];
      uint8_t* row = dst + row_off(d);
      const int b = MODE == MODE_ROWS ? row_width(d) : MODE;
      if (b == 16) {
        store4_f16(row, lane, S[s], active);
      } else {
        const float ir = rowIR[i];
        const float Q = (float)q_of_width(b);
        const float magic = kMagic + (float)(1 << (b - 1));
        float y[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float v = __fmaf_rn(__fmul_rn(S[s][e], ir), ic[e], magic);
          y[e] = fminf(fmaxf(v, magic - Q), magic + Q);
        }
        switch (b) {
          case 2: store4<2>(row, lane, y, active); break;
          case 4: store4<4>(row, lane, y, active); break;
          case 6: store4<6>(row, lane, y, active); break;
          default: store4<8>(row, lane, y, active); break;
        }
      }
    }
  }
  return true;
}

__device__ __forceinline__ bool requant_store_any(int mode, const float (&S)[kRows][4],
                                                  uint8_t* dst, const uint32_t* rows, int warp,
                                                  int lane, int dk, int dv, const float* rowR,
                                                  float* rowIR, float* col, int* bad) {
  switch (mode) {
    case MODE_W2: return requant_store<MODE_W2>(S, dst, rows, warp, lane, dk, dv, rowR, rowIR, col, bad);
    case MODE_W4: return requant_store<MODE_W4>(S, dst, rows, warp, lane, dk, dv, rowR, rowIR, col, bad);
    case MODE_W6: return requant_store<MODE_W6>(S, dst, rows, warp, lane, dk, dv, rowR, rowIR, col, bad);
    case MODE_W8: return requant_store<MODE_W8>(S, dst, rows, warp, lane, dk, dv, rowR, rowIR, col, bad);
    default: return requant_store<MODE_ROWS>(S, dst, rows, warp, lane, dk, dv, rowR, rowIR, col, bad);
  }
}

// fp16 pivot head: all 4 values per row rounded to fp16 and stored row-major. Contains
// __syncthreads; false (nothing stored) if a value overflows fp16.
__device__ __forceinline__ bool store_pivot_head(const float (&S)[kRows][4], uint8_t* dst,
                                                 int warp, int lane, int dk, int dv, int* bad) {
  const bool active = 4 * lane < dv;
  bool of = false;
#pragma unroll
  for (int s = 0; s < kRows; ++s)
    if (warp * kRows + s < dk && active) of |= f16_overflows(S[s]);
  if (of) atomicOr(bad, 1);
  __syncthreads();
  if (*bad) return false;
#pragma unroll
  for (int s = 0; s < kRows; ++s) {
    const int i = warp * kRows + s;
    if (i < dk) store4_f16(dst + (size_t)i * 2 * dv, lane, S[s], active);
  }
  return true;
}

// Unpack the warp's rows of a staged head block into S (exact codes, or fp16 values for pivot
// rows), zero outside the tile.
template <int MODE>
__device__ __forceinline__ void unpack_tile(float (&S)[kRows][4], const uint8_t* blk,
                                            const uint32_t* rows, int warp, int lane, int dk,
                                            int dv) {
#pragma unroll
  for (int s = 0; s < kRows; ++s) {
    const int i = warp * kRows + s;
    if (i < dk && 4 * lane < dv) {
      const uint32_t d = rows[i];
      const uint8_t* row = blk + row_off(d);
      if constexpr (MODE == MODE_ROWS)
        unpack4_rt(row_width(d), row, lane, S[s]);
      else
        unpack4<MODE>(row, lane, S[s]);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) S[s][e] = 0.f;
    }
  }
}

__device__ __forceinline__ void unpack_tile_any(int mode, float (&S)[kRows][4],
                                                const uint8_t* blk, const uint32_t* rows,
                                                int warp, int lane, int dk, int dv) {
  switch (mode) {
    case MODE_W2: unpack_tile<MODE_W2>(S, blk, rows, warp, lane, dk, dv); break;
    case MODE_W4: unpack_tile<MODE_W4>(S, blk, rows, warp, lane, dk, dv); break;
    case MODE_W6: unpack_tile<MODE_W6>(S, blk, rows, warp, lane, dk, dv); break;
    case MODE_W8: unpack_tile<MODE_W8>(S, blk, rows, warp, lane, dk, dv); break;
    case MODE_PIVOT: unpack_tile<MODE_PIVOT>(S, blk, rows, warp, lane, dk, dv); break;
    default: unpack_tile<MODE_ROWS>(S, blk, rows, warp, lane, dk, dv); break;
  }
}

__device__ __forceinline__ int mode_of(const HeadDesc& hd) {
  return hd.pivot_head ? MODE_PIVOT : (int)hd.width;  // width 0 = per-row widths
}

// ---------------------------------------------------------------------------------------------
// Decode step: persistent CTAs over (request, head) items, two-stage bulk-copy pipeline.
// ---------------------------------------------------------------------------------------------
template <int GATE, int IO, bool WANT_STATE>
__global__ void __launch_bounds__(kThreads, 2) k_decode(const StepArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  const Plan P(a.dk, a.dv, IO, GATE, a.stage_bytes);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + P.off_bar);
  float* red = reinterpret_cast<float*>(smem + P.off_red);
  float4* rowA = reinterpret_cast<float4*>(smem + P.off_rowA);
  float* rowW = reinterpret_cast<float*>(smem + P.off_rowW);
  float* rowR = reinterpret_cast<float*>(smem + P.off_rowR);
  float* rowIR = reinterpret_cast<float*>(smem + P.off_rowIR);
  float* rowtmp = reinterpret_cast<float*>(smem + P.off_rowtmp);
  float* col = reinterpret_cast<float*>(smem + P.off_col);
  int* misc = reinterpret_cast<int*>(smem + P.off_misc);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H, dk = a.dk, dv = a.dv;
  const int n_items = a.batch * H;

  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](int item, int s) {  // thread 0: stage item `item` into stage s
    uint8_t* st = smem + s * P.stage;
    StageHdr* hdr = reinterpret_cast<StageHdr*>(st);
    const int b = item / H, h = item % H;
    const int slot = a.slot_idx[b];
    const bool valid = slot >= 0 && slot < a.n_slots;
    hdr->valid = valid;
    hdr->slot = slot;
    hdr->beta = a.beta[item];
    hdr->alpha = GATE == 0 ? a.alpha[item] : 0.f;
    const HeadDesc hd = a.heads[h];
    mbar_arrive_expect_tx(&bar[s], P.kqv + (valid ? hd.bytes : 0u));
    uint8_t* kqv = st + 16;
    const uint8_t* kb = static_cast<const uint8_t*>(a.k) + (size_t)item * dk * P.esz;
    const uint8_t* qb = static_cast<const uint8_t*>(a.q) + (size_t)item * dk * P.esz;
    const uint8_t* vb = static_cast<const uint8_t*>(a.v) + (size_t)item * dv * P.esz;
    bulk_load(kqv + P.k_off, kb, dk * P.esz, &bar[s]);
    bulk_load(kqv + P.q_off, qb, dk * P.esz, &bar[s]);
    bulk_load(kqv + P.v_off, vb, dv * P.esz, &bar[s]);
    if (GATE == 1) bulk_load(kqv + P.al_off, a.alpha + (size_t)item * dk, 4u * dk, &bar[s]);
    if (valid)
      bulk_load(st + 16 + P.kqv, a.pool + (size_t)slot * a.slot_bytes + hd.off, hd.bytes,
                &bar[s]);
  };

  if (tid == 0 && (int)blockIdx.x < n_items) issue(blockIdx.x, 0);

  int it = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
    const int s = it & 1;
    // Stage s^1 was last read during the previous item, which every thread has finished.
    if (tid == 0 && item + (int)gridDim.x < n_items) issue(item + gridDim.x, s ^ 1);
    if (!mbar_wait_bounded(&bar[s], (it >> 1) & 1)) {
      if (tid == 0) atomicOr(a.flag, 8);
      return;
    }
    const uint8_t* st = smem + s * P.stage;
    const StageHdr hdr = *reinterpret_cast<const StageHdr*>(st);
    const uint8_t* kqv = st + 16;
    const uint8_t* blk = st + 16 + P.kqv;
    const int h = item % H;
    const HeadDesc hd = a.heads[h];
    const uint32_t* rows = a.rows + (size_t)h * dk;
    const bool pivot_head = hd.pivot_head != 0;
    const int mode = mode_of(hd);

    // ---- per-item setup: row factors A_i = alpha_i r16_i, column scales, input checks ----
    if (tid == 0) {
      misc[MISC_SLOT] = hdr.valid ? 0 : 1;
      misc[MISC_INPUT] = 0;
      misc[MISC_RANGE] = 0;
    }
    __syncthreads();
    bool bad_in = !isfinite(hdr.beta) || (GATE == 0 && !isfinite(hdr.alpha));
    if (hdr.valid) {
      if (tid < dk) {
        const int i = tid;
        const float ki = ld_io(kqv + P.k_off, IO, i), qi = ld_io(kqv + P.q_off, IO, i);
        const float ai = GATE == 0 ? hdr.alpha : reinterpret_cast<const float*>(kqv + P.al_off)[i];
        bad_in |= !isfinite(ki) || !isfinite(qi) || !isfinite(ai);
        float A = ai;
        if (!pivot_head && row_width(rows[i]) != 16)
          A = ai * __half2float(reinterpret_cast<const __half*>(blk)[i]);
        rowA[i] = make_float4(A, A * ki, A * qi, ki);
      }
      if (tid < dv) {
        const int j = tid;
        const float vj = ld_io(kqv + P.v_off, IO, j);
        bad_in |= !isfinite(vj);
        const float c = pivot_head ? 1.f : __half2float(reinterpret_cast<const __half*>(blk)[dk + j]);
        col[COL_C * kMaxD + j] = c;
        col[COL_IC * kMaxD + j] = __frcp_rn(c);
        col[COL_V * kMaxD + j] = vj;
      } else if (tid < kMaxD) {  // columns past d_v: neutral values for the idle lanes
        col[COL_C * kMaxD + tid] = 1.f;
        col[COL_IC * kMaxD + tid] = 1.f;
        col[COL_V * kMaxD + tid] = 0.f;
        col[COL_B * kMaxD + tid] = 0.f;
        col[COL_P * kMaxD + tid] = 0.f;
      }
      if (warp == 0) {
        float kq = 0.f;
        for (int i = lane; i < dk; i += 32)
          kq = __fmaf_rn(ld_io(kqv + P.k_off, IO, i), ld_io(kqv + P.q_off, IO, i), kq);
        kq = warp_sum(kq);
        if (lane == 0) misc[MISC_KQ] = __float_as_int(kq);
      }
      if (bad_in) atomicOr(&misc[MISC_INPUT], 1);
    }
    __syncthreads();
    float* out = a.out + (size_t)item * dv;
    if (misc[MISC_SLOT] | misc[MISC_INPUT]) {  // skip: flag it and fill the output with NaN
      if (tid == 0) atomicOr(a.flag, misc[MISC_SLOT] ? 1 : 2);
      if (tid < dv) out[tid] = __int_as_float(0x7fc00000);
      __syncthreads();
      continue;
    }

    const float4 c4 = *reinterpret_cast<const float4*>(col + COL_C * kMaxD + 4 * lane);
    const float4 ic4 = *reinterpret_cast<const float4*>(col + COL_IC * kMaxD + 4 * lane);
    const float c[4] = {c4.x, c4.y, c4.z, c4.w};
    const float icv[4] = {ic4.x, ic4.y, ic4.z, ic4.w};

    // ---- pass A: codes; U_j = sum_i x_ij A_i k_i, P_j = sum_i x_ij A_i q_i ----
    float S[kRows][4];
    unpack_tile_any(mode, S, blk, rows, warp, lane, dk, dv);
    float U[4] = {0.f, 0.f, 0.f, 0.f}, Pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s2 = 0; s2 < kRows; ++s2) {
      const int i = warp * kRows + s2;
      if (i < dk) {
        if (!pivot_head && row_width(rows[i]) == 16) {  // fp16 pivot row inside a scaled head
#pragma unroll
          for (int e = 0; e < 4; ++e) S[s2][e] *= icv[e];
        }
        const float4 ra = rowA[i];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          U[e] = __fmaf_rn(S[s2][e], ra.y, U[e]);
          Pq[e] = __fmaf_rn(S[s2][e], ra.z, Pq[e]);
        }
      }
    }
    *reinterpret_cast<float4*>(red + warp * 2 * kMaxD + 4 * lane) =
        make_float4(U[0], U[1], U[2], U[3]);
    *reinterpret_cast<float4*>(red + warp * 2 * kMaxD + kMaxD + 4 * lane) =
        make_float4(Pq[0], Pq[1], Pq[2], Pq[3]);
    __syncthreads();
    if (tid < 2 * dv) {
      const int which = tid / dv, j = tid % dv;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) sum += red[w * 2 * kMaxD + which * kMaxD + j];
      const float cj = col[COL_C * kMaxD + j];
      if (which == 0)
        col[COL_B * kMaxD + j] = hdr.beta * (col[COL_V * kMaxD + j] - cj * sum);
      else
        col[COL_P * kMaxD + j] = cj * sum;
    }
    __syncthreads();
    if (tid < dv)
      out[tid] = __fmaf_rn(col[COL_B * kMaxD + tid], __int_as_float(misc[MISC_KQ]),
                           col[COL_P * kMaxD + tid]);
    const float4 b4 = *reinterpret_cast<const float4*>(col + COL_B * kMaxD + 4 * lane);
    const float bv[4] = {b4.x, b4.y, b4.z, b4.w};

    // ---- pass B: M_new_ij = x_ij (A_i c_j) + k_i b_j ----
#pragma unroll
    for (int s2 = 0; s2 < kRows; ++s2) {
      const int i = warp * kRows + s2;
      if (i < dk && 4 * lane < dv) {
        const float4 ra = rowA[i];
#pragma unroll
        for (int e = 0; e < 4; ++e) S[s2][e] = __fmaf_rn(S[s2][e], ra.x * c[e], ra.w * bv[e]);
      }
    }
    if (WANT_STATE) {
      float* sn = a.s_new + (size_t)item * dk * dv;
#pragma unroll
      for (int s2 = 0; s2 < kRows; ++s2) {
        const int i = warp * kRows + s2;
        if (i < dk && 4 * lane < dv)
          *reinterpret_cast<float4*>(sn + (size_t)i * dv + 4 * lane) =
              make_float4(S[s2][0], S[s2][1], S[s2][2], S[s2][3]);
      }
    }

    // ---- refit, requantize, store in place ----
    uint8_t* dst = a.pool + (size_t)hdr.slot * a.slot_bytes + hd.off;
    bool ok;
    if (pivot_head) {
      ok = store_pivot_head(S, dst, warp, lane, dk, dv, &misc[MISC_RANGE]);
    } else {
      fit_scales(S, a.fit_iters, warp, lane, dk, dv, rows, rowW, rowR, rowtmp, red, col);
      ok = requant_store_any(mode, S, dst, rows, warp, lane, dk, dv, rowR, rowIR, col,
                             &misc[MISC_RANGE]);
    }
    if (!ok && tid == 0) atomicOr(a.flag, 4);
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------------------
// Top-n entries of |S| over the quantized rows (ties to the lower flat index i*dv + j), by n
// rounds of a CTA-wide arg-max. Selected elements are recorded in `sel` (bit s*4+e per thread)
// and their (index, value) pairs in out_idx / out_val (smem, n entries, in selection order).
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void select_top(const float (&S)[kRows][4], int n, int warp, int lane,
                                           int dk, int dv, const uint32_t* rows, uint64_t& sel,
                                           unsigned long long* wbest, int* out_idx,
                                           float* out_val) {
  sel = 0;
  for (int r = 0; r < n; ++r) {
    unsigned long long best = 0;
#pragma unroll
    for (int s = 0; s < kRows; ++s) {
      const int i = warp * kRows + s;
      if (i < dk && 4 * lane < dv && row_width(rows[i]) != 16) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if ((sel >> (s * 4 + e)) & 1) continue;
          const uint32_t idx = (uint32_t)(i * dv + 4 * lane + e);
          const unsigned long long key =
              ((unsigned long long)__float_as_uint(fabsf(S[s][e])) << 32) | (0xffffffffu - idx);
          best = key > best ? key : best;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long other = __shfl_xor_sync(0xffffffffu, best, o);
      best = other > best ? other : best;
    }
    if (lane == 0) wbest[warp] = best;
    __syncthreads();
    unsigned long long win = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) win = wbest[w] > win ? wbest[w] : win;
    const uint32_t idx = 0xffffffffu - (uint32_t)(win & 0xffffffffu);
    const int wi = (int)(idx / dv), wj = (int)(idx % dv);
    if (win != 0 && wi / kRows == warp && wj / 4 == lane) {
      const int s = wi % kRows, e = wj % 4;
      sel |= 1ull << (s * 4 + e);
      out_idx[r] = (int)idx;
      float v = 0.f;
#pragma unroll
      for (int s2 = 0; s2 < kRows; ++s2)
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2)
          if (s2 == s && e2 == e) v = S[s2][e2];
      out_val[r] = v;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------------------
// Quantize dense fp32 states into slots: one CTA per (slot, head).
// ---------------------------------------------------------------------------------------------
constexpr int kMaxOutliers = 64;

struct QSmem {
  float red[kWarps * 2 * kMaxD];
  float rowW[kMaxD], rowR[kMaxD], rowIR[kMaxD], rowtmp[kWarps * kRows];
  float col[N_COL * kMaxD];
  unsigned long long wbest[kWarps];
  int oidx[kMaxOutliers];
  float oval[kMaxOutliers];
  int misc[4];
};

__global__ void __launch_bounds__(kThreads) k_quantize(const QuantArgs a) {
  __shared__ QSmem sm;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = blockIdx.x, dk = a.dk, dv = a.dv;
  const int b = item / a.H, h = item % a.H;
  const int slot = a.slot_idx[b];
  if (slot < 0 || slot >= a.n_slots) {
    if (tid == 0) atomicOr(a.flag, 1);
    return;
  }
  const HeadDesc hd = a.heads[h];
  const uint32_t* rows = a.rows + (size_t)h * dk;
  const float* src = a.S + (size_t)item * dk * dv;
  if (tid == 0) sm.misc[0] = sm.misc[1] = 0;
  float S[kRows][4];
  bool nonfinite = false;
#pragma unroll
  for (int s = 0; s < kRows; ++s) {
    const int i = warp * kRows + s;
    if (i < dk && 4 * lane < dv) {
      const float4 v = *reinterpret_cast<const float4*>(src + (size_t)i * dv + 4 * lane);
      S[s][0] = v.x;
      S[s][1] = v.y;
      S[s][2] = v.z;
      S[s][3] = v.w;
#pragma unroll
      for (int e = 0; e < 4; ++e) nonfinite |= !isfinite(S[s][e]);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) S[s][e] = 0.f;
    }
  }
  __syncthreads();
  if (nonfinite) atomicOr(&sm.misc[1], 1);
  __syncthreads();
  if (sm.misc[1]) {
    if (tid == 0) atomicOr(a.flag, 2);
    return;
  }
  uint8_t* dst = a.pool + (size_t)slot * a.slot_bytes + hd.off;
  bool ok;
  if (hd.pivot_head) {
    ok = store_pivot_head(S, dst, warp, lane, dk, dv, &sm.misc[0]);
  } else {
    const int n_out = a.n_outliers;
    uint64_t sel = 0;
    if (n_out > 0) {
      select_top(S, n_out, warp, lane, dk, dv, rows, sel, sm.wbest, sm.oidx, sm.oval);
#pragma unroll
      for (int s = 0; s < kRows; ++s)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if ((sel >> (s * 4 + e)) & 1) S[s][e] = 0.f;  // outliers: out of the fit, code 0
    }
    fit_scales(S, a.fit_iters, warp, lane, dk, dv, rows, sm.rowW, sm.rowR, sm.rowtmp, sm.red,
               sm.col);
    if (n_out > 0 && tid < n_out) {
      if (__hisinf(__float2half_rn(sm.oval[tid]))) atomicOr(&sm.misc[0], 1);
    }
    ok = requant_store_any(mode_of(hd), S, dst, rows, warp, lane, dk, dv, sm.rowR, sm.rowIR,
                           sm.col, &sm.misc[0]);
    if (ok && n_out > 0 && tid == 0) {
      // outlier list in ascending index order (insertion sort of <= 64 entries)
      uint8_t* o = dst + row_off(rows[dk - 1]) + (size_t)dv * row_width(rows[dk - 1]) / 8;
      for (int x = 0; x < n_out; ++x) {
        int bi = -1;
        for (int y = 0; y < n_out; ++y) {
          if (sm.oidx[y] < 0) continue;
          if (bi < 0 || sm.oidx[y] < sm.oidx[bi]) bi = y;
        }
        const __half hv = __float2half_rn(sm.oval[bi]);
        reinterpret_cast<uint16_t*>(o)[2 * x] = (uint16_t)sm.oidx[bi];
        reinterpret_cast<__half*>(o)[2 * x + 1] = hv;
        sm.oidx[bi] = -1;
      }
    }
  }
  if (!ok && tid == 0) atomicOr(a.flag, 4);
  if (a.side && tid == 0 && h == 0) {  // close the slot's window
    *reinterpret_cast<int32_t*>(a.side + (size_t)slot * a.side_slot_bytes) = 0;
  }
}

// ---------------------------------------------------------------------------------------------
// Dequantize slots to dense fp32: one CTA per (slot, head).
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads) k_dequantize(const QuantArgs a) {
  extern __shared__ __align__(16) uint8_t blk[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = blockIdx.x, dk = a.dk, dv = a.dv;
  const int b = item / a.H, h = item % a.H;
  const int slot = a.slot_idx[b];
  float* out = a.S_out + (size_t)item * dk * dv;
  if (slot < 0 || slot >= a.n_slots) {
    if (tid == 0) atomicOr(a.flag, 1);
    return;
  }
  const HeadDesc hd = a.heads[h];
  const uint32_t* rows = a.rows + (size_t)h * dk;
  const uint4* src = reinterpret_cast<const uint4*>(a.pool + (size_t)slot * a.slot_bytes + hd.off);
  for (uint32_t x = tid; x < hd.bytes / 16; x += kThreads) reinterpret_cast<uint4*>(blk)[x] = src[x];
  __syncthreads();
  float S[kRows][4];
  unpack_tile_any(mode_of(hd), S, blk, rows, warp, lane, dk, dv);
  float c[4] = {1.f, 1.f, 1.f, 1.f};
  if (!hd.pivot_head && 4 * lane < dv) {
#pragma unroll
    for (int e = 0; e < 4; ++e) c[e] = __half2float(reinterpret_cast<const __half*>(blk)[dk + 4 * lane + e]);
  }
#pragma unroll
  for (int s = 0; s < kRows; ++s) {
    const int i = warp * kRows + s;
    if (i < dk && 4 * lane < dv) {
      float d[4];
      if (!hd.pivot_head && row_width(rows[i]) != 16) {
        const float r = __half2float(reinterpret_cast<const __half*>(blk)[i]);
#pragma unroll
        for (int e = 0; e < 4; ++e) d[e] = S[s][e] * (r * c[e]);  // r*c is exact in fp32
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) d[e] = S[s][e];
      }
      *reinterpret_cast<float4*>(out + (size_t)i * dv + 4 * lane) = make_float4(d[0], d[1], d[2], d[3]);
    }
  }
  if (a.n_outliers > 0 && !hd.pivot_head) {
    __syncthreads();
    const uint8_t* o = blk + row_off(rows[dk - 1]) + (size_t)dv * row_width(rows[dk - 1]) / 8;
    if (tid < a.n_outliers) {
      const uint32_t idx = reinterpret_cast<const uint16_t*>(o)[2 * tid];
      const float v = __half2float(reinterpret_cast<const __half*>(o)[2 * tid + 1]);
      if (idx < (uint32_t)(dk * dv)) out[idx] = v;
      else atomicOr(a.flag, 1);
    }
  }
}

template <int GATE, int IO, bool WS>
cudaError_t launch_decode_t(const StepArgs& a, int num_sms, cudaStream_t st) {
  const Plan P(a.dk, a.dv, IO, GATE, a.stage_bytes);
  auto fn = k_decode<GATE, IO, WS>;
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, P.total);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, P.total);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const int items = a.batch * a.H;
  int grid = num_sms * per_sm;
  if (grid > items) grid = items;
  if (grid < 1) return cudaSuccess;
  fn<<<grid, kThreads, P.total, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const StepArgs& a, int gate, int io, bool want_state, int num_sms,
                          cudaStream_t st) {
  if (gate == 0 && io == 0) return want_state ? launch_decode_t<0, 0, true>(a, num_sms, st) : launch_decode_t<0, 0, false>(a, num_sms, st);
  if (gate == 0 && io == 1) return want_state ? launch_decode_t<0, 1, true>(a, num_sms, st) : launch_decode_t<0, 1, false>(a, num_sms, st);
  if (gate == 1 && io == 0) return want_state ? launch_decode_t<1, 0, true>(a, num_sms, st) : launch_decode_t<1, 0, false>(a, num_sms, st);
  return want_state ? launch_decode_t<1, 1, true>(a, num_sms, st) : launch_decode_t<1, 1, false>(a, num_sms, st);
}

cudaError_t launch_quantize(const QuantArgs& a, cudaStream_t st) {
  if (a.n * a.H < 1) return cudaSuccess;
  k_quantize<<<a.n * a.H, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const QuantArgs& a, cudaStream_t st) {
  if (a.n * a.H < 1) return cudaSuccess;
  const uint32_t smem_bytes = round16(a.stage_bytes + kSlack);
  cudaError_t e = cudaFuncSetAttribute(k_dequantize, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem_bytes);
  if (e != cudaSuccess) return e;
  k_dequantize<<<a.n * a.H, kThreads, smem_bytes, st>>>(a);
  return cudaGetLastError();
}

}  // namespace sq
