// sq_tile.cuh -- shared device code of libsq's kernels (sm_100a): the tile mapping, the
// alternating dual-axis fit, requantize + pack, and the top-n compensation entries.
//
// One CTA of 256 threads handles one (request, head) state tile at a time: warp w owns key
// rows [16w, 16w+16), lane l owns value columns [4l, 4l+4), so every thread keeps 16 x 4 fp32
// state values in registers and each packed row is read and written by one warp (a row's
// width is warp-uniform even when widths vary per key row).
#pragma once
#include <cuda_runtime.h>
#include <math.h>

#include <type_traits>

#include "sq_device.cuh"
#include "sq_internal.h"

namespace sq {
namespace tile {

constexpr int kWarps = kThreads / 32;
constexpr int kRows = 16;  // rows per warp
enum { MODE_ROWS = 0, MODE_W2 = 2, MODE_W4 = 4, MODE_W6 = 6, MODE_W8 = 8, MODE_PIVOT = 16 };
template <int M>
using ModeT = std::integral_constant<int, M>;

__host__ __device__ constexpr uint32_t round16(uint32_t x) { return (x + 15u) & ~15u; }

// Column arrays in shared memory (kMaxD floats each).
enum { COL_C = 0, COL_IC, COL_B, COL_P, COL_X, COL_INV, COL_IC16, COL_V, N_COL };

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
// Row weights (omega, per row of the head, in (0, 1], or null; impact-weighted pools): a row
// weighted below 1 counts in the column passes with w_i = fl(omega_i fl(1 / fl(r_i Q_i))), so
// the column scales follow the high-impact rows, and after the last alternation it is fit once
// more against the final column scales, r_i = max(r_i, fl(max_j fl(|S_ij| fl(1/c_j)) / Q_i)).
__device__ __forceinline__ void fit_scales(const float (&S)[kRows][4], int fit_iters, int warp,
                                           int lane, int dk, int dv, const uint32_t* rows,
                                           const float* omega, float* rowW, float* rowR,
                                           float* rowtmp, float* red, float* col) {
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
          const float q = __fdiv_rn(tmp[lane], (float)Q);
          r = fmaxf(q, kScaleFloor);
          w = rcp_rn(__fmul_rn(r, (float)Q));
          if (omega && omega[i] < 1.f) w = __fmul_rn(omega[i], w);
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
      col[COL_INV * kMaxD + t] = rcp_rn(c);
    } else if (t < kMaxD) {  // columns past d_v: neutral values for the idle lanes
      col[COL_X * kMaxD + t] = kScaleFloor;
      col[COL_INV * kMaxD + t] = 1.f;
    }
    __syncthreads();
    if (it + 1 < fit_iters || omega) {
      const float4 iv = *reinterpret_cast<const float4*>(col + COL_INV * kMaxD + 4 * lane);
      inv_c[0] = iv.x;
      inv_c[1] = iv.y;
      inv_c[2] = iv.z;
      inv_c[3] = iv.w;
    }
  }
  if (omega) {  // rows weighted below 1: fit once more against the final column scales
    float rm[kRows];
#pragma unroll
    for (int s = 0; s < kRows; ++s)
      rm[s] = warp_max_nonneg(fmaxf(fmaxf(fabsf(S[s][0]) * inv_c[0], fabsf(S[s][1]) * inv_c[1]),
                                    fmaxf(fabsf(S[s][2]) * inv_c[2], fabsf(S[s][3]) * inv_c[3])));
    if (lane == 0) {
#pragma unroll
      for (int s = 0; s < kRows; s += 4)
        *reinterpret_cast<float4*>(tmp + s) = make_float4(rm[s], rm[s + 1], rm[s + 2], rm[s + 3]);
    }
    __syncwarp();
    if (lane < kRows) {
      const int i = warp * kRows + lane;
      if (i < dk && omega[i] < 1.f) {
        const int Q = q_of_width(row_width(rows[i]));
        if (Q > 0) rowR[i] = fmaxf(rowR[i], __fdiv_rn(tmp[lane], (float)Q));
      }
    }
    __syncthreads();
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
        ir = rcp_f16val(__half2float(r16));
      }
      rowIR[i] = ir;
    }
  }
  if (t < dv) {
    const __half c16 = __float2half_rn(col[COL_X * kMaxD + t]);
    if (__hisinf(c16)) atomicOr(bad, 1);
    col[COL_IC16 * kMaxD + t] = rcp_f16val(__half2float(c16));
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
// Shared scratch of the quantize-type kernels (cold quantize, window flush).
// ---------------------------------------------------------------------------------------------
constexpr int kMaxOutliers = 64;
constexpr int kMaxCand = 256;

struct __align__(16) TileSmem {
  float red[kWarps * 2 * kMaxD];
  float rowW[kMaxD], rowR[kMaxD], rowIR[kMaxD], rowtmp[kWarps * kRows];
  float col[N_COL * kMaxD];
  unsigned long long wbest[kWarps];
  uint32_t tkey[kThreads];  // per-thread max key
  uint32_t thr;             // candidate threshold key
  int ncand;
  int cand_idx[kMaxCand];
  float cand_val[kMaxCand];
  int oidx[kMaxOutliers];
  float oval[kMaxOutliers];
  int misc[4];
};

// Key of an element for the top-n choice: larger |value| first; 0 marks "not eligible".
__device__ __forceinline__ uint32_t abs_key(float v) { return (__float_as_uint(v) & 0x7fffffffu) + 1u; }

// The n entries of largest |S| among the quantized rows (ties to the lower flat index), exact.
// Candidate threshold: the n-th largest per-thread maximum is at most the n-th largest element
// (fewer than n threads can hold an element above the latter), so every selected entry is
// among the elements at or above it. Falls back to n rounds of CTA arg-max if more than
// kMaxCand elements reach the threshold. Result in sm.oidx / sm.oval (ascending index) and in
// `sel` (bit s*4+e of the owning thread). Contains __syncthreads.
__device__ __forceinline__ void select_top_fast(const float (&S)[kRows][4], int n, int warp,
                                                int lane, int dk, int dv, const uint32_t* rows,
                                                uint64_t& sel, TileSmem& sm) {
  const int tid = threadIdx.x;
  uint32_t tmax = 0;
#pragma unroll
  for (int s = 0; s < kRows; ++s) {
    const int i = warp * kRows + s;
    if (i < dk && 4 * lane < dv && row_width(rows[i]) != 16) {
#pragma unroll
      for (int e = 0; e < 4; ++e) tmax = max(tmax, abs_key(S[s][e]));
    }
  }
  sm.tkey[tid] = tmax;
  if (tid == 0) sm.ncand = 0;
  __syncthreads();
  if (warp == 0) {  // n-th largest of the 256 thread maxima
    uint32_t v[kThreads / 32];
#pragma unroll
    for (int t = 0; t < kThreads / 32; ++t) v[t] = sm.tkey[lane * (kThreads / 32) + t];
    uint32_t last = 0;
    for (int r = 0; r < n; ++r) {
      uint32_t m = 0;
#pragma unroll
      for (int t = 0; t < kThreads / 32; ++t) m = max(m, v[t]);
      const uint32_t wm = __reduce_max_sync(0xffffffffu, m);
      last = wm;
      if (wm == 0) break;
      const uint32_t owner = __ffs(__ballot_sync(0xffffffffu, m == wm)) - 1;
      if (lane == (int)owner) {
        bool done = false;
#pragma unroll
        for (int t = 0; t < kThreads / 32; ++t)
          if (!done && v[t] == wm) {
            v[t] = 0;
            done = true;
          }
      }
    }
    if (lane == 0) sm.thr = last;
  }
  __syncthreads();
  const uint32_t thr = sm.thr;
#pragma unroll
  for (int s = 0; s < kRows; ++s) {
    const int i = warp * kRows + s;
    if (i < dk && 4 * lane < dv && row_width(rows[i]) != 16) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (abs_key(S[s][e]) >= thr) {
          const int pos = atomicAdd(&sm.ncand, 1);
          if (pos < kMaxCand) {
            sm.cand_idx[pos] = i * dv + 4 * lane + e;
            sm.cand_val[pos] = S[s][e];
          }
        }
      }
    }
  }
  __syncthreads();
  if (sm.ncand > kMaxCand) {  // many equal values: exact rounds of arg-max
    select_top(S, n, warp, lane, dk, dv, rows, sel, sm.wbest, sm.oidx, sm.oval);
  } else {
    if (warp == 0) {  // top n of the candidates by (|v| desc, index asc)
      const int nc = sm.ncand;
      for (int r = 0; r < n; ++r) {
        unsigned long long best = 0;
        int bpos = -1;
        for (int p = lane; p < nc; p += 32) {
          const int idx = sm.cand_idx[p];
          if (idx < 0) continue;
          const unsigned long long key =
              ((unsigned long long)abs_key(sm.cand_val[p]) << 32) | (0xffffffffu - (uint32_t)idx);
          if (key > best) {
            best = key;
            bpos = p;
          }
        }
        unsigned long long wb = best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const unsigned long long other = __shfl_xor_sync(0xffffffffu, wb, o);
          wb = other > wb ? other : wb;
        }
        if (best == wb && bpos >= 0 && wb != 0) {
          sm.oidx[r] = sm.cand_idx[bpos];
          sm.oval[r] = sm.cand_val[bpos];
          sm.cand_idx[bpos] = -1;
        }
        __syncwarp();
      }
    }
    __syncthreads();
    sel = 0;
    for (int r = 0; r < n; ++r) {
      const int idx = sm.oidx[r], wi = idx / dv, wj = idx % dv;
      if (wi / kRows == warp && wj / 4 == lane) sel |= 1ull << ((wi % kRows) * 4 + wj % 4);
    }
  }
  __syncthreads();
  if (tid == 0) {  // ascending index order
    for (int x = 1; x < n; ++x) {
      const int ki = sm.oidx[x];
      const float kv = sm.oval[x];
      int y = x - 1;
      while (y >= 0 && sm.oidx[y] > ki) {
        sm.oidx[y + 1] = sm.oidx[y];
        sm.oval[y + 1] = sm.oval[y];
        --y;
      }
      sm.oidx[y + 1] = ki;
      sm.oval[y + 1] = kv;
    }
  }
  __syncthreads();
}

// Quantize a register tile into the head block at dst: the n_out compensation entries (if
// any) are chosen and stored in fp16, the rest is fit and packed. Returns false (nothing
// stored) on an fp16 range overflow. Contains __syncthreads; sm.misc[0] must be 0 on entry.
__device__ __forceinline__ bool quantize_tile(float (&S)[kRows][4], uint8_t* dst,
                                              const HeadDesc& hd, const uint32_t* rows,
                                              const float* omega, int n_out, int fit_iters,
                                              int warp, int lane, int dk, int dv, TileSmem& sm) {
  if (hd.pivot_head) return store_pivot_head(S, dst, warp, lane, dk, dv, &sm.misc[0]);
  if (n_out > 0) {
    uint64_t sel = 0;
    select_top_fast(S, n_out, warp, lane, dk, dv, rows, sel, sm);
#pragma unroll
    for (int s = 0; s < kRows; ++s)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if ((sel >> (s * 4 + e)) & 1) S[s][e] = 0.f;  // outliers: out of the fit, code 0
    if ((int)threadIdx.x < n_out && __hisinf(__float2half_rn(sm.oval[threadIdx.x])))
      atomicOr(&sm.misc[0], 1);
  }
  fit_scales(S, fit_iters, warp, lane, dk, dv, rows, omega, sm.rowW, sm.rowR, sm.rowtmp, sm.red,
             sm.col);
  const bool ok = requant_store_any(mode_of(hd), S, dst, rows, warp, lane, dk, dv, sm.rowR,
                                    sm.rowIR, sm.col, &sm.misc[0]);
  if (ok && n_out > 0 && (int)threadIdx.x < n_out) {
    uint8_t* o = dst + row_off(rows[dk - 1]) + (size_t)dv * row_width(rows[dk - 1]) / 8;
    const int x = threadIdx.x;
    reinterpret_cast<uint16_t*>(o)[2 * x] = (uint16_t)sm.oidx[x];
    reinterpret_cast<__half*>(o)[2 * x + 1] = __float2half_rn(sm.oval[x]);
  }
  return ok;
}
}  // namespace tile
}  // namespace sq
