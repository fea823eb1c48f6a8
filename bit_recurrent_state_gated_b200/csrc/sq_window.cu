// sq_window.cu -- windowed variant of the decode step (LeapQuant news, 研究の概要: quantize
// only at the end of a window of tokens; inside it the output comes from the frozen low-bit
// state plus the update held at high precision; a few large entries are kept as
// high-precision "compensation" elements on the same update path).
//
// The exact state inside a window is S_t = frozen + delta_t. The delta is held per (slot,
// head) as low-rank factors in the pool's side region: with the cumulative gate g_t (per key
// channel) and the tokens' (k_hat_s, b_s),
//     S_t = diag(g_t) (Sbar + sum_s k_hat_s b_s^T),     k_hat_s = k_s / g_s,
// because each step is S_t = D_t S_{t-1} + k_t b_t^T. Then, with y = g_t k and z = g_t q,
//     u = Sbar^T y + sum_{s<t} b_s (k_hat_s . y),   b_t = beta (v - u),
//     o = Sbar^T z + sum_{s<t} b_s (k_hat_s . z) + b_t (k . q).
// A step reads the frozen block and the factors and appends one factor pair; after the W-th
// token the state is materialized, the compensation entries are chosen, and it is refit and
// requantized (sq_tile.cuh), as in the per-step path.
//
// Side block of one (slot, head): see SideFmt (sq_internal.h). For the scalar gate a term holds
// the token's k and b / g_s, whose product is the same rank-one term k_hat_s b_s^T.
#include "sq_pair.cuh"
#include "sq_tile.cuh"

namespace sq {
namespace {
using namespace tile;

constexpr int kMaxWindow = 64;

struct __align__(16) WSmem {
  TileSmem t;
  float k[kMaxD], q[kMaxD], y[kMaxD], z[kMaxD], g[kMaxD], A[kMaxD];
  float colC[kMaxD], colU[kMaxD], colP[kMaxD], colB[kMaxD], v[kMaxD];
  float lr[kMaxWindow][2];
  float kq, beta;
  int bad, cnt, flush;
};

__device__ __forceinline__ uint8_t* side_of(const StepArgs& a, int slot, int h) {
  return a.side + (size_t)slot * a.side_slot_bytes + (size_t)h * a.side_head_bytes;
}

// Copy `bytes` (a multiple of 16) from global to shared memory with all threads. Misaligned
// pointers are refused (status bit 16) rather than dereferenced.
__device__ __forceinline__ void copy16(void* dst, const void* src, uint32_t bytes, int32_t* flag) {
  if (((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) & 15) != 0) {
    if (threadIdx.x == 0) atomicOr(flag, 16);
    return;
  }
  for (uint32_t x = threadIdx.x; x < bytes / 16; x += kThreads)
    reinterpret_cast<uint4*>(dst)[x] = reinterpret_cast<const uint4*>(src)[x];
}

// Dequantized frozen state of the warp's rows in the tile (outliers included).
template <bool WITH_OUTLIERS>
__device__ __forceinline__ void frozen_tile(float (&S)[kRows][4], const uint8_t* blk,
                                            const HeadDesc& hd, const uint32_t* rows, int n_out,
                                            int warp, int lane, int dk, int dv) {
  unpack_tile_any(mode_of(hd), S, blk, rows, warp, lane, dk, dv);
  if (hd.pivot_head) return;
  float c[4] = {1.f, 1.f, 1.f, 1.f};
  if (4 * lane < dv) {
#pragma unroll
    for (int e = 0; e < 4; ++e) c[e] = __half2float(reinterpret_cast<const __half*>(blk)[dk + 4 * lane + e]);
  }
#pragma unroll
  for (int s = 0; s < kRows; ++s) {
    const int i = warp * kRows + s;
    if (i < dk && row_width(rows[i]) != 16) {
      const float r = __half2float(reinterpret_cast<const __half*>(blk)[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) S[s][e] = S[s][e] * (r * c[e]);
    }
  }
  if (WITH_OUTLIERS && n_out > 0) {
    const uint8_t* o = blk + row_off(rows[dk - 1]) + (size_t)dv * row_width(rows[dk - 1]) / 8;
    for (int t = 0; t < n_out; ++t) {
      const int idx = reinterpret_cast<const uint16_t*>(o)[2 * t];
      const int wi = idx / dv, wj = idx % dv;
      if (wi / kRows == warp && wj / 4 == lane) {
        const float p = __half2float(reinterpret_cast<const __half*>(o)[2 * t + 1]);
#pragma unroll
        for (int s = 0; s < kRows; ++s)
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (s == wi % kRows && e == wj % 4) S[s][e] = p;
      }
    }
  }
}

// Materialize S = g_i (Sbar_ij + sum_{s<n} khat_s[i] b_s[j]) (+ k_i b_j for a new token), then
// choose the compensation entries, refit, requantize and store; close the window.
// kk, bcol: the new token's k and b (add_new only).
__device__ __forceinline__ void flush_tile(const StepArgs& a, TileSmem& ts, const uint8_t* blk,
                                           const float* terms, int nterms, const float* g,
                                           bool add_new, const float* kk, const float* bcol,
                                           uint8_t* dst, const HeadDesc& hd,
                                           const uint32_t* rows, const float* omega,
                                           int32_t* count) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, dk = a.dk, dv = a.dv;
  float S[kRows][4];
  frozen_tile<true>(S, blk, hd, rows, a.n_outliers, warp, lane, dk, dv);
  const int tstride = dk + dv;  // terms: k part [d_k], b part [d_v], fp32
  if (4 * lane < dv) {
    for (int t = 0; t < nterms; ++t) {
      const float* kh = terms + (size_t)t * tstride;
      const float4 bb = *reinterpret_cast<const float4*>(kh + dk + 4 * lane);
      const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
      for (int s = 0; s < kRows; ++s) {
        const int i = warp * kRows + s;
        if (i < dk) {
          const float kv = kh[i];
#pragma unroll
          for (int e = 0; e < 4; ++e) S[s][e] = __fmaf_rn(kv, bv[e], S[s][e]);
        }
      }
    }
#pragma unroll
    for (int s = 0; s < kRows; ++s) {
      const int i = warp * kRows + s;
      if (i < dk) {
        const float gi = g[i];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          S[s][e] *= gi;
          if (add_new) S[s][e] = __fmaf_rn(kk[i], bcol[4 * lane + e], S[s][e]);
        }
      }
    }
  }
  if (tid == 0) ts.misc[0] = 0;
  __syncthreads();
  const bool ok = quantize_tile(S, dst, hd, rows, omega, a.n_outliers, a.fit_iters, warp, lane, dk,
                                dv, ts);
  if (!ok && tid == 0) atomicOr(a.flag, SQ_FLAG_RANGE_BIT);
  if (tid == 0) *count = 0;
}

// Fold each listed slot's open window into its block now (no-op at count 0).
__global__ void __launch_bounds__(kThreads) k_window_flush(const StepArgs a, int gate, int io) {
  extern __shared__ __align__(16) uint8_t dyn[];
  __shared__ WSmem sm;
  const int tid = threadIdx.x, dk = a.dk, dv = a.dv, H = a.H, W = a.window;
  const int item = blockIdx.x, b = item / H, h = item % H;
  const int slot = a.slot_idx[b];
  if (slot < 0 || slot >= a.n_slots) {
    if (tid == 0) atomicOr(a.flag, SQ_FLAG_BAD_SLOT_BIT);
    return;
  }
  const HeadDesc hd = a.heads[h];
  const uint32_t* rows = a.rows + (size_t)h * dk;
  uint8_t* dst = a.pool + (size_t)slot * a.slot_bytes + hd.off;
  uint8_t* side = side_of(a, slot, h);
  int32_t* count = reinterpret_cast<int32_t*>(side);
  const int cnt = *count;
  if (cnt <= 0 || cnt >= W) return;  // closed (or unreadable) window: nothing to fold
  uint8_t* blk = dyn;
  float* terms = reinterpret_cast<float*>(dyn + round16(a.stage_bytes + kSlack));
  copy16(blk, dst, hd.bytes, a.flag);
  const SideFmt f(dk, dv, gate, io);
  if (gate == 1) {  // the terms as stored: k_hat and b, fp32
    copy16(terms, side + f.head, (uint32_t)cnt * f.stride, a.flag);
    copy16(sm.g, side + 16, dk * 4, a.flag);
  } else {  // the token's k (I/O type) and b / g_s, to fp32 terms; one gate for every row
    for (int x = tid; x < cnt * (dk + dv); x += kThreads) {
      const int t = x / (dk + dv), e = x % (dk + dv);
      const uint8_t* tp = side + f.head + (size_t)t * f.stride;
      terms[x] = e >= dk ? reinterpret_cast<const float*>(tp + f.kbytes)[e - dk]
                         : f.k16 ? __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(tp)[e] << 16)
                                 : reinterpret_cast<const float*>(tp)[e];
    }
    for (int i = tid; i < dk; i += kThreads) sm.g[i] = reinterpret_cast<const float*>(side)[1];
  }
  __syncthreads();
  flush_tile(a, sm.t, blk, terms, cnt, sm.g, false, nullptr, nullptr, dst, hd, rows,
             a.omega ? a.omega + (size_t)h * dk : nullptr, count);
  (void)tid;
}

}  // namespace

cudaError_t launch_window_flush(const StepArgs& a, int gate, int io, cudaStream_t st) {
  if (a.window > kMaxWindow) return cudaErrorInvalidValue;
  const int items = a.batch * a.H;
  if (items < 1) return cudaSuccess;
  const uint32_t dyn = round16(a.stage_bytes + kSlack) + (uint32_t)a.window * (a.dk + a.dv) * 4;
  cudaError_t e = cudaFuncSetAttribute(k_window_flush, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (e != cudaSuccess) return e;
  k_window_flush<<<items, kThreads, dyn, st>>>(a, gate, io);
  return cudaGetLastError();
}

}  // namespace sq
