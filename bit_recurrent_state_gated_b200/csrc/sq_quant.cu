// sq_quant.cu -- cold quantize (fp32 state -> packed slot) and dequantize (packed -> fp32)
// kernels of libsq: one CTA per (slot, head), the tile mapping and fit of sq_tile.cuh,
// bit-exact with the CPU oracle.
#include "sq_tile.cuh"

namespace sq {
namespace {
using namespace tile;

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

}  // namespace

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
