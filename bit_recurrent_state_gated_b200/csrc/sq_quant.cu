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
__global__ void __launch_bounds__(kThreads) k_quantize(const QuantArgs a) {
  __shared__ TileSmem sm;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = blockIdx.x, dk = a.dk, dv = a.dv;
  const int b = item / a.H, h = item % a.H;
  const int slot = a.slot_idx[b];
  if (slot < 0 || slot >= a.n_slots) {
    if (tid == 0) atomicOr(a.flag, SQ_FLAG_BAD_SLOT_BIT);
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
    if (tid == 0) atomicOr(a.flag, SQ_FLAG_NONFINITE_BIT);
    return;
  }
  uint8_t* dst = a.pool + (size_t)slot * a.slot_bytes + hd.off;
  const float* omega = a.omega ? a.omega + (size_t)h * dk : nullptr;
  const bool ok = quantize_tile(S, dst, hd, rows, omega, a.n_outliers, a.fit_iters, warp, lane, dk,
                                dv, sm);
  if (!ok && tid == 0) atomicOr(a.flag, SQ_FLAG_RANGE_BIT);
  if (a.side && tid == 0)  // close this head's window
    *reinterpret_cast<int32_t*>(a.side + (size_t)slot * a.side_slot_bytes +
                                (size_t)h * a.side_head_bytes) = 0;
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
