// sq_pair.cuh -- device helpers shared by libsq's decode and windowed kernels: fp32x2 pair
// construction, 4-byte cp.async, and the unpack of one lane's four columns of TWO packed rows
// into register pairs (row a, row b) of exact codes, so the packed fp32x2 instructions work on
// two rows at once.
#pragma once
#include <cuda_fp16.h>
#include <stdint.h>

#include "sq_device.cuh"

namespace sq {

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 lo(const float4& v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi(const float4& v) { return make_float2(v.z, v.w); }
__device__ __forceinline__ float2 dup(float a) { return make_float2(a, a); }

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// ---- unpack: the lane's four columns of two rows (a, b) as pairs (a_e, b_e) of exact codes
// (f2u, the magic-number pair constructor, is in sq_device.cuh) ----
template <int B>
__device__ __forceinline__ void unpack_pair(const uint8_t* ra, const uint8_t* rb, int lane,
                                            float2 (&x)[4]);

template <>
__device__ __forceinline__ void unpack_pair<2>(const uint8_t* ra, const uint8_t* rb, int lane,
                                               float2 (&x)[4]) {
  const uint32_t va = ra[lane], vb = rb[lane];  // f = 2^23 + u 4^e ; code = f 4^-e - (2^(23-2e) + 2)
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t m = 3u << (2 * e);
    x[e] = __ffma2_rn(f2u(kMagicBits | (va & m), kMagicBits | (vb & m)),
                      dup(1.0f / float(1u << (2 * e))), dup(-(float(1u << (23 - 2 * e)) + 2.0f)));
  }
}

template <>
__device__ __forceinline__ void unpack_pair<4>(const uint8_t* ra, const uint8_t* rb, int lane,
                                               float2 (&x)[4]) {
  const uint32_t va = reinterpret_cast<const uint16_t*>(ra)[lane];
  const uint32_t vb = reinterpret_cast<const uint16_t*>(rb)[lane];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t m = 15u << (4 * e);
    x[e] = __ffma2_rn(f2u(kMagicBits | (va & m), kMagicBits | (vb & m)),
                      dup(1.0f / float(1u << (4 * e))), dup(-(float(1u << (23 - 4 * e)) + 8.0f)));
  }
}

__device__ __forceinline__ uint32_t bits24(const uint8_t* row, int lane) {  // 6-bit: lane's 24 bits
  const int byte = 3 * lane;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(row + (byte & ~3));
  return __funnelshift_r(w[0], w[1], (byte & 3) * 8);
}

template <>
__device__ __forceinline__ void unpack_pair<6>(const uint8_t* ra, const uint8_t* rb, int lane,
                                               float2 (&x)[4]) {
  const uint32_t va = bits24(ra, lane), vb = bits24(rb, lane);
  const uint32_t ha = va >> 12, hb = vb >> 12;
  const float2 s1 = dup(1.0f / 64.0f);
  const float2 o0 = dup(-(8388608.f + 32.f)), o1 = dup(-(131072.f + 32.f));
  x[0] = __fadd2_rn(f2u(kMagicBits | (va & 63u), kMagicBits | (vb & 63u)), o0);
  x[1] = __ffma2_rn(f2u(kMagicBits | (va & (63u << 6)), kMagicBits | (vb & (63u << 6))), s1, o1);
  x[2] = __fadd2_rn(f2u(kMagicBits | (ha & 63u), kMagicBits | (hb & 63u)), o0);
  x[3] = __ffma2_rn(f2u(kMagicBits | (ha & (63u << 6)), kMagicBits | (hb & (63u << 6))), s1, o1);
}

template <>
__device__ __forceinline__ void unpack_pair<8>(const uint8_t* ra, const uint8_t* rb, int lane,
                                               float2 (&x)[4]) {
  const uint32_t va = reinterpret_cast<const uint32_t*>(ra)[lane];
  const uint32_t vb = reinterpret_cast<const uint32_t*>(rb)[lane];
  const float2 m = dup(-(kMagic + 128.f));
#pragma unroll
  for (int e = 0; e < 4; ++e)
    x[e] = __fadd2_rn(f2u(__byte_perm(va, kMagicBits, 0x7540u + e),
                          __byte_perm(vb, kMagicBits, 0x7540u + e)), m);
}

template <>
__device__ __forceinline__ void unpack_pair<16>(const uint8_t* ra, const uint8_t* rb, int lane,
                                                float2 (&x)[4]) {
  // fp16 rows start on 4-byte boundaries: two 32-bit loads per row
  const uint32_t* wa = reinterpret_cast<const uint32_t*>(ra) + 2 * lane;
  const uint32_t* wb = reinterpret_cast<const uint32_t*>(rb) + 2 * lane;
  const uint32_t a0 = wa[0], a1 = wa[1], b0 = wb[0], b1 = wb[1];
  const __half2 ha0 = *reinterpret_cast<const __half2*>(&a0), ha1 = *reinterpret_cast<const __half2*>(&a1);
  const __half2 hb0 = *reinterpret_cast<const __half2*>(&b0), hb1 = *reinterpret_cast<const __half2*>(&b1);
  x[0] = f2(__low2float(ha0), __low2float(hb0));
  x[1] = f2(__high2float(ha0), __high2float(hb0));
  x[2] = f2(__low2float(ha1), __low2float(hb1));
  x[3] = f2(__high2float(ha1), __high2float(hb1));
}

}  // namespace sq
