// sq_decode.cu -- the fused decode-step kernel of libsq (sm_100a).
//
// STEPQuant explainer, experimental-setup paragraph: at every decode step the packed state is
// unpacked, updated and written back by one fused kernel, and the row / column scales are
// refit on the updated state. Per (request, head) item:
//   the packed head block and q, k, v (alpha) arrive in shared memory by bulk copy, two items
//   ahead; unpack exact codes x; U_j = sum_i x_ij A_i k_i and P_j = sum_i x_ij A_i q_i
//   (A_i = alpha_i r16_i, so S'^T k = c * U); b = beta (v - c U); o = c P + b (k.q);
//   M_new_ij = x_ij (A_i c_j) + k_i b_j in registers; refit the dual-axis scales by
//   alternating max-abs passes; requantize, repack and store in place.
//
// Tile mapping (sq_tile.cuh): warp w owns key rows 16w..16w+15, lane l owns value columns
// 4l..4l+3. Row work stays inside a warp (warp redux for row maxima, per-row factors in
// warp-private shared memory); column sums and maxima combine the 8 warps' partials, which
// every lane reads for its own 4 columns. That leaves three CTA barriers per item, and
// rotating partial buffers let warps run into the next item without a closing barrier.
// Element pairs use the packed fp32x2 instructions of sm_100. Items run head-major with heads
// sorted by width, so the CTAs of an SM execute the same width-specialized code; 128 x 128
// tiles get a variant with a compile-time shape.
//
// Arithmetic: the refit follows the oracle's rule (row max / Q, w = 1/(r Q), column max of
// |S| w, fp16 rounding once) with hardware reciprocals (within 1 ulp) for the intermediate
// factors; the code multipliers 1/r16 and 1/c16 are correctly rounded as in the oracle. The
// state here is the GPU's own fp32 update, so its scales are compared with the oracle's
// through the codes they produce.
#include "sq_tile.cuh"

namespace sq {
namespace {
using namespace tile;

struct StageHdr {
  int32_t valid, slot, b, h;
  float beta, alpha;
  int32_t mode;  // width of the head's rows (0: per-row widths, 16: fp16 head)
  uint32_t off;  // byte offset of the head block within a slot
};

// Per-request metadata of the item whose copies are issued next; filled by cp.async one item
// earlier, so no thread waits on a dependent global load.
struct Meta {
  int32_t slot;
  float beta, alpha;
  int32_t pad;
};

// Flag words (per item parity): [0] non-finite input, [1] fp16 range overflow, [2] k.q.
enum { F_INPUT = 0, F_RANGE = 1, F_KQ = 2 };

// Shared memory: fixed-size arrays at compile-time offsets, then the two item stages.
constexpr uint32_t OFF_BAR = 0;                                  // 2 mbarriers
constexpr uint32_t OFF_FLAGS = 16;                               // [2 parities][4] ints
constexpr uint32_t OFF_META = 48;                                // Meta of the item to issue next
constexpr uint32_t OFF_REDA = 96;                                // [8 warps][2][128] U, P partials
constexpr uint32_t OFF_REDC = OFF_REDA + kWarps * 2 * kMaxD * 4;  // [2][8 warps][128] column maxima
constexpr uint32_t OFF_ROWG = OFF_REDC + 2 * kWarps * kMaxD * 4;  // float4 (gk, gk, gq, gq)
constexpr uint32_t OFF_ROWU = OFF_ROWG + kMaxD * 16;             // float4 (A, A, k, k)
constexpr uint32_t OFF_ROWW2 = OFF_ROWU + kMaxD * 16;            // float2 (w, w)
constexpr uint32_t OFF_ROWIR2 = OFF_ROWW2 + kMaxD * 8;           // float2 (1/r16, 1/r16)
constexpr uint32_t OFF_ROWTAB = OFF_ROWIR2 + kMaxD * 8;          // row descriptors (key-row units)
constexpr uint32_t OFF_ROWTMP = OFF_ROWTAB + kMaxD * 4;          // per warp: 16 maxima / fp16 scales
constexpr uint32_t OFF_COLC = OFF_ROWTMP + kWarps * kRows * 4;   // c16 of the item, as float
constexpr uint32_t OFF_COLV = OFF_COLC + kMaxD * 4;              // v of the item, as float
constexpr uint32_t OFF_STAGES = OFF_COLV + kMaxD * 4;            // multiple of 16

// One stage: header, k, q, v, (alpha), (row table), head block.
struct DPlan {
  uint32_t esz, k_off, q_off, v_off, al_off, rt_off, blk_off, stage, tab, total;
  __host__ __device__ DPlan(int dk, int dv, int io, int gate, int per_row, uint32_t stage_bytes,
                            int n_heads) {
    esz = io == 1 ? 2u : 4u;
    k_off = sizeof(StageHdr);
    q_off = k_off + dk * esz;
    v_off = q_off + dk * esz;
    al_off = v_off + dv * esz;
    rt_off = al_off + (gate == 1 ? 4u * dk : 0u);
    blk_off = rt_off + (per_row ? 4u * dk : 0u);  // all offsets multiples of 16
    stage = blk_off + round16(stage_bytes + kSlack);
    tab = OFF_STAGES + 2 * stage;  // head table: H HeadDesc, then H int32 (head order)
    total = tab + round16(20u * (uint32_t)n_heads);
  }
  __host__ __device__ uint32_t kqv_bytes() const { return blk_off - k_off; }
};

extern __shared__ __align__(16) uint8_t smem[];
template <typename T>
__device__ __forceinline__ T* sp(uint32_t off) {
  return reinterpret_cast<T*>(smem + off);
}

// Row geometry of a head block: fixed width (head units, pivot heads) or the row table.
template <int MODE>
struct Geo {
  uint32_t base, rb;
  __device__ Geo(int dk, int dv, const uint32_t*)
      : base(MODE == MODE_PIVOT ? 0u : 2u * (dk + dv)), rb((uint32_t)dv * MODE / 8) {}
  __device__ uint32_t off(int i) const { return base + (uint32_t)i * rb; }
  __device__ int width(int) const { return MODE; }
};
template <>
struct Geo<MODE_ROWS> {
  const uint32_t* tab;
  __device__ Geo(int, int, const uint32_t* t) : tab(t) {}
  __device__ uint32_t off(int i) const { return row_off(tab[i]); }
  __device__ int width(int i) const { return row_width(tab[i]); }
};

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 lo(const float4& v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi(const float4& v) { return make_float2(v.z, v.w); }

__device__ __forceinline__ float max3abs(float a, float b, float c) {  // max(|a|, |b|, |c|)
  float d;
  asm("max.abs.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float rcp_fast(float x) {  // |error| <= 1 ulp; x normal
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}
// The mbarrier's current phase also waits for this thread's earlier cp.async copies.
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Thread context; FULL = compile-time 128 x 128 tile (every row and lane in range).
template <bool FULL>
struct Ctx {
  int tid, warp, lane, dk_, dv_;
  bool act;
  uint32_t blk_off;  // shared-memory offset of the current head block
  int par;           // item parity: selects the flag words
  __device__ int dk() const { return FULL ? kMaxD : dk_; }
  __device__ int dv() const { return FULL ? kMaxD : dv_; }
  __device__ bool row_ok(int i) const { return FULL || i < dk_; }
  __device__ bool active() const { return FULL || act; }
  __device__ const uint8_t* blk() const { return smem + blk_off; }
  __device__ uint32_t* rowtab() const { return sp<uint32_t>(OFF_ROWTAB); }
  __device__ float4* rowG() const { return sp<float4>(OFF_ROWG); }
  __device__ float4* rowU() const { return sp<float4>(OFF_ROWU); }
  __device__ float2* rowW2() const { return sp<float2>(OFF_ROWW2); }
  __device__ float2* rowIR2() const { return sp<float2>(OFF_ROWIR2); }
  __device__ float* rowtmp() const { return sp<float>(OFF_ROWTMP); }
  __device__ float* redA() const { return sp<float>(OFF_REDA); }
  __device__ float* redC() const { return sp<float>(OFF_REDC); }
  __device__ int* flags() const { return sp<int>(OFF_FLAGS) + 4 * par; }
};

// Sum over the 8 warps of the partials in red[w * stride + 4 lane .. +3].
__device__ __forceinline__ float4 sum8(const float* red, int stride, int lane) {
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const float4 v = *reinterpret_cast<const float4*>(red + w * stride + 4 * lane);
    s.x += v.x;
    s.y += v.y;
    s.z += v.z;
    s.w += v.w;
  }
  return s;
}

__device__ __forceinline__ float4 max8(const float* red, int lane) {
  float4 m = *reinterpret_cast<const float4*>(red + 4 * lane);
#pragma unroll
  for (int w = 1; w < kWarps; w += 2) {
    const float4 a = *reinterpret_cast<const float4*>(red + w * kMaxD + 4 * lane);
    const float4 b = *reinterpret_cast<const float4*>(red + (w + 1 < kWarps ? w + 1 : w) * kMaxD + 4 * lane);
    m.x = max3(m.x, a.x, b.x);
    m.y = max3(m.y, a.y, b.y);
    m.z = max3(m.z, a.z, b.z);
    m.w = max3(m.w, a.w, b.w);
  }
  return make_float4(fmaxf(m.x, kScaleFloor), fmaxf(m.y, kScaleFloor), fmaxf(m.z, kScaleFloor),
                     fmaxf(m.w, kScaleFloor));
}

// Row pass of one alternation: r_i = max(max_j |S_ij| inv_c_j / Q_i, 2^-14), w_i = 1/(r_i Q_i)
// for the warp's 16 rows; lanes 0..15 hold r_i of row 16w + lane on return (0 for fp16 rows).
template <int MODE, bool FULL, bool FIRST>
__device__ __forceinline__ float row_pass(const float2 (&S)[kRows][2], const float4& icv,
                                          const Ctx<FULL>& c, const Geo<MODE>& geo,
                                          bool check_range) {
  float* tmp = c.rowtmp() + c.warp * kRows;
  float rm[kRows];
#pragma unroll
  for (int s = 0; s < kRows; ++s) {
    float2 p = S[s][0], q = S[s][1];
    if (!FIRST) {
      p = __fmul2_rn(p, lo(icv));
      q = __fmul2_rn(q, hi(icv));
    }
    rm[s] = warp_max_nonneg(fmaxf(max3abs(p.x, p.y, q.x), fabsf(q.y)));
  }
  if (c.lane == 0) {
#pragma unroll
    for (int s = 0; s < kRows; s += 4)
      *reinterpret_cast<float4*>(tmp + s) = make_float4(rm[s], rm[s + 1], rm[s + 2], rm[s + 3]);
  }
  __syncwarp();
  float r = 0.f;
  if (c.lane < kRows) {
    const int i = c.warp * kRows + c.lane;
    float w = 0.f;
    if (c.row_ok(i)) {
      const int b = geo.width(i);
      const float m = tmp[c.lane];
      if (b != 16) {
        const float Q = (float)q_of_width(b);
        const float invQ = MODE == MODE_ROWS ? rcp_fast(Q) : 1.0f / (float)q_of_width(MODE);
        r = fmaxf(m * invQ, kScaleFloor);
        w = rcp_fast(r * Q);
        if (check_range && r >= 65520.f) atomicOr(&c.flags()[F_RANGE], 1);
        r = fminf(r, 65504.f);  // the largest finite fp16 value
      } else if (check_range && m >= 65520.f) {
        atomicOr(&c.flags()[F_RANGE], 1);
      }
    }
    c.rowW2()[i] = f2(w, w);
  }
  __syncwarp();
  return r;
}

// Column pass partials: max_i |S_ij| w_i over the warp's rows, written to red[warp].
template <bool FULL>
__device__ __forceinline__ void col_pass(const float2 (&S)[kRows][2], const Ctx<FULL>& c,
                                         float* red) {
  float cm0 = 0.f, cm1 = 0.f, cm2 = 0.f, cm3 = 0.f;
  const float4* w2 = reinterpret_cast<const float4*>(c.rowW2() + c.warp * kRows);
#pragma unroll
  for (int s = 0; s < kRows; s += 2) {
    const float4 ww = w2[s / 2];  // (w_s, w_s, w_s+1, w_s+1)
    const float2 a0 = __fmul2_rn(S[s][0], lo(ww));
    const float2 b0 = __fmul2_rn(S[s + 1][0], hi(ww));
    const float2 a1 = __fmul2_rn(S[s][1], lo(ww));
    const float2 b1 = __fmul2_rn(S[s + 1][1], hi(ww));
    cm0 = max3abs(cm0, a0.x, b0.x);
    cm1 = max3abs(cm1, a0.y, b0.y);
    cm2 = max3abs(cm2, a1.x, b1.x);
    cm3 = max3abs(cm3, a1.y, b1.y);
  }
  *reinterpret_cast<float4*>(red + c.warp * kMaxD + 4 * c.lane) = make_float4(cm0, cm1, cm2, cm3);
}

// The width-specialized part of one item. Returns after storing the requantized block (or
// skipping it on a flagged item). Contains exactly three __syncthreads for fit_iters = 2
// (1 + fit_iters in general); `after_first_barrier` runs right after the first.
template <int MODE, bool FULL, bool WANT_STATE, class AfterFirst>
__device__ __forceinline__ void item_body(const StepArgs& a, const Ctx<FULL>& c, float beta,
                                          int io, uint8_t* dst, AfterFirst after_first_barrier) {
  const Geo<MODE> geo(c.dk(), c.dv(), c.rowtab());

  // ---- pass A: exact codes, partial dot products ----
  float2 S[kRows][2];
  {
    float4 icv = make_float4(1.f, 1.f, 1.f, 1.f);
    if (MODE == MODE_ROWS && c.active()) {  // 1/c16 of the lane's columns, for fp16 rows
      const uint2 ch = reinterpret_cast<const uint2*>(c.blk() + 2 * c.dk())[c.lane];
      const float2 a01 = __half22float2(*reinterpret_cast<const __half2*>(&ch.x));
      const float2 a23 = __half22float2(*reinterpret_cast<const __half2*>(&ch.y));
      icv = make_float4(rcp_fast(a01.x), rcp_fast(a01.y), rcp_fast(a23.x), rcp_fast(a23.y));
    }
    float2 U0 = f2(0.f, 0.f), U1 = U0, P0 = U0, P1 = U0;
#pragma unroll
    for (int s = 0; s < kRows; ++s) {
      const int i = c.warp * kRows + s;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (c.row_ok(i)) {
        const int b = geo.width(i);
        if (c.active()) {
          const uint8_t* row = c.blk() + geo.off(i);
          if constexpr (MODE == MODE_ROWS)
            unpack4_rt(b, row, c.lane, x);
          else
            unpack4<MODE>(row, c.lane, x);
        }
        S[s][0] = f2(x[0], x[1]);
        S[s][1] = f2(x[2], x[3]);
        if (MODE == MODE_ROWS && b == 16) {  // fp16 row inside a scaled head: x = value / c_j
          S[s][0] = __fmul2_rn(S[s][0], lo(icv));
          S[s][1] = __fmul2_rn(S[s][1], hi(icv));
        }
        const float4 g = c.rowG()[i];  // (gk, gk, gq, gq)
        U0 = __ffma2_rn(S[s][0], lo(g), U0);
        U1 = __ffma2_rn(S[s][1], lo(g), U1);
        P0 = __ffma2_rn(S[s][0], hi(g), P0);
        P1 = __ffma2_rn(S[s][1], hi(g), P1);
      } else {
        S[s][0] = S[s][1] = f2(0.f, 0.f);
      }
    }
    *reinterpret_cast<float4*>(c.redA() + c.warp * 2 * kMaxD + 4 * c.lane) =
        make_float4(U0.x, U0.y, U1.x, U1.y);
    *reinterpret_cast<float4*>(c.redA() + c.warp * 2 * kMaxD + kMaxD + 4 * c.lane) =
        make_float4(P0.x, P0.y, P1.x, P1.y);
  }
  __syncthreads();  // barrier 1: partial dot products, input flags
  after_first_barrier();
  if (c.flags()[F_INPUT]) {  // non-finite input somewhere in the item: skip it
    if (c.tid == 0) atomicOr(a.flag, SQ_FLAG_NONFINITE_BIT);
    if (c.warp == 0 && c.active())
      *reinterpret_cast<float4*>(a.out + (size_t)io * c.dv() + 4 * c.lane) =
          make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                      __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
    return;
  }
  const float4 cv = sp<float4>(OFF_COLC)[c.lane];
  const float kq = __int_as_float(c.flags()[F_KQ]);
  float4 bv;
  {
    const float4 vv = sp<float4>(OFF_COLV)[c.lane];
    const float4 U = sum8(c.redA(), 2 * kMaxD, c.lane);
    const float4 Pp = sum8(c.redA() + kMaxD, 2 * kMaxD, c.lane);
    bv = make_float4(beta * (vv.x - cv.x * U.x), beta * (vv.y - cv.y * U.y),
                     beta * (vv.z - cv.z * U.z), beta * (vv.w - cv.w * U.w));
    if (c.warp == 0 && c.active())
      *reinterpret_cast<float4*>(a.out + (size_t)io * c.dv() + 4 * c.lane) =
          make_float4(__fmaf_rn(bv.x, kq, cv.x * Pp.x), __fmaf_rn(bv.y, kq, cv.y * Pp.y),
                      __fmaf_rn(bv.z, kq, cv.z * Pp.z), __fmaf_rn(bv.w, kq, cv.w * Pp.w));
  }

  // ---- pass B: M_new = x (A_i c_j) + k_i b_j ----
#pragma unroll
  for (int s = 0; s < kRows; ++s) {
    const int i = c.warp * kRows + s;
    if (c.row_ok(i) && c.active()) {
      const float4 u = c.rowU()[i];  // (A, A, k, k)
      S[s][0] = __ffma2_rn(S[s][0], __fmul2_rn(lo(u), lo(cv)), __fmul2_rn(hi(u), lo(bv)));
      S[s][1] = __ffma2_rn(S[s][1], __fmul2_rn(lo(u), hi(cv)), __fmul2_rn(hi(u), hi(bv)));
    }
  }
  if (WANT_STATE) {
    float* sn = a.s_new + (size_t)io * c.dk() * c.dv();
#pragma unroll
    for (int s = 0; s < kRows; ++s) {
      const int i = c.warp * kRows + s;
      if (c.row_ok(i) && c.active())
        *reinterpret_cast<float4*>(sn + (size_t)i * c.dv() + 4 * c.lane) =
            make_float4(S[s][0].x, S[s][0].y, S[s][1].x, S[s][1].y);
    }
  }

  if constexpr (MODE == MODE_PIVOT) {
    // fp16 head: range check, then round and store
    bool of = false;
#pragma unroll
    for (int s = 0; s < kRows; ++s) {
      const float v[4] = {S[s][0].x, S[s][0].y, S[s][1].x, S[s][1].y};
      if (c.row_ok(c.warp * kRows + s) && c.active()) of |= f16_overflows(v);
    }
    if (of) atomicOr(&c.flags()[F_RANGE], 1);
    __syncthreads();
    if (c.flags()[F_RANGE]) {
      if (c.tid == 0) atomicOr(a.flag, SQ_FLAG_RANGE_BIT);
      return;
    }
#pragma unroll
    for (int s = 0; s < kRows; ++s) {
      const int i = c.warp * kRows + s;
      const float v[4] = {S[s][0].x, S[s][0].y, S[s][1].x, S[s][1].y};
      if (c.row_ok(i)) store4_f16(dst + geo.off(i), c.lane, v, c.active());
    }
  } else {
    // ---- refit: alternating row / column max-abs passes ----
    float r = row_pass<MODE, FULL, true>(S, make_float4(1.f, 1.f, 1.f, 1.f), c, geo, true);
    if (MODE == MODE_ROWS) {  // fp16 rows must fit in fp16
      bool of = false;
#pragma unroll
      for (int s = 0; s < kRows; ++s) {
        const int i = c.warp * kRows + s;
        const float v[4] = {S[s][0].x, S[s][0].y, S[s][1].x, S[s][1].y};
        if (c.row_ok(i) && c.active() && geo.width(i) == 16) of |= f16_overflows(v);
      }
      if (of) atomicOr(&c.flags()[F_RANGE], 1);
    }
    col_pass(S, c, c.redC());
    __syncthreads();  // barrier 2
    float4 cm = max8(c.redC(), c.lane);
    for (int it = 1; it < a.fit_iters; ++it) {
      const float4 icv = make_float4(rcp_fast(cm.x), rcp_fast(cm.y), rcp_fast(cm.z), rcp_fast(cm.w));
      r = row_pass<MODE, FULL, false>(S, icv, c, geo, false);
      float* red = c.redC() + (it & 1) * kWarps * kMaxD;
      col_pass(S, c, red);
      __syncthreads();  // barrier 3 (fit_iters = 2)
      cm = max8(red, c.lane);
    }
    if (c.flags()[F_RANGE]) {
      if (c.tid == 0) atomicOr(a.flag, SQ_FLAG_RANGE_BIT);
      return;
    }
    // ---- fp16 scales, quantize, pack, store ----
    const __half2 c01 = __floats2half2_rn(cm.x, cm.y), c23 = __floats2half2_rn(cm.z, cm.w);
    const float2 fc01 = __half22float2(c01), fc23 = __half22float2(c23);
    // the code multipliers are correctly rounded, as in the oracle
    const float2 ic01 = f2(__frcp_rn(fc01.x), __frcp_rn(fc01.y));
    const float2 ic23 = f2(__frcp_rn(fc23.x), __frcp_rn(fc23.y));
    __half* r16s = reinterpret_cast<__half*>(c.rowtmp() + c.warp * kRows);
    if (c.lane < kRows) {
      const int i = c.warp * kRows + c.lane;
      const __half r16 = __float2half_rn(r);
      const float ir = r > 0.f ? __frcp_rn(__half2float(r16)) : 0.f;
      c.rowIR2()[i] = f2(ir, ir);
      r16s[c.lane] = r16;
    }
    __syncwarp();
    if (c.lane < 2 && c.row_ok(c.warp * kRows + 8 * c.lane))
      reinterpret_cast<uint4*>(dst)[2 * c.warp + c.lane] = reinterpret_cast<const uint4*>(r16s)[c.lane];
    if (c.warp == 0 && c.active()) {
      uint2 cc;
      cc.x = *reinterpret_cast<const uint32_t*>(&c01);
      cc.y = *reinterpret_cast<const uint32_t*>(&c23);
      reinterpret_cast<uint2*>(dst + 2 * c.dk())[c.lane] = cc;
    }
#pragma unroll
    for (int s = 0; s < kRows; ++s) {
      const int i = c.warp * kRows + s;
      if (c.row_ok(i)) {
        uint8_t* row = dst + geo.off(i);
        const int b = geo.width(i);
        if (MODE == MODE_ROWS && b == 16) {
          const float v[4] = {S[s][0].x, S[s][0].y, S[s][1].x, S[s][1].y};
          store4_f16(row, c.lane, v, c.active());
        } else {
          const float2 ir = c.rowIR2()[i];
          const float mgv = kMagic + (float)(1 << (b - 1));
          const float2 mg = f2(mgv, mgv);
          const float2 y0 = __ffma2_rn(__fmul2_rn(S[s][0], ir), ic01, mg);
          const float2 y1 = __ffma2_rn(__fmul2_rn(S[s][1], ir), ic23, mg);
          const float y[4] = {y0.x, y0.y, y1.x, y1.y};
          if constexpr (MODE == MODE_ROWS) {
            switch (b) {
              case 2: store4<2>(row, c.lane, y, c.active()); break;
              case 4: store4<4>(row, c.lane, y, c.active()); break;
              case 6: store4<6>(row, c.lane, y, c.active()); break;
              default: store4<8>(row, c.lane, y, c.active()); break;
            }
          } else {
            store4<MODE>(row, c.lane, y, c.active());
          }
        }
      }
    }
  }
}

template <int GATE, int IO, bool WANT_STATE, bool FULL>
__global__ void __launch_bounds__(kThreads, 2) k_decode(const StepArgs a) {
  const DPlan P(FULL ? kMaxD : a.dk, FULL ? kMaxD : a.dv, IO, GATE, a.per_row, a.stage_bytes, a.H);
  uint64_t* bar = sp<uint64_t>(OFF_BAR);
  Ctx<FULL> c;
  c.tid = threadIdx.x;
  c.warp = c.tid >> 5;
  c.lane = c.tid & 31;
  c.dk_ = a.dk;
  c.dv_ = a.dv;
  c.act = 4 * c.lane < a.dv;
  const int H = a.H, B = a.batch, dk = c.dk(), dv = c.dv(), tid = c.tid;
  const int n_items = B * H;
  const int stride = gridDim.x;

  if (tid == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  if (tid < 8) sp<int>(OFF_FLAGS)[tid] = 0;
  __syncthreads();

  // Head descriptors and head order, staged once per CTA.
  HeadDesc* htab = reinterpret_cast<HeadDesc*>(smem + P.tab);
  int32_t* otab = reinterpret_cast<int32_t*>(smem + P.tab + 16u * H);
  for (int h = tid; h < H; h += kThreads) {
    htab[h] = a.heads[h];
    otab[h] = a.order[h];
  }
  __syncthreads();

  // Items run head-major in the order of otab: item = hh * B + b.
  Meta* meta = sp<Meta>(OFF_META);
  auto fetch_meta = [&](int item) {  // thread 0: async copies of the item's per-request words
    const int hh = item / B, b = item - hh * B, io = b * H + otab[hh];
    cp_async4(&meta->slot, a.slot_idx + b);
    cp_async4(&meta->beta, a.beta + io);
    if (GATE == 0) cp_async4(&meta->alpha, a.alpha + io);
    cp_async_commit();
  };
  // Warp 0: stage an item into stage s. The per-request words of the item are in *meta
  // (copied by lane 0 one item earlier). q, k, v, alpha and the row table move as 16-byte
  // cp.async chunks spread over the warp, tracked by the stage's mbarrier; lane 0 issues the
  // bulk copy of the head block.
  auto issue = [&](int item, int s) {
    if (c.lane == 0) cp_async_wait_all();
    __syncwarp();
    const int hh = item / B, b = item - hh * B, h = otab[hh], io = b * H + h;
    const HeadDesc hd = htab[h];
    uint8_t* st = smem + OFF_STAGES + s * P.stage;
    const int slot = meta->slot;
    const bool valid = slot >= 0 && slot < a.n_slots;
    const int nk = dk * P.esz / 16, nv = dv * P.esz / 16, na = GATE == 1 ? dk / 4 : 0;
    const int nr = a.per_row ? dk / 4 : 0;
    const int total = 2 * nk + nv + na + nr;
    for (int ch = c.lane; ch < total; ch += 32) {
      const uint8_t* src;
      uint8_t* dst;
      int x = ch;
      if (x < nk) {
        src = static_cast<const uint8_t*>(a.k) + (size_t)io * dk * P.esz;
        dst = st + P.k_off;
      } else if ((x -= nk) < nk) {
        src = static_cast<const uint8_t*>(a.q) + (size_t)io * dk * P.esz;
        dst = st + P.q_off;
      } else if ((x -= nk) < nv) {
        src = static_cast<const uint8_t*>(a.v) + (size_t)io * dv * P.esz;
        dst = st + P.v_off;
      } else if ((x -= nv) < na) {
        src = reinterpret_cast<const uint8_t*>(a.alpha + (size_t)io * dk);
        dst = st + P.al_off;
      } else {
        x -= na;
        src = reinterpret_cast<const uint8_t*>(a.rows + (size_t)h * dk);
        dst = st + P.rt_off;
      }
      cp_async16(dst + 16 * x, src + 16 * x);
    }
    cp_async_mbar_arrive(&bar[s]);
    __syncwarp();
    if (c.lane == 0) {
      StageHdr* hdr = reinterpret_cast<StageHdr*>(st);
      hdr->valid = valid;
      hdr->slot = slot;
      hdr->b = b;
      hdr->h = h;
      hdr->beta = meta->beta;
      hdr->alpha = GATE == 0 ? meta->alpha : 0.f;
      hdr->mode = hd.pivot_head ? (int)MODE_PIVOT : (int)hd.width;
      hdr->off = hd.off;
      mbar_arrive_expect_tx(&bar[s], valid ? hd.bytes : 0u);
      if (valid)
        bulk_load(st + P.blk_off, a.pool + (size_t)slot * a.slot_bytes + hd.off, hd.bytes, &bar[s]);
    }
  };

  // Prologue: this CTA's first two items in flight, the third one's words on their way.
  const int first = blockIdx.x;
  if (c.warp == 0) {
    if (first < n_items) {
      if (c.lane == 0) fetch_meta(first);
      issue(first, 0);
    }
    if (first + stride < n_items) {
      if (c.lane == 0) fetch_meta(first + stride);
      issue(first + stride, 1);
    }
    if (first + 2 * stride < n_items && c.lane == 0) fetch_meta(first + 2 * stride);
  }

  int it = 0;
  for (int item = first; item < n_items; item += stride, ++it) {
    const int s = it & 1;
    if (!mbar_wait_bounded(&bar[s], (it >> 1) & 1)) {
      if (tid == 0) atomicOr(a.flag, SQ_FLAG_TIMEOUT_BIT);
      return;
    }
    const uint32_t st_off = OFF_STAGES + s * P.stage;
    const uint8_t* st = smem + st_off;
    const StageHdr hdr = *reinterpret_cast<const StageHdr*>(st);
    const int io = hdr.b * H + hdr.h;
    c.blk_off = st_off + P.blk_off;
    c.par = s;
    const bool pivot_head = hdr.mode == MODE_PIVOT;

    // Issued after the first barrier of the item, when no thread reads stage s any more: the
    // item two strides ahead into stage s, and the metadata of the one after it.
    auto refill = [&]() {
      if (c.warp == 0) {
        if (item + 2 * stride < n_items) issue(item + 2 * stride, s);
        if (c.lane == 0) {
          if (item + 3 * stride < n_items) fetch_meta(item + 3 * stride);
          int* f = sp<int>(OFF_FLAGS) + 4 * (s ^ 1);  // the next item's words
          f[F_INPUT] = f[F_RANGE] = 0;
        }
      }
    };

    if (!hdr.valid) {  // bad slot: skip the item
      if (tid == 0) atomicOr(a.flag, SQ_FLAG_BAD_SLOT_BIT);
      if (tid < dv) a.out[(size_t)io * dv + tid] = __int_as_float(0x7fc00000);
      __syncthreads();
      refill();
      continue;
    }

    // ---- per-item setup: each warp its own rows' factors; warp 0 the column data ----
    const uint8_t* kq = st + P.k_off;
    const uint8_t* qq = st + P.q_off;
    bool bad_in = false;
    if (c.lane < kRows) {
      const int i = c.warp * kRows + c.lane;
      float4 g = make_float4(0.f, 0.f, 0.f, 0.f), u = g;
      if (c.row_ok(i)) {
        uint32_t desc = 0;
        if (a.per_row) {
          desc = reinterpret_cast<const uint32_t*>(st + P.rt_off)[i];
          c.rowtab()[i] = desc;
        }
        const float ki = ld_io(kq, IO, i), qi = ld_io(qq, IO, i);
        const float ai = GATE == 0 ? hdr.alpha : reinterpret_cast<const float*>(st + P.al_off)[i];
        bad_in |= !isfinite(ki) || !isfinite(qi) || !isfinite(ai);
        const bool qrow = !pivot_head && (!a.per_row || row_width(desc) != 16);
        const float A = qrow ? ai * __half2float(reinterpret_cast<const __half*>(c.blk())[i]) : ai;
        g = make_float4(A * ki, A * ki, A * qi, A * qi);
        u = make_float4(A, A, ki, ki);
      }
      c.rowG()[i] = g;
      c.rowU()[i] = u;
    }
    if (c.warp == 0) {
      float4 cv = make_float4(1.f, 1.f, 1.f, 1.f), vv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c.active()) {
        if (!pivot_head) {
          const uint2 ch = reinterpret_cast<const uint2*>(c.blk() + 2 * dk)[c.lane];
          const float2 a01 = __half22float2(*reinterpret_cast<const __half2*>(&ch.x));
          const float2 a23 = __half22float2(*reinterpret_cast<const __half2*>(&ch.y));
          cv = make_float4(a01.x, a01.y, a23.x, a23.y);
        }
        const uint8_t* vq = st + P.v_off;
        vv = make_float4(ld_io(vq, IO, 4 * c.lane), ld_io(vq, IO, 4 * c.lane + 1),
                         ld_io(vq, IO, 4 * c.lane + 2), ld_io(vq, IO, 4 * c.lane + 3));
        bad_in |= !(isfinite(vv.x) && isfinite(vv.y) && isfinite(vv.z) && isfinite(vv.w));
      }
      sp<float4>(OFF_COLC)[c.lane] = cv;
      sp<float4>(OFF_COLV)[c.lane] = vv;
      bad_in |= !isfinite(hdr.beta) || (GATE == 0 && !isfinite(hdr.alpha));
    }
    if (bad_in) atomicOr(&c.flags()[F_INPUT], 1);
    if (c.warp == 0) {  // k.q, read by every warp after the first barrier
      float kqs = 0.f;
#pragma unroll
      for (int t = 0; t < kMaxD / 32; ++t) {
        const int i = c.lane + 32 * t;
        if (FULL || i < dk) kqs = __fmaf_rn(ld_io(kq, IO, i), ld_io(qq, IO, i), kqs);
      }
      kqs = warp_sum(kqs);
      if (c.lane == 0) c.flags()[F_KQ] = __float_as_int(kqs);
    }
    __syncwarp();

    const float beta = hdr.beta;
    uint8_t* dst = a.pool + (size_t)hdr.slot * a.slot_bytes + hdr.off;
    switch (hdr.mode) {
      case MODE_W2: item_body<MODE_W2, FULL, WANT_STATE>(a, c, beta, io, dst, refill); break;
      case MODE_W4: item_body<MODE_W4, FULL, WANT_STATE>(a, c, beta, io, dst, refill); break;
      case MODE_W6: item_body<MODE_W6, FULL, WANT_STATE>(a, c, beta, io, dst, refill); break;
      case MODE_W8: item_body<MODE_W8, FULL, WANT_STATE>(a, c, beta, io, dst, refill); break;
      case MODE_PIVOT: item_body<MODE_PIVOT, FULL, WANT_STATE>(a, c, beta, io, dst, refill); break;
      default: item_body<MODE_ROWS, FULL, WANT_STATE>(a, c, beta, io, dst, refill); break;
    }
  }
}

template <int GATE, int IO, bool WS, bool FULL>
cudaError_t launch_t(const StepArgs& a, int num_sms, cudaStream_t st) {
  const DPlan P(a.dk, a.dv, IO, GATE, a.per_row, a.stage_bytes, a.H);
  auto fn = k_decode<GATE, IO, WS, FULL>;
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

template <int GATE, int IO, bool WS>
cudaError_t launch_shape(const StepArgs& a, int num_sms, cudaStream_t st) {
  if (a.dk == kMaxD && a.dv == kMaxD) return launch_t<GATE, IO, WS, true>(a, num_sms, st);
  return launch_t<GATE, IO, WS, false>(a, num_sms, st);
}

}  // namespace

cudaError_t launch_decode(const StepArgs& a, int gate, int io, bool want_state, int num_sms,
                          cudaStream_t st) {
  if (gate == 0 && io == 0)
    return want_state ? launch_shape<0, 0, true>(a, num_sms, st) : launch_shape<0, 0, false>(a, num_sms, st);
  if (gate == 0 && io == 1)
    return want_state ? launch_shape<0, 1, true>(a, num_sms, st) : launch_shape<0, 1, false>(a, num_sms, st);
  if (gate == 1 && io == 0)
    return want_state ? launch_shape<1, 0, true>(a, num_sms, st) : launch_shape<1, 0, false>(a, num_sms, st);
  return want_state ? launch_shape<1, 1, true>(a, num_sms, st) : launch_shape<1, 1, false>(a, num_sms, st);
}

}  // namespace sq
