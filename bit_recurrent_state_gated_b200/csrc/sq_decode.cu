// sq_decode.cu -- the fused decode-step kernel of libsq (sm_100a).
//
// STEPQuant explainer, experimental-setup paragraph: at every decode step the packed state is
// unpacked, updated and written back by one fused kernel, and the row / column scales are
// refit on the updated state. Per (request, head) item:
//   the packed head block and q, k, v (alpha) arrive in shared memory by bulk copy; unpack
//   exact codes x; U_j = sum_i x_ij A_i k_i and P_j = sum_i x_ij A_i q_i (A_i = alpha_i r16_i,
//   so S'^T k = c * U); b = beta (v - c U); o = c P + b (k.q); M_new_ij = x_ij (A_i c_j) +
//   k_i b_j; refit the dual-axis scales by alternating max-abs passes; requantize, repack and
//   store in place.
//
// Where the tile lives. Each thread owns 16 key rows x 4 value columns of the 128 x 128 fp32
// tile (warp w: rows 16w..16w+15, lane l: columns 4l..4l+3), and keeps its 64 values in the
// SM's tensor memory, not in registers: the CTA allocates 128 tensor-memory columns, and
// thread t of warp w uses columns 64 (w / 4) .. + 63 of lane 32 (w % 4) + t. Every pass over
// the tile streams 4-row chunks (16 values) through registers with one tcgen05.ld and, where
// the pass changes the tile, one tcgen05.st. With the tile out of the register file a CTA
// needs few registers, so three or four CTAs share an SM (four tiles fill the 512 columns)
// and each one's barrier and load latency is covered by the others' passes; the passes are
// loops, which keeps the instruction footprint small.
//
// Row work stays inside a warp (warp redux for row maxima, per-row factors in warp-private
// shared memory); column sums and maxima combine the 8 warps' partials. Three CTA barriers per
// item (fit_iters = 2). One lane issues the bulk copies of the next item into the single
// stage right after the first barrier, so the copy overlaps the item's remaining passes.
//
// Arithmetic: the refit follows the oracle's rule step for step with correctly rounded
// operations (r_i = max(m_i / Q_i, 2^-14), w_i = 1/(r_i Q_i), c_j = max(max_i |S_ij| w_i,
// 2^-14), v_j = 1/c_j, fp16 rounding once); the code multipliers 1/r16 and 1/c16 are correctly
// rounded as well. The state is the GPU's own fp32 update (fused multiply-adds), so its scales
// and codes are compared with the oracle's within the stated agreement.
#include "sq_tile.cuh"

namespace sq {
namespace {
using namespace tile;

constexpr uint32_t kTmemCols = 128;  // 8 warps x 32 lanes x 64 values = 128 lanes x 128 columns
constexpr int kMaxCtasPerSm = 4;     // 4 x 128 columns: the SM's whole tensor memory
constexpr int kChunks = kRows / 4;   // 4-row chunks per warp and pass

struct StageHdr {
  int32_t valid, slot, b, h;
  float beta, alpha;
  int32_t mode;  // width of the head's rows (0: per-row widths, 16: fp16 head)
  uint32_t off;  // byte offset of the head block within a slot
};

// Per-request words of the item issued next; copied by cp.async one item earlier.
struct Meta {
  int32_t slot;
  float beta, alpha;
  int32_t pad;
};

// Flag words of an item: [0] non-finite input, [1] fp16 range overflow.
enum { F_INPUT = 0, F_RANGE = 1 };

// Shared memory: fixed-size arrays at compile-time offsets, then the stage and the head table.
constexpr uint32_t OFF_BAR = 0;                                   // stage mbarriers (<= 2)
constexpr uint32_t OFF_TMEM = 16;                                 // tensor-memory base address
constexpr uint32_t OFF_FLAGS = 32;                                // [4 items][4] ints
constexpr uint32_t OFF_META = 96;                                 // Meta
constexpr uint32_t OFF_REDA = 112;                                // [8 warps][2][128] U, P
constexpr uint32_t OFF_REDC = OFF_REDA + kWarps * 2 * kMaxD * 4;  // [2][8 warps][128] col maxima
constexpr uint32_t OFF_ROWG = OFF_REDC + 2 * kWarps * kMaxD * 4;  // float4 (gk, gk, gq, gq)
constexpr uint32_t OFF_ROWU = OFF_ROWG + kMaxD * 16;              // float4 (A, A, k, k)
constexpr uint32_t OFF_ROWW2 = OFF_ROWU + kMaxD * 16;             // float2 (w, w)
constexpr uint32_t OFF_ROWIR2 = OFF_ROWW2 + kMaxD * 8;            // float2 (1/r16, 1/r16)
constexpr uint32_t OFF_ROWTAB = OFF_ROWIR2 + kMaxD * 8;           // row descriptors
constexpr uint32_t OFF_ROWTMP = OFF_ROWTAB + kMaxD * 4;           // per warp: 16 maxima / r16
constexpr uint32_t OFF_COLC = OFF_ROWTMP + kWarps * kRows * 4;    // c16 of the item, as float
constexpr uint32_t OFF_COLV = OFF_COLC + kMaxD * 4;               // v of the item, as float
constexpr uint32_t OFF_KQP = OFF_COLV + kMaxD * 4;                // per-warp partials of k.q
constexpr uint32_t OFF_STAGE = OFF_KQP + kWarps * 4;              // multiple of 16
static_assert(OFF_STAGE % 16 == 0 && OFF_REDA % 16 == 0, "16-byte aligned regions");

// A stage: header, k, q, v, (alpha), (row table), head block (offsets within the stage); one
// or two stages, then the head table.
struct DPlan {
  uint32_t esz, k_off, q_off, v_off, al_off, rt_off, blk_off, stage, tab, total;
  __host__ __device__ DPlan(int dk, int dv, int io, int gate, int per_row, uint32_t stage_bytes,
                            int n_heads, int n_stages) {
    esz = io == 1 ? 2u : 4u;
    k_off = (uint32_t)sizeof(StageHdr);
    q_off = k_off + dk * esz;
    v_off = q_off + dk * esz;
    al_off = v_off + dv * esz;
    rt_off = al_off + (gate == 1 ? 4u * dk : 0u);
    blk_off = rt_off + (per_row ? 4u * dk : 0u);  // all offsets multiples of 16
    stage = blk_off + round16(stage_bytes + kSlack);
    tab = OFF_STAGE + (uint32_t)n_stages * stage;
    total = tab + round16(20u * (uint32_t)n_heads);
  }
};

extern __shared__ __align__(16) uint8_t smem[];
template <typename T>
__device__ __forceinline__ T* sp(uint32_t off) {
  return reinterpret_cast<T*>(smem + off);
}

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

__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_addr(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Thread context of one item; FULL = compile-time 128 x 128 tile (every row and lane active).
template <bool FULL>
struct Ctx {
  int tid, warp, lane, dk_, dv_;
  bool act_;   // the lane's columns are < d_v
  bool wact_;  // the warp's rows are < d_k (d_k is a multiple of 16)
  __device__ int dk() const { return FULL ? kMaxD : dk_; }
  __device__ int dv() const { return FULL ? kMaxD : dv_; }
  __device__ bool act() const { return FULL || act_; }
  __device__ bool wact() const { return FULL || wact_; }
  const uint8_t* blk;
  int* flags;  // the item's flag words
  uint32_t tm;  // tensor-memory address of the thread's 64 values
  __device__ float4* rowG() const { return sp<float4>(OFF_ROWG); }
  __device__ float4* rowU() const { return sp<float4>(OFF_ROWU); }
  __device__ float2* rowW2() const { return sp<float2>(OFF_ROWW2); }
  __device__ float2* rowIR2() const { return sp<float2>(OFF_ROWIR2); }
  __device__ uint32_t* rowtab() const { return sp<uint32_t>(OFF_ROWTAB); }
  __device__ float* rowtmp() const { return sp<float>(OFF_ROWTMP) + warp * kRows; }
  __device__ int row0() const { return warp * kRows; }
};

// Row geometry of a head block: fixed width (head units, fp16 heads) or the row table.
template <int MODE>
struct Geo {
  uint32_t base, rb;
  template <bool FULL>
  __device__ Geo(const Ctx<FULL>& c)
      : base(MODE == MODE_PIVOT ? 0u : 2u * (c.dk() + c.dv())), rb((uint32_t)c.dv() * MODE / 8) {}
  __device__ uint32_t off(int i) const { return base + (uint32_t)i * rb; }
  __device__ int width(int) const { return MODE; }
};
template <>
struct Geo<MODE_ROWS> {
  const uint32_t* tab;
  template <bool FULL>
  __device__ Geo(const Ctx<FULL>& c) : tab(c.rowtab()) {}
  __device__ uint32_t off(int i) const { return row_off(tab[i]); }
  __device__ int width(int i) const { return row_width(tab[i]); }
};

// Sum / max over the 8 warps of the partials in red[w * stride + 4 lane .. +3].
__device__ __forceinline__ float4 sum8(const float* red, int stride, int lane) {
  float2 a = f2(0.f, 0.f), b = a;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    const float4 v = *reinterpret_cast<const float4*>(red + w * stride + 4 * lane);
    a = __fadd2_rn(a, lo(v));
    b = __fadd2_rn(b, hi(v));
  }
  return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float4 max8(const float* red, int lane) {
  float4 m = *reinterpret_cast<const float4*>(red + 4 * lane);
#pragma unroll
  for (int w = 1; w < kWarps; w += 2) {
    const float4 a = *reinterpret_cast<const float4*>(red + w * kMaxD + 4 * lane);
    const float4 b =
        *reinterpret_cast<const float4*>(red + (w + 1 < kWarps ? w + 1 : w) * kMaxD + 4 * lane);
    m.x = max3(m.x, a.x, b.x);
    m.y = max3(m.y, a.y, b.y);
    m.z = max3(m.z, a.z, b.z);
    m.w = max3(m.w, a.w, b.w);
  }
  return make_float4(fmaxf(m.x, kScaleFloor), fmaxf(m.y, kScaleFloor), fmaxf(m.z, kScaleFloor),
                     fmaxf(m.w, kScaleFloor));
}

// ---- pass A: exact codes into tensor memory, partial dot products -------------------------
template <int MODE, bool FULL>
__device__ __forceinline__ void pass_a(const Ctx<FULL>& c) {
  const Geo<MODE> geo(c);
  // two accumulator sets (even / odd rows) halve the dependent-add chains
  float2 U0 = f2(0.f, 0.f), U1 = U0, P0 = U0, P1 = U0, U2 = U0, U3 = U0, P2 = U0, P3 = U0;
  if (c.wact()) {
    float4 icv = make_float4(1.f, 1.f, 1.f, 1.f);
    if (MODE == MODE_ROWS && c.act()) {  // 1/c16 of the lane's columns, for fp16 rows
      const uint2 ch = reinterpret_cast<const uint2*>(c.blk + 2 * c.dk())[c.lane];
      const float2 a01 = __half22float2(*reinterpret_cast<const __half2*>(&ch.x));
      const float2 a23 = __half22float2(*reinterpret_cast<const __half2*>(&ch.y));
      icv = make_float4(rcp_f16val(a01.x), rcp_f16val(a01.y), rcp_f16val(a23.x), rcp_f16val(a23.y));
    }
#pragma unroll 1
    for (int ch = 0; ch < kChunks; ++ch) {
      float2 v[8];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = c.row0() + 4 * ch + r;
        float2 x01 = f2(0.f, 0.f), x23 = x01;
        const int b = geo.width(i);
        if (c.act()) {
          const uint8_t* row = c.blk + geo.off(i);
          if constexpr (MODE == MODE_ROWS)
            unpack4x2_rt(b, row, c.lane, x01, x23);
          else
            unpack4x2<MODE>(row, c.lane, x01, x23);
        }
        if (MODE == MODE_ROWS && b == 16) {  // fp16 row inside a scaled head: x = value / c_j
          x01 = __fmul2_rn(x01, lo(icv));
          x23 = __fmul2_rn(x23, hi(icv));
        }
        v[2 * r] = x01;
        v[2 * r + 1] = x23;
        const float4 g = c.rowG()[i];  // (gk, gk, gq, gq)
        if (r & 1) {
          U2 = __ffma2_rn(x01, lo(g), U2);
          U3 = __ffma2_rn(x23, lo(g), U3);
          P2 = __ffma2_rn(x01, hi(g), P2);
          P3 = __ffma2_rn(x23, hi(g), P3);
        } else {
          U0 = __ffma2_rn(x01, lo(g), U0);
          U1 = __ffma2_rn(x23, lo(g), U1);
          P0 = __ffma2_rn(x01, hi(g), P0);
          P1 = __ffma2_rn(x23, hi(g), P1);
        }
      }
      tmem_st16x2(c.tm + 16 * ch, v);
    }
  }
  U0 = __fadd2_rn(U0, U2);
  U1 = __fadd2_rn(U1, U3);
  P0 = __fadd2_rn(P0, P2);
  P1 = __fadd2_rn(P1, P3);
  float* red = sp<float>(OFF_REDA) + c.warp * 2 * kMaxD + 4 * c.lane;
  *reinterpret_cast<float4*>(red) = make_float4(U0.x, U0.y, U1.x, U1.y);
  *reinterpret_cast<float4*>(red + kMaxD) = make_float4(P0.x, P0.y, P1.x, P1.y);
}

// ---- pass B: M_new = x (A_i c_j) + k_i b_j, row maxima of |M_new| -------------------------
// check16: 0 no fp16 rows, 1 every row is fp16 (fp16 head), 2 per the row table.
template <bool FULL>
__device__ __forceinline__ void pass_b(const Ctx<FULL>& c, const float4& cv, const float4& bv,
                                       float* s_new, int check16, bool fit) {
  bool of = false;
  if (c.wact()) {
#pragma unroll 1
    for (int ch = 0; ch < kChunks; ++ch) {
      float2 v[8];
      tmem_ld16x2(c.tm + 16 * ch, v);
      float rm[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int i = c.row0() + 4 * ch + r;
        const float4 u = c.rowU()[i];  // (A, A, k, k)
        const float2 s0 = __ffma2_rn(v[2 * r], __fmul2_rn(lo(u), lo(cv)), __fmul2_rn(hi(u), lo(bv)));
        const float2 s1 = __ffma2_rn(v[2 * r + 1], __fmul2_rn(lo(u), hi(cv)), __fmul2_rn(hi(u), hi(bv)));
        v[2 * r] = s0;
        v[2 * r + 1] = s1;
        if (fit) rm[r] = warp_max_nonneg(fmaxf(max3abs(s0.x, s0.y, s1.x), fabsf(s1.y)));
        if (check16 == 1 || (check16 == 2 && row_width(c.rowtab()[i]) == 16))  // RN16 -> inf
          if (c.act()) of |= !(fmaxf(max3abs(s0.x, s0.y, s1.x), fabsf(s1.y)) < 65520.f);
        if (s_new != nullptr && c.act())
          *reinterpret_cast<float4*>(s_new + (size_t)i * c.dv() + 4 * c.lane) =
              make_float4(s0.x, s0.y, s1.x, s1.y);
      }
      tmem_st16x2(c.tm + 16 * ch, v);
      if (fit && c.lane == 0)
        *reinterpret_cast<float4*>(c.rowtmp() + 4 * ch) = make_float4(rm[0], rm[1], rm[2], rm[3]);
    }
  }
  if (of) atomicOr(&c.flags[F_RANGE], 1);
  tmem_wait_st();
  __syncwarp();
}

// Row scales from the row maxima in rowtmp: r_i = max(m_i / Q_i, 2^-14), w_i = 1 / (r_i Q_i);
// fp16 rows get r = w = 0. Lane s < 16 returns r of row 16w + s.
template <bool FULL>
__device__ __forceinline__ float row_scales(const Ctx<FULL>& c, int mode, bool check) {
  float r = 0.f;
  if (c.lane < kRows) {
    const int i = c.row0() + c.lane;
    float w = 0.f;
    if (c.wact()) {
      const int b = mode == MODE_ROWS ? row_width(c.rowtab()[i]) : mode;
      if (b != 16) {
        const float Q = (float)q_of_width(b);
        const float inv_q = b == 2 ? 1.0f : b == 4 ? 1.0f / 7.0f : b == 6 ? 1.0f / 31.0f : 1.0f / 127.0f;
        const float rq = div_q(c.rowtmp()[c.lane], Q, inv_q);  // exactly m / Q
        if (check && !(rq < 65520.f)) atomicOr(&c.flags[F_RANGE], 1);
        r = fminf(fmaxf(rq, kScaleFloor), 65504.f);  // 65504: the largest finite fp16 value
        w = rcp_approx(__fmul_rn(r, Q));
      }
    }
    c.rowW2()[i] = f2(w, w);
  }
  __syncwarp();
  return r;
}

// Column pass: max_i |S_ij| w_i over the warp's rows, into red[warp].
template <bool FULL>
__device__ __forceinline__ void col_pass(const Ctx<FULL>& c, float* red) {
  float cm0 = 0.f, cm1 = 0.f, cm2 = 0.f, cm3 = 0.f, cn0 = 0.f, cn1 = 0.f, cn2 = 0.f, cn3 = 0.f;
  if (c.wact()) {
    const float4* w2 = reinterpret_cast<const float4*>(c.rowW2() + c.row0());
#pragma unroll 1
    for (int ch = 0; ch < kChunks; ++ch) {
      float2 v[8];
      tmem_ld16x2(c.tm + 16 * ch, v);
#pragma unroll
      for (int r = 0; r < 4; r += 2) {
        const float4 ww = w2[2 * ch + r / 2];  // (w_s, w_s, w_s+1, w_s+1)
        const float2 a0 = __fmul2_rn(v[2 * r], lo(ww));
        const float2 a1 = __fmul2_rn(v[2 * r + 1], lo(ww));
        const float2 b0 = __fmul2_rn(v[2 * r + 2], hi(ww));
        const float2 b1 = __fmul2_rn(v[2 * r + 3], hi(ww));
        if (r == 0) {
          cm0 = max3abs(cm0, a0.x, b0.x);
          cm1 = max3abs(cm1, a0.y, b0.y);
          cm2 = max3abs(cm2, a1.x, b1.x);
          cm3 = max3abs(cm3, a1.y, b1.y);
        } else {
          cn0 = max3abs(cn0, a0.x, b0.x);
          cn1 = max3abs(cn1, a0.y, b0.y);
          cn2 = max3abs(cn2, a1.x, b1.x);
          cn3 = max3abs(cn3, a1.y, b1.y);
        }
      }
    }
  }
  *reinterpret_cast<float4*>(red + c.warp * kMaxD + 4 * c.lane) =
      make_float4(fmaxf(cm0, cn0), fmaxf(cm1, cn1), fmaxf(cm2, cn2), fmaxf(cm3, cn3));
}

// Row pass of a later alternation: row maxima of |S_ij| v_j into rowtmp.
template <bool FULL>
__device__ __forceinline__ void row_pass(const Ctx<FULL>& c, const float4& icv) {
  if (c.wact()) {
#pragma unroll 1
    for (int ch = 0; ch < kChunks; ++ch) {
      float2 v[8];
      tmem_ld16x2(c.tm + 16 * ch, v);
      float rm[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float2 p = __fmul2_rn(v[2 * r], lo(icv));
        const float2 q = __fmul2_rn(v[2 * r + 1], hi(icv));
        rm[r] = warp_max_nonneg(fmaxf(max3abs(p.x, p.y, q.x), fabsf(q.y)));
      }
      if (c.lane == 0)
        *reinterpret_cast<float4*>(c.rowtmp() + 4 * ch) = make_float4(rm[0], rm[1], rm[2], rm[3]);
    }
  }
  __syncwarp();
}

// ---- requantize, pack and store the scaled head ---------------------------------------------
template <int MODE, bool FULL>
__device__ __forceinline__ void requant(const Ctx<FULL>& c, uint8_t* dst, const float4& cm, float r) {
  const Geo<MODE> geo(c);
  const __half2 c01 = __floats2half2_rn(cm.x, cm.y), c23 = __floats2half2_rn(cm.z, cm.w);
  const float2 fc01 = __half22float2(c01), fc23 = __half22float2(c23);
  const float2 ic01 = f2(rcp_f16val(fc01.x), rcp_f16val(fc01.y));  // correctly rounded
  const float2 ic23 = f2(rcp_f16val(fc23.x), rcp_f16val(fc23.y));
  __half* r16s = reinterpret_cast<__half*>(c.rowtmp());
  if (c.lane < kRows) {
    const __half r16 = __float2half_rn(r);
    const float ir = r > 0.f ? rcp_f16val(__half2float(r16)) : 0.f;
    c.rowIR2()[c.row0() + c.lane] = f2(ir, ir);
    r16s[c.lane] = r16;
  }
  __syncwarp();
  if (c.wact() && c.lane < 2)
    reinterpret_cast<uint4*>(dst)[2 * c.warp + c.lane] = reinterpret_cast<const uint4*>(r16s)[c.lane];
  if (c.warp == 0 && c.act()) {
    uint2 cc;
    cc.x = *reinterpret_cast<const uint32_t*>(&c01);
    cc.y = *reinterpret_cast<const uint32_t*>(&c23);
    reinterpret_cast<uint2*>(dst + 2 * c.dk())[c.lane] = cc;
  }
  if (!c.wact()) return;
#pragma unroll 1
  for (int ch = 0; ch < kChunks; ++ch) {
    float2 v[8];
    tmem_ld16x2(c.tm + 16 * ch, v);
#pragma unroll
    for (int r2 = 0; r2 < 4; ++r2) {
      const int i = c.row0() + 4 * ch + r2;
      uint8_t* row = dst + geo.off(i);
      const int b = geo.width(i);
      if (MODE == MODE_ROWS && b == 16) {
        store4_f16x2(row, c.lane, v[2 * r2], v[2 * r2 + 1], c.act());
      } else {
        const float2 ir = c.rowIR2()[i];
        const float mgv = kMagic + (float)(1 << (b - 1));
        const float2 mg = f2(mgv, mgv);
        const float2 y0 = __ffma2_rn(__fmul2_rn(v[2 * r2], ir), ic01, mg);
        const float2 y1 = __ffma2_rn(__fmul2_rn(v[2 * r2 + 1], ir), ic23, mg);
        const float y[4] = {y0.x, y0.y, y1.x, y1.y};
        if constexpr (MODE == MODE_ROWS) {
          switch (b) {
            case 2: store4<2>(row, c.lane, y, c.act()); break;
            case 4: store4<4>(row, c.lane, y, c.act()); break;
            case 6: store4<6>(row, c.lane, y, c.act()); break;
            default: store4<8>(row, c.lane, y, c.act()); break;
          }
        } else {
          store4<MODE>(row, c.lane, y, c.act());
        }
      }
    }
  }
}

// fp16 head: round and store the updated tile.
template <bool FULL>
__device__ __forceinline__ void store_pivot(const Ctx<FULL>& c, uint8_t* dst) {
  if (!c.wact()) return;
  const Geo<MODE_PIVOT> geo(c);
#pragma unroll 1
  for (int ch = 0; ch < kChunks; ++ch) {
    float2 v[8];
    tmem_ld16x2(c.tm + 16 * ch, v);
#pragma unroll
    for (int r = 0; r < 4; ++r)
      store4_f16x2(dst + geo.off(c.row0() + 4 * ch + r), c.lane, v[2 * r], v[2 * r + 1], c.act());
  }
}

__device__ __forceinline__ void nan_out(float* out, int dv, int tid) {
  if (tid < dv) out[tid] = __int_as_float(0x7fc00000);
}

template <int GATE, int IO, bool WANT_STATE, bool FULL>
__global__ void __launch_bounds__(kThreads, 3) k_decode(const StepArgs a) {
  const int nst = a.n_stages;
  const DPlan P(a.dk, a.dv, IO, GATE, a.per_row, a.stage_bytes, a.H, nst);
  uint64_t* bars = sp<uint64_t>(OFF_BAR);
  Ctx<FULL> c;
  c.tid = threadIdx.x;
  c.warp = c.tid >> 5;
  c.lane = c.tid & 31;
  c.dk_ = a.dk;
  c.dv_ = a.dv;
  c.act_ = 4 * c.lane < a.dv;
  c.wact_ = c.warp * kRows < a.dk;
  const int H = a.H, B = a.batch, dk = c.dk(), dv = c.dv(), tid = c.tid;
  const int n_items = B * H;
  const int stride = gridDim.x;

  if (c.warp == 0) {
    tmem_alloc(sp<uint32_t>(OFF_TMEM), kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < nst; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  if (tid < 16) sp<int>(OFF_FLAGS)[tid] = 0;
  HeadDesc* htab = reinterpret_cast<HeadDesc*>(smem + P.tab);
  int32_t* otab = reinterpret_cast<int32_t*>(smem + P.tab + 16u * H);
  for (int h = tid; h < H; h += kThreads) {
    htab[h] = a.heads[h];
    otab[h] = a.order[h];
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tbase = *sp<uint32_t>(OFF_TMEM);
  c.tm = tbase + ((uint32_t)(32 * (c.warp & 3)) << 16) + 64u * (uint32_t)(c.warp >> 2);

  // Items run head-major in the order of otab: item = hh * B + b. The last warp stages them;
  // its cursors advance by the grid stride without divisions.
  Meta* meta = sp<Meta>(OFF_META);
  int* flag_base = sp<int>(OFF_FLAGS);
  const bool producer = c.warp == kWarps - 1;
  const int first = blockIdx.x;
  const int step_hh = stride / B, step_b = stride - step_hh * B;
  struct Cursor {
    int item, hh, b;
  };
  auto advance = [&](Cursor& k) {
    k.item += stride;
    k.hh += step_hh;
    k.b += step_b;
    if (k.b >= B) {
      k.b -= B;
      ++k.hh;
    }
  };
  Cursor next_issue{first, first / B, first % B};  // the item to stage next
  Cursor next_meta = next_issue;                    // the item whose words to fetch next
  // Producer lanes 0..2: async copies of an item's slot index, beta and (scalar) alpha.
  auto fetch_meta = [&](Cursor& k) {
    if (c.lane < 3) {
      const int io = k.b * H + otab[k.hh];
      if (c.lane == 0) cp_async4(&meta->slot, a.slot_idx + k.b);
      if (c.lane == 1) cp_async4(&meta->beta, a.beta + io);
      if (c.lane == 2 && GATE == 0) cp_async4(&meta->alpha, a.alpha + io);
      cp_async_commit();
    }
    advance(k);
  };
  // Producer warp: stage an item into stage s (its words are in *meta). Lane 0 clears the
  // item's flag words, writes the header and arrives on the stage's mbarrier with the byte
  // count (the arrive publishes both); lanes 1..6 issue one bulk copy each.
  auto issue = [&](Cursor& k, int s, int* nflags) {
    if (c.lane < 3) cp_async_wait_all();
    __syncwarp();
    uint8_t* st = smem + OFF_STAGE + s * P.stage;
    uint64_t* bar = &bars[s];
    const int h = otab[k.hh], io = k.b * H + h;
    const HeadDesc hd = htab[h];
    const Meta m = *meta;
    const bool valid = m.slot >= 0 && m.slot < a.n_slots;
    const uint32_t kb = (uint32_t)dk * P.esz, vb = (uint32_t)dv * P.esz;
    const uint32_t ab = GATE == 1 ? 4u * dk : 0u, rb = a.per_row ? 4u * dk : 0u;
    if (c.lane == 0) {
      nflags[F_INPUT] = nflags[F_RANGE] = 0;
      StageHdr* shdr = reinterpret_cast<StageHdr*>(st);
      *reinterpret_cast<int4*>(shdr) = make_int4(valid, m.slot, k.b, h);
      *(reinterpret_cast<int4*>(shdr) + 1) =
          make_int4(__float_as_int(m.beta), __float_as_int(GATE == 0 ? m.alpha : 0.f),
                    hd.pivot_head ? (int)MODE_PIVOT : (int)hd.width, (int)hd.off);
      mbar_arrive_expect_tx(bar, valid ? 2 * kb + vb + ab + rb + hd.bytes : 0u);
    }
    if (valid && c.lane >= 1 && c.lane <= 6) {
      uint8_t* dst = st;
      const uint8_t* src = nullptr;
      uint32_t n = 0;
      switch (c.lane) {
        case 1: dst += P.k_off, src = static_cast<const uint8_t*>(a.k) + (size_t)io * kb, n = kb; break;
        case 2: dst += P.q_off, src = static_cast<const uint8_t*>(a.q) + (size_t)io * kb, n = kb; break;
        case 3: dst += P.v_off, src = static_cast<const uint8_t*>(a.v) + (size_t)io * vb, n = vb; break;
        case 4: dst += P.al_off, src = reinterpret_cast<const uint8_t*>(a.alpha + (size_t)io * dk), n = ab; break;
        case 5: dst += P.rt_off, src = reinterpret_cast<const uint8_t*>(a.rows + (size_t)h * dk), n = rb; break;
        default: dst += P.blk_off, src = a.pool + (size_t)m.slot * a.slot_bytes + hd.off, n = hd.bytes; break;
      }
      if (n) bulk_load(dst, src, n, bar);
    }
    __syncwarp();  // every lane has read *meta before lanes 0..2 fetch the next words into it
    advance(k);
  };

  if (producer) {  // the first n_stages items in flight, the next one's words on their way
    for (int s = 0; s < nst && next_issue.item < n_items; ++s) {
      fetch_meta(next_meta);
      issue(next_issue, s, flag_base + 4 * s);
    }
    if (next_meta.item < n_items) fetch_meta(next_meta);
  }

  int it = 0;
  bool timed_out = false;
  for (int item = first; item < n_items; item += stride, ++it) {
    // warp-uniform, so the warp-collective tensor-memory instructions below never diverge
    const int s = nst == 1 ? 0 : (it & 1);
    const uint32_t phase = (uint32_t)(nst == 1 ? it : it >> 1) & 1u;
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&bars[s], phase));
    c.flags = flag_base + 4 * (it & 3);
    const uint8_t* st = smem + OFF_STAGE + s * P.stage;
    c.blk = st + P.blk_off;
    StageHdr hdr = *reinterpret_cast<const StageHdr*>(st);
    if (!ok) hdr.valid = 0;
    const int io = hdr.b * H + hdr.h;
    const bool pivot_head = hdr.mode == MODE_PIVOT;

    // ---- setup (each warp its own rows' factors and k.q partial; warps 0 and 1 the column
    // data) and pass A ----
    if (hdr.valid) {
      const uint8_t* kq = st + P.k_off;
      const uint8_t* qq = st + P.q_off;
      bool bad_in = false;
      float kqp = 0.f;
      if (c.wact() && c.lane < kRows) {
        const int i = c.row0() + c.lane;
        uint32_t desc = 0;
        if (a.per_row) {
          desc = reinterpret_cast<const uint32_t*>(st + P.rt_off)[i];
          c.rowtab()[i] = desc;
        }
        const float ki = ld_io(kq, IO, i), qi = ld_io(qq, IO, i);
        const float ai = GATE == 0 ? hdr.alpha : reinterpret_cast<const float*>(st + P.al_off)[i];
        bad_in |= !isfinite(ki) || !isfinite(qi) || !isfinite(ai);
        const bool qrow = !pivot_head && (!a.per_row || row_width(desc) != 16);
        const float A = qrow ? ai * __half2float(reinterpret_cast<const __half*>(c.blk)[i]) : ai;
        c.rowG()[i] = make_float4(A * ki, A * ki, A * qi, A * qi);
        c.rowU()[i] = make_float4(A, A, ki, ki);
        kqp = ki * qi;
      }
      kqp = warp_sum(kqp);
      if (c.lane == 0) sp<float>(OFF_KQP)[c.warp] = kqp;
      if (c.warp == 0) {
        float4 cv = make_float4(1.f, 1.f, 1.f, 1.f);
        if (c.act() && !pivot_head) {
          const uint2 ch = reinterpret_cast<const uint2*>(c.blk + 2 * dk)[c.lane];
          const float2 a01 = __half22float2(*reinterpret_cast<const __half2*>(&ch.x));
          const float2 a23 = __half22float2(*reinterpret_cast<const __half2*>(&ch.y));
          cv = make_float4(a01.x, a01.y, a23.x, a23.y);
        }
        sp<float4>(OFF_COLC)[c.lane] = cv;
        bad_in |= !isfinite(hdr.beta) || (GATE == 0 && !isfinite(hdr.alpha));
      } else if (c.warp == 1) {
        float4 vv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c.act()) {
          const uint8_t* vq = st + P.v_off;
          vv = make_float4(ld_io(vq, IO, 4 * c.lane), ld_io(vq, IO, 4 * c.lane + 1),
                           ld_io(vq, IO, 4 * c.lane + 2), ld_io(vq, IO, 4 * c.lane + 3));
          bad_in |= !(isfinite(vv.x) && isfinite(vv.y) && isfinite(vv.z) && isfinite(vv.w));
        }
        sp<float4>(OFF_COLV)[c.lane] = vv;
      }
      if (bad_in) atomicOr(&c.flags[F_INPUT], 1);
      __syncwarp();
      switch (hdr.mode) {
        case MODE_W2: pass_a<MODE_W2>(c); break;
        case MODE_W4: pass_a<MODE_W4>(c); break;
        case MODE_W6: pass_a<MODE_W6>(c); break;
        case MODE_W8: pass_a<MODE_W8>(c); break;
        case MODE_PIVOT: pass_a<MODE_PIVOT>(c); break;
        default: pass_a<MODE_ROWS>(c); break;
      }
      tmem_wait_st();
    }
    // barrier 1: partial dot products, input flags; the stage is free afterwards
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      break;
    }
    if (producer && next_issue.item < n_items) {  // refill this stage (item + nst strides)
      issue(next_issue, s, flag_base + 4 * ((it + nst) & 3));
      if (next_meta.item < n_items) fetch_meta(next_meta);
    }
    float* out = a.out + (size_t)io * dv;
    if (!hdr.valid) {  // bad slot: skip the item
      if (tid == 0) atomicOr(a.flag, SQ_FLAG_BAD_SLOT_BIT);
      nan_out(out, dv, tid);
      continue;
    }
    if (c.flags[F_INPUT]) {  // non-finite input somewhere in the item: skip it
      if (tid == 0) atomicOr(a.flag, SQ_FLAG_NONFINITE_BIT);
      nan_out(out, dv, tid);
      continue;
    }

    // ---- b, o ----
    const float4 cv = sp<float4>(OFF_COLC)[c.lane];
    float4 bv;
    {
      const float4 kq0 = sp<float4>(OFF_KQP)[0], kq1 = sp<float4>(OFF_KQP)[1];
      const float kqv = ((kq0.x + kq0.y) + (kq0.z + kq0.w)) + ((kq1.x + kq1.y) + (kq1.z + kq1.w));
      const float4 vv = sp<float4>(OFF_COLV)[c.lane];
      const float4 U = sum8(sp<float>(OFF_REDA), 2 * kMaxD, c.lane);
      const float beta = hdr.beta;
      bv = make_float4(beta * (vv.x - cv.x * U.x), beta * (vv.y - cv.y * U.y),
                       beta * (vv.z - cv.z * U.z), beta * (vv.w - cv.w * U.w));
      if (c.warp == 0 && c.act()) {
        const float4 Pp = sum8(sp<float>(OFF_REDA) + kMaxD, 2 * kMaxD, c.lane);
        *reinterpret_cast<float4*>(out + 4 * c.lane) =
            make_float4(__fmaf_rn(bv.x, kqv, cv.x * Pp.x), __fmaf_rn(bv.y, kqv, cv.y * Pp.y),
                        __fmaf_rn(bv.z, kqv, cv.z * Pp.z), __fmaf_rn(bv.w, kqv, cv.w * Pp.w));
      }
    }
    float* s_new = WANT_STATE ? a.s_new + (size_t)io * dk * dv : nullptr;
    uint8_t* dst = a.pool + (size_t)hdr.slot * a.slot_bytes + hdr.off;

    if (pivot_head) {
      pass_b(c, cv, bv, s_new, 1, false);
      __syncthreads();
      if (c.flags[F_RANGE]) {
        if (tid == 0) atomicOr(a.flag, SQ_FLAG_RANGE_BIT);
        continue;
      }
      store_pivot(c, dst);
      continue;
    }

    // ---- refit: alternating row / column max-abs passes ----
    pass_b(c, cv, bv, s_new, a.per_row ? 2 : 0, true);
    float r = row_scales(c, hdr.mode, true);
    col_pass(c, sp<float>(OFF_REDC));
    __syncthreads();  // barrier 2
    float4 cm = max8(sp<float>(OFF_REDC), c.lane);
    for (int f = 1; f < a.fit_iters; ++f) {
      const float4 icv = make_float4(rcp_approx(cm.x), rcp_approx(cm.y), rcp_approx(cm.z), rcp_approx(cm.w));
      row_pass(c, icv);
      r = row_scales(c, hdr.mode, false);
      float* red = sp<float>(OFF_REDC) + (f & 1) * kWarps * kMaxD;
      col_pass(c, red);
      __syncthreads();  // barrier 3 (fit_iters = 2)
      cm = max8(red, c.lane);
    }
    if (c.flags[F_RANGE]) {
      if (tid == 0) atomicOr(a.flag, SQ_FLAG_RANGE_BIT);
      continue;
    }
    switch (hdr.mode) {
      case MODE_W2: requant<MODE_W2>(c, dst, cm, r); break;
      case MODE_W4: requant<MODE_W4>(c, dst, cm, r); break;
      case MODE_W6: requant<MODE_W6>(c, dst, cm, r); break;
      case MODE_W8: requant<MODE_W8>(c, dst, cm, r); break;
      default: requant<MODE_ROWS>(c, dst, cm, r); break;
    }
  }

  if (timed_out) {
    if (tid == 0) atomicOr(a.flag, SQ_FLAG_TIMEOUT_BIT);
    // let copies still in flight land before the CTA exits
    const int s = nst == 1 ? 0 : (it & 1);
    mbar_wait_bounded(&bars[s], (uint32_t)(nst == 1 ? it : it >> 1) & 1u);
    const int item = first + it * stride;
    if (nst == 2 && item + stride < n_items) mbar_wait_bounded(&bars[s ^ 1], (uint32_t)((it + 1) >> 1) & 1u);
    if (producer && c.lane < 3) cp_async_wait_all();
  }
  tmem_fence_before_sync();
  __syncthreads();
  if (c.warp == 0) {
    tmem_fence_after_sync();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// Resident CTAs of kThreads threads per SM, from the registers and shared memory a CTA holds.
cudaError_t resident_ctas(const void* fn, uint32_t smem_bytes, int* per_sm) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, fn);
  if (e != cudaSuccess) return e;
  int dev = 0, smem_sm = 0, regs_sm = 0, thr_sm = 0, reserved = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&thr_sm, cudaDevAttrMaxThreadsPerMultiProcessor, dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess) return e;
  const int regs_cta = ((fa.numRegs + 7) / 8 * 8) * kThreads;  // allocated per warp in units of 8 per thread
  int n = thr_sm / kThreads;
  if (regs_cta > 0 && regs_sm / regs_cta < n) n = regs_sm / regs_cta;
  const int smem_cta = (int)smem_bytes + (int)fa.sharedSizeBytes + reserved;
  if (smem_sm / smem_cta < n) n = smem_sm / smem_cta;
  *per_sm = n < 1 ? 1 : n;
  return cudaSuccess;
}

template <int GATE, int IO, bool WS, bool FULL>
cudaError_t launch_t(const StepArgs& a, int num_sms, cudaStream_t st) {
  auto fn = k_decode<GATE, IO, WS, FULL>;
  // Two stages where they still leave three CTAs on an SM, else one. Shared memory of at least
  // a fifth of the SM's keeps at most four CTAs on an SM, so the tensor-memory allocations
  // (128 columns each) always fit. CTAs per SM come from the kernel's registers and shared
  // memory: the runtime's occupancy query answers 1 for kernels that allocate tensor memory.
  StepArgs b = a;
  uint32_t smem_bytes = 0;
  int per_sm = 0;
  for (int nst = 2; nst >= 1; --nst) {  // the most CTAs per SM, then the most stages
    const DPlan P(a.dk, a.dv, IO, GATE, a.per_row, a.stage_bytes, a.H, nst);
    const uint32_t sb = P.total > 47u * 1024u ? P.total : 47u * 1024u;
    int n = 0;
    const cudaError_t e = resident_ctas(reinterpret_cast<const void*>(fn), sb, &n);
    if (e != cudaSuccess) return e;
    if (n > kMaxCtasPerSm) n = kMaxCtasPerSm;
    if (n > per_sm) {
      per_sm = n;
      smem_bytes = sb;
      b.n_stages = nst;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return e;
  const int items = a.batch * a.H;
  int grid = num_sms * per_sm;
  if (grid > items) grid = items;
  if (grid < 1) return cudaSuccess;
  fn<<<grid, kThreads, smem_bytes, st>>>(b);
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
