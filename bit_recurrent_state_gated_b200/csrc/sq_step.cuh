// sq_step.cuh -- the per-item machinery shared by libsq's per-step kernels (sm_100a): the
// shared-memory map, the tensor-memory tile of one (request, head) item and the passes over it
// (unpack with the dot products, the gated delta update, the row / column max-abs fit passes,
// requantize and pack), used by the decode step (sq_decode.cu), the windowed step
// (sq_window_step.cu) and the multi-token chunk (sq_chunk.cu).
//
// Mapping. A CTA of four warps handles one item at a time; warp w owns 32 key rows, lane l
// owns value columns 4l .. 4l+3, so every thread holds 32 x 4 fp32 state values. They live in
// the SM's tensor memory: the CTA allocates 128 columns and thread t of warp w keeps its values
// in columns 0..127 of lane 32 w + t, written and read 16 at a time (four rows) with tcgen05.st
// / tcgen05.ld. Rows are processed in pairs: a register pair holds the same column of two rows,
// so one shared-memory broadcast serves two rows' factors and the packed fp32x2 instructions do
// two elements at a time.
#pragma once
#include "sq_pair.cuh"
#include "sq_tile.cuh"

namespace sq {
namespace {
using tile::ld_io;
using tile::q_of_width;
using tile::round16;

constexpr int kW = 4;                 // warps per CTA
constexpr int kT = 32 * kW;           // threads per CTA
constexpr int kRW = 32;               // key rows per warp
constexpr int kMaxCh = kRW / 4;       // four-row chunks per warp
constexpr uint32_t kTmemCols = 128;   // 32 rows x 4 columns per thread
constexpr int kMaxCtasPerSm = 4;      // 4 x 128 columns: the SM's whole tensor memory
constexpr int MODE_ROWS = 0, MODE_PIVOT = 16;

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

enum { F_INPUT = 0, F_RANGE = 1, F_BADA = 3 };

// Fixed shared memory (byte offsets).
constexpr uint32_t S_BAR = 0;                 // stage mbarrier
constexpr uint32_t S_TMEM = 8;                // tensor-memory base address
constexpr uint32_t S_FLAGS = 16;              // [4 items][4] int
constexpr uint32_t S_META = 80;               // Meta
constexpr uint32_t S_KQ = 96;                 // per-warp partials of k.q
constexpr uint32_t S_GKQ = 128;               // float4 per row pair (gk_a, gk_b, gq_a, gq_b)
constexpr uint32_t S_AK = S_GKQ + 1024;       // float4 per row pair (A_a, A_b, k_a, k_b)
constexpr uint32_t S_W = S_AK + 1024;         // float per row: w_i (column passes)
constexpr uint32_t S_IR = S_W + 512;          // float per row: 1 / r16_i
constexpr uint32_t S_RT = S_IR + 512;         // float per row: row maxima
constexpr uint32_t S_RD = S_RT + 512;         // uint32 per row: descriptor (processing order)
constexpr uint32_t S_REDU = S_RD + 512;       // [4 warps][128] partial U
constexpr uint32_t S_REDP = S_REDU + 2048;    // [4 warps][128] partial P
constexpr uint32_t S_REDC = S_REDP + 2048;    // [2][4 warps][128] partial column maxima
constexpr uint32_t S_KT = S_REDC + 4096;      // float per row: k_i / A_i
constexpr uint32_t S_TR = S_KT + 512;         // float per row: t_i, the tile holds M_ij / t_i
constexpr uint32_t S_FIT = S_TR + 512;        // [4] per-warp change of the column multipliers,
                                              // [4] slack of the column scales (last column pass)
constexpr uint32_t S_STAGE = S_FIT + 32;      // staging buffer, then the head table
static_assert(S_STAGE % 16 == 0 && S_GKQ % 16 == 0 && S_REDU % 16 == 0, "16-byte aligned");

// Row descriptor, processing order: original row << 24 | byte offset in the block << 8 |
// uniform << 7 | width, where the uniform bit marks every row of a key-row unit's four-row chunk
// whose rows share one width (set when the pool is made).
__device__ __forceinline__ int rd_row(uint32_t d) { return (int)(d >> 24); }
__device__ __forceinline__ uint32_t rd_off(uint32_t d) { return (d >> 8) & 0xffffu; }
__device__ __forceinline__ int rd_width(uint32_t d) { return (int)(d & 0x1fu); }
__device__ __forceinline__ bool rd_uniform(uint32_t d) { return (d & 0x80u) != 0u; }

// Stage: header, k, q, v, (alpha), (row table), head block.
struct DPlan {
  uint32_t esz, k_off, q_off, v_off, al_off, rt_off, blk_off, stage, tab, total;
  __host__ __device__ DPlan(int dk, int dv, int io, int gate, int per_row, uint32_t stage_bytes,
                            int n_heads) {
    esz = io == 1 ? 2u : 4u;
    k_off = (uint32_t)sizeof(StageHdr);
    q_off = k_off + dk * esz;
    v_off = q_off + dk * esz;
    al_off = v_off + dv * esz;
    rt_off = al_off + (gate == 1 ? 4u * dk : 0u);
    blk_off = rt_off + (per_row ? 4u * dk : 0u);  // all offsets multiples of 16
    stage = blk_off + round16(stage_bytes + kSlack);
    tab = S_STAGE + stage;
    total = tab + round16(20u * (uint32_t)n_heads);
  }
};

extern __shared__ __align__(16) uint8_t smem[];
template <typename T>
__device__ __forceinline__ T* sp(uint32_t off) {
  return reinterpret_cast<T*>(smem + off);
}

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
// max |.| over the four columns of row a (.x) or row b (.y) of a pair group
__device__ __forceinline__ float rowmax_x(const float2* v) {
  return fmaxf(max3abs(v[0].x, v[1].x, v[2].x), fabsf(v[3].x));
}
__device__ __forceinline__ float rowmax_y(const float2* v) {
  return fmaxf(max3abs(v[0].y, v[1].y, v[2].y), fabsf(v[3].y));
}

// ---- tensor memory, one chunk (16 columns) at a time, loads issued ahead of their use -------
__device__ __forceinline__ void tm_issue(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// Wait for every load this thread issued; the registers are operands of the wait, so nothing
// reads them earlier. Then view them as 8 pairs.
__device__ __forceinline__ void tm_take(uint32_t (&r)[16], float2 (&v)[8]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                 "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                 "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
               :
               : "memory");
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
}

// Run body(ch, v) over chunks 0..nch-1 (nch even) of the thread's tile, each chunk's load in
// flight while the previous chunk is processed.
template <class F>
__device__ __forceinline__ void sweep_ahead(uint32_t tm, int nch, F&& body) {
  uint32_t ra[16], rb[16];
  if (nch <= 0) return;
  tm_issue(tm, ra);
#pragma unroll 1
  for (int ch = 0; ch < nch; ch += 2) {
    float2 v[8];
    tm_take(ra, v);
    tm_issue(tm + 16u * (ch + 1), rb);
    body(ch, v);
    float2 w[8];
    tm_take(rb, w);
    if (ch + 2 < nch) tm_issue(tm + 16u * (ch + 2), ra);
    body(ch + 1, w);
  }
}

// The same, one chunk at a time (a smaller loop: the key-row kernels, whose bodies dispatch
// on row widths, run faster this way).
template <class F>
__device__ __forceinline__ void sweep_each(uint32_t tm, int nch, F&& body) {
#pragma unroll 1
  for (int ch = 0; ch < nch; ++ch) {
    uint32_t r[16];
    float2 v[8];
    tm_issue(tm + 16u * ch, r);
    tm_take(r, v);
    body(ch, v);
  }
}

template <class C, class F>
__device__ __forceinline__ void sweep(const C& c, F&& body) {
  if (C::kAhead)
    sweep_ahead(c.tm, c.nch(), body);
  else
    sweep_each(c.tm, c.nch(), body);
}

// Either row of a pair with its own width (key-row units, rows of two widths).
__device__ __forceinline__ void unpack_mixed(int wa, const uint8_t* ra, int wb, const uint8_t* rb,
                                             int lane, float2 (&x)[4]) {
  float xa[4], xb[4];
  unpack4_rt(wa, ra, lane, xa);
  unpack4_rt(wb, rb, lane, xb);
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = f2(xa[e], xb[e]);
}

template <int B>
__device__ __forceinline__ constexpr uint32_t row_bytes_of(int dv) {
  return (uint32_t)dv * B / 8;
}

// Thread context of one item; FULL = compile-time 128 x 128 tile; AHEAD: sweeps load the next
// chunk while the current one is processed.
template <bool FULL, bool AHEAD = true>
struct Ctx {
  static constexpr bool kAhead = AHEAD;
  int tid, warp, lane, dk_, dv_, nch_;
  bool act_;  // the lane's columns are < d_v
  uint32_t tm;
  int* flags;
  __device__ int dk() const { return FULL ? kMaxD : dk_; }
  __device__ int dv() const { return FULL ? kMaxD : dv_; }
  __device__ bool act() const { return FULL || act_; }
  __device__ int nch() const { return FULL ? kMaxCh : nch_; }  // chunks of the warp's rows
  __device__ int row0() const { return warp * kRW; }
};

// ---- pass A: exact codes into tensor memory, partial U and P ------------------------------
// Head units of width B (16: fp16 head): rows in key order, row p at base + p * rb.
template <int B, class C>
__device__ __forceinline__ void pass_a_head(const C& c, const uint8_t* blk) {
  const int dv = c.dv();
  const uint32_t rb = row_bytes_of<B>(dv);
  const uint8_t* row0 = blk + (B == 16 ? 0u : 2u * (c.dk() + dv)) + (uint32_t)c.row0() * rb;
  const float4* gkq = sp<float4>(S_GKQ) + c.row0() / 2;
  float2 U[4], P[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) U[e] = P[e] = f2(0.f, 0.f);
#pragma unroll 2
  for (int ch = 0; ch < c.nch(); ++ch) {
    float2 v[8];
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const uint8_t* ra = row0 + (uint32_t)(4 * ch + 2 * pr) * rb;
      float2 x[4];
      if (c.act()) {
        unpack_pair<B>(ra, ra + rb, c.lane, x);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = f2(0.f, 0.f);
      }
      const float4 g = gkq[2 * ch + pr];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        U[e] = __ffma2_rn(x[e], lo(g), U[e]);
        P[e] = __ffma2_rn(x[e], hi(g), P[e]);
        v[4 * pr + e] = x[e];
      }
    }
    tmem_st16x2(c.tm + 16u * ch, v);
  }
  *reinterpret_cast<float4*>(sp<float>(S_REDU) + c.warp * kMaxD + 4 * c.lane) =
      make_float4(U[0].x + U[0].y, U[1].x + U[1].y, U[2].x + U[2].y, U[3].x + U[3].y);
  *reinterpret_cast<float4*>(sp<float>(S_REDP) + c.warp * kMaxD + 4 * c.lane) =
      make_float4(P[0].x + P[0].y, P[1].x + P[1].y, P[2].x + P[2].y, P[3].x + P[3].y);
}

// Key-row units: one width dispatch per chunk whose four rows share a width (the uniform bit),
// per row pair otherwise; fp16 rows are scaled by 1/c_j.
__device__ __forceinline__ void unpack_pair_rt(uint32_t da, uint32_t db, const uint8_t* blk,
                                               int lane, const float (&ic)[4], float2 (&x)[4]) {
  const int wa = rd_width(da), wb = rd_width(db);
  const uint8_t* ra = blk + rd_off(da);
  const uint8_t* rbp = blk + rd_off(db);
  if (wa == wb) {
    switch (wa) {
      case 2: unpack_pair<2>(ra, rbp, lane, x); break;
      case 4: unpack_pair<4>(ra, rbp, lane, x); break;
      case 6: unpack_pair<6>(ra, rbp, lane, x); break;
      case 8: unpack_pair<8>(ra, rbp, lane, x); break;
      default: unpack_pair<16>(ra, rbp, lane, x); break;
    }
  } else {
    unpack_mixed(wa, ra, wb, rbp, lane, x);
  }
  if (wa == 16 || wb == 16) {  // fp16 rows hold values: x = value / c_j
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = f2(wa == 16 ? x[e].x * ic[e] : x[e].x, wb == 16 ? x[e].y * ic[e] : x[e].y);
  }
}

template <int B>
__device__ __forceinline__ void unpack_chunk(const uint4& d, const uint8_t* blk, int lane,
                                             float2 (&x0)[4], float2 (&x1)[4]) {
  unpack_pair<B>(blk + rd_off(d.x), blk + rd_off(d.y), lane, x0);
  unpack_pair<B>(blk + rd_off(d.z), blk + rd_off(d.w), lane, x1);
}

template <class C>
__device__ __forceinline__ void pass_a_rows(const C& c, const uint8_t* blk, const float4& icv) {
  const float4* gkq = sp<float4>(S_GKQ) + c.row0() / 2;
  const uint4* rd4 = reinterpret_cast<const uint4*>(sp<uint32_t>(S_RD) + c.row0());
  float2 U[4], P[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) U[e] = P[e] = f2(0.f, 0.f);
  const float ic[4] = {icv.x, icv.y, icv.z, icv.w};
#pragma unroll 1
  for (int ch = 0; ch < c.nch(); ++ch) {
    const uint4 d = rd4[ch];
    float2 x0[4], x1[4];
    if (!c.act()) {
#pragma unroll
      for (int e = 0; e < 4; ++e) x0[e] = x1[e] = f2(0.f, 0.f);
    } else if (rd_uniform(d.x)) {
      switch (rd_width(d.x)) {
        case 2: unpack_chunk<2>(d, blk, c.lane, x0, x1); break;
        case 4: unpack_chunk<4>(d, blk, c.lane, x0, x1); break;
        case 6: unpack_chunk<6>(d, blk, c.lane, x0, x1); break;
        case 8: unpack_chunk<8>(d, blk, c.lane, x0, x1); break;
        default:  // fp16 rows hold values: x = value / c_j
          unpack_chunk<16>(d, blk, c.lane, x0, x1);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            x0[e] = __fmul2_rn(x0[e], dup(ic[e]));
            x1[e] = __fmul2_rn(x1[e], dup(ic[e]));
          }
          break;
      }
    } else {
      unpack_pair_rt(d.x, d.y, blk, c.lane, ic, x0);
      unpack_pair_rt(d.z, d.w, blk, c.lane, ic, x1);
    }
    const float4 g0 = gkq[2 * ch], g1 = gkq[2 * ch + 1];
    float2 v[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      U[e] = __ffma2_rn(x0[e], lo(g0), U[e]);
      P[e] = __ffma2_rn(x0[e], hi(g0), P[e]);
      U[e] = __ffma2_rn(x1[e], lo(g1), U[e]);
      P[e] = __ffma2_rn(x1[e], hi(g1), P[e]);
      v[e] = x0[e];
      v[4 + e] = x1[e];
    }
    tmem_st16x2(c.tm + 16u * ch, v);
  }
  *reinterpret_cast<float4*>(sp<float>(S_REDU) + c.warp * kMaxD + 4 * c.lane) =
      make_float4(U[0].x + U[0].y, U[1].x + U[1].y, U[2].x + U[2].y, U[3].x + U[3].y);
  *reinterpret_cast<float4*>(sp<float>(S_REDP) + c.warp * kMaxD + 4 * c.lane) =
      make_float4(P[0].x + P[0].y, P[1].x + P[1].y, P[2].x + P[2].y, P[3].x + P[3].y);
}

// ---- pass B: the updated state in place, row maxima of the tile into S_RT ----------------
// TILDE: the tile holds M_new / A_i = x_ij c_j + (k_i / A_i) b_j (one multiply and one fused
// multiply-add per pair of elements); otherwise M_new = x_ij (A_i c_j) + k_i b_j. S_TR holds the
// row factor t_i (A_i or 1) by which a tile row is the state; the fit and the requantization take
// it into their row factors.
// KIND 0: quantized head (row maxima); 1: fp16 head (fp16 range check, no maxima); 2: key-row
// units (row maxima; row_scales checks the fp16 rows' range on them).
template <int KIND, bool WS, bool TILDE, class C>
__device__ __forceinline__ void pass_b(const C& c, const float4& cv, const float4& bv,
                                       float* s_new) {
  const float2 cc[4] = {dup(cv.x), dup(cv.y), dup(cv.z), dup(cv.w)};
  const float2 bb[4] = {dup(bv.x), dup(bv.y), dup(bv.z), dup(bv.w)};
  const float4* ak = sp<float4>(S_AK) + c.row0() / 2;
  const float2* kt = reinterpret_cast<const float2*>(sp<float>(S_KT) + c.row0());
  const float4* tr4 = reinterpret_cast<const float4*>(sp<float>(S_TR) + c.row0());
  float4* rt = reinterpret_cast<float4*>(sp<float>(S_RT) + c.row0());
  const uint4* rd4 = reinterpret_cast<const uint4*>(sp<uint32_t>(S_RD) + c.row0());
  const int dv = c.dv();
  bool of = false;
  sweep(c, [&](int ch, float2 (&v)[8]) {
    float rm[4];
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      if (TILDE) {
        const float2 k2 = kt[2 * ch + pr];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[4 * pr + e] = __ffma2_rn(k2, bb[e], __fmul2_rn(v[4 * pr + e], cc[e]));
      } else {
        const float4 f = ak[2 * ch + pr];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          v[4 * pr + e] = __ffma2_rn(v[4 * pr + e], __fmul2_rn(lo(f), cc[e]), __fmul2_rn(hi(f), bb[e]));
      }
      if (KIND != 1) {
        rm[2 * pr] = warp_max_nonneg(rowmax_x(v + 4 * pr));
        rm[2 * pr + 1] = warp_max_nonneg(rowmax_y(v + 4 * pr));
      }
    }
    if (KIND == 1) {
      float m = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) m = max3abs(m, v[e].x, v[e].y);
      of |= !(m < 65520.f);
    }
    if (KIND != 1 && c.lane == 0) rt[ch] = make_float4(rm[0], rm[1], rm[2], rm[3]);
    if (WS) {
      const uint4 d = rd4[ch];
      const uint32_t ds[4] = {d.x, d.y, d.z, d.w};
      const float4 t4 = tr4[ch];
      const float ts[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float2* g = v + 4 * (r >> 1);
        const float t = KIND == 1 ? 1.f : ts[r];
        const float4 row = (r & 1) ? make_float4(g[0].y, g[1].y, g[2].y, g[3].y)
                                   : make_float4(g[0].x, g[1].x, g[2].x, g[3].x);
        if (c.act())
          *reinterpret_cast<float4*>(s_new + (size_t)rd_row(ds[r]) * dv + 4 * c.lane) =
              make_float4(t * row.x, t * row.y, t * row.z, t * row.w);
      }
    }
    tmem_st16x2(c.tm + 16u * ch, v);
  });
  if (of) atomicOr(&c.flags[F_RANGE], 1);
  tmem_wait_st();
  __syncwarp();
}

// Row scales from the row maxima in S_RT, one row per lane: m = t max |tile row|,
// r = max(m / Q, 2^-14) (at most the largest fp16), w = 1 / (r Q); S_W gets t w, the factor of
// the tile row in the column passes; fp16 rows get r = w = 0, and with `check` their values
// must round to finite fp16 (m < 65520). Returns the lane's r.
// omega: this row's weight in the column passes, in (0, 1] (1 without an impact table): a row
// weighted below 1 counts with w = fl(omega fl(1 / (r Q))), so it sets the column scales less.
template <class C>
__device__ __forceinline__ float row_scale_of(const C& c, int p, float tile_max, bool check,
                                              float omega, float& w) {
  float r = 0.f;
  w = 0.f;
  const int b = rd_width(sp<uint32_t>(S_RD)[p]);
  if (b != 16) {
    const float Q = (float)q_of_width(b);
    const float inv_q = b == 2 ? 1.0f : b == 4 ? 1.0f / 7.0f : b == 6 ? 1.0f / 31.0f : 1.0f / 127.0f;
    const float t = sp<float>(S_TR)[p];
    const float rq = div_q(__fmul_rn(t, tile_max), Q, inv_q);  // exactly m / Q
    if (check && !(rq < 65520.f)) atomicOr(&c.flags[F_RANGE], 1);
    r = fminf(fmaxf(rq, kScaleFloor), 65504.f);
    float wi = rcp_rn(__fmul_rn(r, Q));
    if (omega < 1.f) wi = __fmul_rn(omega, wi);
    w = __fmul_rn(t, wi);
  } else if (check && !(__fmul_rn(sp<float>(S_TR)[p], tile_max) < 65520.f)) {
    atomicOr(&c.flags[F_RANGE], 1);
  }
  return r;
}

template <class C>
__device__ __forceinline__ float row_scales(const C& c, bool check, float omega) {
  const int p = c.row0() + c.lane;
  float r = 0.f, w = 0.f;
  if (p < c.dk()) r = row_scale_of(c, p, sp<float>(S_RT)[p], check, omega, w);
  sp<float>(S_W)[p] = w;
  __syncwarp();
  return r;
}

// After the last alternation of an impact-weighted fit, with S_RT holding the row maxima of
// |S_ij| / c_j (row_pass with the final column scales): a row weighted below 1 widens its
// scale to fit them, r = max(r, m / Q), so none of its codes leaves [-Q, Q]. Other rows keep r.
template <class C>
__device__ __forceinline__ float row_refit(const C& c, float r, float omega) {
  const int p = c.row0() + c.lane;
  if (p < c.dk() && omega < 1.f) {
    const int b = rd_width(sp<uint32_t>(S_RD)[p]);
    if (b != 16) {
      const float Q = (float)q_of_width(b);
      const float inv_q = b == 2 ? 1.0f : b == 4 ? 1.0f / 7.0f : b == 6 ? 1.0f / 31.0f : 1.0f / 127.0f;
      const float rq = div_q(__fmul_rn(sp<float>(S_TR)[p], sp<float>(S_RT)[p]), Q, inv_q);
      if (!(rq < 65520.f)) atomicOr(&c.flags[F_RANGE], 1);
      r = fmaxf(r, rq);
    }
  }
  return r;
}

// Column pass: max_i |S_ij| w_i over the warp's rows into red[warp].
template <class C>
__device__ __forceinline__ void col_pass(const C& c, float* red) {
  const float2* w2 = reinterpret_cast<const float2*>(sp<float>(S_W) + c.row0());
  float m0[4] = {0.f, 0.f, 0.f, 0.f}, m1[4] = {0.f, 0.f, 0.f, 0.f};
  sweep(c, [&](int ch, float2 (&v)[8]) {
    const float2 wa = w2[2 * ch], wb = w2[2 * ch + 1];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 p = __fmul2_rn(v[e], wa);
      const float2 q = __fmul2_rn(v[4 + e], wb);
      m0[e] = max3abs(m0[e], p.x, p.y);
      m1[e] = max3abs(m1[e], q.x, q.y);
    }
  });
  *reinterpret_cast<float4*>(red + c.warp * kMaxD + 4 * c.lane) =
      make_float4(fmaxf(m0[0], m1[0]), fmaxf(m0[1], m1[1]), fmaxf(m0[2], m1[2]), fmaxf(m0[3], m1[3]));
}

// Row pass of a later alternation: row maxima of |S_ij| v_j into S_RT.
template <class C>
__device__ __forceinline__ void row_pass(const C& c, const float4& icv) {
  const float2 ic[4] = {dup(icv.x), dup(icv.y), dup(icv.z), dup(icv.w)};
  float4* rt = reinterpret_cast<float4*>(sp<float>(S_RT) + c.row0());
  sweep(c, [&](int ch, float2 (&v)[8]) {
    float rm[4];
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      float2 p[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) p[e] = __fmul2_rn(v[4 * pr + e], ic[e]);
      rm[2 * pr] = warp_max_nonneg(rowmax_x(p));
      rm[2 * pr + 1] = warp_max_nonneg(rowmax_y(p));
    }
    if (c.lane == 0) rt[ch] = make_float4(rm[0], rm[1], rm[2], rm[3]);
  });
  __syncwarp();
}

// ---- skipping the last column pass when it cannot change an fp16 column scale ----------------
// The last column pass recomputes c'_j = max(max_i fl(|S_ij| w'_i), 2^-14) with the multipliers
// w'_i of the last row pass, where the previous column pass used w_i. If every w'_i lies within a
// factor (1 +- delta) of w_i, then c'_j lies within c_j (1 +- (delta + 2.1 u)), u = 2^-24 (each
// product rounds once, and max and the floor are monotone). If that interval holds no fp16
// rounding boundary, RN_fp16(c'_j) = RN_fp16(c_j), and the stored column scales (rounded once,
// at the end) are exactly what the full pass would give. The row scales come from the last row
// pass either way. So: warp 0 takes the slack of every column (its relative distance from c_j to
// the nearest fp16 rounding boundary), every warp its largest relative change of w, and the pass
// is skipped when the largest change stays below the smallest slack minus 2^-21 (> 2.1 u).

// Relative distance from c (>= 2^-14, rounding to a normal fp16 value) to the nearest fp16
// rounding boundary, rounded down; a value on a boundary gets 0.
__device__ __forceinline__ float fp16_slack(float c) {
  const __half h = __float2half_rn(c);
  const unsigned short hb = __half_as_ushort(h);
  const float hf = __half2float(h);
  const float up = __half2float(__ushort_as_half((unsigned short)(hb + 1)));
  const float dn = __half2float(__ushort_as_half((unsigned short)(hb - 1)));
  const float mid_hi = 0.5f * (hf + up), mid_lo = 0.5f * (hf + dn);  // exact
  const float dist = c <= kScaleFloor ? mid_hi - c : fminf(mid_hi - c, c - mid_lo);  // exact
  return fmaxf(dist, 0.f) * rcp_approx(c) * (1.0f - 0x1p-20f);
}

// Distance of x's fp32 bit pattern from the nearest fp16 rounding boundary, in units of x's last
// place: for x in the normal fp16 range the boundaries are exactly the fp32 values whose low 13
// bits are 0x1000. Since x / ulp(x) < 2^24, a distance of d ulps is a relative distance above
// d 2^-24.
__device__ __forceinline__ int fp16_margin_ulps(float x) {
  return abs((int)(__float_as_uint(x) & 0x1fffu) - 0x1000);
}

// Skipping the whole second alternation (fit_iters = 2) without looking at it. Following the
// rounding chain of the rule (u = 2^-24; each operation rounds once; the row maxima m_i, the
// column scales c_j <= (1 + u)^3 / (1 - u)^3, v_j = 1/c_j): the second row pass gives
// m'_i in m_i [1 - 10 u, 1 + 8 u], hence r'_i in r_i [1 - 12 u, 1 + 10 u] for rows above the
// 2^-14 floor (floored rows stay within [2^-14, 2^-14 (1 + 10 u)]), the multipliers
// w'_i in w_i [1 - 16 u, 1 + 18 u], and the second column pass c'_j in c_j [1 - 18 u, 1 + 20 u].
// So when every row scale lies more than 16 ulps and every column scale more than 24 ulps from
// an fp16 rounding boundary (and no row scale is near the fp16 range's end), the second
// alternation cannot change any fp16 scale: the stored bytes are those of the full fit.
__device__ __forceinline__ bool row_scale_settled(float r) {
  return r == 0.f || (r < 32768.f && fp16_margin_ulps(r) > 16);  // r == 0: an fp16 row
}
__device__ __forceinline__ bool column_scales_settled(const float4& cm) {
  return fp16_margin_ulps(cm.x) > 24 && fp16_margin_ulps(cm.y) > 24 &&
         fp16_margin_ulps(cm.z) > 24 && fp16_margin_ulps(cm.w) > 24;
}

// Warp 0: the smallest slack over the lane's four columns and the warp (all 128 columns), less
// the margin, into S_FIT[4].
__device__ __forceinline__ void column_slack(int warp, int lane, const float4& cm, bool act) {
  if (warp != 0) return;
  float t = act ? fminf(fminf(fp16_slack(cm.x), fp16_slack(cm.y)),
                        fminf(fp16_slack(cm.z), fp16_slack(cm.w)))
                : 1.f;
  t = __uint_as_float(__reduce_min_sync(0xffffffffu, __float_as_uint(t)));  // t >= 0
  if (lane == 0) sp<float>(S_FIT)[4] = t - 0x1p-21f;
}

// The lane's row: relative change of its column multiplier, rounded up (infinite when a zero
// multiplier became nonzero); the warp's largest into S_FIT[warp].
__device__ __forceinline__ void multiplier_change(int warp, int lane, float w_old, float w_new) {
  float d = 0.f;
  if (w_new != w_old) d = w_old > 0.f ? fabsf(w_new - w_old) * rcp_approx(w_old) * (1.0f + 0x1p-20f)
                                      : __int_as_float(0x7f800000);
  d = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(d)));  // d >= 0
  if (lane == 0) sp<float>(S_FIT)[warp] = d;
}

// Max over the four warps' partial column maxima of the lane's columns, floored at 2^-14.
__device__ __forceinline__ float4 max4(const float* red, int lane) {
  const float4 a = *reinterpret_cast<const float4*>(red + 4 * lane);
  const float4 b = *reinterpret_cast<const float4*>(red + kMaxD + 4 * lane);
  const float4 c = *reinterpret_cast<const float4*>(red + 2 * kMaxD + 4 * lane);
  const float4 d = *reinterpret_cast<const float4*>(red + 3 * kMaxD + 4 * lane);
  return make_float4(max3(fmaxf(a.x, b.x), c.x, fmaxf(d.x, kScaleFloor)),
                     max3(fmaxf(a.y, b.y), c.y, fmaxf(d.y, kScaleFloor)),
                     max3(fmaxf(a.z, b.z), c.z, fmaxf(d.z, kScaleFloor)),
                     max3(fmaxf(a.w, b.w), c.w, fmaxf(d.w, kScaleFloor)));
}

__device__ __forceinline__ float4 sum4(const float* red, int lane) {
  const float4 a = *reinterpret_cast<const float4*>(red + 4 * lane);
  const float4 b = *reinterpret_cast<const float4*>(red + kMaxD + 4 * lane);
  const float4 c = *reinterpret_cast<const float4*>(red + 2 * kMaxD + 4 * lane);
  const float4 d = *reinterpret_cast<const float4*>(red + 3 * kMaxD + 4 * lane);
  const float2 x = __fadd2_rn(__fadd2_rn(lo(a), lo(b)), __fadd2_rn(lo(c), lo(d)));
  const float2 y = __fadd2_rn(__fadd2_rn(hi(a), hi(b)), __fadd2_rn(hi(c), hi(d)));
  return make_float4(x.x, x.y, y.x, y.y);
}

// The second row pass for those rows of the warp whose scale lies within the margin of an fp16
// rounding boundary (row_scale_settled), taken as row_pass and row_scales take it: the row's
// maximum of fl(|T_ij| fl(1/c_j)) over its columns (the chunk holding the row loaded from tensor
// memory, the lane's four columns, then the warp), then its scale. When every column scale is
// settled, these are the only scales the second alternation can change. Returns the lane's r.
template <class C>
__device__ __forceinline__ float refit_unsettled_rows(const C& c, const float4& cm, float r) {
  const float ic[4] = {rcp_rn(cm.x), rcp_rn(cm.y), rcp_rn(cm.z), rcp_rn(cm.w)};
  const int p0 = c.row0();
  unsigned m = __ballot_sync(0xffffffffu, p0 + c.lane < c.dk() && !row_scale_settled(r));
  while (m) {
    const int l = __ffs(m) - 1;  // the row's lane in the warp
    m &= m - 1;
    uint32_t regs[16];
    float2 v[8];
    tm_issue(c.tm + 16u * (uint32_t)(l >> 2), regs);
    tm_take(regs, v);
    // the row's four values by selects on fixed indices (an index computed at run time would
    // move v to local memory)
    const bool second_pair = (l >> 1) & 1, odd = l & 1;
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 g = second_pair ? v[4 + e] : v[e];
      mx = fmaxf(mx, fabsf(__fmul_rn(odd ? g.y : g.x, ic[e])));
    }
    mx = warp_max_nonneg(mx);
    if (c.lane == l) {
      float w;
      r = row_scale_of(c, p0 + l, mx, false, 1.f, w);
    }
  }
  return r;
}

// The scale fit of an item after the row maxima are in S_RT (all threads; fit_iters
// alternations of row and column max-abs passes): returns the lane's row scale r and the lane's
// four column scales in cm, fp32, as the rule computes them, except where the fp16 values
// provably cannot differ (the exact shortcuts below). Two or three CTA barriers for
// fit_iters = 2.
template <class C>
__device__ __forceinline__ float fit_scales(const C& c, const StepArgs& a, float omega, float4& cm) {
  float r = row_scales(c, true, omega);
  // the second (and last) alternation may be provably unable to change an fp16 scale (see
  // row_scale_settled); not with row weights, whose closing refit needs the exact fp32 scales
  const bool may_settle = a.fit_iters == 2 && !a.omega && !a.full_fit;
  col_pass(c, sp<float>(S_REDC));
  const bool unsettled_row = __syncthreads_or(may_settle && !row_scale_settled(r));
  cm = max4(sp<float>(S_REDC), c.lane);
  const bool columns_settled =  // the same in every warp: each holds every column scale
      may_settle && __all_sync(0xffffffffu, !c.act() || column_scales_settled(cm));
  // with every column scale settled, only the rows near an fp16 boundary can change: their
  // second row pass alone, row by row (no barrier)
  if (columns_settled) return unsettled_row ? refit_unsettled_rows(c, cm, r) : r;
  for (int f = 1; f < a.fit_iters; ++f) {
    // the last column pass may be skipped (see column_slack); not with row weights
    const bool maybe_skip = f + 1 == a.fit_iters && !a.omega && !a.full_fit;
    if (maybe_skip) column_slack(c.warp, c.lane, cm, c.act());
    const float w_old = sp<float>(S_W)[c.row0() + c.lane];
    row_pass(c, make_float4(rcp_rn(cm.x), rcp_rn(cm.y), rcp_rn(cm.z), rcp_rn(cm.w)));
    r = row_scales(c, false, omega);
    if (maybe_skip) {
      multiplier_change(c.warp, c.lane, w_old, sp<float>(S_W)[c.row0() + c.lane]);
      __syncthreads();  // slack and changes of every warp
      const float4 d4 = *sp<float4>(S_FIT);
      if (fmaxf(fmaxf(d4.x, d4.y), fmaxf(d4.z, d4.w)) <= sp<float>(S_FIT)[4]) break;
    }
    float* red = sp<float>(S_REDC) + (f & 1) * kW * kMaxD;
    col_pass(c, red);
    __syncthreads();
    cm = max4(red, c.lane);
  }
  if (a.omega) {  // rows weighted below 1: fit once more against the final column scales
    row_pass(c, make_float4(rcp_rn(cm.x), rcp_rn(cm.y), rcp_rn(cm.z), rcp_rn(cm.w)));
    r = row_refit(c, r, omega);
    __syncthreads();  // every warp sees the range flags the refit may have set
  }
  return r;
}


// ---- requantize, pack and store ----------------------------------------------------------
// Row scales: r16_i to the block (at the original row), t_i / r16_i into S_IR (t_i for fp16
// rows); column scales: c16.
// Returns the lane's correctly rounded 1/c16 of its four columns.
template <class C>
__device__ __forceinline__ float4 store_scales(const C& c, uint8_t* dst, const float4& cm, float r) {
  const int p = c.row0() + c.lane;
  if (p < c.dk()) {
    const uint32_t d = sp<uint32_t>(S_RD)[p];
    const bool q = rd_width(d) != 16;
    const __half r16 = __float2half_rn(q ? r : 0.f);
    const float t = sp<float>(S_TR)[p];  // fp16 rows: the factor of the stored value
    sp<float>(S_IR)[p] = q ? __fmul_rn(t, rcp_f16val(__half2float(r16))) : t;
    reinterpret_cast<__half*>(dst)[rd_row(d)] = r16;
  }
  const __half2 c01 = __floats2half2_rn(cm.x, cm.y), c23 = __floats2half2_rn(cm.z, cm.w);
  if (c.warp == 0 && c.act()) {
    uint2 cc;
    cc.x = *reinterpret_cast<const uint32_t*>(&c01);
    cc.y = *reinterpret_cast<const uint32_t*>(&c23);
    reinterpret_cast<uint2*>(dst + 2 * c.dk())[c.lane] = cc;
  }
  __syncwarp();
  const float2 f01 = __half22float2(c01), f23 = __half22float2(c23);
  return make_float4(rcp_f16val(f01.x), rcp_f16val(f01.y), rcp_f16val(f23.x), rcp_f16val(f23.y));
}

// The lane's packed codes of one row (y: floats whose low bits hold the offset codes) at p,
// which already points at the lane's bytes of the row (2, 4, 8 bits).
template <int B>
__device__ __forceinline__ void store_lane(uint8_t* p, const float (&y)[4], bool act) {
  const uint32_t y0 = __float_as_uint(y[0]), y1 = __float_as_uint(y[1]);
  const uint32_t y2 = __float_as_uint(y[2]), y3 = __float_as_uint(y[3]);
  if (B == 8) {
    const uint32_t w = __byte_perm(__byte_perm(y0, y1, 0x0040u), __byte_perm(y2, y3, 0x0040u), 0x5410u);
    if (act) *reinterpret_cast<uint32_t*>(p) = w;
  } else if (B == 4) {
    const uint32_t t = y0 + (y1 << 4) + (y2 << 8) + (y3 << 12);
    if (act) *reinterpret_cast<uint16_t*>(p) = static_cast<uint16_t>(t);
  } else {
    const uint32_t t = y0 + (y1 << 2) + (y2 << 4) + (y3 << 6);
    if (act) *p = static_cast<uint8_t>(t);
  }
}

// Codes of one pair group (rows a, b of a chunk): y = fl(S fl(1/r16)) * fl(1/c16) + magic.
__device__ __forceinline__ void quant_pair(const float2* v, float2 ir, const float2 (&ic)[4],
                                           float mgv, float ya[4], float yb[4]) {
  const float2 mg = dup(mgv);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 y = __ffma2_rn(__fmul2_rn(v[e], ir), ic[e], mg);
    ya[e] = y.x;
    yb[e] = y.y;
  }
}

template <int B>
__device__ __forceinline__ float magic_of() {
  return kMagic + (float)(1 << (B - 1));
}

// Head units of width B.
template <int B, class C>
__device__ __forceinline__ void requant_head(const C& c, uint8_t* dst, const float4& icv) {
  const float2 ic[4] = {dup(icv.x), dup(icv.y), dup(icv.z), dup(icv.w)};
  const uint32_t rb = row_bytes_of<B>(c.dv());
  const float2* ir2 = reinterpret_cast<const float2*>(sp<float>(S_IR) + c.row0());
  const bool act = c.act();
  const int lane = c.lane;
  // the lane's bytes of the warp's first row (6-bit rows: the row start; store4<6> places them)
  uint8_t* base = dst + 2u * (c.dk() + c.dv()) + (uint32_t)c.row0() * rb +
                  (B == 6 ? 0u : (uint32_t)lane * (B / 2));
  sweep(c, [&](int ch, float2 (&v)[8]) {
    uint8_t* cb = base + (uint32_t)ch * 4u * rb;
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      float ya[4], yb[4];
      quant_pair(v + 4 * pr, ir2[2 * ch + pr], ic, magic_of<B>(), ya, yb);
      uint8_t* ra = cb + (uint32_t)(2 * pr) * rb;
      if (B == 6) {
        store4<6>(ra, lane, ya, act);
        store4<6>(ra + rb, lane, yb, act);
      } else {
        store_lane<B>(ra, ya, act);
        store_lane<B>(ra + rb, yb, act);
      }
    }
  });
}

// Key-row units: per-row width (chunk-level dispatch when the chunk has one width).
__device__ __forceinline__ void store_row_rt(int b, uint8_t* row, int lane, const float2* g,
                                             bool odd, float ir, const float (&ic)[4], bool act) {
  float s[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) s[e] = odd ? g[e].y : g[e].x;
  if (b == 16) {  // ir = t: the state value
#pragma unroll
    for (int e = 0; e < 4; ++e) s[e] *= ir;
    store4_f16(row, lane, s, act);
    return;
  }
  // any width 2..8: the lane's 4b bits go bytewise to byte lane * b / 2 of the row (rows of
  // mixed-width chunks only; one code path keeps the kernel small)
  const float mg = kMagic + (float)(1 << (b - 1));
  const uint32_t mask = (1u << b) - 1u;
  uint32_t t = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    t |= (__float_as_uint(__fmaf_rn(__fmul_rn(s[e], ir), ic[e], mg)) & mask) << (e * b);
  if (!act) return;
  uint8_t* p = row + (uint32_t)lane * (uint32_t)b / 2u;
#pragma unroll 1
  for (int j = 0; j < b / 2; ++j) p[j] = (uint8_t)(t >> (8 * j));
}

template <int B>
__device__ __forceinline__ void requant_chunk_uniform(const float2 (&v)[8], const uint32_t (&ds)[4],
                                                      uint8_t* dst, const float2* ir2, int ch,
                                                      const float2 (&ic)[4], int lane, bool act) {
#pragma unroll
  for (int pr = 0; pr < 2; ++pr) {
    float ya[4], yb[4];
    quant_pair(v + 4 * pr, ir2[2 * ch + pr], ic, magic_of<B>(), ya, yb);
    store4<B>(dst + rd_off(ds[2 * pr]), lane, ya, act);
    store4<B>(dst + rd_off(ds[2 * pr + 1]), lane, yb, act);
  }
}

template <class C>
__device__ __forceinline__ void requant_rows(const C& c, uint8_t* dst, const float4& icv) {
  const float2 ic2[4] = {dup(icv.x), dup(icv.y), dup(icv.z), dup(icv.w)};
  const float ic[4] = {icv.x, icv.y, icv.z, icv.w};
  const float* irs = sp<float>(S_IR) + c.row0();
  const float2* ir2 = reinterpret_cast<const float2*>(irs);
  const uint4* rd4 = reinterpret_cast<const uint4*>(sp<uint32_t>(S_RD) + c.row0());
  const bool act = c.act();
  const int lane = c.lane;
  sweep(c, [&](int ch, float2 (&v)[8]) {
    const uint4 d = rd4[ch];
    const uint32_t ds[4] = {d.x, d.y, d.z, d.w};
    const int b0 = rd_width(ds[0]);
    const bool uni = rd_uniform(ds[0]);
    if (uni && b0 == 2) {
      requant_chunk_uniform<2>(v, ds, dst, ir2, ch, ic2, lane, act);
    } else if (uni && b0 == 4) {
      requant_chunk_uniform<4>(v, ds, dst, ir2, ch, ic2, lane, act);
    } else if (uni && b0 == 6) {
      requant_chunk_uniform<6>(v, ds, dst, ir2, ch, ic2, lane, act);
    } else if (uni && b0 == 8) {
      requant_chunk_uniform<8>(v, ds, dst, ir2, ch, ic2, lane, act);
    } else {
#pragma unroll
      for (int r = 0; r < 4; ++r)
        store_row_rt(rd_width(ds[r]), dst + rd_off(ds[r]), lane, v + 4 * (r >> 1), r & 1,
                     irs[4 * ch + r], ic, act);
    }
  });
}

// fp16 head: round and store the updated tile.
template <class C>
__device__ __forceinline__ void store_pivot(const C& c, uint8_t* dst) {
  const uint32_t rb = 2u * c.dv();
  uint8_t* row0 = dst + (uint32_t)c.row0() * rb;
  const bool act = c.act();
  const int lane = c.lane;
  sweep(c, [&](int ch, float2 (&v)[8]) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float2* g = v + 4 * (r >> 1);
      const float s[4] = {(r & 1) ? g[0].y : g[0].x, (r & 1) ? g[1].y : g[1].x,
                          (r & 1) ? g[2].y : g[2].x, (r & 1) ? g[3].y : g[3].x};
      store4_f16(row0 + (uint32_t)(4 * ch + r) * rb, lane, s, act);
    }
  });
}

__device__ __forceinline__ void nan_out(float* out, int dv, int tid) {
  if (tid < dv) out[tid] = __int_as_float(0x7fc00000);
}

// Resident CTAs of kT threads per SM, from the registers and shared memory a CTA holds.
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
  const int regs_cta = ((fa.numRegs + 7) / 8 * 8) * kT;  // allocated per warp in units of 8 per thread
  int n = thr_sm / kT;
  if (regs_cta > 0 && regs_sm / regs_cta < n) n = regs_sm / regs_cta;
  const int smem_cta = (int)smem_bytes + (int)fa.sharedSizeBytes + reserved;
  if (smem_sm / smem_cta < n) n = smem_sm / smem_cta;
  *per_sm = n < 1 ? 1 : n;
  return cudaSuccess;
}

}  // namespace
}  // namespace sq
