// sq_decode.cu -- the fused decode-step kernel of libsq (sm_100a).
//
// STEPQuant explainer, experimental-setup paragraph: at every decode step the packed state is
// unpacked, updated and written back by one fused kernel, and the row / column scales are
// refit on the updated state. Per (request, head) item, with x the exact integer codes of the
// packed head, A_i = alpha_i r16_i and c_j = c16_j (so S'_ij = A_i x_ij c_j):
//   pass A  unpack x; U_j = sum_i x_ij A_i k_i, P_j = sum_i x_ij A_i q_i (S'^T k = c U);
//   ----    b = beta (v - c U);  o = c P + b (k.q)
//   pass B  M_new_ij = x_ij (A_i c_j) + k_i b_j, row maxima of |M_new|
//   fit     alternating row / column max-abs passes (fit_iters alternations)
//   pass Q  requantize, repack and store in place.
//
// Mapping. A CTA of four warps handles one item at a time; warp w owns 32 key rows, lane l
// owns value columns 4l .. 4l+3, so every thread holds 32 x 4 fp32 state values. They live in
// the SM's tensor memory: the CTA allocates 128 columns and thread t of warp w keeps its values
// in columns 0..127 of lane 32 w + t, written and read 16 at a time (four rows) with tcgen05.st
// / tcgen05.ld. With the tile out of the register file four CTAs (four items) share an SM and
// fill its 512 tensor-memory columns. Rows are processed in pairs: a register pair holds the
// same column of two rows, so one shared-memory broadcast serves two rows' factors and the
// packed fp32x2 instructions do two elements at a time. Key-row units are processed in an
// order that groups rows of equal width (a per-head permutation fixed when the pool is made),
// so almost every row pair and four-row chunk has one width.
//
// Row work stays inside a warp (redux for row maxima; per-row scalars computed by the lane
// whose index is the row); column sums and maxima combine the four warps' partials after a CTA
// barrier, three per item for fit_iters = 2. Tensor-memory loads are issued one chunk ahead of
// their use. The packed head block and q, k, v (alpha, row table) of the next item arrive by
// bulk copies issued right after the current item's first barrier, when the single staging
// buffer is free again.
//
// Arithmetic: the refit follows the oracle's rule step for step: r_i = max(m_i / Q_i, 2^-14)
// correctly rounded, c_j = max(max_i |S_ij| w_i, 2^-14), fp16 rounding once; w_i = 1/(r_i Q_i)
// and v_j = 1/c_j use the hardware's approximate reciprocal, the code multipliers 1/r16 and
// 1/c16 are correctly rounded. Codes need no clamp: every |S_ij| w_i <= c_j, so the quotient
// S_ij / (r16_i c16_j) is at most Q (1 + 2^-10) in magnitude, less than Q + 1/2 for Q <= 127.
// The state is the GPU's own fp32 update (fused multiply-adds), so its scales and codes are
// compared with the oracle's within the stated agreement.
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
constexpr uint32_t S_STAGE = S_TR + 512;      // staging buffer, then the head table
static_assert(S_STAGE % 16 == 0 && S_GKQ % 16 == 0 && S_REDU % 16 == 0, "16-byte aligned");

// Row descriptor, processing order: original row << 24 | byte offset in the block << 8 | width.
__device__ __forceinline__ int rd_row(uint32_t d) { return (int)(d >> 24); }
__device__ __forceinline__ uint32_t rd_off(uint32_t d) { return (d >> 8) & 0xffffu; }
__device__ __forceinline__ int rd_width(uint32_t d) { return (int)(d & 0xffu); }

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
__device__ __forceinline__ void sweep(uint32_t tm, int nch, F&& body) {
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

// Thread context of one item; FULL = compile-time 128 x 128 tile.
template <bool FULL>
struct Ctx {
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
template <int B, bool FULL>
__device__ __forceinline__ void pass_a_head(const Ctx<FULL>& c, const uint8_t* blk) {
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

// Key-row units: per-chunk width dispatch (rows are width-sorted), fp16 rows scaled by 1/c_j.
template <bool FULL>
__device__ __forceinline__ void pass_a_rows(const Ctx<FULL>& c, const uint8_t* blk, const float4& icv) {
  const float4* gkq = sp<float4>(S_GKQ) + c.row0() / 2;
  const uint4* rd4 = reinterpret_cast<const uint4*>(sp<uint32_t>(S_RD) + c.row0());
  float2 U[4], P[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) U[e] = P[e] = f2(0.f, 0.f);
  const float ic[4] = {icv.x, icv.y, icv.z, icv.w};
#pragma unroll 1
  for (int ch = 0; ch < c.nch(); ++ch) {
    const uint4 d = rd4[ch];
    const uint32_t ds[4] = {d.x, d.y, d.z, d.w};
    float2 v[8];
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const uint32_t da = ds[2 * pr], db = ds[2 * pr + 1];
      const int wa = rd_width(da), wb = rd_width(db);
      const uint8_t* ra = blk + rd_off(da);
      const uint8_t* rbp = blk + rd_off(db);
      float2 x[4];
      if (!c.act()) {
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = f2(0.f, 0.f);
      } else if (wa == wb) {
        switch (wa) {
          case 2: unpack_pair<2>(ra, rbp, c.lane, x); break;
          case 4: unpack_pair<4>(ra, rbp, c.lane, x); break;
          case 6: unpack_pair<6>(ra, rbp, c.lane, x); break;
          case 8: unpack_pair<8>(ra, rbp, c.lane, x); break;
          default: unpack_pair<16>(ra, rbp, c.lane, x); break;
        }
      } else {
        unpack_mixed(wa, ra, wb, rbp, c.lane, x);
      }
      if (wa == 16 || wb == 16) {  // fp16 rows hold values: x = value / c_j
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = f2(wa == 16 ? x[e].x * ic[e] : x[e].x, wb == 16 ? x[e].y * ic[e] : x[e].y);
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

// ---- pass B: the updated state in place, row maxima of the tile into S_RT ----------------
// TILDE: the tile holds M_new / A_i = x_ij c_j + (k_i / A_i) b_j (one multiply and one fused
// multiply-add per pair of elements); otherwise M_new = x_ij (A_i c_j) + k_i b_j. S_TR holds the
// row factor t_i (A_i or 1) by which a tile row is the state; the fit and the requantization take
// it into their row factors.
// KIND 0: quantized head (row maxima); 1: fp16 head (fp16 range check, no maxima); 2: key-row
// units (row maxima; range check of the fp16 rows).
template <int KIND, bool WS, bool TILDE, bool FULL>
__device__ __forceinline__ void pass_b(const Ctx<FULL>& c, const float4& cv, const float4& bv,
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
  sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
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
    if (KIND == 2 || WS) {
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
        if (KIND == 2 && rd_width(ds[r]) == 16 && c.act())  // |t x| < 65520
          of |= !(t * fmaxf(max3abs(row.x, row.y, row.z), fabsf(row.w)) < 65520.f);
        if (WS && c.act())
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
// the tile row in the column passes; fp16 rows get r = w = 0. Returns the lane's r.
// rho: this row's impact weight in (0, 1] (1 without an impact table): the scale widens to
// min(fl(q / rho), 65504) when that exceeds q = m / Q.
template <bool FULL>
__device__ __forceinline__ float row_scales(const Ctx<FULL>& c, bool check, float rho) {
  const int p = c.row0() + c.lane;
  float r = 0.f, w = 0.f;
  if (p < c.dk()) {
    const int b = rd_width(sp<uint32_t>(S_RD)[p]);
    if (b != 16) {
      const float Q = (float)q_of_width(b);
      const float inv_q = b == 2 ? 1.0f : b == 4 ? 1.0f / 7.0f : b == 6 ? 1.0f / 31.0f : 1.0f / 127.0f;
      const float t = sp<float>(S_TR)[p];
      const float rq = div_q(__fmul_rn(t, sp<float>(S_RT)[p]), Q, inv_q);  // exactly m / Q
      if (check && !(rq < 65520.f)) atomicOr(&c.flags[F_RANGE], 1);
      r = fmaxf(rq, kScaleFloor);
      if (rho != 1.f) r = fmaxf(r, fminf(__fdiv_rn(rq, rho), 65504.f));
      r = fminf(r, 65504.f);
      w = __fmul_rn(t, rcp_approx(__fmul_rn(r, Q)));
    }
  }
  sp<float>(S_W)[p] = w;
  __syncwarp();
  return r;
}

// Column pass: max_i |S_ij| w_i over the warp's rows into red[warp].
template <bool FULL>
__device__ __forceinline__ void col_pass(const Ctx<FULL>& c, float* red) {
  const float2* w2 = reinterpret_cast<const float2*>(sp<float>(S_W) + c.row0());
  float m0[4] = {0.f, 0.f, 0.f, 0.f}, m1[4] = {0.f, 0.f, 0.f, 0.f};
  sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
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
template <bool FULL>
__device__ __forceinline__ void row_pass(const Ctx<FULL>& c, const float4& icv) {
  const float2 ic[4] = {dup(icv.x), dup(icv.y), dup(icv.z), dup(icv.w)};
  float4* rt = reinterpret_cast<float4*>(sp<float>(S_RT) + c.row0());
  sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
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

// ---- requantize, pack and store ----------------------------------------------------------
// Row scales: r16_i to the block (at the original row), t_i / r16_i into S_IR (t_i for fp16
// rows); column scales: c16.
// Returns the lane's correctly rounded 1/c16 of its four columns.
template <bool FULL>
__device__ __forceinline__ float4 store_scales(const Ctx<FULL>& c, uint8_t* dst, const float4& cm, float r) {
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
template <int B, bool FULL>
__device__ __forceinline__ void requant_head(const Ctx<FULL>& c, uint8_t* dst, const float4& icv) {
  const float2 ic[4] = {dup(icv.x), dup(icv.y), dup(icv.z), dup(icv.w)};
  const uint32_t rb = row_bytes_of<B>(c.dv());
  const float2* ir2 = reinterpret_cast<const float2*>(sp<float>(S_IR) + c.row0());
  const bool act = c.act();
  const int lane = c.lane;
  // the lane's bytes of the warp's first row (6-bit rows: the row start; store4<6> places them)
  uint8_t* base = dst + 2u * (c.dk() + c.dv()) + (uint32_t)c.row0() * rb +
                  (B == 6 ? 0u : (uint32_t)lane * (B / 2));
  sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
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

template <bool FULL>
__device__ __forceinline__ void requant_rows(const Ctx<FULL>& c, uint8_t* dst, const float4& icv) {
  const float2 ic2[4] = {dup(icv.x), dup(icv.y), dup(icv.z), dup(icv.w)};
  const float ic[4] = {icv.x, icv.y, icv.z, icv.w};
  const float* irs = sp<float>(S_IR) + c.row0();
  const float2* ir2 = reinterpret_cast<const float2*>(irs);
  const uint4* rd4 = reinterpret_cast<const uint4*>(sp<uint32_t>(S_RD) + c.row0());
  const bool act = c.act();
  const int lane = c.lane;
  sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
    const uint4 d = rd4[ch];
    const uint32_t ds[4] = {d.x, d.y, d.z, d.w};
    const int b0 = rd_width(ds[0]);
    const bool uni = b0 == rd_width(ds[1]) && b0 == rd_width(ds[2]) && b0 == rd_width(ds[3]);
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
template <bool FULL>
__device__ __forceinline__ void store_pivot(const Ctx<FULL>& c, uint8_t* dst) {
  const uint32_t rb = 2u * c.dv();
  uint8_t* row0 = dst + (uint32_t)c.row0() * rb;
  const bool act = c.act();
  const int lane = c.lane;
  sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
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

// ROWS: key-row units (per-row widths; every head block has row and column scales); else head
// units (one width per head, fp16 pivot heads).
template <int GATE, int IO, bool WS, bool FULL, bool ROWS>
__global__ void __launch_bounds__(kT, kMaxCtasPerSm) k_decode(const StepArgs a) {
  const DPlan P(a.dk, a.dv, IO, GATE, ROWS, a.stage_bytes, a.H);
  uint64_t* bar = sp<uint64_t>(S_BAR);
  Ctx<FULL> c;
  c.tid = threadIdx.x;
  c.warp = c.tid >> 5;
  c.lane = c.tid & 31;
  c.dk_ = a.dk;
  c.dv_ = a.dv;
  c.act_ = 4 * c.lane < a.dv;
  {
    const int rows = a.dk - c.warp * kRW;
    c.nch_ = rows <= 0 ? 0 : (rows >= kRW ? kMaxCh : rows / 4);
  }
  const int H = a.H, B = a.batch, dk = c.dk(), dv = c.dv(), tid = c.tid;
  const int n_items = B * H;
  const int stride = gridDim.x;

  if (c.warp == 0) {
    tmem_alloc(sp<uint32_t>(S_TMEM), kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (tid < 16) sp<int>(S_FLAGS)[tid] = 0;
  HeadDesc* htab = reinterpret_cast<HeadDesc*>(smem + P.tab);
  int32_t* otab = reinterpret_cast<int32_t*>(smem + P.tab + 16u * H);
  for (int h = tid; h < H; h += kT) {
    htab[h] = a.heads[h];
    otab[h] = a.order[h];
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tbase = *sp<uint32_t>(S_TMEM);
  c.tm = tbase + ((uint32_t)(32 * c.warp) << 16);

  // Items run head-major in the order of otab: item = hh * B + b. The last warp stages them;
  // its cursors advance by the grid stride without divisions.
  Meta* meta = sp<Meta>(S_META);
  int* flag_base = sp<int>(S_FLAGS);
  const bool producer = c.warp == kW - 1;
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
  Cursor next_issue{first, first / B, first % B};
  Cursor next_meta = next_issue;
  auto fetch_meta = [&](Cursor& k) {  // producer lanes 0..2: the item's slot, beta, alpha
    if (c.lane < 3) {
      const int io = k.b * H + otab[k.hh];
      if (c.lane == 0) cp_async4(&meta->slot, a.slot_idx + k.b);
      if (c.lane == 1) cp_async4(&meta->beta, a.beta + io);
      if (c.lane == 2 && GATE == 0) cp_async4(&meta->alpha, a.alpha + io);
      cp_async_commit();
    }
    advance(k);
  };
  // Producer warp: stage an item (its words are in *meta). Lane 0 clears the item's flag words,
  // writes the header and arrives on the mbarrier with the byte count; lanes 1..6 issue one
  // bulk copy each.
  auto issue = [&](Cursor& k, int* nflags) {
    if (c.lane < 3) cp_async_wait_all();
    __syncwarp();
    uint8_t* st = smem + S_STAGE;
    const int h = otab[k.hh], io = k.b * H + h;
    const HeadDesc hd = htab[h];
    const Meta m = *meta;
    const bool valid = m.slot >= 0 && m.slot < a.n_slots;
    const uint32_t kb = (uint32_t)dk * P.esz, vb = (uint32_t)dv * P.esz;
    const uint32_t ab = GATE == 1 ? 4u * dk : 0u, rb = ROWS ? 4u * dk : 0u;
    if (c.lane == 0) {
      nflags[F_INPUT] = nflags[F_RANGE] = nflags[F_BADA] = 0;
      StageHdr* shdr = reinterpret_cast<StageHdr*>(st);
      *reinterpret_cast<int4*>(shdr) = make_int4(valid, m.slot, k.b, h);
      *(reinterpret_cast<int4*>(shdr) + 1) =
          make_int4(__float_as_int(m.beta), __float_as_int(GATE == 0 ? m.alpha : 0.f),
                    hd.pivot_head ? MODE_PIVOT : (int)hd.width, (int)hd.off);
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
        case 5: dst += P.rt_off, src = reinterpret_cast<const uint8_t*>(a.srows + (size_t)h * dk), n = rb; break;
        default: dst += P.blk_off, src = a.pool + (size_t)m.slot * a.slot_bytes + hd.off, n = hd.bytes; break;
      }
      if (n) bulk_load(dst, src, n, bar);
    }
    __syncwarp();  // every lane has read *meta before lanes 0..2 fetch the next words into it
    advance(k);
  };

  if (producer && next_issue.item < n_items) {
    fetch_meta(next_meta);
    issue(next_issue, flag_base);
    if (next_meta.item < n_items) fetch_meta(next_meta);
  }

  int it = 0;
  bool timed_out = false;
  const uint8_t* st = smem + S_STAGE;
  const uint8_t* blk = st + P.blk_off;
  for (int item = first; item < n_items; item += stride, ++it) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar, (uint32_t)it & 1u));
    c.flags = flag_base + 4 * (it & 3);
    StageHdr hdr = *reinterpret_cast<const StageHdr*>(st);
    if (!ok) hdr.valid = 0;
    const int io = hdr.b * H + hdr.h;
    const int mode = ROWS ? MODE_ROWS : hdr.mode;
    const bool pivot_head = !ROWS && mode == MODE_PIVOT;

    // ---- setup: thread t takes processing row t (its factors) and every lane its four
    // columns' old scale and v, before the stage is handed back ----
    float4 cv = make_float4(1.f, 1.f, 1.f, 1.f), vv = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 icv = make_float4(1.f, 1.f, 1.f, 1.f);
    float rho = 1.f;  // this row's impact weight (used by the refit, loaded early)
    if (hdr.valid) {
      bool bad_in = false, bad_a = false;
      float kqp = 0.f;
      const int p = tid;
      if (p < dk) {
        uint32_t d;
        if (ROWS) {
          d = reinterpret_cast<const uint32_t*>(st + P.rt_off)[p];
        } else {
          const uint32_t off = pivot_head ? (uint32_t)p * 2u * dv
                                          : 2u * (dk + dv) + (uint32_t)p * dv * mode / 8u;
          d = (uint32_t)p << 24 | off << 8 | (uint32_t)mode;
        }
        sp<uint32_t>(S_RD)[p] = d;
        const int i = rd_row(d);
        if (a.rho) rho = __ldg(a.rho + (size_t)hdr.h * dk + i);
        const float ki = ld_io(st + P.k_off, IO, i), qi = ld_io(st + P.q_off, IO, i);
        const float ai = GATE == 0 ? hdr.alpha : reinterpret_cast<const float*>(st + P.al_off)[i];
        bad_in |= !isfinite(ki) || !isfinite(qi) || !isfinite(ai);
        const float A = rd_width(d) != 16 ? ai * __half2float(reinterpret_cast<const __half*>(blk)[i]) : ai;
        float* gkq = sp<float>(S_GKQ) + 4 * (p >> 1) + (p & 1);
        gkq[0] = A * ki;
        gkq[2] = A * qi;
        float* akp = sp<float>(S_AK) + 4 * (p >> 1) + (p & 1);
        akp[0] = A;
        akp[2] = ki;
        const bool okA = A >= 0x1p-60f && A <= 0x1p60f;  // k / A representable to full precision
        sp<float>(S_KT)[p] = okA ? __fdiv_rn(ki, A) : 0.f;
        bad_a = !okA;
        kqp = ki * qi;
      }
      kqp = warp_sum(kqp);
      if (c.lane == 0) sp<float>(S_KQ)[c.warp] = kqp;
      if (c.act()) {
        if (!pivot_head) {
          const uint2 ch = reinterpret_cast<const uint2*>(blk + 2 * dk)[c.lane];
          const float2 a01 = __half22float2(*reinterpret_cast<const __half2*>(&ch.x));
          const float2 a23 = __half22float2(*reinterpret_cast<const __half2*>(&ch.y));
          cv = make_float4(a01.x, a01.y, a23.x, a23.y);
          if (ROWS)
            icv = make_float4(rcp_f16val(cv.x), rcp_f16val(cv.y), rcp_f16val(cv.z), rcp_f16val(cv.w));
        }
        const uint8_t* vq = st + P.v_off;
        vv = make_float4(ld_io(vq, IO, 4 * c.lane), ld_io(vq, IO, 4 * c.lane + 1),
                         ld_io(vq, IO, 4 * c.lane + 2), ld_io(vq, IO, 4 * c.lane + 3));
        if (c.warp == 0)
          bad_in |= !(isfinite(vv.x) && isfinite(vv.y) && isfinite(vv.z) && isfinite(vv.w));
      }
      if (tid == 0) bad_in |= !isfinite(hdr.beta) || (GATE == 0 && !isfinite(hdr.alpha));
      if (bad_in) atomicOr(&c.flags[F_INPUT], 1);
      if (bad_a) atomicOr(&c.flags[F_BADA], 1);
      __syncwarp();
      if (ROWS) {
        pass_a_rows(c, blk, icv);
      } else {
        switch (mode) {
          case 2: pass_a_head<2>(c, blk); break;
          case 4: pass_a_head<4>(c, blk); break;
          case 6: pass_a_head<6>(c, blk); break;
          case 8: pass_a_head<8>(c, blk); break;
          default: pass_a_head<16>(c, blk); break;
        }
      }
      tmem_wait_st();
    }
    // barrier 1: partial dot products and flags; the stage is free afterwards
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      break;
    }
    if (producer && next_issue.item < n_items) {  // stage the next item
      issue(next_issue, flag_base + 4 * ((it + 1) & 3));
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
      if (WS && a.update_only && tid == 0) a.s_new[(size_t)io * dk * dv] = __int_as_float(0x7fc00000);
      nan_out(out, dv, tid);
      continue;
    }

    // ---- b, o ----
    float4 bv;
    {
      const float4 kq4 = *sp<float4>(S_KQ);
      const float kqv = (kq4.x + kq4.y) + (kq4.z + kq4.w);
      const float4 U = sum4(sp<float>(S_REDU), c.lane);
      const float beta = hdr.beta;
      bv = make_float4(beta * (vv.x - cv.x * U.x), beta * (vv.y - cv.y * U.y),
                       beta * (vv.z - cv.z * U.z), beta * (vv.w - cv.w * U.w));
      if (c.warp == 0 && c.act()) {
        const float4 Pp = sum4(sp<float>(S_REDP), c.lane);
        *reinterpret_cast<float4*>(out + 4 * c.lane) =
            make_float4(__fmaf_rn(bv.x, kqv, cv.x * Pp.x), __fmaf_rn(bv.y, kqv, cv.y * Pp.y),
                        __fmaf_rn(bv.z, kqv, cv.z * Pp.z), __fmaf_rn(bv.w, kqv, cv.w * Pp.w));
      }
    }
    float* s_new = WS ? a.s_new + (size_t)io * dk * dv : nullptr;
    uint8_t* dst = a.pool + (size_t)hdr.slot * a.slot_bytes + hdr.off;

    if (!ROWS && pivot_head) {
      if (tid < dk) sp<float>(S_TR)[tid] = 1.f;
      __syncwarp();
      pass_b<1, WS, false>(c, cv, bv, s_new);
      __syncthreads();
      if (WS && a.update_only) continue;
      if (c.flags[F_RANGE]) {
        if (tid == 0) atomicOr(a.flag, SQ_FLAG_RANGE_BIT);
        continue;
      }
      store_pivot(c, dst);
      continue;
    }

    // ---- refit: alternating row / column max-abs passes ----
    // head units: every row factor A_i in [2^-60, 2^60] (key-row units keep the direct form,
    // which makes their kernels smaller)
    const bool tilde = !ROWS && !c.flags[F_BADA];
    if (tid < dk) sp<float>(S_TR)[tid] = tilde ? sp<float>(S_AK)[4 * (tid >> 1) + (tid & 1)] : 1.f;
    __syncwarp();
    if (!ROWS && tilde)
      pass_b<ROWS ? 2 : 0, WS, !ROWS>(c, cv, bv, s_new);
    else
      pass_b<ROWS ? 2 : 0, WS, false>(c, cv, bv, s_new);
    if (WS && a.update_only) {  // the refit and requantization run elsewhere
      __syncthreads();
      continue;
    }
    float r = row_scales(c, true, rho);
    col_pass(c, sp<float>(S_REDC));
    __syncthreads();  // barrier 2
    float4 cm = max4(sp<float>(S_REDC), c.lane);
    for (int f = 1; f < a.fit_iters; ++f) {
      row_pass(c, make_float4(rcp_approx(cm.x), rcp_approx(cm.y), rcp_approx(cm.z), rcp_approx(cm.w)));
      r = row_scales(c, false, rho);
      float* red = sp<float>(S_REDC) + (f & 1) * kW * kMaxD;
      col_pass(c, red);
      __syncthreads();  // barrier 3 (fit_iters = 2)
      cm = max4(red, c.lane);
    }
    if (c.flags[F_RANGE]) {
      if (tid == 0) atomicOr(a.flag, SQ_FLAG_RANGE_BIT);
      continue;
    }
    const float4 icn = store_scales(c, dst, cm, r);
    if (ROWS) {
      requant_rows(c, dst, icn);
    } else {
      switch (mode) {
        case 2: requant_head<2>(c, dst, icn); break;
        case 4: requant_head<4>(c, dst, icn); break;
        case 6: requant_head<6>(c, dst, icn); break;
        default: requant_head<8>(c, dst, icn); break;
      }
    }
  }

  if (timed_out) {
    if (tid == 0) atomicOr(a.flag, SQ_FLAG_TIMEOUT_BIT);
    // let copies still in flight land before the CTA exits
    mbar_wait_bounded(bar, (uint32_t)it & 1u);
    if (producer && c.lane < 3) cp_async_wait_all();
  }
  tmem_fence_before_sync();
  __syncthreads();
  if (c.warp == 0) {
    tmem_fence_after_sync();
    tmem_dealloc(tbase, kTmemCols);
  }
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

template <int GATE, int IO, bool WS, bool FULL, bool ROWS>
cudaError_t launch_t(const StepArgs& a, int num_sms, cudaStream_t st) {
  auto fn = k_decode<GATE, IO, WS, FULL, ROWS>;
  // Shared memory of at least a fifth of the SM's keeps at most four CTAs on an SM, so the
  // tensor-memory allocations (128 columns each) always fit. CTAs per SM come from the
  // kernel's registers and shared memory: the runtime's occupancy query answers 1 for kernels
  // that allocate tensor memory.
  const DPlan P(a.dk, a.dv, IO, GATE, a.per_row, a.stage_bytes, a.H);
  const uint32_t smem_bytes = P.total > 47u * 1024u ? P.total : 47u * 1024u;
  int per_sm = 0;
  cudaError_t e = resident_ctas(reinterpret_cast<const void*>(fn), smem_bytes, &per_sm);
  if (e != cudaSuccess) return e;
  if (per_sm > kMaxCtasPerSm) per_sm = kMaxCtasPerSm;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return e;
  const int items = a.batch * a.H;
  int grid = num_sms * per_sm;
  if (grid > items) grid = items;
  if (grid < 1) return cudaSuccess;
  fn<<<grid, kT, smem_bytes, st>>>(a);
  return cudaGetLastError();
}

// The 128 x 128 tile has its own compile-time-shaped kernels, except for the debug variant
// that also writes the fp32 state.
template <int GATE, int IO, bool WS>
cudaError_t launch_shape(const StepArgs& a, int num_sms, cudaStream_t st) {
  const bool full = !WS && a.dk == kMaxD && a.dv == kMaxD;
  if (a.per_row)
    return full ? launch_t<GATE, IO, false, true, true>(a, num_sms, st)
                : launch_t<GATE, IO, WS, false, true>(a, num_sms, st);
  return full ? launch_t<GATE, IO, false, true, false>(a, num_sms, st)
              : launch_t<GATE, IO, WS, false, false>(a, num_sms, st);
}


// =============================================================================================
// Windowed variant (LeapQuant news, 研究の概要: quantize only at the end of a window of tokens;
// inside it the output comes from the frozen low-bit state plus the update held at high
// precision; a few large entries are kept as high-precision "compensation" elements).
//
// The exact state inside a window is S_t = diag(g_t) (Sbar + sum_{s<t} k_hat_s b_s^T) with the
// cumulative gate g_t and k_hat_s = k_s / g_s; with y = g_t k and z = g_t q,
//     u = Sbar^T y + sum_s b_s (k_hat_s . y),  b = beta (v - u),
//     o = Sbar^T z + sum_s b_s (k_hat_s . z) + b (k . q).
// Sbar^T y and Sbar^T z are pass A of the per-step kernel with the row factors A_i y_i and
// A_i z_i (A_i = r16_i, 1 for fp16 rows); the codes it leaves in tensor memory serve the fold
// at the window's end, which materializes S (dequantized block, low-rank terms, gate, the new
// token), takes the n largest |S| of the quantized rows as fp16 compensation entries, and runs
// the per-step kernel's fit and requantize passes on the rest.
//
// Side block of one (slot, head): int32 count | pad to 16 B | g [d_k] fp32 |
// (W - 1) x (k_hat [d_k] fp32, b [d_v] fp32). Two stages hold the next items' q, k, v
// (alpha, row table), side header + g and frozen block; the low-rank terms, whose count is known
// only once the header has landed, follow into their own buffer while pass A runs.
// =============================================================================================
constexpr int kMaxWin = 64;
constexpr int kMaxCand = 256;  // candidate entries for the compensation choice

// Window-only shared memory, after the per-step kernel's fixed arrays.
constexpr uint32_t W_BAR = S_STAGE;          // full[2], tfull
constexpr uint32_t W_Y = W_BAR + 32;         // y, z, k, g by original row
constexpr uint32_t W_Z = W_Y + 512;
constexpr uint32_t W_K = W_Z + 512;
constexpr uint32_t W_GN = W_K + 512;
constexpr uint32_t W_GNP = W_GN + 512;       // g by processing row
constexpr uint32_t W_INV = W_GNP + 512;      // processing row of each original row
constexpr uint32_t W_OU = W_INV + 512;       // compensation entries' contributions to u, o
constexpr uint32_t W_OP = W_OU + 512;
constexpr uint32_t W_LR = W_OP + 512;        // [64][2] (k_hat_s . y, k_hat_s . z)
constexpr uint32_t W_TKEY = W_LR + 512;      // per-thread largest key
constexpr uint32_t W_OIDX = W_TKEY + 512;    // chosen entries: flat index, position, value
constexpr uint32_t W_OPOS = W_OIDX + 256;
constexpr uint32_t W_OVAL = W_OPOS + 256;
constexpr uint32_t W_MISC = W_OVAL + 256;    // [0] candidates, [1] threshold key, [2] entries'
                                             // byte offset, [4..5] items issued per stage
constexpr uint32_t W_OE = W_MISC + 64;       // the frozen block's compensation entries:
                                             // flat index [64] int, value [64] float
constexpr uint32_t W_STAGE = W_OE + 512;
static_assert(W_STAGE % 16 == 0, "16-byte aligned");
// Candidates of the compensation choice share the column-maxima buffer (used later).
constexpr uint32_t W_CIDX = S_REDC, W_CPOS = S_REDC + 4 * kMaxCand, W_CVAL = S_REDC + 8 * kMaxCand;
constexpr uint32_t W_CSEL = S_REDC + 12 * kMaxCand;  // the chosen n in key order: idx, pos, value
static_assert(12 * kMaxCand + 3 * 64 * 4 <= 4096, "candidates fit the column-maxima buffer");

enum { F_UNDER = 2 };

// Stage: header, k, q, v, (alpha), (row table), side header + g, block; two stages, then the
// low-rank term buffer and the head table.
struct WDPlan {
  uint32_t esz, k_off, q_off, v_off, al_off, rt_off, sh_off, blk_off, stage, terms, tab, total;
  __host__ __device__ WDPlan(int dk, int dv, int io, int gate, int per_row, uint32_t stage_bytes,
                             int n_heads, int window) {
    esz = io == 1 ? 2u : 4u;
    k_off = (uint32_t)sizeof(StageHdr);
    q_off = k_off + dk * esz;
    v_off = q_off + dk * esz;
    al_off = v_off + dv * esz;
    rt_off = al_off + (gate == 1 ? 4u * dk : 0u);
    sh_off = rt_off + (per_row ? 4u * dk : 0u);
    blk_off = sh_off + 16u + 4u * dk;
    stage = blk_off + round16(stage_bytes + kSlack);
    terms = W_STAGE + 2u * stage;
    tab = terms + (uint32_t)(window - 1) * 4u * (dk + dv);
    total = tab + round16(20u * (uint32_t)n_heads);
  }
};

// Add `add` to element (row r of the chunk, column e) of the pairs v (r, e uniform or not).
__device__ __forceinline__ void chunk_add(float2 (&v)[8], int r, int e, float add, bool set) {
#pragma unroll
  for (int rr = 0; rr < 4; ++rr)
#pragma unroll
    for (int ee = 0; ee < 4; ++ee)
      if (rr == r && ee == e) {
        float& x = (rr & 1) ? v[4 * (rr >> 1) + ee].y : v[4 * (rr >> 1) + ee].x;
        x = set ? add : x + add;
      }
}

// One element of the tensor-memory tile, by processing row p and column j: its owner warp loads
// the chunk, the owner lane changes the element (x += add, or x = add), the warp stores it.
// Returns the element's new value to the owner lane (0 elsewhere).
template <bool FULL>
__device__ __forceinline__ float tile_patch(const Ctx<FULL>& c, int p, int j, float add, bool set) {
  if (p / kRW != c.warp) return 0.f;  // warp-uniform
  const int ch = (p % kRW) / 4;
  uint32_t r[16];
  float2 v[8];
  tm_issue(c.tm + 16u * ch, r);
  tm_take(r, v);
  float nv = 0.f;
  if (c.lane == j / 4) {
    chunk_add(v, p % 4, j % 4, add, set);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
      for (int ee = 0; ee < 4; ++ee)
        if (rr == p % 4 && ee == j % 4) nv = (rr & 1) ? v[4 * (rr >> 1) + ee].y : v[4 * (rr >> 1) + ee].x;
  }
  tmem_st16x2(c.tm + 16u * ch, v);
  tmem_wait_st();
  return nv;
}

// Key of an element for the compensation choice: larger |value| first; 0 = not eligible.
__device__ __forceinline__ uint32_t wkey(float v) { return (__float_as_uint(v) & 0x7fffffffu) + 1u; }

// The fold at the window's end (all threads). v of the lane's columns: cv (old c16), bv (b).
template <int GATE, bool FULL, bool ROWS>
__device__ __forceinline__ void window_fold(const Ctx<FULL>& c, const StepArgs& a, const uint8_t* blk,
                                            const float* terms, int cnt, int mode,
                                            const float4& cv, const float4& bv, uint8_t* dst,
                                            float rho, int32_t* count) {
  const int dk = c.dk(), dv = c.dv(), tid = c.tid, lane = c.lane;
  const bool pivot_head = !ROWS && mode == MODE_PIVOT;
  const int n_out = pivot_head ? 0 : a.n_outliers;
  const uint32_t ts = (uint32_t)(dk + dv);
  const float2 cc[4] = {dup(cv.x), dup(cv.y), dup(cv.z), dup(cv.w)};
  const float2 bb[4] = {dup(bv.x), dup(bv.y), dup(bv.z), dup(bv.w)};
  const float4* ak = sp<float4>(S_AK) + c.row0() / 2;
  const float2* gnp = reinterpret_cast<const float2*>(sp<float>(W_GNP) + c.row0());
  const uint4* rd4 = reinterpret_cast<const uint4*>(sp<uint32_t>(S_RD) + c.row0());
  // ---- materialize S = g (x A c + sum_s k_hat_s b_s^T) + k b^T in tensor memory; the thread's
  // largest |S| over the rows eligible for compensation entries ----
  float tmaxf = 0.f;
  sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
    const uint4 d = rd4[ch];
    const int orow[4] = {rd_row(d.x), rd_row(d.y), rd_row(d.z), rd_row(d.w)};
    float2 acc[8];
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const float4 f = ak[2 * ch + pr];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[4 * pr + e] = __fmul2_rn(v[4 * pr + e], __fmul2_rn(lo(f), cc[e]));
    }
#pragma unroll 1
    for (int s = 0; s < cnt; ++s) {
      const float* t = terms + (size_t)s * ts;
      const float4 b4 = c.act() ? *reinterpret_cast<const float4*>(t + dk + 4 * lane)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
      const float2 bs[4] = {dup(b4.x), dup(b4.y), dup(b4.z), dup(b4.w)};
      float4 k4;  // k_hat of the chunk's four rows (head units: rows 4ch..4ch+3, one load)
      if (ROWS)
        k4 = make_float4(t[orow[0]], t[orow[1]], t[orow[2]], t[orow[3]]);
      else
        k4 = *reinterpret_cast<const float4*>(t + orow[0]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[e] = __ffma2_rn(lo(k4), bs[e], acc[e]);
        acc[4 + e] = __ffma2_rn(hi(k4), bs[e], acc[4 + e]);
      }
    }
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const float4 f = ak[2 * ch + pr];
      const float2 g = gnp[2 * ch + pr];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[4 * pr + e] = __ffma2_rn(acc[4 * pr + e], g, __fmul2_rn(hi(f), bb[e]));
    }
    if (ROWS) {  // fp16 rows are not eligible for the compensation entries
#pragma unroll
      for (int r = 0; r < 4; ++r)
        if (rd_width((&d.x)[r]) != 16) tmaxf = fmaxf(tmaxf, (r & 1) ? rowmax_y(v + 4 * (r >> 1)) : rowmax_x(v + 4 * (r >> 1)));
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) tmaxf = max3abs(tmaxf, v[e].x, v[e].y);
    }
    tmem_st16x2(c.tm + 16u * ch, v);
  });
  tmem_wait_st();
  __syncwarp();
  // ---- the frozen compensation entries: S_ij += g_i value (their code is 0) ----
  if (!pivot_head) {
    for (int o = 0; o < a.n_outliers; ++o) {
      const int idx = sp<int>(W_OE)[o];
      if (idx >= dk * dv) continue;
      const float pv = sp<float>(W_OE)[64 + o];
      const int i = idx / dv, j = idx % dv;
      tmaxf = fmaxf(tmaxf, fabsf(tile_patch(c, sp<int>(W_INV)[i], j, sp<float>(W_GN)[i] * pv, false)));
    }
  }
  // ---- the n largest |S| of the quantized rows: fp16 compensation entries ----
  int* misc = sp<int>(W_MISC);
  int* oidx = sp<int>(W_OIDX);
  int* opos = sp<int>(W_OPOS);
  float* oval = sp<float>(W_OVAL);
  if (n_out > 0) {
    sp<uint32_t>(W_TKEY)[tid] = c.act() ? wkey(tmaxf) : 0u;
    if (tid == 0) misc[0] = 0;
    __syncthreads();
    if (c.warp == 0) {  // n-th largest of the 128 thread maxima: a lower bound of the n-th element
      uint32_t kv[kT / 32];
#pragma unroll
      for (int t = 0; t < kT / 32; ++t) kv[t] = sp<uint32_t>(W_TKEY)[lane * (kT / 32) + t];
      uint32_t last = 0;
      for (int r = 0; r < n_out; ++r) {
        uint32_t m = 0;
#pragma unroll
        for (int t = 0; t < kT / 32; ++t) m = max(m, kv[t]);
        const uint32_t wm = __reduce_max_sync(0xffffffffu, m);
        last = wm;
        if (wm == 0) break;
        const uint32_t owner = __ffs(__ballot_sync(0xffffffffu, m == wm)) - 1;
        if (lane == (int)owner) {
          bool done = false;
#pragma unroll
          for (int t = 0; t < kT / 32; ++t)
            if (!done && kv[t] == wm) {
              kv[t] = 0;
              done = true;
            }
        }
      }
      if (lane == 0) misc[1] = (int)(last ? last : 1u);
    }
    __syncthreads();
    const uint32_t thr = (uint32_t)misc[1];
    sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
      float cmx = 0.f;  // the chunk's largest |S| (all rows) bounds its candidates
#pragma unroll
      for (int e = 0; e < 8; ++e) cmx = max3abs(cmx, v[e].x, v[e].y);
      if (!c.act() || wkey(cmx) < thr) return;
      const uint4 d = rd4[ch];
      const uint32_t ds[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (ROWS && rd_width(ds[r]) == 16) continue;
        const float2* g = v + 4 * (r >> 1);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x = (r & 1) ? g[e].y : g[e].x;
          if (c.act() && wkey(x) >= thr) {
            const int pos = atomicAdd(&misc[0], 1);
            if (pos < kMaxCand) {
              const int p = c.row0() + 4 * ch + r, j = 4 * lane + e;
              sp<int>(W_CIDX)[pos] = rd_row(ds[r]) * dv + j;
              sp<int>(W_CPOS)[pos] = p << 8 | j;
              sp<float>(W_CVAL)[pos] = x;
            }
          }
        }
      }
    });
    __syncthreads();
    // The thread maxima can exceed the tile's current values (an element changed by a frozen
    // entry's patch after its maximum was taken), so the threshold may lie above the n-th
    // largest element; then fewer than n candidates exist and the exact path below decides.
    // With n or more candidates every element of the top n is among them.
    const int nc = misc[0];
    const bool ranked = nc >= n_out && nc <= kMaxCand;
    if (ranked) {
      // rank of each candidate by (|v| desc, flat index asc); the first n go to the stage
      // arrays in that order, then to oidx/opos/oval in ascending flat index
      int* sidx = sp<int>(W_CSEL);
      int* spos = sidx + 64;
      float* sval = reinterpret_cast<float*>(sidx + 128);
      for (int q = tid; q < nc; q += kT) {
        const int qi = sp<int>(W_CIDX)[q];
        const uint32_t qk = wkey(sp<float>(W_CVAL)[q]);
        int rank = 0;
        for (int u = 0; u < nc; ++u) {
          const uint32_t uk = wkey(sp<float>(W_CVAL)[u]);
          rank += (uk > qk || (uk == qk && sp<int>(W_CIDX)[u] < qi)) ? 1 : 0;
        }
        if (rank < n_out) {
          sidx[rank] = qi;
          spos[rank] = sp<int>(W_CPOS)[q];
          sval[rank] = sp<float>(W_CVAL)[q];
        }
      }
      __syncthreads();
      if (tid < n_out) {
        const int mi = sidx[tid];
        int rank = 0;
        for (int u = 0; u < n_out; ++u) rank += sidx[u] < mi ? 1 : 0;
        oidx[rank] = mi;
        opos[rank] = spos[tid];
        oval[rank] = sval[tid];
      }
    } else {  // many equal values, or too few candidates: n rounds of an exact arg-max
      for (int r = 0; r < n_out; ++r) {
        unsigned long long best = 0;
        int bp = 0;
        float bvx = 0.f;
        sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
          const uint4 d = rd4[ch];
          const uint32_t ds[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
          for (int rr = 0; rr < 4; ++rr) {
            if (ROWS && rd_width(ds[rr]) == 16) continue;
            const float2* g = v + 4 * (rr >> 1);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x = (rr & 1) ? g[e].y : g[e].x;
              const int j = 4 * lane + e, idx = rd_row(ds[rr]) * dv + j;
              bool taken = false;
              for (int q = 0; q < r; ++q) taken |= oidx[q] == idx;
              if (!c.act() || taken) continue;
              const unsigned long long key =
                  ((unsigned long long)wkey(x) << 32) | (0xffffffffu - (uint32_t)idx);
              if (key > best) {
                best = key;
                bp = (c.row0() + 4 * ch + rr) << 8 | j;
                bvx = x;
              }
            }
          }
        });
        unsigned long long wb = best;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const unsigned long long other = __shfl_xor_sync(0xffffffffu, wb, o);
          wb = other > wb ? other : wb;
        }
        unsigned long long* wbest = reinterpret_cast<unsigned long long*>(sp<float>(W_TKEY));
        if (lane == 0) wbest[c.warp] = wb;
        __syncthreads();
        unsigned long long win = 0;
        for (int w = 0; w < kW; ++w) win = wbest[w] > win ? wbest[w] : win;
        if (win != 0 && best == win) {
          oidx[r] = (int)(0xffffffffu - (uint32_t)(win & 0xffffffffu));
          opos[r] = bp;
          oval[r] = bvx;
        }
        __syncthreads();
      }
    }
    __syncthreads();
    if (!ranked && tid == 0) {  // exact path: ascending flat index
      for (int x = 1; x < n_out; ++x) {
        const int ki = oidx[x], kp = opos[x];
        const float kv = oval[x];
        int y = x - 1;
        while (y >= 0 && oidx[y] > ki) {
          oidx[y + 1] = oidx[y];
          opos[y + 1] = opos[y];
          oval[y + 1] = oval[y];
          --y;
        }
        oidx[y + 1] = ki;
        opos[y + 1] = kp;
        oval[y + 1] = kv;
      }
    }
    __syncthreads();
    for (int o = 0; o < n_out; ++o)  // out of the fit, code 0
      tile_patch(c, opos[o] >> 8, opos[o] & 0xff, 0.f, true);
    if (tid < n_out && __hisinf(__float2half_rn(oval[tid]))) atomicOr(&c.flags[F_RANGE], 1);
  }
  // ---- refit and requantize (pivot heads: round to fp16) ----
  if (pivot_head) {
    bool of = false;
    sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
      float m = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) m = max3abs(m, v[e].x, v[e].y);
      of |= !(m < 65520.f);
    });
    if (of) atomicOr(&c.flags[F_RANGE], 1);
    __syncthreads();
    if (c.flags[F_RANGE]) {
      if (tid == 0) atomicOr(a.flag, SQ_FLAG_RANGE_BIT);
    } else {
      store_pivot(c, dst);
    }
    if (tid == 0) *count = 0;
    return;
  }
  {  // row maxima (fp16 rows: range check)
    float4* rtab = reinterpret_cast<float4*>(sp<float>(S_RT) + c.row0());
    bool of = false;
    sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
      float rm[4];
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        rm[2 * pr] = warp_max_nonneg(rowmax_x(v + 4 * pr));
        rm[2 * pr + 1] = warp_max_nonneg(rowmax_y(v + 4 * pr));
      }
      if (lane == 0) rtab[ch] = make_float4(rm[0], rm[1], rm[2], rm[3]);
      if (ROWS) {
        const uint4 d = rd4[ch];
        const uint32_t ds[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
        for (int r = 0; r < 4; ++r)
          if (rd_width(ds[r]) == 16 && !(rm[r] < 65520.f)) of = true;
      }
    });
    if (of) atomicOr(&c.flags[F_RANGE], 1);
    __syncwarp();
  }
  float r = row_scales(c, true, rho);
  col_pass(c, sp<float>(S_REDC));
  __syncthreads();
  float4 cm = max4(sp<float>(S_REDC), lane);
  for (int f = 1; f < a.fit_iters; ++f) {
    row_pass(c, make_float4(rcp_approx(cm.x), rcp_approx(cm.y), rcp_approx(cm.z), rcp_approx(cm.w)));
    r = row_scales(c, false, rho);
    float* red = sp<float>(S_REDC) + (f & 1) * kW * kMaxD;
    col_pass(c, red);
    __syncthreads();
    cm = max4(red, lane);
  }
  if (c.flags[F_RANGE]) {
    if (tid == 0) {
      atomicOr(a.flag, SQ_FLAG_RANGE_BIT);
      *count = 0;
    }
    return;
  }
  const float4 icn = store_scales(c, dst, cm, r);
  if (ROWS) {
    requant_rows(c, dst, icn);
  } else {
    switch (mode) {
      case 2: requant_head<2>(c, dst, icn); break;
      case 4: requant_head<4>(c, dst, icn); break;
      case 6: requant_head<6>(c, dst, icn); break;
      default: requant_head<8>(c, dst, icn); break;
    }
  }
  if (tid < n_out) {
    uint8_t* o = dst + sp<int>(W_MISC)[2];
    reinterpret_cast<uint16_t*>(o)[2 * tid] = (uint16_t)oidx[tid];
    reinterpret_cast<__half*>(o)[2 * tid + 1] = __float2half_rn(oval[tid]);
  }
  if (tid == 0) *count = 0;
}

template <int GATE, int IO, bool FULL, bool ROWS>
__global__ void __launch_bounds__(kT, 3) k_window(const StepArgs a) {
  const WDPlan P(a.dk, a.dv, IO, GATE, ROWS, a.stage_bytes, a.H, a.window);
  uint64_t* full = sp<uint64_t>(W_BAR);
  uint64_t* tfull = full + 2;
  Ctx<FULL> c;
  c.tid = threadIdx.x;
  c.warp = c.tid >> 5;
  c.lane = c.tid & 31;
  c.dk_ = a.dk;
  c.dv_ = a.dv;
  c.act_ = 4 * c.lane < a.dv;
  {
    const int rows = a.dk - c.warp * kRW;
    c.nch_ = rows <= 0 ? 0 : (rows >= kRW ? kMaxCh : rows / 4);
  }
  const int H = a.H, B = a.batch, dk = c.dk(), dv = c.dv(), tid = c.tid, W = a.window;
  const int n_items = B * H;
  const int stride = gridDim.x;
  const uint32_t tbytes = 4u * (uint32_t)(dk + dv);
  float* terms = reinterpret_cast<float*>(smem + P.terms);

  if (c.warp == 0) {
    tmem_alloc(sp<uint32_t>(S_TMEM), kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < 3; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  if (tid < 16) sp<int>(S_FLAGS)[tid] = 0;
  HeadDesc* htab = reinterpret_cast<HeadDesc*>(smem + P.tab);
  int32_t* otab = reinterpret_cast<int32_t*>(smem + P.tab + 16u * H);
  for (int h = tid; h < H; h += kT) {
    htab[h] = a.heads[h];
    otab[h] = a.order[h];
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tbase = *sp<uint32_t>(S_TMEM);
  c.tm = tbase + ((uint32_t)(32 * c.warp) << 16);

  Meta* meta = sp<Meta>(S_META);
  int* flag_base = sp<int>(S_FLAGS);
  const bool producer = c.warp == kW - 1;
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
  Cursor next_issue{first, first / B, first % B};
  Cursor next_meta = next_issue;
  auto fetch_meta = [&](Cursor& k) {
    if (c.lane < 3 && k.item < n_items) {
      const int io = k.b * H + otab[k.hh];
      if (c.lane == 0) cp_async4(&meta->slot, a.slot_idx + k.b);
      if (c.lane == 1) cp_async4(&meta->beta, a.beta + io);
      if (c.lane == 2 && GATE == 0) cp_async4(&meta->alpha, a.alpha + io);
      cp_async_commit();
    }
    advance(k);
  };
  auto issue = [&](Cursor& k, int s, int fslot) {
    if (c.lane < 3) cp_async_wait_all();
    __syncwarp();
    uint8_t* st = smem + W_STAGE + s * P.stage;
    const int h = otab[k.hh], io = k.b * H + h;
    const HeadDesc hd = htab[h];
    const Meta m = *meta;
    const bool valid = m.slot >= 0 && m.slot < a.n_slots;
    const uint32_t kb = (uint32_t)dk * P.esz, vb = (uint32_t)dv * P.esz;
    const uint32_t ab = GATE == 1 ? 4u * dk : 0u, rb = ROWS ? 4u * dk : 0u, shb = 16u + 4u * dk;
    if (c.lane == 0) {
      int* nf = flag_base + 4 * fslot;
      nf[F_INPUT] = nf[F_RANGE] = nf[F_UNDER] = 0;
      ++sp<int>(W_MISC)[4 + s];
      StageHdr* shdr = reinterpret_cast<StageHdr*>(st);
      *reinterpret_cast<int4*>(shdr) = make_int4(valid, m.slot, k.b, h);
      *(reinterpret_cast<int4*>(shdr) + 1) =
          make_int4(__float_as_int(m.beta), __float_as_int(GATE == 0 ? m.alpha : 0.f),
                    hd.pivot_head ? MODE_PIVOT : (int)hd.width, (int)hd.off);
      mbar_arrive_expect_tx(&full[s], valid ? 2 * kb + vb + ab + rb + shb + hd.bytes : 0u);
    }
    if (valid && c.lane >= 1 && c.lane <= 7) {
      uint8_t* dst = st;
      const uint8_t* src = nullptr;
      uint32_t n = 0;
      switch (c.lane) {
        case 1: dst += P.k_off, src = static_cast<const uint8_t*>(a.k) + (size_t)io * kb, n = kb; break;
        case 2: dst += P.q_off, src = static_cast<const uint8_t*>(a.q) + (size_t)io * kb, n = kb; break;
        case 3: dst += P.v_off, src = static_cast<const uint8_t*>(a.v) + (size_t)io * vb, n = vb; break;
        case 4: dst += P.al_off, src = reinterpret_cast<const uint8_t*>(a.alpha + (size_t)io * dk), n = ab; break;
        case 5: dst += P.rt_off, src = reinterpret_cast<const uint8_t*>(a.srows + (size_t)h * dk), n = rb; break;
        case 6:
          dst += P.sh_off;
          src = a.side + (size_t)m.slot * a.side_slot_bytes + (size_t)h * a.side_head_bytes;
          n = shb;
          break;
        default: dst += P.blk_off, src = a.pool + (size_t)m.slot * a.slot_bytes + hd.off, n = hd.bytes; break;
      }
      if (n) bulk_load(dst, src, n, &full[s]);
    }
    __syncwarp();
    advance(k);
  };

  if (tid == 0) sp<int>(W_MISC)[4] = sp<int>(W_MISC)[5] = 0;
  __syncthreads();
  if (producer) {
    fetch_meta(next_meta);
    for (int s = 0; s < 2 && next_issue.item < n_items; ++s) {
      issue(next_issue, s, s);
      fetch_meta(next_meta);
    }
  }

  int it = 0;
  bool timed_out = false;
  for (int item = first; item < n_items; item += stride, ++it) {
    const int s = it & 1;
    const uint8_t* st = smem + W_STAGE + s * P.stage;
    const uint8_t* blk = st + P.blk_off;
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full[s], (uint32_t)(it >> 1) & 1u));
    c.flags = flag_base + 4 * (it & 3);
    StageHdr hdr = *reinterpret_cast<const StageHdr*>(st);
    if (!ok) hdr.valid = 0;
    int cnt = *reinterpret_cast<const int32_t*>(st + P.sh_off);
    if (cnt < 0 || cnt >= W || !hdr.valid) cnt = 0;  // a closed or unreadable window restarts
    if (tid == 0) {  // the item's low-rank terms
      mbar_arrive_expect_tx(tfull, (uint32_t)cnt * tbytes);
      if (cnt > 0)
        bulk_load(terms,
                  a.side + (size_t)hdr.slot * a.side_slot_bytes + (size_t)hdr.h * a.side_head_bytes +
                      16u + 4u * dk,
                  (uint32_t)cnt * tbytes, tfull);
    }
    const int io = hdr.b * H + hdr.h;
    const int mode = ROWS ? MODE_ROWS : hdr.mode;
    const bool pivot_head = !ROWS && mode == MODE_PIVOT;

    // ---- setup: thread t takes processing row t and value column t ----
    float tc = 1.f, tv = 0.f, rho = 1.f;
    float4 cv = make_float4(1.f, 1.f, 1.f, 1.f);
    if (hdr.valid) {
      bool bad_in = false, under = false;
      float kqp = 0.f;
      const int p = tid;
      if (p < dk) {
        uint32_t d;
        if (ROWS) {
          d = reinterpret_cast<const uint32_t*>(st + P.rt_off)[p];
        } else {
          const uint32_t off = pivot_head ? (uint32_t)p * 2u * dv
                                          : 2u * (dk + dv) + (uint32_t)p * dv * mode / 8u;
          d = (uint32_t)p << 24 | off << 8 | (uint32_t)mode;
        }
        sp<uint32_t>(S_RD)[p] = d;
        const int i = rd_row(d);
        if (a.rho) rho = __ldg(a.rho + (size_t)hdr.h * dk + i);
        sp<int>(W_INV)[i] = p;
        const float ki = ld_io(st + P.k_off, IO, i), qi = ld_io(st + P.q_off, IO, i);
        const float ai = GATE == 0 ? hdr.alpha : reinterpret_cast<const float*>(st + P.al_off)[i];
        bad_in |= !isfinite(ki) || !isfinite(qi) || !isfinite(ai);
        const float gold = cnt > 0 ? reinterpret_cast<const float*>(st + P.sh_off + 16)[i] : 1.f;
        const float gn = gold * ai;
        under |= gn < 1e-30f;
        const float yi = gn * ki, zi = gn * qi;
        const float A = (!pivot_head && rd_width(d) != 16) ? __half2float(reinterpret_cast<const __half*>(blk)[i]) : 1.f;
        float* gkq = sp<float>(S_GKQ) + 4 * (p >> 1) + (p & 1);
        gkq[0] = A * yi;
        gkq[2] = A * zi;
        float* akp = sp<float>(S_AK) + 4 * (p >> 1) + (p & 1);
        akp[0] = A;
        akp[2] = ki;
        sp<float>(W_GNP)[p] = gn;
        sp<float>(S_TR)[p] = 1.f;  // the fold's tile holds the state itself
        sp<float>(W_Y)[i] = yi;
        sp<float>(W_Z)[i] = zi;
        sp<float>(W_K)[i] = ki;
        sp<float>(W_GN)[i] = gn;
        kqp = ki * qi;
      }
      kqp = warp_sum(kqp);
      if (c.lane == 0) sp<float>(S_KQ)[c.warp] = kqp;
      sp<float>(W_OU)[tid] = 0.f;
      sp<float>(W_OP)[tid] = 0.f;
      if (tid < dv) {
        if (!pivot_head) tc = __half2float(reinterpret_cast<const __half*>(blk)[dk + tid]);
        tv = ld_io(st + P.v_off, IO, tid);
        bad_in |= !isfinite(tv);
      }
      if (c.act() && !pivot_head) {  // the lane's old column scales (the fold's c)
        const uint2 ch = reinterpret_cast<const uint2*>(blk + 2 * dk)[c.lane];
        const float2 a01 = __half22float2(*reinterpret_cast<const __half2*>(&ch.x));
        const float2 a23 = __half22float2(*reinterpret_cast<const __half2*>(&ch.y));
        cv = make_float4(a01.x, a01.y, a23.x, a23.y);
      }
      if (!pivot_head && tid < a.n_outliers) {  // the block's compensation entries
        const uint32_t dl = ROWS ? a.rows[(size_t)hdr.h * dk + dk - 1]
                                 : (uint32_t)(2 * (dk + dv) + (dk - 1) * dv * mode / 8) << 8 | (uint32_t)mode;
        const uint32_t roff = row_off(dl) + (uint32_t)dv * (uint32_t)row_width(dl) / 8u;
        const uint8_t* o = blk + roff;
        sp<int>(W_OE)[tid] = reinterpret_cast<const uint16_t*>(o)[2 * tid];
        sp<float>(W_OE)[64 + tid] = __half2float(reinterpret_cast<const __half*>(o)[2 * tid + 1]);
        if (tid == 0) sp<int>(W_MISC)[2] = (int)roff;
      }
      float4 icv = make_float4(1.f, 1.f, 1.f, 1.f);
      if (ROWS && c.act()) {
        const uint2 ch = reinterpret_cast<const uint2*>(blk + 2 * dk)[c.lane];
        const float2 a01 = __half22float2(*reinterpret_cast<const __half2*>(&ch.x));
        const float2 a23 = __half22float2(*reinterpret_cast<const __half2*>(&ch.y));
        icv = make_float4(rcp_f16val(a01.x), rcp_f16val(a01.y), rcp_f16val(a23.x), rcp_f16val(a23.y));
      }
      if (tid == 0) bad_in |= !isfinite(hdr.beta) || (GATE == 0 && !isfinite(hdr.alpha));
      if (bad_in) atomicOr(&c.flags[F_INPUT], 1);
      if (under) atomicOr(&c.flags[F_UNDER], 1);
      __syncwarp();
      // ---- pass A: Sbar^T y and Sbar^T z (c_j applied below); the codes stay in tensor memory
      if (ROWS) {
        pass_a_rows(c, blk, icv);
      } else {
        switch (mode) {
          case 2: pass_a_head<2>(c, blk); break;
          case 4: pass_a_head<4>(c, blk); break;
          case 6: pass_a_head<6>(c, blk); break;
          case 8: pass_a_head<8>(c, blk); break;
          default: pass_a_head<16>(c, blk); break;
        }
      }
      tmem_wait_st();
    }
    if (__syncthreads_or(!ok)) {  // barrier: partial sums, flags, y and z of every row
      timed_out = true;
      break;
    }
    const bool skip = !hdr.valid || c.flags[F_INPUT];
    float u0 = 0.f, p0 = 0.f;  // c_t (Sbar^T y)_t / c_t, (Sbar^T z)_t of column t
    if (!skip && tid < dv) {
      const float* ru = sp<float>(S_REDU) + tid;
      const float* rp = sp<float>(S_REDP) + tid;
      u0 = tc * ((ru[0] + ru[kMaxD]) + (ru[2 * kMaxD] + ru[3 * kMaxD]));
      p0 = tc * ((rp[0] + rp[kMaxD]) + (rp[2 * kMaxD] + rp[3 * kMaxD]));
    }
    // the frozen block is no longer read: stage the item after next into its buffer
    if (producer && next_issue.item < n_items) {
      issue(next_issue, s, (it + 2) & 3);
      fetch_meta(next_meta);
    }
    // frozen compensation entries' share of u and o
    if (!skip && !pivot_head && tid < a.n_outliers) {
      const int idx = sp<int>(W_OE)[tid];
      const float pv = sp<float>(W_OE)[64 + tid];
      if (idx < dk * dv) {
        atomicAdd(sp<float>(W_OU) + idx % dv, pv * sp<float>(W_Y)[idx / dv]);
        atomicAdd(sp<float>(W_OP) + idx % dv, pv * sp<float>(W_Z)[idx / dv]);
      }
    }
    const bool tok = __all_sync(0xffffffffu, mbar_wait_bounded(tfull, (uint32_t)it & 1u));
    if (!skip) {  // low-rank coefficients, one term per warp at a time
      for (int t = c.warp; t < cnt; t += kW) {
        float dy = 0.f, dz = 0.f;
        if (4 * c.lane < dk) {
          const float4 kh = *reinterpret_cast<const float4*>(terms + (size_t)t * (dk + dv) + 4 * c.lane);
          const float4 y4 = *reinterpret_cast<const float4*>(sp<float>(W_Y) + 4 * c.lane);
          const float4 z4 = *reinterpret_cast<const float4*>(sp<float>(W_Z) + 4 * c.lane);
          dy = __fmaf_rn(kh.x, y4.x, __fmaf_rn(kh.y, y4.y, __fmaf_rn(kh.z, y4.z, kh.w * y4.w)));
          dz = __fmaf_rn(kh.x, z4.x, __fmaf_rn(kh.y, z4.y, __fmaf_rn(kh.z, z4.z, kh.w * z4.w)));
        }
        dy = warp_sum(dy);
        dz = warp_sum(dz);
        if (c.lane == 0) {
          sp<float>(W_LR)[2 * t] = dy;
          sp<float>(W_LR)[2 * t + 1] = dz;
        }
      }
    }
    if (__syncthreads_or(!tok)) {
      timed_out = true;
      break;
    }
    float* out = a.out + (size_t)io * dv;
    if (skip) {
      if (tid == 0) atomicOr(a.flag, hdr.valid ? SQ_FLAG_NONFINITE_BIT : SQ_FLAG_BAD_SLOT_BIT);
      nan_out(out, dv, tid);
    } else {
      // ---- u, b, o of column t ----
      const bool fold = cnt + 1 >= W || c.flags[F_UNDER] != 0;
      uint8_t* side = a.side + (size_t)hdr.slot * a.side_slot_bytes + (size_t)hdr.h * a.side_head_bytes;
      float* tnew = reinterpret_cast<float*>(side + 16 + 4 * dk) + (size_t)cnt * (dk + dv);
      if (tid < dv) {
        float u = u0 + sp<float>(W_OU)[tid], pq = p0 + sp<float>(W_OP)[tid];
        const float2* lr = reinterpret_cast<const float2*>(sp<float>(W_LR));
        for (int t = 0; t < cnt; ++t) {
          const float bt = terms[(size_t)t * (dk + dv) + dk + tid];
          const float2 l = lr[t];
          u = __fmaf_rn(l.x, bt, u);
          pq = __fmaf_rn(l.y, bt, pq);
        }
        const float4 kq4 = *sp<float4>(S_KQ);
        const float kqv = (kq4.x + kq4.y) + (kq4.z + kq4.w);
        const float bj = hdr.beta * (tv - u);
        out[tid] = __fmaf_rn(bj, kqv, pq);
        if (fold)
          sp<float>(W_OU)[tid] = bj;  // b for the fold (the column's share of u is used up)
        else
          tnew[dk + tid] = bj;
      }
      if (!fold) {  // append this token's factors, keep the window open
        if (tid < dk) {
          tnew[tid] = sp<float>(W_K)[tid] / sp<float>(W_GN)[tid];
          reinterpret_cast<float*>(side + 16)[tid] = sp<float>(W_GN)[tid];
        }
        if (tid == 0) *reinterpret_cast<int32_t*>(side) = cnt + 1;
      } else {  // end of the window: fold everything into the block
        __syncthreads();
        float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c.act()) bv = *reinterpret_cast<const float4*>(sp<float>(W_OU) + 4 * c.lane);
        uint8_t* dst = a.pool + (size_t)hdr.slot * a.slot_bytes + hdr.off;
        window_fold<GATE, FULL, ROWS>(c, a, blk, terms, cnt, mode, cv, bv, dst, rho,
                                      reinterpret_cast<int32_t*>(side));
      }
    }
    __syncthreads();  // the term buffer and this item's shared arrays are free
  }

  if (timed_out) {
    if (tid == 0) atomicOr(a.flag, SQ_FLAG_TIMEOUT_BIT);
    // let copies still in flight land before the CTA exits: stage s has received
    // W_MISC[4 + s] copies, of which the items before `it` consumed (it + 1 - s) / 2
    __syncthreads();
    for (int s2 = 0; s2 < 2; ++s2) {
      const int issued = sp<int>(W_MISC)[4 + s2], used = (it + 1 - s2) / 2;
      for (int u = used; u < issued; ++u) mbar_wait_bounded(&full[s2], (uint32_t)u & 1u);
    }
    mbar_wait_bounded(tfull, (uint32_t)it & 1u);
    if (producer && c.lane < 3) cp_async_wait_all();
  }
  tmem_fence_before_sync();
  __syncthreads();
  if (c.warp == 0) {
    tmem_fence_after_sync();
    tmem_dealloc(tbase, kTmemCols);
  }
}

template <int GATE, int IO, bool FULL, bool ROWS>
cudaError_t launch_w(const StepArgs& a, int num_sms, cudaStream_t st) {
  auto fn = k_window<GATE, IO, FULL, ROWS>;
  const WDPlan P(a.dk, a.dv, IO, GATE, ROWS, a.stage_bytes, a.H, a.window);
  const uint32_t smem_bytes = P.total > 47u * 1024u ? P.total : 47u * 1024u;
  int per_sm = 0;
  cudaError_t e = resident_ctas(reinterpret_cast<const void*>(fn), smem_bytes, &per_sm);
  if (e != cudaSuccess) return e;
  if (per_sm > kMaxCtasPerSm) per_sm = kMaxCtasPerSm;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return e;
  const int items = a.batch * a.H;
  int grid = num_sms * per_sm;
  if (grid > items) grid = items;
  if (grid < 1) return cudaSuccess;
  fn<<<grid, kT, smem_bytes, st>>>(a);
  return cudaGetLastError();
}

template <int GATE, int IO>
cudaError_t launch_w_shape(const StepArgs& a, int num_sms, cudaStream_t st) {
  const bool full = a.dk == kMaxD && a.dv == kMaxD;
  if (a.per_row)
    return full ? launch_w<GATE, IO, true, true>(a, num_sms, st) : launch_w<GATE, IO, false, true>(a, num_sms, st);
  return full ? launch_w<GATE, IO, true, false>(a, num_sms, st) : launch_w<GATE, IO, false, false>(a, num_sms, st);
}


// =============================================================================================
// Multi-token chunk: T consecutive tokens of each request advance its state, which is read
// from the pool once and requantized once, after the T-th token (prefill or speculative decode
// into a quantized state). The state within the chunk is exactly the windowed variant's
// S_t = diag(g_t) (Sbar + sum_{s<t} k_hat_s b_s^T) with W = T, held on chip: the codes of Sbar
// in tensor memory (unpacked once), the low-rank terms in shared memory. Per token: the row
// factors A_i y_i, A_i z_i, one pass over the codes for Sbar^T y and Sbar^T z, the low-rank
// coefficients, then u, b, o one column per thread. After the last token the state is folded
// and requantized by the windowed variant's fold (without compensation entries).
// Inputs of request b, head h, token t: q, k at [b][h][t][d_k], v at [b][h][t][d_v], alpha at
// [b][h][t] (scalar gate) or [b][h][t][d_k], beta at [b][h][t]; o at [b][h][t][d_v].
// =============================================================================================
constexpr int kMaxChunk = 16;

// Stage: header, q, k, v, (alpha per key channel), (alpha per token), beta, (row table),
// block; then the low-rank term buffer and the head table.
struct CPlan {
  uint32_t esz, q_off, k_off, v_off, al_off, as_off, bs_off, rt_off, blk_off, stage, terms, tab,
      total;
  __host__ __device__ CPlan(int dk, int dv, int io, int gate, int per_row, uint32_t stage_bytes,
                            int n_heads, int T) {
    esz = io == 1 ? 2u : 4u;
    q_off = (uint32_t)sizeof(StageHdr);
    k_off = q_off + (uint32_t)T * dk * esz;
    v_off = k_off + (uint32_t)T * dk * esz;
    al_off = v_off + (uint32_t)T * dv * esz;
    as_off = al_off + (gate == 1 ? 4u * T * dk : 0u);
    bs_off = as_off + (gate == 1 ? 0u : round16(4u * T));
    rt_off = bs_off + round16(4u * T);
    blk_off = rt_off + (per_row ? 4u * dk : 0u);
    stage = blk_off + round16(stage_bytes + kSlack);
    terms = W_STAGE + stage;
    tab = terms + (uint32_t)(T > 1 ? T - 1 : 1) * 4u * (dk + dv);
    total = tab + round16(20u * (uint32_t)n_heads);
  }
};

// Arrive on `bar` when this thread's cp.async copies so far have landed (the arrival is counted
// in advance, so the phase cannot complete before they do).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Pass A of a later token: Sbar^T y and Sbar^T z from the codes held in tensor memory.
template <bool FULL>
__device__ __forceinline__ void pass_a_tmem(const Ctx<FULL>& c) {
  const float4* gkq = sp<float4>(S_GKQ) + c.row0() / 2;
  float2 U[4], P[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) U[e] = P[e] = f2(0.f, 0.f);
  sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const float4 g = gkq[2 * ch + pr];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        U[e] = __ffma2_rn(v[4 * pr + e], lo(g), U[e]);
        P[e] = __ffma2_rn(v[4 * pr + e], hi(g), P[e]);
      }
    }
  });
  *reinterpret_cast<float4*>(sp<float>(S_REDU) + c.warp * kMaxD + 4 * c.lane) =
      make_float4(U[0].x + U[0].y, U[1].x + U[1].y, U[2].x + U[2].y, U[3].x + U[3].y);
  *reinterpret_cast<float4*>(sp<float>(S_REDP) + c.warp * kMaxD + 4 * c.lane) =
      make_float4(P[0].x + P[0].y, P[1].x + P[1].y, P[2].x + P[2].y, P[3].x + P[3].y);
}

// Pass A of the first token: the codes unpacked into tensor memory, with Sbar^T y and Sbar^T z.
template <bool FULL, bool ROWS>
__device__ __forceinline__ void pass_a_codes(const Ctx<FULL>& c, const uint8_t* blk, int mode,
                                             const float4& icv) {
  if (ROWS) {
    pass_a_rows(c, blk, icv);
  } else {
    switch (mode) {
      case 2: pass_a_head<2>(c, blk); break;
      case 4: pass_a_head<4>(c, blk); break;
      case 6: pass_a_head<6>(c, blk); break;
      case 8: pass_a_head<8>(c, blk); break;
      default: pass_a_head<16>(c, blk); break;
    }
  }
  tmem_wait_st();
}

// The tile takes the state itself: x <- g (x A c + sum_{s < cnt} k_hat_s b_s^T), g per row from
// the processing-row table, A from the row-pair factors.
template <bool FULL, bool ROWS>
__device__ __forceinline__ void rebase_tile(const Ctx<FULL>& c, const float* terms, int cnt,
                                            const float4& cv) {
  const int dk = c.dk(), lane = c.lane;
  const uint32_t ts = (uint32_t)(dk + c.dv());
  const float2 cc[4] = {dup(cv.x), dup(cv.y), dup(cv.z), dup(cv.w)};
  const float4* ak = sp<float4>(S_AK) + c.row0() / 2;
  const float2* gnp = reinterpret_cast<const float2*>(sp<float>(W_GNP) + c.row0());
  const uint4* rd4 = reinterpret_cast<const uint4*>(sp<uint32_t>(S_RD) + c.row0());
  sweep(c.tm, c.nch(), [&](int ch, float2 (&v)[8]) {
    const uint4 d = rd4[ch];
    float2 acc[8];
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const float4 f = ak[2 * ch + pr];
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[4 * pr + e] = __fmul2_rn(v[4 * pr + e], __fmul2_rn(lo(f), cc[e]));
    }
#pragma unroll 1
    for (int s = 0; s < cnt; ++s) {
      const float* t = terms + (size_t)s * ts;
      const float4 b4 = c.act() ? *reinterpret_cast<const float4*>(t + dk + 4 * lane)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
      const float2 bs[4] = {dup(b4.x), dup(b4.y), dup(b4.z), dup(b4.w)};
      const float4 k4 = make_float4(t[rd_row(d.x)], t[rd_row(d.y)], t[rd_row(d.z)], t[rd_row(d.w)]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[e] = __ffma2_rn(lo(k4), bs[e], acc[e]);
        acc[4 + e] = __ffma2_rn(hi(k4), bs[e], acc[4 + e]);
      }
    }
#pragma unroll
    for (int pr = 0; pr < 2; ++pr) {
      const float2 g = gnp[2 * ch + pr];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[4 * pr + e] = __fmul2_rn(acc[4 * pr + e], g);
    }
    tmem_st16x2(c.tm + 16u * ch, v);
  });
  tmem_wait_st();
  __syncwarp();
}

// Head units: 3 CTAs per SM (shared memory holds a pivot head's 32 KB tile); key-row units: 4.
template <int GATE, int IO, bool FULL, bool ROWS>
__global__ void __launch_bounds__(kT, ROWS ? 4 : 3) k_chunk(const StepArgs a) {
  const int T = a.n_tok;
  const CPlan P(a.dk, a.dv, IO, GATE, ROWS, a.stage_bytes, a.H, T);
  uint64_t* full = sp<uint64_t>(W_BAR);
  Ctx<FULL> c;
  c.tid = threadIdx.x;
  c.warp = c.tid >> 5;
  c.lane = c.tid & 31;
  c.dk_ = a.dk;
  c.dv_ = a.dv;
  c.act_ = 4 * c.lane < a.dv;
  {
    const int rows = a.dk - c.warp * kRW;
    c.nch_ = rows <= 0 ? 0 : (rows >= kRW ? kMaxCh : rows / 4);
  }
  const int H = a.H, B = a.batch, dk = c.dk(), dv = c.dv(), tid = c.tid;
  const int n_items = B * H;
  const int stride = gridDim.x;
  float* terms = reinterpret_cast<float*>(smem + P.terms);
  const uint8_t* st = smem + W_STAGE;
  const uint8_t* blk = st + P.blk_off;

  if (c.warp == 0) {
    tmem_alloc(sp<uint32_t>(S_TMEM), kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(full, 1);
    fence_mbar_init();
  }
  if (tid < 16) sp<int>(S_FLAGS)[tid] = 0;
  HeadDesc* htab = reinterpret_cast<HeadDesc*>(smem + P.tab);
  int32_t* otab = reinterpret_cast<int32_t*>(smem + P.tab + 16u * H);
  for (int h = tid; h < H; h += kT) {
    htab[h] = a.heads[h];
    otab[h] = a.order[h];
  }
  tmem_fence_before_sync();
  __syncthreads();
  tmem_fence_after_sync();
  const uint32_t tbase = *sp<uint32_t>(S_TMEM);
  c.tm = tbase + ((uint32_t)(32 * c.warp) << 16);

  Meta* meta = sp<Meta>(S_META);
  int* flag_base = sp<int>(S_FLAGS);
  const bool producer = c.warp == kW - 1;
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
  Cursor next_issue{first, first / B, first % B};
  Cursor next_meta = next_issue;
  auto fetch_meta = [&](Cursor& k) {  // the item's slot, one item ahead
    if (c.lane == 0 && k.item < n_items) {
      cp_async4(&meta->slot, a.slot_idx + k.b);
      cp_async_commit();
    }
    advance(k);
  };
  // Stage an item: lanes < T copy its per-token scalars by cp.async (their arrival is tied to
  // the stage barrier), lane 0 writes the header and arrives with the byte count, lanes 1..6
  // issue the bulk copies.
  auto issue = [&](Cursor& k, int fslot) {
    if (c.lane == 0) cp_async_wait_all();
    __syncwarp();
    uint8_t* s = smem + W_STAGE;
    const int h = otab[k.hh], io = k.b * H + h;
    const HeadDesc hd = htab[h];
    const int32_t slot = meta->slot;
    const bool valid = slot >= 0 && slot < a.n_slots;
    __syncwarp();
    const uint32_t qb = (uint32_t)T * dk * P.esz, vb = (uint32_t)T * dv * P.esz;
    const uint32_t ab = GATE == 1 ? 4u * T * dk : 0u, rb = ROWS ? 4u * dk : 0u;
    if (valid && c.lane < T) {
      if (GATE == 0) cp_async4(s + P.as_off + 4 * c.lane, a.alpha + (size_t)io * T + c.lane);
      cp_async4(s + P.bs_off + 4 * c.lane, a.beta + (size_t)io * T + c.lane);
      cp_async_commit();
      cp_async_arrive(full);
    }
    __syncwarp();
    if (c.lane == 0) {
      int* nf = flag_base + 4 * fslot;
      nf[F_INPUT] = nf[F_RANGE] = nf[F_UNDER] = 0;
      StageHdr* shdr = reinterpret_cast<StageHdr*>(s);
      *reinterpret_cast<int4*>(shdr) = make_int4(valid, slot, k.b, h);
      *(reinterpret_cast<int4*>(shdr) + 1) =
          make_int4(0, 0, hd.pivot_head ? MODE_PIVOT : (int)hd.width, (int)hd.off);
      mbar_arrive_expect_tx(full, valid ? 2 * qb + vb + ab + rb + hd.bytes : 0u);
    }
    if (valid && c.lane >= 1 && c.lane <= 6) {
      uint8_t* dst = s;
      const uint8_t* src = nullptr;
      uint32_t n = 0;
      switch (c.lane) {
        case 1: dst += P.q_off, src = static_cast<const uint8_t*>(a.q) + (size_t)io * qb, n = qb; break;
        case 2: dst += P.k_off, src = static_cast<const uint8_t*>(a.k) + (size_t)io * qb, n = qb; break;
        case 3: dst += P.v_off, src = static_cast<const uint8_t*>(a.v) + (size_t)io * vb, n = vb; break;
        case 4: dst += P.al_off, src = reinterpret_cast<const uint8_t*>(a.alpha + (size_t)io * T * dk), n = ab; break;
        case 5: dst += P.rt_off, src = reinterpret_cast<const uint8_t*>(a.srows + (size_t)h * dk), n = rb; break;
        default: dst += P.blk_off, src = a.pool + (size_t)slot * a.slot_bytes + hd.off, n = hd.bytes; break;
      }
      if (n) bulk_load(dst, src, n, full);
    }
    __syncwarp();
    advance(k);
  };

  if (producer && next_issue.item < n_items) {
    fetch_meta(next_meta);
    issue(next_issue, 0);
    fetch_meta(next_meta);
  }

  int it = 0;
  bool timed_out = false;
  int32_t dummy_count = 0;
  for (int item = first; item < n_items; item += stride, ++it) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(full, (uint32_t)it & 1u));
    c.flags = flag_base + 4 * (it & 3);
    StageHdr hdr = *reinterpret_cast<const StageHdr*>(st);
    if (!ok) hdr.valid = 0;
    const int io = hdr.b * H + hdr.h;
    const int mode = ROWS ? MODE_ROWS : hdr.mode;
    const bool pivot_head = !ROWS && mode == MODE_PIVOT;
    const float* bs = reinterpret_cast<const float*>(st + P.bs_off);
    const float* as = reinterpret_cast<const float*>(st + P.as_off);

    // ---- token-independent setup, and every token's inputs checked ----
    float tc = 1.f, g = 1.f, A = 1.f, rho = 1.f;
    float4 cv = make_float4(1.f, 1.f, 1.f, 1.f), icv = make_float4(1.f, 1.f, 1.f, 1.f);
    int i = 0;
    if (hdr.valid) {
      bool bad_in = false;
      const int p = tid;
      if (p < dk) {
        uint32_t d;
        if (ROWS) {
          d = reinterpret_cast<const uint32_t*>(st + P.rt_off)[p];
        } else {
          const uint32_t off = pivot_head ? (uint32_t)p * 2u * dv
                                          : 2u * (dk + dv) + (uint32_t)p * dv * mode / 8u;
          d = (uint32_t)p << 24 | off << 8 | (uint32_t)mode;
        }
        sp<uint32_t>(S_RD)[p] = d;
        i = rd_row(d);
        if (a.rho) rho = __ldg(a.rho + (size_t)hdr.h * dk + i);
        sp<int>(W_INV)[i] = p;
        sp<float>(S_TR)[p] = 1.f;  // the fold's tile holds the state itself
        A = (!pivot_head && rd_width(d) != 16) ? __half2float(reinterpret_cast<const __half*>(blk)[i]) : 1.f;
        float* akp = sp<float>(S_AK) + 4 * (p >> 1) + (p & 1);
        akp[0] = A;
        akp[2] = 0.f;
        for (int t = 0; t < T; ++t) {
          const float kt = ld_io(st + P.k_off, IO, t * dk + i), qt = ld_io(st + P.q_off, IO, t * dk + i);
          const float at = GATE == 0 ? as[t] : reinterpret_cast<const float*>(st + P.al_off)[t * dk + i];
          bad_in |= !isfinite(kt) || !isfinite(qt) || !isfinite(at);
        }
      }
      if (tid < dv) {
        if (!pivot_head) tc = __half2float(reinterpret_cast<const __half*>(blk)[dk + tid]);
        for (int t = 0; t < T; ++t) bad_in |= !isfinite(ld_io(st + P.v_off, IO, t * dv + tid));
      }
      if (tid < T) bad_in |= !isfinite(bs[tid]);
      if (c.act() && !pivot_head) {
        const uint2 ch = reinterpret_cast<const uint2*>(blk + 2 * dk)[c.lane];
        const float2 a01 = __half22float2(*reinterpret_cast<const __half2*>(&ch.x));
        const float2 a23 = __half22float2(*reinterpret_cast<const __half2*>(&ch.y));
        cv = make_float4(a01.x, a01.y, a23.x, a23.y);
        if (ROWS) icv = make_float4(rcp_f16val(cv.x), rcp_f16val(cv.y), rcp_f16val(cv.z), rcp_f16val(cv.w));
      }
      if (bad_in) atomicOr(&c.flags[F_INPUT], 1);
    }
    if (__syncthreads_or(!ok)) {
      timed_out = true;
      break;
    }
    const bool skip = !hdr.valid || c.flags[F_INPUT];

    // ---- the tokens; terms held: tokens t0 .. t-1 ----
    int t0 = 0;
    bool rebased = false;
    for (int t = 0; t < T && !skip; ++t) {
      float gn = g, kt = 0.f, qt = 0.f;
      if (tid < dk) {
        kt = ld_io(st + P.k_off, IO, t * dk + i);
        qt = ld_io(st + P.q_off, IO, t * dk + i);
        gn = g * (GATE == 0 ? as[t] : reinterpret_cast<const float*>(st + P.al_off)[t * dk + i]);
      }
      // The previous token's term is complete. A gate product outside [1e-30, 1e30] would put
      // k_hat = k / g out of range: the tile then takes the gated state S' itself (exact up to
      // one fp32 rounding per element) and the factors restart with A = c = g = 1.
      if (__syncthreads_or(tid < dk && !(fabsf(gn) >= 1e-30f && fabsf(gn) <= 1e30f))) {
        float* gkq = sp<float>(S_GKQ) + 4 * (tid >> 1) + (tid & 1);
        if (t == 0) {  // the codes are not in tensor memory yet
          if (tid < dk) gkq[0] = gkq[2] = 0.f;
          __syncwarp();
          pass_a_codes<FULL, ROWS>(c, blk, mode, icv);
        }
        if (tid < dk) sp<float>(W_GNP)[tid] = gn;
        __syncwarp();
        rebase_tile<FULL, ROWS>(c, terms, t - t0, cv);
        if (tid < dk) sp<float>(S_AK)[4 * (tid >> 1) + (tid & 1)] = 1.f;
        __syncwarp();
        A = 1.f;
        tc = 1.f;
        cv = make_float4(1.f, 1.f, 1.f, 1.f);
        gn = 1.f;
        t0 = t;
        rebased = true;
      }
      g = gn;
      const int tt = t - t0;  // this token's term index
      float kqp = 0.f;
      if (tid < dk) {
        const float yi = g * kt, zi = g * qt;
        float* gkq = sp<float>(S_GKQ) + 4 * (tid >> 1) + (tid & 1);
        gkq[0] = A * yi;
        gkq[2] = A * zi;
        sp<float>(W_Y)[i] = yi;
        sp<float>(W_Z)[i] = zi;
        if (t + 1 < T) {
          terms[(size_t)tt * (dk + dv) + i] = kt / g;
        } else {  // the last token's k and g, for the fold
          sp<float>(S_AK)[4 * (tid >> 1) + (tid & 1) + 2] = kt;
          sp<float>(W_GNP)[tid] = g;
        }
        kqp = kt * qt;
      }
      kqp = warp_sum(kqp);
      if (c.lane == 0) sp<float>(S_KQ)[c.warp] = kqp;
      __syncwarp();
      if (t == 0 && !rebased) {
        pass_a_codes<FULL, ROWS>(c, blk, mode, icv);
      } else {
        pass_a_tmem(c);
      }
      __syncthreads();  // partial sums, y, z
      float u0 = 0.f, p0 = 0.f;
      if (tid < dv) {
        const float* ru = sp<float>(S_REDU) + tid;
        const float* rp = sp<float>(S_REDP) + tid;
        u0 = tc * ((ru[0] + ru[kMaxD]) + (ru[2 * kMaxD] + ru[3 * kMaxD]));
        p0 = tc * ((rp[0] + rp[kMaxD]) + (rp[2 * kMaxD] + rp[3 * kMaxD]));
      }
      for (int s2 = c.warp; s2 < tt; s2 += kW) {  // low-rank coefficients
        float dy = 0.f, dz = 0.f;
        if (4 * c.lane < dk) {
          const float4 kh = *reinterpret_cast<const float4*>(terms + (size_t)s2 * (dk + dv) + 4 * c.lane);
          const float4 y4 = *reinterpret_cast<const float4*>(sp<float>(W_Y) + 4 * c.lane);
          const float4 z4 = *reinterpret_cast<const float4*>(sp<float>(W_Z) + 4 * c.lane);
          dy = __fmaf_rn(kh.x, y4.x, __fmaf_rn(kh.y, y4.y, __fmaf_rn(kh.z, y4.z, kh.w * y4.w)));
          dz = __fmaf_rn(kh.x, z4.x, __fmaf_rn(kh.y, z4.y, __fmaf_rn(kh.z, z4.z, kh.w * z4.w)));
        }
        dy = warp_sum(dy);
        dz = warp_sum(dz);
        if (c.lane == 0) {
          sp<float>(W_LR)[2 * s2] = dy;
          sp<float>(W_LR)[2 * s2 + 1] = dz;
        }
      }
      __syncthreads();  // coefficients, k.q
      if (tid < dv) {
        float u = u0, pq = p0;
        const float2* lr = reinterpret_cast<const float2*>(sp<float>(W_LR));
        for (int s2 = 0; s2 < tt; ++s2) {
          const float bt = terms[(size_t)s2 * (dk + dv) + dk + tid];
          const float2 l = lr[s2];
          u = __fmaf_rn(l.x, bt, u);
          pq = __fmaf_rn(l.y, bt, pq);
        }
        const float4 kq4 = *sp<float4>(S_KQ);
        const float kqv = (kq4.x + kq4.y) + (kq4.z + kq4.w);
        const float bj = bs[t] * (ld_io(st + P.v_off, IO, t * dv + tid) - u);
        a.out[((size_t)io * T + t) * dv + tid] = __fmaf_rn(bj, kqv, pq);
        if (t + 1 < T)
          terms[(size_t)tt * (dk + dv) + dk + tid] = bj;
        else
          sp<float>(W_OU)[tid] = bj;
      }
    }
    __syncthreads();  // the last token's term; the stage is no longer read
    if (producer && next_issue.item < n_items) {  // stage the next item
      issue(next_issue, (it + 1) & 3);
      fetch_meta(next_meta);
    }
    if (skip) {
      if (tid == 0)
        if (tid == 0) atomicOr(a.flag, hdr.valid ? SQ_FLAG_NONFINITE_BIT : SQ_FLAG_BAD_SLOT_BIT);
      for (int x = tid; x < T * dv; x += kT) a.out[(size_t)io * T * dv + x] = __int_as_float(0x7fc00000);
    } else {  // fold the chunk into the block
      float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c.act()) bv = *reinterpret_cast<const float4*>(sp<float>(W_OU) + 4 * c.lane);
      uint8_t* dst = a.pool + (size_t)hdr.slot * a.slot_bytes + hdr.off;
      window_fold<GATE, FULL, ROWS>(c, a, blk, terms, T - 1 - t0, mode, cv, bv, dst, rho,
                                    &dummy_count);
    }
    __syncthreads();
  }
  if (timed_out) {
    if (tid == 0) atomicOr(a.flag, SQ_FLAG_TIMEOUT_BIT);
    mbar_wait_bounded(full, (uint32_t)it & 1u);  // the copy in flight, if any
    if (producer && c.lane < 32) cp_async_wait_all();
  }
  tmem_fence_before_sync();
  __syncthreads();
  if (c.warp == 0) {
    tmem_fence_after_sync();
    tmem_dealloc(tbase, kTmemCols);
  }
}

template <int GATE, int IO, bool FULL, bool ROWS>
cudaError_t launch_c(const StepArgs& a, int num_sms, cudaStream_t st) {
  auto fn = k_chunk<GATE, IO, FULL, ROWS>;
  const CPlan P(a.dk, a.dv, IO, GATE, ROWS, a.stage_bytes, a.H, a.n_tok);
  const uint32_t smem_bytes = P.total > 47u * 1024u ? P.total : 47u * 1024u;
  int per_sm = 0;
  cudaError_t e = resident_ctas(reinterpret_cast<const void*>(fn), smem_bytes, &per_sm);
  if (e != cudaSuccess) return e;
  if (per_sm > kMaxCtasPerSm) per_sm = kMaxCtasPerSm;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return e;
  const int items = a.batch * a.H;
  int grid = num_sms * per_sm;
  if (grid > items) grid = items;
  if (grid < 1) return cudaSuccess;
  fn<<<grid, kT, smem_bytes, st>>>(a);
  return cudaGetLastError();
}

template <int GATE, int IO>
cudaError_t launch_c_shape(const StepArgs& a, int num_sms, cudaStream_t st) {
  const bool full = a.dk == kMaxD && a.dv == kMaxD;
  if (a.per_row)
    return full ? launch_c<GATE, IO, true, true>(a, num_sms, st) : launch_c<GATE, IO, false, true>(a, num_sms, st);
  return full ? launch_c<GATE, IO, true, false>(a, num_sms, st) : launch_c<GATE, IO, false, false>(a, num_sms, st);
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

cudaError_t launch_window_step(const StepArgs& a, int gate, int io, int num_sms, cudaStream_t st) {
  if (a.window > kMaxWin) return cudaErrorInvalidValue;
  if (gate == 0 && io == 0) return launch_w_shape<0, 0>(a, num_sms, st);
  if (gate == 0 && io == 1) return launch_w_shape<0, 1>(a, num_sms, st);
  if (gate == 1 && io == 0) return launch_w_shape<1, 0>(a, num_sms, st);
  return launch_w_shape<1, 1>(a, num_sms, st);
}

cudaError_t launch_chunk(const StepArgs& a, int gate, int io, int num_sms, cudaStream_t st) {
  if (a.n_tok < 1 || a.n_tok > kMaxChunk) return cudaErrorInvalidValue;
  if (gate == 0 && io == 0) return launch_c_shape<0, 0>(a, num_sms, st);
  if (gate == 0 && io == 1) return launch_c_shape<0, 1>(a, num_sms, st);
  if (gate == 1 && io == 0) return launch_c_shape<1, 0>(a, num_sms, st);
  return launch_c_shape<1, 1>(a, num_sms, st);
}

}  // namespace sq
