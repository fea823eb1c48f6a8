// sq_fold.cuh -- the window-end fold shared by the windowed step (sq_window_step.cu) and the
// multi-token chunk (sq_chunk.cu): materialize the full-precision state in tensor memory, choose
// the compensation entries, refit and requantize.
#pragma once
#include "sq_step.cuh"

namespace sq {
namespace {

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
// Side block of one (slot, head): see SideFmt (sq_internal.h); for the scalar gate a term holds
// the token's k in the I/O type and b_s / g_s, whose product is k_hat_s b_s^T. The staging
// buffer holds the next item's q, k, v (alpha, row table), side header (+ g) and frozen block;
// the low-rank terms, whose count is known only once the header has landed, follow into their
// own buffer while pass A runs.
// =============================================================================================
constexpr int kMaxWin = 64;
constexpr int kMaxCand = 256;  // candidate entries for the compensation choice

// Window-only shared memory, after the per-step kernel's fixed arrays.
constexpr uint32_t W_BAR = S_STAGE;          // full (stage), tfull (terms)
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
                                             // byte offset, [4] items staged
constexpr uint32_t W_OE = W_MISC + 64;       // the frozen block's compensation entries:
                                             // flat index [64] int, value [64] float
constexpr uint32_t W_STAGE = W_OE + 512;
static_assert(W_STAGE % 16 == 0, "16-byte aligned");
// Candidates of the compensation choice share the column-maxima buffer (used later).
constexpr uint32_t W_CIDX = S_REDC, W_CPOS = S_REDC + 4 * kMaxCand, W_CVAL = S_REDC + 8 * kMaxCand;
constexpr uint32_t W_CSEL = S_REDC + 12 * kMaxCand;  // the chosen n in key order: idx, pos, value
static_assert(12 * kMaxCand + 3 * 64 * 4 <= 4096, "candidates fit the column-maxima buffer");

enum { F_UNDER = 2 };

// Stage: header, k, q, v, (alpha), (row table), side header (+ g), block; then the low-rank term
// buffer and the head table.
struct WDPlan {
  uint32_t esz, k_off, q_off, v_off, al_off, rt_off, sh_off, blk_off, stage, terms, tab, total;
  SideFmt side;
  __host__ __device__ WDPlan(int dk, int dv, int io, int gate, int per_row, uint32_t stage_bytes,
                             int n_heads, int window)
      : side(dk, dv, gate, io) {
    esz = io == 1 ? 2u : 4u;
    k_off = (uint32_t)sizeof(StageHdr);
    q_off = k_off + dk * esz;
    v_off = q_off + dk * esz;
    al_off = v_off + dv * esz;
    rt_off = al_off + (gate == 1 ? 4u * dk : 0u);
    sh_off = rt_off + (per_row ? 4u * dk : 0u);
    blk_off = sh_off + side.head;
    stage = blk_off + round16(stage_bytes + kSlack);
    terms = W_STAGE + stage;
    tab = terms + (uint32_t)(window - 1) * side.stride;
    total = tab + round16(20u * (uint32_t)n_heads);
  }
};

// The k part of four rows of a term: fp32, or bf16 (K16); head units' four rows are consecutive
// (one load), key-row units' are gathered by original row.
template <bool K16, bool ROWS>
__device__ __forceinline__ float4 term_k4(const uint8_t* t, const int (&orow)[4]) {
  if (K16) {
    if (ROWS) return make_float4(ld_io(t, 1, orow[0]), ld_io(t, 1, orow[1]), ld_io(t, 1, orow[2]), ld_io(t, 1, orow[3]));
    const uint2 w = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(t) + orow[0]);
    return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                       __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
  }
  const float* k = reinterpret_cast<const float*>(t);
  if (ROWS) return make_float4(k[orow[0]], k[orow[1]], k[orow[2]], k[orow[3]]);
  return *reinterpret_cast<const float4*>(k + orow[0]);
}

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
template <class C>
__device__ __forceinline__ float tile_patch(const C& c, int p, int j, float add, bool set,
                                            float* old = nullptr) {
  if (p / kRW != c.warp) return 0.f;  // warp-uniform
  const int ch = (p % kRW) / 4;
  uint32_t r[16];
  float2 v[8];
  tm_issue(c.tm + 16u * ch, r);
  tm_take(r, v);
  float nv = 0.f, ov = 0.f;
  if (c.lane == j / 4) {
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
      for (int ee = 0; ee < 4; ++ee)
        if (rr == p % 4 && ee == j % 4) ov = (rr & 1) ? v[4 * (rr >> 1) + ee].y : v[4 * (rr >> 1) + ee].x;
    chunk_add(v, p % 4, j % 4, add, set);
#pragma unroll
    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
      for (int ee = 0; ee < 4; ++ee)
        if (rr == p % 4 && ee == j % 4) nv = (rr & 1) ? v[4 * (rr >> 1) + ee].y : v[4 * (rr >> 1) + ee].x;
  }
  tmem_st16x2(c.tm + 16u * ch, v);
  tmem_wait_st();
  if (old) *old = ov;
  return nv;
}

// Key of an element for the compensation choice: larger |value| first; 0 = not eligible.
__device__ __forceinline__ uint32_t wkey(float v) { return (__float_as_uint(v) & 0x7fffffffu) + 1u; }

// The fold at the window's end (all threads). v of the lane's columns: cv (old c16), bv (b).
// terms: cnt terms of `tstride` bytes, the k part (bf16 if K16, else fp32) then at `boff` the b
// part, fp32; each contributes the rank-one product of its parts.
template <int GATE, bool FULL, bool ROWS, bool K16>
__device__ __forceinline__ void window_fold(const Ctx<FULL>& c, const StepArgs& a, const uint8_t* blk,
                                            const uint8_t* terms, uint32_t tstride, uint32_t boff,
                                            int cnt, int mode, const float4& cv, const float4& bv,
                                            uint8_t* dst, float omega, int32_t* count) {
  const int dk = c.dk(), dv = c.dv(), tid = c.tid, lane = c.lane;
  const bool pivot_head = !ROWS && mode == MODE_PIVOT;
  const int n_out = pivot_head ? 0 : a.n_outliers;
  const float2 cc[4] = {dup(cv.x), dup(cv.y), dup(cv.z), dup(cv.w)};
  const float2 bb[4] = {dup(bv.x), dup(bv.y), dup(bv.z), dup(bv.w)};
  const float4* ak = sp<float4>(S_AK) + c.row0() / 2;
  const float2* gnp = reinterpret_cast<const float2*>(sp<float>(W_GNP) + c.row0());
  const uint4* rd4 = reinterpret_cast<const uint4*>(sp<uint32_t>(S_RD) + c.row0());
  // ---- materialize S = g (x A c + sum_s k_hat_s b_s^T) + k b^T in tensor memory; the thread's
  // largest |S| over the rows eligible for compensation entries ----
  float tmaxf = 0.f;
  sweep(c, [&](int ch, float2 (&v)[8]) {
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
      const uint8_t* t = terms + (size_t)s * tstride;
      const float4 b4 = c.act() ? reinterpret_cast<const float4*>(t + boff)[lane]
                                : make_float4(0.f, 0.f, 0.f, 0.f);
      const float2 bs[4] = {dup(b4.x), dup(b4.y), dup(b4.z), dup(b4.w)};
      const float4 k4 = term_k4<K16, ROWS>(t, orow);  // the chunk's four rows
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
    bool lowered = false;  // a patch lowered the element that held the thread's maximum
    for (int o = 0; o < a.n_outliers; ++o) {
      const int idx = sp<int>(W_OE)[o];
      if (idx >= dk * dv) continue;
      const float pv = sp<float>(W_OE)[64 + o];
      const int i = idx / dv, j = idx % dv;
      float ov = 0.f;
      const float nv = fabsf(tile_patch(c, sp<int>(W_INV)[i], j, sp<float>(W_GN)[i] * pv, false, &ov));
      lowered |= nv < fabsf(ov) && fabsf(ov) >= tmaxf;
      tmaxf = fmaxf(tmaxf, nv);
    }
    // then the recorded maximum may exceed every element of the thread: that warp rescans its
    // tile, so that the thread maxima below are exact and the n-th largest of them bounds the
    // n-th largest element from below
    if (__any_sync(0xffffffffu, lowered)) {
      tmaxf = 0.f;
      sweep(c, [&](int ch, float2 (&v)[8]) {
        if (ROWS) {
          const uint4 d = rd4[ch];
#pragma unroll
          for (int r = 0; r < 4; ++r)
            if (rd_width((&d.x)[r]) != 16)
              tmaxf = fmaxf(tmaxf, (r & 1) ? rowmax_y(v + 4 * (r >> 1)) : rowmax_x(v + 4 * (r >> 1)));
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) tmaxf = max3abs(tmaxf, v[e].x, v[e].y);
        }
      });
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
    sweep(c, [&](int ch, float2 (&v)[8]) {
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
    // The thread maxima are exact (a warp whose patch lowered a thread's largest element
    // rescanned above), so at least n elements reach the threshold and every element of the top
    // n is among the candidates; the exact path below only serves more than kMaxCand ties.
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
      // Entries start empty (an index no element has, sorted last, never patched): the layout
      // guarantees at least n eligible elements, so every round fills one, and an entry left
      // empty would be skipped rather than read as stale shared memory.
      if (tid < n_out) {
        oidx[tid] = 0x7fffffff;
        opos[tid] = -1;
        oval[tid] = 0.f;
      }
      __syncthreads();
      for (int r = 0; r < n_out; ++r) {
        unsigned long long best = 0;
        int bp = 0;
        float bvx = 0.f;
        sweep(c, [&](int ch, float2 (&v)[8]) {
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
      if (opos[o] >= 0) tile_patch(c, opos[o] >> 8, opos[o] & 0xff, 0.f, true);
    if (tid < n_out && __hisinf(__float2half_rn(oval[tid]))) atomicOr(&c.flags[F_RANGE], 1);
  }
  // ---- refit and requantize (pivot heads: round to fp16) ----
  if (pivot_head) {
    bool of = false;
    sweep(c, [&](int ch, float2 (&v)[8]) {
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
  {  // row maxima (row_scales checks the fp16 rows' range on them)
    float4* rtab = reinterpret_cast<float4*>(sp<float>(S_RT) + c.row0());
    sweep(c, [&](int ch, float2 (&v)[8]) {
      float rm[4];
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {
        rm[2 * pr] = warp_max_nonneg(rowmax_x(v + 4 * pr));
        rm[2 * pr + 1] = warp_max_nonneg(rowmax_y(v + 4 * pr));
      }
      if (lane == 0) rtab[ch] = make_float4(rm[0], rm[1], rm[2], rm[3]);
    });
    __syncwarp();
  }
  float4 cm;
  const float r = fit_scales(c, a, omega, cm);
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
    reinterpret_cast<uint16_t*>(o)[2 * tid] = (uint16_t)min(oidx[tid], 0xffff);
    reinterpret_cast<__half*>(o)[2 * tid + 1] = __float2half_rn(oval[tid]);
  }
  if (tid == 0) *count = 0;
}

}  // namespace
}  // namespace sq
