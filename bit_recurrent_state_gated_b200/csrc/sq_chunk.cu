// sq_chunk.cu -- the multi-token chunk step of libsq (sm_100a).
#include "sq_fold.cuh"

namespace sq {
namespace {

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
template <class C>
__device__ __forceinline__ void pass_a_tmem(const C& c) {
  const float4* gkq = sp<float4>(S_GKQ) + c.row0() / 2;
  float2 U[4], P[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) U[e] = P[e] = f2(0.f, 0.f);
  sweep(c, [&](int ch, float2 (&v)[8]) {
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
  sweep(c, [&](int ch, float2 (&v)[8]) {
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
      mbar_arrive_expect_tx(full, valid ? 2 * qb + vb + ab + rb + hd.bytes + a.extra_tx : 0u);
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
  const uint64_t wait_ns = a.wait_ns ? a.wait_ns : kWaitLimitNs;
  int32_t dummy_count = 0;
  for (int item = first; item < n_items; item += stride, ++it) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(full, (uint32_t)it & 1u, wait_ns));
    c.flags = flag_base + 4 * (it & 3);
    StageHdr hdr = *reinterpret_cast<const StageHdr*>(st);
    if (!ok) hdr.valid = 0;
    const int io = hdr.b * H + hdr.h;
    const int mode = ROWS ? MODE_ROWS : hdr.mode;
    const bool pivot_head = !ROWS && mode == MODE_PIVOT;
    const float* bs = reinterpret_cast<const float*>(st + P.bs_off);
    const float* as = reinterpret_cast<const float*>(st + P.as_off);

    // ---- token-independent setup, and every token's inputs checked ----
    float tc = 1.f, g = 1.f, A = 1.f, omega = 1.f;
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
        if (a.omega) omega = __ldg(a.omega + (size_t)hdr.h * dk + i);
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
      if (tid == 0) atomicOr(a.flag, hdr.valid ? SQ_FLAG_NONFINITE_BIT : SQ_FLAG_BAD_SLOT_BIT);
      for (int x = tid; x < T * dv; x += kT) a.out[(size_t)io * T * dv + x] = __int_as_float(0x7fc00000);
    } else {  // fold the chunk into the block
      float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c.act()) bv = *reinterpret_cast<const float4*>(sp<float>(W_OU) + 4 * c.lane);
      uint8_t* dst = a.pool + (size_t)hdr.slot * a.slot_bytes + hdr.off;
      window_fold<GATE, FULL, ROWS, false>(c, a, blk, reinterpret_cast<const uint8_t*>(terms),
                                           4u * (uint32_t)(dk + dv), 4u * (uint32_t)dk,
                                           T - 1 - t0, mode, cv, bv, dst, omega, &dummy_count);
    }
    __syncthreads();
  }
  if (timed_out) {
    if (tid == 0) atomicOr(a.flag, SQ_FLAG_TIMEOUT_BIT);
    mbar_wait_bounded(full, (uint32_t)it & 1u, wait_ns);  // the copy in flight, if any
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

cudaError_t launch_chunk(const StepArgs& a, int gate, int io, int num_sms, cudaStream_t st) {
  if (a.n_tok < 1 || a.n_tok > kMaxChunk) return cudaErrorInvalidValue;
  if (gate == 0 && io == 0) return launch_c_shape<0, 0>(a, num_sms, st);
  if (gate == 0 && io == 1) return launch_c_shape<0, 1>(a, num_sms, st);
  if (gate == 1 && io == 0) return launch_c_shape<1, 0>(a, num_sms, st);
  return launch_c_shape<1, 1>(a, num_sms, st);
}

}  // namespace sq
