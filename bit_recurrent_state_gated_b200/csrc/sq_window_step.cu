// sq_window_step.cu -- the windowed decode step of libsq (sm_100a): the frozen low-bit block
// plus a low-rank full-precision update per (slot, head), folded and requantized every W tokens.
#include "sq_fold.cuh"

namespace sq {
namespace {

// One staging buffer, refilled with the next item right after the current item's first barrier
// (as in the decode kernel): with the term buffer that keeps a CTA within a quarter of the SM's
// shared memory and 128 registers, so four CTAs (sixteen warps) share an SM. The in-window token
// is bound by latency, not by issue, so the extra warps matter more than the shorter lead of the
// copies (two staging buffers at three CTAs per SM: 75 us per in-window token at 256 x 32).
template <int GATE, int IO, bool FULL, bool ROWS>
__global__ void __launch_bounds__(kT, 4) k_window(const StepArgs a) {
  const WDPlan P(a.dk, a.dv, IO, GATE, ROWS, a.stage_bytes, a.H, a.window);
  uint64_t* full = sp<uint64_t>(W_BAR);
  uint64_t* tfull = full + 1;
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
  const uint32_t tbytes = P.side.stride, kbytes = P.side.kbytes;
  uint8_t* terms = smem + P.terms;

  if (c.warp == 0) {
    tmem_alloc(sp<uint32_t>(S_TMEM), kTmemCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < 2; ++s) mbar_init(&full[s], 1);
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
    const uint32_t ab = GATE == 1 ? 4u * dk : 0u, rb = ROWS ? 4u * dk : 0u, shb = P.side.head;
    if (c.lane == 0) {
      int* nf = flag_base + 4 * fslot;
      nf[F_INPUT] = nf[F_RANGE] = nf[F_UNDER] = 0;
      ++sp<int>(W_MISC)[4 + s];
      StageHdr* shdr = reinterpret_cast<StageHdr*>(st);
      *reinterpret_cast<int4*>(shdr) = make_int4(valid, m.slot, k.b, h);
      *(reinterpret_cast<int4*>(shdr) + 1) =
          make_int4(__float_as_int(m.beta), __float_as_int(GATE == 0 ? m.alpha : 0.f),
                    hd.pivot_head ? MODE_PIVOT : (int)hd.width, (int)hd.off);
      mbar_arrive_expect_tx(&full[s], valid ? 2 * kb + vb + ab + rb + shb + hd.bytes + a.extra_tx : 0u);
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

  if (tid == 0) sp<int>(W_MISC)[4] = 0;
  __syncthreads();
  if (producer) {
    fetch_meta(next_meta);
    if (next_issue.item < n_items) {
      issue(next_issue, 0, 0);
      fetch_meta(next_meta);
    }
  }

  int it = 0;
  bool timed_out = false;
  const uint64_t wait_ns = a.wait_ns ? a.wait_ns : kWaitLimitNs;
  for (int item = first; item < n_items; item += stride, ++it) {
    const int s = 0;
    const uint8_t* st = smem + W_STAGE;
    const uint8_t* blk = st + P.blk_off;
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(&full[s], (uint32_t)it & 1u, wait_ns));
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
                      P.side.head,
                  (uint32_t)cnt * tbytes, tfull);
    }
    const int io = hdr.b * H + hdr.h;
    const int mode = ROWS ? MODE_ROWS : hdr.mode;
    const bool pivot_head = !ROWS && mode == MODE_PIVOT;

    // ---- setup: thread t takes processing row t and value column t ----
    float tc = 1.f, tv = 0.f, omega = 1.f;
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
        if (a.omega) omega = __ldg(a.omega + (size_t)hdr.h * dk + i);
        sp<int>(W_INV)[i] = p;
        const float ki = ld_io(st + P.k_off, IO, i), qi = ld_io(st + P.q_off, IO, i);
        const float ai = GATE == 0 ? hdr.alpha : reinterpret_cast<const float*>(st + P.al_off)[i];
        bad_in |= !isfinite(ki) || !isfinite(qi) || !isfinite(ai);
        const float gold = cnt == 0 ? 1.f
                           : GATE == 1 ? reinterpret_cast<const float*>(st + P.sh_off + 16)[i]
                                       : reinterpret_cast<const float*>(st + P.sh_off)[1];
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
    // the stage is no longer read: stage the next item
    if (producer && next_issue.item < n_items) {
      issue(next_issue, s, (it + 1) & 3);
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
    const bool tok = __all_sync(0xffffffffu, mbar_wait_bounded(tfull, (uint32_t)it & 1u, wait_ns));
    if (!skip) {  // low-rank coefficients, one term per warp at a time
      for (int t = c.warp; t < cnt; t += kW) {
        float dy = 0.f, dz = 0.f;
        if (4 * c.lane < dk) {
          const int rows4[4] = {4 * c.lane, 4 * c.lane + 1, 4 * c.lane + 2, 4 * c.lane + 3};
          const float4 kh = term_k4<GATE == 0 && IO == 1, false>(terms + (size_t)t * tbytes, rows4);
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
      uint8_t* tnew = side + P.side.head + (size_t)cnt * tbytes;
      if (tid < dv) {
        float u = u0 + sp<float>(W_OU)[tid], pq = p0 + sp<float>(W_OP)[tid];
        const float2* lr = reinterpret_cast<const float2*>(sp<float>(W_LR));
        for (int t = 0; t < cnt; ++t) {
          const float bt = reinterpret_cast<const float*>(terms + (size_t)t * tbytes + kbytes)[tid];
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
        else  // the b part: b, or b / g for the scalar gate
          reinterpret_cast<float*>(tnew + kbytes)[tid] = GATE == 1 ? bj : bj / sp<float>(W_GN)[0];
      }
      if (!fold) {  // append this token's factors, keep the window open
        if (GATE == 1) {  // k_hat = k / g and the gates
          if (tid < dk) {
            reinterpret_cast<float*>(tnew)[tid] = sp<float>(W_K)[tid] / sp<float>(W_GN)[tid];
            reinterpret_cast<float*>(side + 16)[tid] = sp<float>(W_GN)[tid];
          }
          if (tid == 0) *reinterpret_cast<int32_t*>(side) = cnt + 1;
        } else {  // the token's k as given (W_K holds it exactly), the gate in the header
          if (tid < dk) {
            if (IO == 1)
              reinterpret_cast<uint16_t*>(tnew)[tid] = (uint16_t)(__float_as_uint(sp<float>(W_K)[tid]) >> 16);
            else
              reinterpret_cast<float*>(tnew)[tid] = sp<float>(W_K)[tid];
          }
          if (tid == 0)
            *reinterpret_cast<int2*>(side) = make_int2(cnt + 1, __float_as_int(sp<float>(W_GN)[0]));
        }
      } else {  // end of the window: fold everything into the block
        __syncthreads();
        float4 bv = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c.act()) bv = *reinterpret_cast<const float4*>(sp<float>(W_OU) + 4 * c.lane);
        uint8_t* dst = a.pool + (size_t)hdr.slot * a.slot_bytes + hdr.off;
        window_fold<GATE, FULL, ROWS, GATE == 0 && IO == 1>(c, a, blk, terms, tbytes, kbytes, cnt,
                                                             mode, cv, bv, dst, omega,
                                                             reinterpret_cast<int32_t*>(side));
      }
    }
    __syncthreads();  // the term buffer and this item's shared arrays are free
  }

  if (timed_out) {
    if (tid == 0) atomicOr(a.flag, SQ_FLAG_TIMEOUT_BIT);
    // let copies still in flight land before the CTA exits: the stage has received W_MISC[4]
    // copies, of which the items before `it` consumed `it`
    __syncthreads();
    for (int u = it; u < sp<int>(W_MISC)[4]; ++u) mbar_wait_bounded(&full[0], (uint32_t)u & 1u, wait_ns);
    mbar_wait_bounded(tfull, (uint32_t)it & 1u, wait_ns);
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

}  // namespace

cudaError_t launch_window_step(const StepArgs& a, int gate, int io, int num_sms, cudaStream_t st) {
  if (a.window > kMaxWin) return cudaErrorInvalidValue;
  if (gate == 0 && io == 0) return launch_w_shape<0, 0>(a, num_sms, st);
  if (gate == 0 && io == 1) return launch_w_shape<0, 1>(a, num_sms, st);
  if (gate == 1 && io == 0) return launch_w_shape<1, 0>(a, num_sms, st);
  return launch_w_shape<1, 1>(a, num_sms, st);
}

}  // namespace sq
