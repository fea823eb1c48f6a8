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
// Arithmetic: the refit follows the oracle's rule step for step, every operation correctly
// rounded: r_i = max(m_i / Q_i, 2^-14), w_i = 1/(r_i Q_i), c_j = max(max_i |S_ij| w_i, 2^-14),
// v_j = 1/c_j, fp16 rounding once at the end; the code multipliers 1/r16 and 1/c16 are correctly
// rounded too. One difference remains for head units: the tile holds T_ij with M_ij = t_i T_ij
// (t_i the row factor), and a product |M_ij| w_i is taken as fl(|T_ij| fl(t_i w_i)) on the tile
// rather than fl(fl(t_i T_ij) w_i), so it can differ from the rule in the last place. Codes need no
// clamp: every |S_ij| w_i <= c_j, so the quotient S_ij / (r16_i c16_j) is at most Q (1 + 2^-10)
// in magnitude, less than Q + 1/2 for Q <= 127. The state is the GPU's own fp32 update (fused
// multiply-adds), so its scales and codes are compared with the oracle's within the stated
// agreement.
#include "sq_step.cuh"

namespace sq {
namespace {

// ROWS: key-row units (per-row widths; every head block has row and column scales); else head
// units (one width per head, fp16 pivot heads).
template <int GATE, int IO, bool WS, bool FULL, bool ROWS>
__global__ void __launch_bounds__(kT, kMaxCtasPerSm) k_decode(const StepArgs a) {
  const DPlan P(a.dk, a.dv, IO, GATE, ROWS, a.stage_bytes, a.H);
  uint64_t* bar = sp<uint64_t>(S_BAR);
  Ctx<FULL, !ROWS> c;
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
      mbar_arrive_expect_tx(bar, valid ? 2 * kb + vb + ab + rb + hd.bytes + a.extra_tx : 0u);
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
  const uint64_t wait_ns = a.wait_ns ? a.wait_ns : kWaitLimitNs;
  const uint8_t* st = smem + S_STAGE;
  const uint8_t* blk = st + P.blk_off;
  for (int item = first; item < n_items; item += stride, ++it) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait_bounded(bar, (uint32_t)it & 1u, wait_ns));
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
    float omega = 1.f;  // this row's weight in the column passes (impact tables), loaded early
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
        if (a.omega) omega = __ldg(a.omega + (size_t)hdr.h * dk + i);
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
        // k / A within 2 ulps (the tile's own factor, not a quantizer decision)
        sp<float>(S_KT)[p] = okA ? ki * rcp_approx(A) : 0.f;
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
    // the row-factored form when every row factor A_i is in [2^-60, 2^60], else the direct one
    const bool tilde = !c.flags[F_BADA];
    if (tid < dk) sp<float>(S_TR)[tid] = tilde ? sp<float>(S_AK)[4 * (tid >> 1) + (tid & 1)] : 1.f;
    __syncwarp();
    if (tilde)
      pass_b<ROWS ? 2 : 0, WS, true>(c, cv, bv, s_new);
    else
      pass_b<ROWS ? 2 : 0, WS, false>(c, cv, bv, s_new);
    if (WS && a.update_only) {  // the refit and requantization run elsewhere
      __syncthreads();
      continue;
    }
    float4 cm;
    const float r = fit_scales(c, a, omega, cm);
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
    mbar_wait_bounded(bar, (uint32_t)it & 1u, wait_ns);
    if (producer && c.lane < 3) cp_async_wait_all();
  }
  tmem_fence_before_sync();
  __syncthreads();
  if (c.warp == 0) {
    tmem_fence_after_sync();
    tmem_dealloc(tbase, kTmemCols);
  }
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
