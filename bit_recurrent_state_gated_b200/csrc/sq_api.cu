// sq_api.cu -- host side of the libsq C ABI (include/sq.h): layout arithmetic, argument
// checks, the pool handle and kernel dispatch. Every exported function returns sq_status and
// never aborts or prints.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <new>
#include <vector>

#include "sq.h"
#include "sq_internal.h"

struct sq_pool {
  sq_layout L;
  std::vector<uint8_t> bits;  // unit widths (16 = pivot)
  std::vector<sq::HeadDesc> heads;
  std::vector<uint32_t> rows;  // [H][d_k] (offset << 8) | width
  std::vector<uint32_t> srows;  // key-row units: [H][d_k] descriptors, rows grouped by width
  size_t slot_bytes = 0, side_slot_bytes = 0, side_head_bytes = 0;
  uint32_t max_head_bytes = 0;
  uint8_t* base = nullptr;  // caller's buffer
  std::vector<int32_t> order;  // heads sorted by width (pivot heads last)
  sq::HeadDesc* d_heads = nullptr;
  uint32_t* d_rows = nullptr;
  uint32_t* d_srows = nullptr;
  int32_t* d_order = nullptr;
  int32_t* d_flag = nullptr;
  int device = 0, num_sms = 0;
  float* d_omega = nullptr;  // column-pass weights [H][d_k] (sq_pool_set_row_impact)
  bool has_omega = false;
  // side-stream split: the last split's requantization, which later calls on the pool wait for
  cudaEvent_t ev_update = nullptr, ev_side = nullptr;
  bool side_pending = false;
  // bounded waits of the decode kernel (sq_debug_set_wait)
  uint64_t wait_ns = 1000000000ull;
  uint32_t extra_tx = 0;
  int32_t full_fit = 0;  // sq_debug_set_full_fit
};

namespace sq {
void pool_dims(const sq_pool* p, int* n_heads, int* d_k, int* d_v) {
  *n_heads = p->L.n_heads;
  *d_k = p->L.d_k;
  *d_v = p->L.d_v;
}
}  // namespace sq

namespace {

bool width_ok(int b) { return b == 2 || b == 4 || b == 6 || b == 8 || b == 16; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t row_bytes(int b, int dv) { return (size_t)dv * (size_t)b / 8; }

// Validate a layout + bit map and compute the per-head geometry.
sq_status plan(const sq_layout* L, const uint8_t* bits, const uint8_t* pivot_mask, sq_pool* P) {
  if (!L || !bits) return SQ_ERR_INVALID_ARG;
  if (L->n_slots < 1 || L->n_heads < 1) return SQ_ERR_INVALID_ARG;
  for (int d : {L->d_k, L->d_v})
    if (d < 16 || d > sq::kMaxD || d % 16) return SQ_ERR_INVALID_ARG;
  if (L->unit != SQ_UNIT_HEAD && L->unit != SQ_UNIT_KEY_ROW) return SQ_ERR_INVALID_ARG;
  if (L->gate != SQ_GATE_SCALAR && L->gate != SQ_GATE_DIAG) return SQ_ERR_INVALID_ARG;
  if (L->io_dtype != SQ_IO_F32 && L->io_dtype != SQ_IO_BF16) return SQ_ERR_INVALID_ARG;
  if (L->fit_iters < 1 || L->fit_iters > 8) return SQ_ERR_INVALID_ARG;
  if (L->window < 1 || L->n_outliers < 0 || L->n_outliers > 64) return SQ_ERR_INVALID_ARG;
  if (L->window == 1 && L->n_outliers != 0) return SQ_ERR_INVALID_ARG;
  const int H = L->n_heads, dk = L->d_k, dv = L->d_v;
  const int n_units = L->unit == SQ_UNIT_HEAD ? H : H * dk;
  for (int u = 0; u < n_units; ++u) {
    if (!width_ok(bits[u])) return SQ_ERR_INVALID_ARG;
    if (pivot_mask && ((pivot_mask[u] != 0) != (bits[u] == 16))) return SQ_ERR_INVALID_ARG;
  }
  P->L = *L;
  P->bits.assign(bits, bits + n_units);
  P->heads.assign(H, sq::HeadDesc{});
  P->rows.assign((size_t)H * dk, 0);
  size_t off = 0;
  uint32_t maxb = 0;
  for (int h = 0; h < H; ++h) {
    sq::HeadDesc& hd = P->heads[h];
    const bool pivot_head = L->unit == SQ_UNIT_HEAD && bits[h] == 16;
    size_t n;
    if (pivot_head) {
      for (int i = 0; i < dk; ++i) P->rows[(size_t)h * dk + i] = (uint32_t)((size_t)i * 2 * dv) << 8 | 16u;
      n = (size_t)2 * dk * dv;
      hd.pivot_head = 1;
      hd.width = 16;
    } else {
      n = (size_t)2 * (dk + dv);
      int eligible = 0;
      for (int i = 0; i < dk; ++i) {
        const int b = L->unit == SQ_UNIT_HEAD ? bits[h] : bits[(size_t)h * dk + i];
        P->rows[(size_t)h * dk + i] = (uint32_t)n << 8 | (uint32_t)b;
        n += row_bytes(b, dv);
        if (b != 16) eligible += dv;
      }
      if (L->n_outliers > eligible) return SQ_ERR_INVALID_ARG;
      n += 4u * (size_t)L->n_outliers;
      hd.pivot_head = 0;
      hd.width = L->unit == SQ_UNIT_HEAD ? bits[h] : 0u;
    }
    n = (n + 15) / 16 * 16;
    if (n >= (1u << 24)) return SQ_ERR_INVALID_ARG;
    hd.off = (uint32_t)off;
    hd.bytes = (uint32_t)n;
    off += n;
    if (n > maxb) maxb = (uint32_t)n;
  }
  P->slot_bytes = off;
  P->max_head_bytes = maxb;
  if (L->unit == SQ_UNIT_KEY_ROW) {
    // Processing order of the decode kernel: each head's rows grouped by width (stable), so
    // that row pairs and four-row chunks almost always share one width; the four-row chunks of
    // that sequence are then dealt to the warps in turn (warp w owns processing rows
    // [32 w, 32 w + 32)), so every warp gets about the same mix of widths and none of them
    // waits long for the others at the item's barriers.
    P->srows.assign((size_t)H * dk, 0);
    const int n_ch = dk / 4, n_warps = (dk + 31) / 32;
    for (int h = 0; h < H; ++h) {
      std::vector<int> idx(dk);
      for (int i = 0; i < dk; ++i) idx[i] = i;
      const uint32_t* rt = &P->rows[(size_t)h * dk];
      std::stable_sort(idx.begin(), idx.end(), [&](int x, int y) {
        return sq::row_width(rt[x]) < sq::row_width(rt[y]);
      });
      // chunk k of the sorted sequence goes to warp k % n_warps as its chunk k / n_warps; with
      // d_k not a multiple of 32 the last warp owns fewer chunks, so the deal skips it once its
      // chunks are full
      std::vector<int> order;
      order.reserve(dk);
      std::vector<std::vector<int>> per_warp(n_warps);
      int w = 0;
      for (int k = 0; k < n_ch; ++k) {
        for (int tries = 0; (int)per_warp[w].size() >= std::min(32, dk - 32 * w) && tries < n_warps; ++tries)
          w = (w + 1) % n_warps;
        for (int r = 0; r < 4; ++r) per_warp[w].push_back(idx[4 * k + r]);
        w = (w + 1) % n_warps;
      }
      for (int ww = 0; ww < n_warps; ++ww) order.insert(order.end(), per_warp[ww].begin(), per_warp[ww].end());
      for (int p = 0; p < dk; ++p) {
        const uint32_t d = rt[order[p]];
        if (sq::row_off(d) >= (1u << 16)) return SQ_ERR_INVALID_ARG;
        const int p0 = p & ~3;  // the four-row chunk of processing row p
        bool uniform = true;
        for (int r = 1; r < 4; ++r)
          uniform &= sq::row_width(rt[order[p0 + r]]) == sq::row_width(rt[order[p0]]);
        P->srows[(size_t)h * dk + p] = (uint32_t)order[p] << 24 | sq::row_off(d) << 8 |
                                       (uniform ? sq::kChunkUniform : 0u) |
                                       (uint32_t)sq::row_width(d);
      }
    }
  }
  P->order.resize(H);
  for (int h = 0; h < H; ++h) P->order[h] = h;
  std::stable_sort(P->order.begin(), P->order.end(), [&](int x, int y) {
    const auto key = [&](int h) { return P->heads[h].pivot_head ? 99 : (int)P->heads[h].width; };
    return key(x) < key(y);
  });
  if (L->window > 1) {
    if (L->window > 64) return SQ_ERR_INVALID_ARG;
    // per (slot, head): header, cumulative gate(s) and `window` low-rank terms (sq::SideFmt)
    const sq::SideFmt f(dk, dv, L->gate, L->io_dtype);
    P->side_head_bytes = f.head + (size_t)L->window * f.stride;
    P->side_head_bytes = (P->side_head_bytes + 15) / 16 * 16;
    P->side_slot_bytes = (size_t)H * P->side_head_bytes;
    P->side_slot_bytes = (P->side_slot_bytes + 255) / 256 * 256;
  }
  return SQ_OK;
}

size_t required_bytes(const sq_pool& P) {
  return (size_t)P.L.n_slots * (P.slot_bytes + P.side_slot_bytes);
}

sq_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SQ_OK;
  if (e == cudaErrorMemoryAllocation) return SQ_ERR_OOM;
  if (e == cudaErrorNoKernelImageForDevice || e == cudaErrorInvalidDeviceFunction ||
      e == cudaErrorNotSupported)
    return SQ_ERR_UNSUPPORTED;
  return SQ_ERR_CUDA;
}

sq::StepArgs step_args(sq_pool* p, const int32_t* slot_idx, int32_t batch, const void* q,
                       const void* k, const void* v, const float* alpha, const float* beta,
                       float* out, float* s_new) {
  sq::StepArgs a{};
  a.pool = p->base;
  a.slot_bytes = (int64_t)p->slot_bytes;
  a.n_slots = p->L.n_slots;
  a.slot_idx = slot_idx;
  a.batch = batch;
  a.q = q;
  a.k = k;
  a.v = v;
  a.alpha = alpha;
  a.beta = beta;
  a.out = out;
  a.s_new = s_new;
  a.heads = p->d_heads;
  a.rows = p->d_rows;
  a.srows = p->d_srows;
  a.order = p->d_order;
  a.H = p->L.n_heads;
  a.dk = p->L.d_k;
  a.dv = p->L.d_v;
  a.fit_iters = p->L.fit_iters;
  a.per_row = p->L.unit == SQ_UNIT_KEY_ROW;
  a.stage_bytes = p->max_head_bytes;
  a.flag = p->d_flag;
  a.side = p->side_slot_bytes ? p->base + (size_t)p->L.n_slots * p->slot_bytes : nullptr;
  a.side_slot_bytes = (int64_t)p->side_slot_bytes;
  a.side_head_bytes = (int64_t)p->side_head_bytes;
  a.window = p->L.window;
  a.n_outliers = p->L.n_outliers;
  a.omega = p->has_omega ? p->d_omega : nullptr;
  a.wait_ns = p->wait_ns;
  a.extra_tx = p->extra_tx;
  a.full_fit = p->full_fit;
  return a;
}

sq::QuantArgs quant_args(sq_pool* p, const int32_t* slot_idx, int32_t n, const float* S,
                         float* S_out) {
  sq::QuantArgs a{};
  a.pool = p->base;
  a.slot_bytes = (int64_t)p->slot_bytes;
  a.n_slots = p->L.n_slots;
  a.slot_idx = slot_idx;
  a.n = n;
  a.S = S;
  a.S_out = S_out;
  a.heads = p->d_heads;
  a.rows = p->d_rows;
  a.H = p->L.n_heads;
  a.dk = p->L.d_k;
  a.dv = p->L.d_v;
  a.fit_iters = p->L.fit_iters;
  a.n_outliers = p->L.n_outliers;
  a.stage_bytes = p->max_head_bytes;
  a.flag = p->d_flag;
  a.side = p->side_slot_bytes ? p->base + (size_t)p->L.n_slots * p->slot_bytes : nullptr;
  a.side_slot_bytes = (int64_t)p->side_slot_bytes;
  a.side_head_bytes = (int64_t)p->side_head_bytes;
  a.omega = p->has_omega ? p->d_omega : nullptr;
  return a;
}

// Order `st` after the requantization a side-stream split left running on the pool.
cudaError_t after_side(sq_pool* p, cudaStream_t st) {
  return p->side_pending ? cudaStreamWaitEvent(st, p->ev_side, 0) : cudaSuccess;
}

sq_status check_step(sq_pool* p, const int32_t* slot_idx, int32_t batch, const void* q,
                     const void* k, const void* v, const float* alpha, const float* beta,
                     const float* out) {
  if (!p || batch < 0) return SQ_ERR_INVALID_ARG;
  if (batch == 0) return SQ_OK;
  const void* ptrs[] = {slot_idx, q, k, v, alpha, beta, out};
  for (const void* x : ptrs)
    if (!x || !aligned(x, 16)) return SQ_ERR_INVALID_ARG;
  return SQ_OK;
}

}  // namespace

extern "C" {

sq_status sq_pool_required_bytes(const sq_layout* layout, const uint8_t* bits_map,
                                 const uint8_t* pivot_mask, size_t* bytes) {
  if (!bytes) return SQ_ERR_INVALID_ARG;
  sq_pool P;
  const sq_status s = plan(layout, bits_map, pivot_mask, &P);
  if (s != SQ_OK) return s;
  *bytes = required_bytes(P);
  return SQ_OK;
}

sq_status sq_state_pool_create(const sq_layout* layout, const uint8_t* bits_map,
                               const uint8_t* pivot_mask, void* device_buf,
                               size_t device_buf_bytes, sq_pool** out) {
  if (!out) return SQ_ERR_INVALID_ARG;
  *out = nullptr;
  sq_pool* p = new (std::nothrow) sq_pool();
  if (!p) return SQ_ERR_OOM;
  sq_status s = plan(layout, bits_map, pivot_mask, p);
  if (s == SQ_OK && (!device_buf || !aligned(device_buf, 256) ||
                     device_buf_bytes < required_bytes(*p)))
    s = SQ_ERR_INVALID_ARG;
  if (s != SQ_OK) {
    delete p;
    return s;
  }
  p->base = static_cast<uint8_t*>(device_buf);
  cudaError_t e = cudaGetDevice(&p->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->device);
  int major = 0;
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, p->device);
  if (e == cudaSuccess && major != 10) {
    delete p;
    return SQ_ERR_UNSUPPORTED;
  }
  if (e == cudaSuccess) e = cudaMalloc(&p->d_heads, sizeof(sq::HeadDesc) * p->heads.size());
  if (e == cudaSuccess) e = cudaMalloc(&p->d_rows, sizeof(uint32_t) * p->rows.size());
  if (e == cudaSuccess && !p->srows.empty())
    e = cudaMalloc(&p->d_srows, sizeof(uint32_t) * p->srows.size());
  if (e == cudaSuccess && !p->srows.empty())
    e = cudaMemcpy(p->d_srows, p->srows.data(), sizeof(uint32_t) * p->srows.size(),
                   cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMalloc(&p->d_flag, sizeof(int32_t));
  if (e == cudaSuccess) e = cudaMalloc(&p->d_order, sizeof(int32_t) * p->order.size());
  if (e == cudaSuccess)
    e = cudaMemcpy(p->d_order, p->order.data(), sizeof(int32_t) * p->order.size(),
                   cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(p->d_heads, p->heads.data(), sizeof(sq::HeadDesc) * p->heads.size(),
                   cudaMemcpyHostToDevice);
  if (e == cudaSuccess)
    e = cudaMemcpy(p->d_rows, p->rows.data(), sizeof(uint32_t) * p->rows.size(),
                   cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemset(p->d_flag, 0, sizeof(int32_t));
  if (e != cudaSuccess) {
    cudaFree(p->d_heads);
    cudaFree(p->d_rows);
    cudaFree(p->d_srows);
    cudaFree(p->d_flag);
    cudaFree(p->d_order);
    delete p;
    return cuda_status(e);
  }
  *out = p;
  return SQ_OK;
}

sq_status sq_state_pool_destroy(sq_pool* pool) {
  if (!pool) return SQ_OK;
  cudaFree(pool->d_heads);
  cudaFree(pool->d_rows);
  cudaFree(pool->d_srows);
  cudaFree(pool->d_flag);
  cudaFree(pool->d_order);
  cudaFree(pool->d_omega);
  if (pool->ev_update) cudaEventDestroy(pool->ev_update);
  if (pool->ev_side) cudaEventDestroy(pool->ev_side);
  delete pool;
  return SQ_OK;
}

sq_status sq_pool_info(const sq_pool* pool, size_t* slot_bytes, size_t* head_offsets,
                       size_t* side_bytes_per_slot) {
  if (!pool) return SQ_ERR_INVALID_ARG;
  if (slot_bytes) *slot_bytes = pool->slot_bytes;
  if (head_offsets)
    for (size_t h = 0; h < pool->heads.size(); ++h) head_offsets[h] = pool->heads[h].off;
  if (side_bytes_per_slot) *side_bytes_per_slot = pool->side_slot_bytes;
  return SQ_OK;
}

sq_status sq_quantize_fp32_state(sq_pool* pool, const int32_t* slot_idx, int32_t n,
                                 const float* S, void* stream) {
  if (!pool || n < 0) return SQ_ERR_INVALID_ARG;
  if (n == 0) return SQ_OK;
  if (!slot_idx || !S || !aligned(slot_idx, 4) || !aligned(S, 16)) return SQ_ERR_INVALID_ARG;
  const sq::QuantArgs a = quant_args(pool, slot_idx, n, S, nullptr);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaError_t e = after_side(pool, st)) return cuda_status(e);
  return cuda_status(sq::launch_quantize(a, st));
}

sq_status sq_dequantize_state(sq_pool* pool, const int32_t* slot_idx, int32_t n, float* S_out,
                              void* stream) {
  if (!pool || n < 0) return SQ_ERR_INVALID_ARG;
  if (n == 0) return SQ_OK;
  if (!slot_idx || !S_out || !aligned(slot_idx, 4) || !aligned(S_out, 16)) return SQ_ERR_INVALID_ARG;
  const sq::QuantArgs a = quant_args(pool, slot_idx, n, nullptr, S_out);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaError_t e = after_side(pool, st)) return cuda_status(e);
  return cuda_status(sq::launch_dequantize(a, st));
}

sq_status sq_decode_step(sq_pool* pool, const int32_t* slot_idx, int32_t batch, const void* q,
                         const void* k, const void* v, const float* alpha, const float* beta,
                         float* out, void* stream) {
  sq_status s = check_step(pool, slot_idx, batch, q, k, v, alpha, beta, out);
  if (s != SQ_OK || batch == 0) return s;
  const sq::StepArgs a = step_args(pool, slot_idx, batch, q, k, v, alpha, beta, out, nullptr);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaError_t e = after_side(pool, st)) return cuda_status(e);
  if (pool->L.window > 1)
    return cuda_status(sq::launch_window_step(a, pool->L.gate, pool->L.io_dtype, pool->num_sms, st));
  return cuda_status(sq::launch_decode(a, pool->L.gate, pool->L.io_dtype, false, pool->num_sms, st));
}

sq_status sq_decode_chunk(sq_pool* pool, const int32_t* slot_idx, int32_t batch, int32_t n_tokens,
                          const void* q, const void* k, const void* v, const float* alpha,
                          const float* beta, float* out, void* stream) {
  if (!pool || n_tokens < 1 || n_tokens > sq::kMaxChunkTokens) return SQ_ERR_INVALID_ARG;
  sq_status s = check_step(pool, slot_idx, batch, q, k, v, alpha, beta, out);
  if (s != SQ_OK || batch == 0) return s;
  if (pool->L.window > 1) return SQ_ERR_UNSUPPORTED;
  sq::StepArgs a = step_args(pool, slot_idx, batch, q, k, v, alpha, beta, out, nullptr);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaError_t e = after_side(pool, st)) return cuda_status(e);
  if (n_tokens == 1)  // one token is the decode step
    return cuda_status(sq::launch_decode(a, pool->L.gate, pool->L.io_dtype, false, pool->num_sms, st));
  a.n_tok = n_tokens;
  return cuda_status(sq::launch_chunk(a, pool->L.gate, pool->L.io_dtype, pool->num_sms, st));
}

sq_status sq_debug_decode_step_fp32(sq_pool* pool, const int32_t* slot_idx, int32_t batch,
                                    const void* q, const void* k, const void* v,
                                    const float* alpha, const float* beta, float* out,
                                    float* s_new, void* stream) {
  sq_status s = check_step(pool, slot_idx, batch, q, k, v, alpha, beta, out);
  if (s != SQ_OK || batch == 0) return s;
  if (pool->L.window > 1) return SQ_ERR_UNSUPPORTED;
  if (!s_new || !aligned(s_new, 16)) return SQ_ERR_INVALID_ARG;
  const sq::StepArgs a = step_args(pool, slot_idx, batch, q, k, v, alpha, beta, out, s_new);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaError_t e = after_side(pool, st)) return cuda_status(e);
  return cuda_status(sq::launch_decode(a, pool->L.gate, pool->L.io_dtype, true, pool->num_sms, st));
}

sq_status sq_decode_step_split(sq_pool* pool, const int32_t* slot_idx, int32_t batch,
                               const void* q, const void* k, const void* v, const float* alpha,
                               const float* beta, float* out, float* staging, void* stream,
                               void* side_stream) {
  sq_status s = check_step(pool, slot_idx, batch, q, k, v, alpha, beta, out);
  if (s != SQ_OK || batch == 0) return s;
  if (pool->L.window > 1) return SQ_ERR_UNSUPPORTED;
  if (!staging || !aligned(staging, 16)) return SQ_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream), side = static_cast<cudaStream_t>(side_stream);
  cudaError_t e = cudaSuccess;
  if (!pool->ev_update) {
    if ((e = cudaEventCreateWithFlags(&pool->ev_update, cudaEventDisableTiming)) ||
        (e = cudaEventCreateWithFlags(&pool->ev_side, cudaEventDisableTiming)))
      return cuda_status(e);
  }
  if ((e = after_side(pool, st))) return cuda_status(e);
  sq::StepArgs a = step_args(pool, slot_idx, batch, q, k, v, alpha, beta, out, staging);
  a.update_only = 1;
  if ((e = sq::launch_decode(a, pool->L.gate, pool->L.io_dtype, true, pool->num_sms, st)) ||
      (e = cudaEventRecord(pool->ev_update, st)) || (e = cudaStreamWaitEvent(side, pool->ev_update, 0)))
    return cuda_status(e);
  const sq::QuantArgs qa = quant_args(pool, slot_idx, batch, staging, nullptr);
  if ((e = sq::launch_quantize(qa, side)) || (e = cudaEventRecord(pool->ev_side, side)))
    return cuda_status(e);
  pool->side_pending = true;
  return SQ_OK;
}

sq_status sq_window_flush(sq_pool* pool, const int32_t* slot_idx, int32_t n, void* stream) {
  if (!pool || n < 0) return SQ_ERR_INVALID_ARG;
  if (n == 0 || pool->L.window == 1) return SQ_OK;
  if (!slot_idx || !aligned(slot_idx, 4)) return SQ_ERR_INVALID_ARG;
  const sq::StepArgs a = step_args(pool, slot_idx, n, nullptr, nullptr, nullptr, nullptr,
                                   nullptr, nullptr, nullptr);
  return cuda_status(sq::launch_window_flush(a, pool->L.gate, pool->L.io_dtype, static_cast<cudaStream_t>(stream)));
}

sq_status sq_pool_set_row_impact(sq_pool* pool, const float* impact) {
  if (!pool) return SQ_ERR_INVALID_ARG;
  if (!impact) {
    pool->has_omega = false;
    return SQ_OK;
  }
  // Weight of row i in the column passes of the fit: min(1, sqrt(impact_i / mean impact of its
  // head)), in double precision, rounded to fp32 once. Lowering a column scale refines that
  // column in every row but widens the row that sets it; with d_v columns of similar scale the
  // trade pays while the widening factor f satisfies f^2 < mean impact / impact_i, so the row
  // counts with 1 / f. Equal impacts give 1 everywhere: the plain fit.
  const int H = pool->L.n_heads, dk = pool->L.d_k;
  std::vector<float> omega((size_t)H * dk);
  for (int h = 0; h < H; ++h) {
    double sum = 0.0;
    for (int i = 0; i < dk; ++i) {
      const double x = impact[(size_t)h * dk + i];
      if (!(x > 0.0) || !std::isfinite(x)) return SQ_ERR_INVALID_ARG;
      sum += x;
    }
    const double mean = sum / dk;
    for (int i = 0; i < dk; ++i) {
      const double x = std::sqrt((double)impact[(size_t)h * dk + i] / mean);
      omega[(size_t)h * dk + i] = (float)(x < 1.0 ? x : 1.0);
    }
  }
  cudaError_t e = cudaDeviceSynchronize();  // no kernel of this pool may still read the table
  if (e == cudaSuccess && !pool->d_omega)
    e = cudaMalloc(&pool->d_omega, omega.size() * sizeof(float));
  if (e == cudaSuccess)
    e = cudaMemcpy(pool->d_omega, omega.data(), omega.size() * sizeof(float), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_status(e);
  pool->has_omega = true;
  return SQ_OK;
}

sq_status sq_pool_status(sq_pool* pool, int32_t* device_flag) {
  if (!pool) return SQ_ERR_INVALID_ARG;
  cudaError_t e = cudaDeviceSynchronize();
  int32_t f = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&f, pool->d_flag, sizeof f, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(pool->d_flag, 0, sizeof f);
  if (e != cudaSuccess) return cuda_status(e);
  if (device_flag) *device_flag = f;
  if (f & SQ_FLAG_TIMEOUT) return SQ_ERR_TIMEOUT;
  return f ? SQ_ERR_DEVICE_FLAG : SQ_OK;
}

sq_status sq_debug_set_wait(sq_pool* pool, uint64_t wait_limit_ns, uint32_t extra_expected_bytes) {
  if (!pool || extra_expected_bytes > 4096u) return SQ_ERR_INVALID_ARG;
  pool->wait_ns = wait_limit_ns ? wait_limit_ns : 1000000000ull;
  pool->extra_tx = extra_expected_bytes;
  return SQ_OK;
}

sq_status sq_debug_set_full_fit(sq_pool* pool, int32_t full_fit) {
  if (!pool || (full_fit != 0 && full_fit != 1)) return SQ_ERR_INVALID_ARG;
  pool->full_fit = full_fit;
  return SQ_OK;
}

const char* sq_status_string(sq_status status) {
  switch (status) {
    case SQ_OK: return "ok";
    case SQ_ERR_INVALID_ARG: return "invalid argument";
    case SQ_ERR_UNSUPPORTED: return "unsupported";
    case SQ_ERR_CUDA: return "CUDA error";
    case SQ_ERR_OOM: return "out of device memory";
    case SQ_ERR_DEVICE_FLAG: return "the GPU flagged a slot, a value or a range";
    case SQ_ERR_TIMEOUT: return "a kernel gave up waiting on a copy";
  }
  return "unknown status";
}

}  // extern "C"
