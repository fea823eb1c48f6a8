"""Helpers for the GPU parity tests: a libsq pool driven through the C ABI next to an oracle
pool fed the same bytes and the same inputs."""
from __future__ import annotations

import numpy as np

import oracle
from bit_recurrent_state_gated_b200 import sq
from bit_recurrent_state_gated_b200 import workloads as W

import packed

ATOL, RTOL = 2e-3, 1e-3  # |gpu - oracle| <= ATOL + RTOL |oracle|


def sq_layout(wl, n_slots=None) -> sq.Layout:
    return sq.Layout(n_slots or wl.slots, wl.n_heads, wl.d_k, wl.d_v, wl.unit, wl.gate,
                     wl.io_dtype, wl.fit_iters, wl.window, wl.n_outliers)


def orc_layout(wl) -> oracle.Layout:
    return oracle.Layout(wl.n_heads, wl.d_k, wl.d_v, wl.unit, wl.gate, wl.fit_iters, wl.window,
                         wl.n_outliers)


def to_dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


class GpuCase:
    """A pool on the GPU for workload `wl`, filled from the workload's initial states."""

    def __init__(self, wl: W.Workload, init=True):
        import torch
        self.wl = wl
        self.bits = wl.bits()
        self.pool = sq.StatePool(sq_layout(wl), self.bits, wl.pivot_mask())
        self.si_np = wl.slot_idx()
        self.si = to_dev(self.si_np)
        if init:
            S0 = to_dev(wl.initial_state(self.si_np))
            self.pool.quantize(self.si, S0)
            torch.cuda.synchronize()

    def slots(self) -> np.ndarray:
        import torch
        torch.cuda.synchronize()
        return self.pool.slots_view().cpu().numpy()

    def device_inputs(self, x: dict):
        import torch
        if self.wl.io_dtype == W.IO_BF16:
            q, k, v = (to_dev(x[n + "_bf16"], torch.bfloat16) for n in ("q", "k", "v"))
        else:
            q, k, v = (to_dev(x[n]) for n in ("q", "k", "v"))
        return q, k, v, to_dev(x["alpha"]), to_dev(x["beta"])

    def step(self, x: dict, want_state=False, slot_idx=None):
        import torch
        wl = self.wl
        si = self.si if slot_idx is None else slot_idx
        B = si.numel()
        q, k, v, a, b = self.device_inputs(x)
        out = torch.empty((B, wl.n_heads, wl.d_v), dtype=torch.float32, device="cuda")
        s_new = (torch.empty((B, wl.n_heads, wl.d_k, wl.d_v), dtype=torch.float32,
                             device="cuda") if want_state else None)
        self.pool.decode_step(si, q, k, v, a, b, out, s_new)
        torch.cuda.synchronize()
        return out.cpu().numpy(), (s_new.cpu().numpy() if want_state else None)


def oracle_pool_from(wl, bits, slot_bytes: np.ndarray) -> oracle.Pool:
    """An oracle pool whose slots 0..n-1 hold the given packed slots."""
    p = oracle.Pool(orc_layout(wl), bits, slot_bytes.shape[0])
    assert p.slot_bytes == slot_bytes.shape[1]
    p.data[:] = slot_bytes.reshape(-1)
    return p


def sub_inputs(x: dict, rows) -> dict:
    return {k: np.ascontiguousarray(v[rows]) for k, v in x.items()}


def close(got, ref, what: str):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance, "
                           f"max err {err.max():.3g}")
    return float(err.max())


def compare_codes(wl, bits, gpu_slots: np.ndarray, orc_slots: np.ndarray, what: str):
    """Codes equal on >= 99.99 % of quantized elements and within 1 LSB elsewhere; the
    dequantized states within tolerance wherever codes match (fp16 entries always). Head
    blocks whose bytes are identical on both sides agree trivially; only the others are
    decoded and compared element by element."""
    H, dk, dv, K = wl.n_heads, wl.d_k, wl.d_v, wl.n_outliers
    ranges = packed.head_ranges(wl.unit, bits, H, dk, dv, K)
    n_mis = total = 0
    max_diff = 0
    for h, (a, b) in enumerate(ranges):
        bh = packed.head_bits(wl.unit, bits, h, dk)
        if wl.unit == W.UNIT_HEAD:
            n_quant = 0 if bh[0] == 16 else dk * dv - K
        else:
            n_quant = int((bh != 16).sum()) * dv - K
        differ = np.nonzero((gpu_slots[:, a:b] != orc_slots[:, a:b]).any(axis=1))[0]
        total += n_quant * gpu_slots.shape[0]
        if differ.size == 0:
            continue
        dg = packed.decode(gpu_slots[differ, a:b], wl.unit, bh, 1, dk, dv, K)
        do = packed.decode(orc_slots[differ, a:b], wl.unit, bh, 1, dk, dv, K)
        quant = ~np.broadcast_to(dg["pivot"][None, :, :, None], dg["codes"].shape)
        if K:
            quant = quant & (dg["f16"] == 0) & (do["f16"] == 0)
        diff = np.abs(dg["codes"] - do["codes"])[quant]
        n_mis += int((diff != 0).sum())
        if diff.size:
            max_diff = max(max_diff, int(diff.max()))
        Dg, Do = packed.dequant(dg), packed.dequant(do)
        same = (dg["codes"] == do["codes"]) | ~quant
        close(Dg[same], Do[same], f"{what} head {h} dequantized state")
    assert max_diff <= 1, f"{what}: code differs by {max_diff} LSB"
    frac = n_mis / max(total, 1)
    if total >= 100_000:  # on small samples one flip exceeds the fraction; callers sum up
        assert frac <= 1e-4, f"{what}: {n_mis} of {total} codes differ ({frac:.2e})"
    return n_mis, total


def code_agreement(wl, bits, slots_a: np.ndarray, slots_b: np.ndarray):
    """Element statistics of two packed copies of the same requests: (quantized elements,
    of them with equal codes, of those whose dequantized values are within tolerance, the
    largest dequantized difference among them). Identical head blocks count as agreeing."""
    H, dk, dv, K = wl.n_heads, wl.d_k, wl.d_v, wl.n_outliers
    n_quant = n_agree = n_ok = 0
    max_err = 0.0
    for h, (a, b) in enumerate(packed.head_ranges(wl.unit, bits, H, dk, dv, K)):
        bh = packed.head_bits(wl.unit, bits, h, dk)
        if wl.unit == W.UNIT_HEAD:
            per = 0 if bh[0] == 16 else dk * dv - K
        else:
            per = int((bh != 16).sum()) * dv - K
        differ = (slots_a[:, a:b] != slots_b[:, a:b]).any(axis=1)
        same_n = int((~differ).sum()) * per
        n_quant, n_agree, n_ok = n_quant + same_n, n_agree + same_n, n_ok + same_n
        idx = np.nonzero(differ)[0]
        if idx.size == 0 or per == 0:
            n_quant += idx.size * per
            continue
        da = packed.decode(slots_a[idx, a:b], wl.unit, bh, 1, dk, dv, K)
        db = packed.decode(slots_b[idx, a:b], wl.unit, bh, 1, dk, dv, K)
        quant = ~np.broadcast_to(da["pivot"][None, :, :, None], da["codes"].shape)
        if K:
            quant = quant & (da["f16"] == 0) & (db["f16"] == 0)
        agree = (da["codes"] == db["codes"]) & quant
        Da, Db = packed.dequant(da).astype(np.float64), packed.dequant(db)
        err = np.abs(Da - Db)[agree]
        n_quant += int(quant.sum())
        n_agree += int(agree.sum())
        n_ok += int((err <= ATOL + RTOL * np.abs(np.asarray(Db, np.float64)[agree])).sum())
        if err.size:
            max_err = max(max_err, float(err.max()))
    return n_quant, n_agree, n_ok, max_err


def lockstep(case: GpuCase, t: int, sample=None, want_state=True, x=None):
    """One GPU step checked against the oracle started from the GPU's own pre-step bytes.
    `sample`: request indices to check (default all); `x`: inputs (default step t's)."""
    wl = case.wl
    x = wl.step_inputs(t) if x is None else x
    pre = case.slots()
    o_gpu, s_gpu = case.step(x, want_state=want_state)
    post = case.slots()
    rows = np.arange(wl.batch) if sample is None else np.asarray(sample)
    slots = case.si_np[rows]
    opool = oracle_pool_from(wl, case.bits, pre[slots])
    xs = sub_inputs(x, rows)
    o_ref, s_ref = opool.decode_step(np.arange(rows.size), xs["q"], xs["k"], xs["v"],
                                     xs["alpha"], xs["beta"], want_state=True)
    close(o_gpu[rows], o_ref, f"step {t} o")
    if want_state:
        close(s_gpu[rows], s_ref, f"step {t} state after update")
    n_mis, n = compare_codes(wl, case.bits, post[slots], opool.data.reshape(rows.size, -1),
                             f"step {t}")
    untouched = np.setdiff1d(np.arange(wl.slots), case.si_np)
    if untouched.size:
        np.testing.assert_array_equal(post[untouched], pre[untouched])
    return n_mis, n
