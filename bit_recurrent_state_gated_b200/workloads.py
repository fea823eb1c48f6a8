"""Seeded synthetic workloads for the quantized decode step.

This module only draws inputs: unit bit widths, pivot positions, the initial fp32 states and
the per-step q, k, v, alpha, beta. It holds none of the method's arithmetic (no fit, no
quantizer, no update), so the CUDA path and the CPU oracle can both consume what it draws.

Shapes follow the workloads the STEPQuant and LeapQuant pages talk about (d_k = d_v = 128
heads of GDN / KDA layers, batches of 64 to 512 concurrent requests, a serving pool with spare
slots); none of them is a public benchmark and nothing here reads a dataset.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np

UNIT_HEAD, UNIT_ROW = 0, 1
GATE_SCALAR, GATE_DIAG = 0, 1
IO_F32, IO_BF16 = 0, 1


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.default_rng([seed, *stream])


_S_INIT, _S_BITS, _S_STEP, _S_PERM = 11, 12, 13, 14


@dataclass(frozen=True)
class Workload:
    """One synthetic decode workload. ``mix`` lists (width, count) for the non-pivot units."""
    name: str
    batch: int
    n_heads: int
    d_k: int
    d_v: int
    steps: int
    gate: int
    unit: int
    io_dtype: int
    mix: tuple
    n_pivots: int
    seed: int
    n_slots: int = 0               # 0: one slot per request, slot_idx = identity
    alpha_mu: float = -3.0         # alpha = exp(-softplus(N(alpha_mu, 1)))
    alpha_min: float = 0.0         # lower clamp on alpha (0 = none)
    normalize_q: bool = True
    fit_iters: int = 2
    window: int = 1
    n_outliers: int = 0
    tokens: int = 1                # tokens per call (> 1: the multi-token chunk step)
    side_stream: bool = False      # refit + requantize on a second stream (the split step)
    init_std: float = 0.1
    notes: str = field(default="", compare=False)

    @property
    def slots(self) -> int:
        return self.n_slots or self.batch

    @property
    def alpha_width(self) -> int:
        return 1 if self.gate == GATE_SCALAR else self.d_k

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)

    # -- unit widths ------------------------------------------------------------------------
    def bits(self) -> np.ndarray:
        """Unit widths: [H] for head units, [H * d_k] for key-row units; 16 marks a pivot."""
        n_units = self.n_heads if self.unit == UNIT_HEAD else self.n_heads * self.d_k
        widths = np.concatenate([np.full(c, w, dtype=np.uint8) for w, c in self.mix]
                                or [np.zeros(0, np.uint8)])
        assert widths.size + self.n_pivots == n_units, (self.name, widths.size, n_units)
        r = _rng(self.seed, _S_BITS)
        widths = r.permutation(widths)
        piv = np.sort(r.choice(n_units, size=self.n_pivots, replace=False))
        out = np.zeros(n_units, dtype=np.uint8)
        mask = np.zeros(n_units, dtype=bool)
        mask[piv] = True
        out[mask] = 16
        out[~mask] = widths
        return out

    def pivot_mask(self) -> np.ndarray:
        return (self.bits() == 16).astype(np.uint8)

    # -- slots ------------------------------------------------------------------------------
    def slot_idx(self) -> np.ndarray:
        """Slot of each request: identity, or the first ``batch`` of a seeded permutation."""
        if not self.n_slots:
            return np.arange(self.batch, dtype=np.int32)
        return _rng(self.seed, _S_PERM).permutation(self.n_slots)[: self.batch].astype(np.int32)

    def initial_state(self, slots) -> np.ndarray:
        """fp32 N(0, init_std) states [len(slots)][H][d_k][d_v], one seeded stream per slot."""
        slots = np.atleast_1d(np.asarray(slots))
        out = np.empty((slots.size, self.n_heads, self.d_k, self.d_v), dtype=np.float32)
        for n, s in enumerate(slots):
            out[n] = _rng(self.seed, _S_INIT, int(s)).normal(
                0.0, self.init_std, (self.n_heads, self.d_k, self.d_v)).astype(np.float32)
        return out

    # -- per-step inputs --------------------------------------------------------------------
    def step_inputs(self, t: int) -> dict:
        """Inputs of decode step t for the whole batch.

        q, k: N(0, 1), L2-normalized per (request, head) in fp32 (q only if normalize_q);
        v: N(0, 1). With bf16 I/O they are then rounded to bf16, and the fp32 arrays hold the
        exact upcast of those bf16 values, so both sides see identical numbers.
        alpha = exp(-softplus(x)), x ~ N(alpha_mu, 1), clamped below at alpha_min;
        one per (request, head) for the scalar gate, per key channel for the diagonal gate.
        beta = sigmoid(N(0, 1)) per (request, head).
        """
        B, H, dk, dv = self.batch, self.n_heads, self.d_k, self.d_v
        r = _rng(self.seed, _S_STEP, t)
        q = r.standard_normal((B, H, dk)).astype(np.float32)
        k = r.standard_normal((B, H, dk)).astype(np.float32)
        v = r.standard_normal((B, H, dv)).astype(np.float32)
        k = k / np.linalg.norm(k, axis=-1, keepdims=True).astype(np.float32)
        if self.normalize_q:
            q = q / np.linalg.norm(q, axis=-1, keepdims=True).astype(np.float32)
        x = r.normal(self.alpha_mu, 1.0, (B, H, self.alpha_width))
        alpha = np.exp(-np.logaddexp(0.0, x))
        if self.alpha_min > 0:
            alpha = np.maximum(alpha, self.alpha_min)
        alpha = alpha.astype(np.float32)
        if self.gate == GATE_SCALAR:
            alpha = alpha.reshape(B, H)
        beta = (1.0 / (1.0 + np.exp(-r.standard_normal((B, H))))).astype(np.float32)
        d = {"alpha": alpha, "beta": beta}
        if self.io_dtype == IO_BF16:
            for name, a in (("q", q), ("k", k), ("v", v)):
                bits = bf16_bits(a)
                d[name + "_bf16"] = bits
                d[name] = bf16_to_f32(bits)
        else:
            d.update(q=np.ascontiguousarray(q), k=np.ascontiguousarray(k),
                     v=np.ascontiguousarray(v))
        return d

    def chunk_inputs(self, t0: int, n: int) -> dict:
        """Steps t0 .. t0+n-1 of step_inputs stacked on a token axis after the head axis:
        q, k [B][H][n][d_k], v [B][H][n][d_v], alpha [B][H][n] or [B][H][n][d_k], beta
        [B][H][n] (and the bf16 patterns with bf16 I/O)."""
        steps = [self.step_inputs(t0 + t) for t in range(n)]
        return {name: np.ascontiguousarray(np.stack([x[name] for x in steps], axis=2))
                for name in steps[0]}


# The workloads: a tiny oracle check, a GDN layer, a KDA layer, a serving pool, the windowed
# variant, the GDN layer in 8-token chunks and the GDN layer with the side-stream split. Bit mixes: averages are over the non-pivot units.
WORKLOADS = {
    "tiny": Workload(
        name="tiny", batch=2, n_heads=2, d_k=16, d_v=16, steps=8, gate=GATE_SCALAR,
        unit=UNIT_HEAD, io_dtype=IO_F32, mix=((6, 2),), n_pivots=0, seed=0,
        alpha_mu=0.0, alpha_min=0.0, normalize_q=False,
        notes="uniform 6-bit, 2 fit alternations, fp32 I/O, q not normalized"),
    "gdn": Workload(
        name="gdn", batch=64, n_heads=32, d_k=128, d_v=128, steps=256, gate=GATE_SCALAR,
        unit=UNIT_HEAD, io_dtype=IO_BF16, mix=((4, 10), (6, 10), (8, 10)), n_pivots=2, seed=1,
        alpha_min=0.9, notes="per-head widths {4,6,8} mean 6 + 2 fp16 pivot heads"),
    "kda": Workload(
        name="kda", batch=128, n_heads=32, d_k=128, d_v=128, steps=256, gate=GATE_DIAG,
        unit=UNIT_ROW, io_dtype=IO_BF16, mix=((2, 1420), (4, 1621), (6, 608), (8, 406)),
        n_pivots=41, seed=2, alpha_min=0.85,
        notes="per-key-row widths {2,4,6,8} mean 4.0 + 41 fp16 pivot rows (1%)"),
    "pool": Workload(
        name="pool", batch=512, n_heads=32, d_k=128, d_v=128, steps=64, gate=GATE_SCALAR,
        unit=UNIT_HEAD, io_dtype=IO_BF16, mix=((2, 8), (4, 14), (6, 8)), n_pivots=2, seed=3,
        n_slots=1024, alpha_min=0.9,
        notes="1024-slot pool, 512 active by seeded permutation, mean 4 bits + 2 pivot heads"),
    "window": Workload(
        name="window", batch=256, n_heads=32, d_k=128, d_v=128, steps=512, gate=GATE_SCALAR,
        unit=UNIT_HEAD, io_dtype=IO_BF16, mix=((8, 32),), n_pivots=0, seed=4, alpha_min=0.9,
        window=16, n_outliers=8,
        notes="8-bit, requantize every 16 tokens, top-8 |S| per head kept fp16"),
    "chunk": Workload(
        name="chunk", batch=64, n_heads=32, d_k=128, d_v=128, steps=256, gate=GATE_SCALAR,
        unit=UNIT_HEAD, io_dtype=IO_BF16, mix=((4, 10), (6, 10), (8, 10)), n_pivots=2, seed=1,
        alpha_min=0.9, tokens=8,
        notes="the GDN layer advanced 8 tokens per call (prefill / speculative decode chunk), "
              "requantized once per call"),
    "split": Workload(
        name="split", batch=64, n_heads=32, d_k=128, d_v=128, steps=256, gate=GATE_SCALAR,
        unit=UNIT_HEAD, io_dtype=IO_BF16, mix=((4, 10), (6, 10), (8, 10)), n_pivots=2, seed=1,
        alpha_min=0.9, side_stream=True,
        notes="the GDN layer with the update on one stream (fp32 state to a staging buffer) "
              "and the refit + requantization on a second"),
}


def small(name: str, batch: int = 3, n_heads: int = 4, d: int = 32, **kw) -> Workload:
    """A reduced copy of a named workload with the same mix proportions (for parity tests)."""
    w = WORKLOADS[name]
    n_units = n_heads if w.unit == UNIT_HEAD else n_heads * d
    full_units = w.n_heads if w.unit == UNIT_HEAD else w.n_heads * w.d_k
    n_piv = kw.pop("n_pivots", max(1, round(w.n_pivots * n_units / full_units))
                   if w.n_pivots else 0)
    rest = n_units - n_piv
    total = sum(c for _, c in w.mix)
    counts = [int(c * rest // total) for _, c in w.mix]
    counts[0] += rest - sum(counts)
    mix = tuple((wd, c) for (wd, _), c in zip(w.mix, counts) if c > 0)
    n_slots = kw.pop("n_slots", 2 * batch if w.n_slots else 0)
    return replace(w, name=f"{name}-small", batch=batch, n_heads=n_heads, d_k=d, d_v=d,
                   mix=mix, n_pivots=n_piv, n_slots=n_slots, **kw)
