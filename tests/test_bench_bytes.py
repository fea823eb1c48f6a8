"""The bench's algorithmic bytes per request-step, derived by hand for each workload.

state: packed slot read + written (r16[d_k] + c16[d_v] + code rows per head); io: q, k, v
(bf16, or fp32 for tiny) + alpha (one per head, or d_k for the diagonal gate) + beta + o (fp32)
per head, plus the 4-byte slot index. A chunk of T tokens reads and writes the state once per
call; a window reads the frozen block every token and writes it once per window.
"""
import pytest

import oracle
import bench
from bit_recurrent_state_gated_b200 import workloads as W

H, D = 32, 128
IO_BF16_SCALAR = H * (3 * D * 2 + 4 + 4 + D * 4) + 4          # 41,220
IO_BF16_DIAG = H * (3 * D * 2 + 4 * D + 4 + D * 4) + 4        # 57,476


def head_bytes(widths_rows):
    """r16 + c16 + rows of one head (d_k = d_v = 128), padded to 16 bytes."""
    n = 2 * (D + D) + sum(D * b // 8 for b in widths_rows)
    return (n + 15) // 16 * 16


@pytest.mark.parametrize("name, state, io", [
    # 10 heads each at 4, 6, 8 bits + 2 fp16 heads (128 x 128 x 2 bytes, no scales)
    ("gdn", 2 * (10 * (head_bytes([4] * D) + head_bytes([6] * D) + head_bytes([8] * D))
                 + 2 * D * D * 2), IO_BF16_SCALAR),
    ("pool", 2 * (8 * head_bytes([2] * D) + 14 * head_bytes([4] * D) + 8 * head_bytes([6] * D)
                  + 2 * D * D * 2), IO_BF16_SCALAR),
    # 4096 key rows: 41 fp16 rows, 1420 x 2, 1621 x 4, 608 x 6, 406 x 8 bits; scales per head
    ("kda", 2 * (H * 2 * (D + D) + (41 * 16 + 1420 * 2 + 1621 * 4 + 608 * 6 + 406 * 8) * D // 8),
     IO_BF16_DIAG),
])
def test_algorithmic_bytes(name, state, io):
    wl = W.WORKLOADS[name]
    lay = oracle.Layout(wl.n_heads, wl.d_k, wl.d_v, wl.unit, wl.gate, wl.fit_iters, wl.window,
                        wl.n_outliers)
    slot = oracle.Pool(lay, wl.bits(), 1).slot_bytes
    ab = bench.algorithmic_bytes(wl, slot)
    assert ab["state"] == state and ab["io"] == io and ab["total"] == state + io


def test_chunk_and_window_amortize_the_state():
    gdn = W.WORKLOADS["gdn"]
    slot = 449_536
    assert bench.algorithmic_bytes(gdn.scaled(tokens=8), slot)["state"] == 2 * slot / 8
    win = W.WORKLOADS["window"]
    ab = bench.algorithmic_bytes(win, 541_696)
    assert ab["state"] == 541_696 + 541_696 / 16  # read every token, written once per window
    # low-rank side state (scalar gate): every token reads the 16-byte header (count, gate) and
    # its t terms of 768 bytes (k in bf16, 256 B; b / g in fp32, 512 B); tokens 0..14 write a
    # term and 8 header bytes, the folding token clears the count: per request-step
    # 32 heads x (16 x 16 + 120 x 768 + 15 x 776 + 4) / 16 = 208,120 B
    assert ab["side"] == 208_120
    # the side state is this implementation's representation: reported apart, not in the total
    assert ab["total"] == 541_696 + 541_696 / 16 + IO_BF16_SCALAR == 616_772
