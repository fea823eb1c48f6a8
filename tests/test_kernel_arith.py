"""Host checks of the decode kernel's short arithmetic sequences (no GPU needed).

The kernel divides a row maximum by Q in three single-precision operations, takes correctly
rounded reciprocals of fp16 scales in three, and of any single-precision value with two Newton
steps in double precision; all are exhaustively compared here,
in C with IEEE single-precision fma and multiplication, with the correctly rounded results
the library division and reciprocal would give (tests/c/kernel_arith.c).
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def test_division_and_fp16_reciprocal_sequences_are_exact(tmp_path):
    src = os.path.join(HERE, "c", "kernel_arith.c")
    exe = str(tmp_path / "kernel_arith")
    subprocess.run(["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", src, "-o", exe, "-lm"],
                   check=True)
    out = subprocess.run([exe], check=True, capture_output=True, text=True).stdout
    fields = dict(kv.split("=") for kv in out.split())
    assert int(fields["cases"]) > 100_000_000
    assert int(fields["div_mismatch"]) == 0
    assert int(fields["rcp_mismatch"]) == 0
    assert int(fields["rcp32_mismatch"]) == 0
