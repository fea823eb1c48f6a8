"""The bench reads a kernel's DRAM traffic from its committed ncu summary only while the
summary's source digest matches that kernel's sources: edits to comments keep the digest, edits
to code change it, and a kernel's digest ignores the other kernels' files."""
import os
import shutil

import bench


def _copy_sources(tmp_path):
    dst = tmp_path / "bit_recurrent_state_gated_b200" / "csrc"
    shutil.copytree(os.path.join(bench.ROOT, "bit_recurrent_state_gated_b200", "csrc"), dst,
                    ignore=shutil.ignore_patterns("*.o"))
    return dst


def _edit(path, old, new):
    text = path.read_text()
    assert old in text
    path.write_text(text.replace(old, new, 1))


def test_code_only_strips_comments_and_whitespace():
    assert bench._code_only("a = 1;  // note\n/* block\ncomment */ b =  2;") == "a = 1; b = 2;"


def test_digest_follows_code_not_comments(tmp_path):
    src = _copy_sources(tmp_path)
    root = str(tmp_path)
    base = {k: bench.source_digest(k, root) for k in bench.KERNEL_SOURCES}
    assert base == {k: bench.source_digest(k) for k in bench.KERNEL_SOURCES}
    _edit(src / "sq_window_step.cu", "// sq_window_step.cu", "// sq_window_step.cu (reworded)")
    assert {k: bench.source_digest(k, root) for k in bench.KERNEL_SOURCES} == base
    _edit(src / "sq_window_step.cu", "const int s = 0;", "const int s = 0 * 1;")
    after = {k: bench.source_digest(k, root) for k in bench.KERNEL_SOURCES}
    assert after["k_window"] != base["k_window"]
    assert after["k_decode"] == base["k_decode"] and after["k_chunk"] == base["k_chunk"]
