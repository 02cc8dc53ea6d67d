"""Host-side arithmetic of bench.py (CPU): the algorithmic bytes its roofline
divides by, and the rule that a committed ncu traffic figure is used only for
the kernel sources it was measured on."""

import os
import shutil

import bench
import sikv_inputs as gen


def test_step_bytes_with_two_bit_values():
    """Per (sequence, KV head) at 4 x 128K: the code rows, k value rows of
    48 bytes instead of 256, the sinks' key and value rows, the codebook."""
    w = gen.config(2)
    per = 16 * (131072 - 64) + 2048 * 48 + 64 * 2 * 128 * 2 + 8192
    assert bench.step_bytes(w, value_row_bytes=48) == per * 32 == 71_532_544
    assert bench.step_bytes(w) - bench.step_bytes(w, value_row_bytes=48) == 32 * 2048 * (256 - 48)


def test_ragged_step_bytes_follow_each_sequence():
    w = gen.config(3)
    want = 0
    for n, k in zip(w.seq_lens, w.topk):
        want += w.num_kv_heads * (16 * (n - 64) + k * 256 + 64 * 2 * 256 + 8192)
    assert bench.step_bytes(w) == want


def test_profiled_traffic_needs_matching_sources(tmp_path, monkeypatch):
    """The figure is read when the summary's source hash equals the hash of
    the kernel's files, and ignored (None) once any of them changes."""
    root = tmp_path / "repo"
    csrc = root / "long_context_decode_sikv_b200" / "csrc"
    csrc.mkdir(parents=True)
    (root / "profiles").mkdir()
    kernel = "decode_fused"
    for name in bench.PROFILED[kernel][1]:
        shutil.copy(os.path.join(bench.ROOT, "long_context_decode_sikv_b200", "csrc", name), csrc / name)
    monkeypatch.setattr(bench, "ROOT", str(root))
    summary = root / "profiles" / bench.PROFILED[kernel][0]
    good = bench.kernel_source_hash(kernel)
    summary.write_text(f"# x\n\n- bench_traffic_bytes_per_launch: 12345\n- bench_traffic_source_hash: {good}\n")
    assert bench.profiled_traffic(kernel) == 12345.0
    first = bench.PROFILED[kernel][1][0]
    with open(csrc / first, "a") as f:
        f.write("\n// edited\n")
    assert bench.kernel_source_hash(kernel) != good
    assert bench.profiled_traffic(kernel) is None
    summary.unlink()
    assert bench.profiled_traffic(kernel) is None
