"""Host-side pieces of the benchmark (CPU only): the byte accounting of the
weight formats and the code hash that attributes DRAM counters to sources."""
import os

import bench
import synthetic


def test_block_bytes_and_expert_bytes():
    wl = synthetic.WORKLOADS["30b"]
    assert wl.block_bytes == 54 and wl.matrix_bytes(768, 2048) == 768 * 8 * 54
    s = synthetic.WORKLOADS["30b-sign"]
    assert s.block_bytes == 34 and s.matrix_bytes(768, 2048) == 768 * 8 * 34
    e = synthetic.WORKLOADS["30b-e16"]
    assert e.block_bytes == 60 and e.matrix_bytes(768, 2048) == 768 * 8 * 60 + 2 * 768
    # one expert = gate + up ([ffn][hidden]) + down ([hidden][ffn])
    assert wl.expert_bytes == 3 * 768 * 2048 // 256 * 54
    assert e.expert_bytes == 2 * (768 * 8 * 60 + 2 * 768) + (2048 * 3 * 60 + 2 * 2048)


def test_kernel_bytes_scale_with_unique_experts():
    wl = synthetic.WORKLOADS["large-b8"]
    a, b = bench.kernel_bytes(wl, 10.0), bench.kernel_bytes(wl, 20.0)
    per_expert = 2 * wl.matrix_bytes(wl.ffn, wl.hidden)
    assert b["gateup"] - a["gateup"] == 10 * per_expert
    assert b["down"] - a["down"] == 10 * wl.matrix_bytes(wl.hidden, wl.ffn)


def test_kernel_bytes_of_the_step_with_a_shared_expert():
    """One token with a shared expert runs as the one-token step alone, so its
    algorithmic bytes are the routed step's plus the shared expert's 8-bit
    weights (three matrices of hidden x ffn_s, 34 bytes per 32) and its
    tagged block words (written and read)."""
    plain, shared = synthetic.WORKLOADS["30b"], synthetic.WORKLOADS["30b-shared"]
    a, b = bench.kernel_bytes(plain, 8.0), bench.kernel_bytes(shared, 8.0)
    H, Fs = shared.hidden, shared.shared_ffn
    assert b["step1"] - a["step1"] == 3 * H * Fs * 34 // 32 + Fs // 32 * 10 * 8 * 2


def test_code_hash_ignores_comments(tmp_path, monkeypatch):
    csrc = tmp_path / "bit_moe_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text('int a = 1; // one\n/* block */ const char* s = "x//y";\n')
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_source_hash()
    (csrc / "k.cu").write_text('int a = 1;   // another comment\nconst char* s = "x//y";  /* c */\n')
    assert bench.kernel_source_hash() == h0
    (csrc / "k.cu").write_text('int a = 2; // one\n/* block */ const char* s = "x//y";\n')
    assert bench.kernel_source_hash() != h0
    (csrc / "k.cu").write_text('int a = 1; // one\n/* block */ const char* s = "x/ /y";\n')
    assert bench.kernel_source_hash() != h0


def test_code_hash_per_kernel_follows_its_includes(tmp_path, monkeypatch):
    """A kernel's hash covers its translation unit and the local headers it
    includes, transitively, and nothing else."""
    csrc = tmp_path / "bit_moe_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "step1.cu").write_text('#include "a.cuh"\n#include "bitmoe.h"\nint s = 1;\n')
    (csrc / "a.cuh").write_text('#include "b.cuh"\nint a = 1;\n')
    (csrc / "b.cuh").write_text("int b = 1;\n")
    (csrc / "decode.cu").write_text("int d = 1;\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0, d0, all0 = bench.kernel_source_hash("step1"), bench.kernel_source_hash("gateup"), bench.kernel_source_hash()
    (csrc / "decode.cu").write_text("int d = 2;\n")
    assert bench.kernel_source_hash("step1") == h0
    assert bench.kernel_source_hash("gateup") != d0 and bench.kernel_source_hash() != all0
    (csrc / "b.cuh").write_text("int b = 2;\n")
    assert bench.kernel_source_hash("step1") != h0


def test_cpu_baseline_reports_host_and_pinning():
    """The oracle's timed CPU baseline on the tiny layer: pinned to one core
    (the affinity is restored afterwards), median of 3 timings, and the host's
    core count and CPU model stated."""
    before = os.sched_getaffinity(0)
    cb = bench.cpu_baseline(synthetic.WORKLOADS["tiny"], repeats=3, n_tok=2)
    assert os.sched_getaffinity(0) == before
    assert cb["cores"] == 1 and cb["kind"] == "oracle" and cb["unit"] == "tok/s"
    assert len(cb["times_s"]) == 3 and cb["value"] == 2 / sorted(cb["times_s"])[1]
    assert cb["pinned_core"] in before
    assert cb["nproc"] >= 1 and isinstance(cb["cpu_model"], str)
