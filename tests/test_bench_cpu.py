"""CPU checks of bench.py's host logic: the launch flags it benchmarks with,
the algorithmic byte count behind every roofline figure, the averaging over a
workload's step cycle, and the rule that a recorded ncu traffic figure is
used only for the kernel sources it was captured on."""
import os

import numpy as np
import pytest

import bench
from paged_attention_decode_pkv_b200 import workloads as W


def test_launch_flags_are_the_documented_ones():
    from paged_attention_decode_pkv_b200 import pkv
    assert bench.launch_flags(pkv) == pkv.LAUNCH_PDL | pkv.LAUNCH_EARLY_TABLES | \
        pkv.LAUNCH_EARLY_PAGES
    assert bench.launch_flags(pkv, early_pages=False) == pkv.LAUNCH_PDL | pkv.LAUNCH_EARLY_TABLES
    assert bench.launch_flags(pkv, pdl=False) == 0


def test_algorithmic_bytes_follow_the_per_sequence_formula():
    # per (sequence, layer): 2048 B per context token (K and V of 8 heads x 64
    # BF16), q 32 x 64 BF16, out 32 x 64 FP32, 4 B per block-table entry, 4 B
    # for the length -- written out sequence by sequence
    lens = np.array([0, 1, 15, 16, 17, 1000, 8192], np.int32)
    want = 0
    for L in lens.tolist():
        want += 2 * 8 * 64 * 2 * L + 32 * 64 * 2 + 32 * 64 * 4 + 4 * -(-L // 16) + 4
    assert bench.alg_bytes_decode(lens) == want
    # T queries: q and out per query; BF16 output halves the out bytes
    want2 = want + len(lens) * (32 * 64 * 2 + 32 * 64 * 4)
    assert bench.alg_bytes_decode(lens, queries=2) == want2
    assert bench.alg_bytes_decode(lens, out_bytes=2) == want - len(lens) * 32 * 64 * 2


class _FakeRunner:
    """Just the state Runner's byte accounting reads (no GPU)."""
    decode_bytes = bench.Runner.decode_bytes
    mean_decode_bytes = bench.Runner.mean_decode_bytes

    def __init__(self, w, fused=True):
        self.w, self.fused, self.queries = w, fused, 1
        self.lens_np = [w.seq_lens(s) for s in range(1, w.num_steps + 1)]

        class _Out:
            @staticmethod
            def element_size():
                return 4
        self.out = _Out()


def test_mean_bytes_over_the_step_cycle_equal_the_brute_force_mean():
    w = W.continuous_batching()
    r = _FakeRunner(w)
    for start, n in [(0, 20), (20, 1000), (5, 3), (17, 16), (0, 1)]:
        brute = sum(r.decode_bytes(i) for i in range(start, start + n)) / n
        assert r.mean_decode_bytes(start, n) == pytest.approx(brute, rel=1e-12)
    # the fused append adds each sequence's new K/V rows read and written
    assert r.decode_bytes(0) == bench.alg_bytes_decode(w.seq_lens(1)) + 4096 * 64


def test_recorded_traffic_only_for_the_captured_sources(tmp_path, monkeypatch):
    digest = bench.kernel_source_digest()
    prof = tmp_path / "profiles"
    prof.mkdir()
    body = "kernel_source_sha256: %s\ndram_bytes_per_launch: 2000\nalg_bytes_of_launch: 1000\n"
    (prof / "decode_traffic_good.txt").write_text(body % digest)
    (prof / "decode_traffic_stale.txt").write_text(body % ("0" * 64))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_digest", lambda: digest)
    assert bench.recorded_traffic("good", 500.0) == pytest.approx(1000.0)   # scaled 2x
    assert bench.recorded_traffic("stale", 500.0) is None
    assert bench.recorded_traffic("missing", 500.0) is None


def test_committed_traffic_records_match_the_kernel_sources():
    # every committed capture names the sources it was taken on; those of the
    # three captured workloads are today's (else bench.py would report null)
    for name in ("continuous_batching_b64", "llama1b_b16", "long_context_b4"):
        assert bench.recorded_traffic(name, 1e6) is not None, name


def test_comment_stripping_keeps_code_and_literals():
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "// not a comment";'
    out = bench._strip_comments(src)
    assert "note" not in out and "block" not in out
    assert '"// not a comment"' in out and "int a = 1;" in out
