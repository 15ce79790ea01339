"""Host-side pieces of bench.py that its figures depend on (no GPU).

- The DRAM traffic recorded from an ncu capture is reported only while the
  kernel's sources hash as they did at capture time.
- The all-cores CPU baseline splits every layer's output rows into contiguous,
  disjoint slices; the oracle on the slices reproduces the whole decode step.
- The timed-block count covers the minimum timed region.
"""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


@pytest.mark.parametrize("n_rows", [1, 7, 2560, 6912])
@pytest.mark.parametrize("parts", [1, 3, 16, 128])
def test_row_slices_cover_every_row_once(n_rows, parts):
    sl = bench.row_slices(n_rows, parts)
    assert len(sl) == parts
    assert sl[0][0] == 0 and sl[-1][1] == n_rows
    for (a0, a1), (b0, b1) in zip(sl, sl[1:]):
        assert a1 == b0
    sizes = [n1 - n0 for n0, n1 in sl]
    assert min(sizes) >= 0 and max(sizes) - min(sizes) <= 1 and sum(sizes) == n_rows


def test_profiled_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    h = bench.kernel_source_hash("gemv")
    f = tmp_path / "traffic.txt"
    f.write_text("# comment decode_2b 1 %s\ndecode_2b 6106112 %s\nstale 123 0000000000000000\n" % (h, h))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.profiled_traffic("decode_2b", "gemv") == 6106112.0
    assert bench.profiled_traffic("stale", "gemv") is None  # taken on other sources
    assert bench.profiled_traffic("absent", "gemv") is None
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(tmp_path / "missing.txt"))
    assert bench.profiled_traffic("decode_2b", "gemv") is None


def test_source_hash_covers_the_kernel_files(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("a")
    monkeypatch.setitem(bench.KERNEL_SOURCES, "probe", [str(src)])
    monkeypatch.setattr(bench, "ROOT", "/")
    h1 = bench.kernel_source_hash("probe")
    src.write_text("b")
    assert bench.kernel_source_hash("probe") != h1


def test_rep_plan_covers_the_minimum_region():
    assert bench.rep_plan(20, 0.8e-3, 0.5) == 625
    assert bench.rep_plan(20, 1.0, 0.05) == 1
    assert bench.rep_plan(20, 1e-9, 0.05, max_reps=100) == 100
    assert bench.rep_plan(20, 0.0, 0.05, max_reps=7) == 7


def test_chain_sample_rows_and_shared_input():
    layers, set_bytes = bench.oracle_chain_layers(rows_div=256)
    assert len(layers) == len(bench.CHAIN_70B)
    assert set_bytes == sum(-(-N // 256) * K // 4 for K, N in bench.CHAIN_70B)
    for (packed, gamma, K, xf), (K2, N) in zip(layers, bench.CHAIN_70B):
        assert packed.shape == (-(-N // 256), K // 4) and K == K2 and xf.shape == (1, K)
    assert layers[3][3] is layers[2][3]  # gate and up take one input


def test_oracle_row_slices_reassemble_the_decode_step():
    import oracle

    layers, set_bytes = bench.oracle_chain_layers(rows_div=256)
    for packed, gamma, K, xf in layers:
        T, ok = oracle.unpack(packed, K)
        acc, y, *_ = oracle.forward(T, gamma, xf)
        parts = []
        for n0, n1 in bench.row_slices(packed.shape[0], 5):
            Ts, _ = oracle.unpack(packed[n0:n1], K)
            acc_s, y_s, *_ = oracle.forward(Ts, gamma, xf)
            parts.append((acc_s, y_s))
        assert np.array_equal(np.concatenate([a for a, _ in parts], axis=1), acc)
        assert np.array_equal(np.concatenate([b for _, b in parts], axis=1), y)
