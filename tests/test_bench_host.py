"""Host-side pieces of bench.py and of the seeded input module (no GPU)."""
import numpy as np

import bench
from block_sparse_attention_15_b200 import inputs as I

NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


def _line(sm, power, reasons=("Not Active",) * 4):
    return f"{sm}, 1965, {power}, " + ", ".join(reasons)


def test_clock_summary_keeps_the_timed_window():
    lines = [(0.5, _line(1200, 100)),            # before the window: ignored
             (1.1, _line(1965, 700)),
             (1.2, _line(1900, 900, ("Not Active", "Not Active", "Not Active", "Active"))),
             (1.3, _line(1965, 800)),
             (2.5, _line(1000, 50))]             # after the window: ignored
    got = bench.summarize_clock_lines(lines, 1.0, 2.0, NAMES)
    assert got["samples"] == 3
    assert got["sm_mhz"] == 1965.0
    assert got["power_w_max"] == 900.0
    assert got["reasons"] == ["sw_power_cap"]


def test_clock_summary_short_window_takes_the_next_sample():
    lines = [(0.5, _line(1200, 100)), (2.5, _line(1800, 300)), (3.0, _line(1700, 300))]
    got = bench.summarize_clock_lines(lines, 1.0, 1.05, NAMES)
    assert got["samples"] == 1 and got["sm_mhz"] == 1800.0
    assert bench.summarize_clock_lines([], 1.0, 2.0, NAMES)["sm_mhz"] is None


def test_varlen_random_selection():
    """Per sequence, block and head: topk_count(frac, n_kv_i) distinct KV
    blocks of that sequence, ascending, -1 after them; seeded."""
    q_lens, kv_lens = (100, 700, 64), (64, 1000, 130)
    idx, num, ks = I.varlen_random_selection(q_lens, kv_lens, 3, 0.5, 7)
    nq = [2, 11, 1]
    nkv = [1, 16, 3]
    assert ks == [I.topk_count(0.5, n) for n in nkv] == [1, 8, 1]
    assert idx.shape == (3, sum(nq), max(ks)) and num.shape == (3, sum(nq))
    row = 0
    for i in range(3):
        for _ in range(nq[i]):
            for h in range(3):
                sel = idx[h, row, :ks[i]]
                assert num[h, row] == ks[i]
                assert np.all(np.diff(sel) > 0) and sel.min() >= 0 and sel.max() < nkv[i]
                assert np.all(idx[h, row, ks[i]:] == -1)
            row += 1
    idx2, num2, _ = I.varlen_random_selection(q_lens, kv_lens, 3, 0.5, 7)
    assert np.array_equal(idx, idx2) and np.array_equal(num, num2)


def test_forward_host_binding_rejects_bad_tensors():
    """The host-buffer binding checks dtypes, devices and shapes before it
    touches the GPU."""
    import pytest
    import torch

    from block_sparse_attention_15_b200 import binding as vsa

    q = torch.zeros((1, 2, 128, 64), dtype=torch.bfloat16)
    k = torch.zeros((1, 2, 192, 64), dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        vsa.vsa_forward_host(q.float(), k, k, topk=1)
    with pytest.raises(ValueError):
        vsa.vsa_forward_host(q, k, k[:, :, :128], topk=1)               # v shape != k shape
    with pytest.raises(ValueError):
        vsa.vsa_forward_host(q, k, k, torch.zeros((1, 128, 3, 64), dtype=torch.bfloat16), topk=1)
    with pytest.raises(ValueError):
        vsa.vsa_forward_host(q, k, k, topk=1, q_block_sizes=[64])     # 2 query blocks


def test_traffic_record_applies_to_its_workload_only():
    """The committed DRAM-traffic record is reported for the workload shape it
    was captured on (with the kernel sources unchanged) and for no other."""
    import dataclasses
    h3 = bench.make_workload("h3")
    assert bench.profiled_traffic(h3) == 1080151296
    assert bench.profiled_traffic(bench.make_workload("vsa128")) is None
    assert bench.profiled_traffic(bench.make_workload("long10")) is None
    assert bench.profiled_traffic(dataclasses.replace(h3, H=16)) is None
