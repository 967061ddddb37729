"""Host-side rules of bench.py (no GPU)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _clocks(sm, mx, reasons):
    return {"sm_mhz": sm, "sm_max_mhz": mx, "reasons": reasons, "samples": 5}


def test_clean_and_power_capped_runs_are_kept():
    assert not bench.clocks_rejected(_clocks(1965.0, 1965.0, []))
    assert not bench.clocks_rejected(_clocks(1852.0, 1965.0, ["sw_power_cap"]))
    # a dense step settling far down under the power cap is still a valid run
    assert not bench.clocks_rejected(_clocks(1300.0, 1965.0, ["sw_power_cap"]))
    assert not bench.clocks_rejected(None)


def test_slowdowns_and_leftover_clock_locks_are_measured_again():
    for reason in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected(_clocks(1965.0, 1965.0, [reason]))
        assert bench.clocks_rejected(_clocks(1500.0, 1965.0, ["sw_power_cap", reason]))
    # well below the maximum with nothing to explain it: a lock someone left behind
    assert bench.clocks_rejected(_clocks(1100.0, 1965.0, []))
    assert not bench.clocks_rejected(_clocks(1800.0, 1965.0, []))


def test_real_token_flops_count_real_query_and_key_tokens():
    """Real-token FLOPs: 4 D (real query tokens) (real key tokens) per listed
    pair; the block-pair count includes the padded slots."""
    import numpy as np
    import oracle
    from block_sparse_video_gather_b200 import workloads
    wl = workloads.custom(T=5, Hg=9, Wg=11, H=1, topk=2)  # partial blocks on every axis
    real = bench.block_real_tokens(wl)
    np.testing.assert_array_equal(real, oracle.block_valid_counts(oracle.geometry_of(wl)))
    idx = np.array([[[[0, 3], [1, -1], [2, 2], [0, 1], [3, 0], [1, 2], [0, 3], [2, 1]]]], dtype=np.int32)
    num = np.array([[[2, 1, 2, 0, 1, 2, 2, 2]]], dtype=np.int32)
    want = 0
    for r in range(8):
        for t in range(num[0, 0, r]):
            want += 4 * 128 * int(real[r]) * int(real[idx[0, 0, r, t]])
    assert bench.real_token_flops(wl, idx, num) == want
    assert bench.selected_flops(wl, num) == 4 * 128 * 256 ** 2 * int(num.sum())
    # prefix tiles count their real tokens too (a partial last prefix tile)
    wl64 = workloads.custom(T=4, Hg=8, Wg=8, block=(4, 4, 4), n_prefix=100, H=1)
    np.testing.assert_array_equal(bench.block_real_tokens(wl64),
                                  oracle.block_valid_counts(oracle.geometry_of(wl64)))


def test_committed_traffic_summaries_parse_and_name_their_workload():
    """Every ncu summary bench.py reads a per-launch DRAM figure from carries the
    three machine-read lines, for the workload it is filed under; the figure is
    used only while the hash of the kernel sources matches."""
    import re
    entries = list(bench.TRAFFIC_PROFILES.items()) + list(bench.FP4_TRAFFIC_PROFILES.items())
    for workload, (path, sources) in entries:
        text = open(path).read()
        assert re.search(r"source_hash:\s*[0-9a-f]{16}", text), path
        assert re.search(r"bench_workload:\s*" + workload + r"\b", text), path
        m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
        assert m and float(m.group(1)) > 0, path
        got = bench.profile_traffic(workload, path, sources)
        fresh = re.search(r"source_hash:\s*([0-9a-f]+)", text).group(1) == bench.attn_source_hash(sources)
        assert (got == float(m.group(1))) if fresh else got is None, path
        assert bench.profile_traffic("tiny", path, sources) is None  # another workload's summary never applies


def test_grouped_products_count_each_q_tiles_union():
    """Executed Q-tile products of the grouped 64-token kernel, on groups built
    to take every shape of the two Q tiles' streams: each Q tile walks the union
    of its two query blocks' selections, two blocks per 128-key tile."""
    import numpy as np
    from tests.test_gpu_grouped64 import _stream_shapes
    idx, num = _stream_shapes(32)
    # per group: ceil(|union of blocks 0-1| / 2) + ceil(|union of blocks 2-3| / 2)
    assert bench.grouped_products(idx, num, 32) == (0 + 3) + (2 + 0) + (4 + 4) + (5 + 2) + (1 + 6) + (5 + 6) \
        + (2 + 2) + (2 + 2)
    # a list that repeats an id: that group walks the four lists as given for both Q tiles
    idx2, num2 = idx.copy(), num.copy()
    idx2[0, 0, 9, :3] = [13, 13, 1]
    num2[0, 0, 9] = 3
    per_list = sum((int(c) + 1) // 2 for c in num2[0, 0, 8:12])
    assert bench.grouped_products(idx2, num2, 32) == bench.grouped_products(idx, num, 32) - 8 + 2 * per_list
    # ids outside [0, NB) are skipped; an all-dense group of two query blocks (NB % 4 == 2)
    dense = np.broadcast_to(np.arange(6, dtype=np.int32), (1, 1, 6, 6)).copy()
    assert bench.grouped_products(dense, np.full((1, 1, 6), 6, np.int32), 6) == 3 + 3 + 3
    dense[0, 0, 5, 0] = 99
    assert bench.grouped_products(dense, np.full((1, 1, 6), 6, np.int32), 6) == 3 + 3 + 3
