"""Host logic of bench.py that needs no GPU: the rotation of inputs that fit in
L2, and the lookup of the committed ncu traffic record."""
import hashlib
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
L2 = 126 * 1000 * 1000


def test_inputs_larger_than_twice_the_l2_are_not_copied():
    assert bench.input_copies(985_006_080 + 65_536) == 1       # b256: logits and tokens
    assert bench.input_copies(2 * L2) == 1


def test_small_inputs_rotate_over_at_least_twice_the_l2():
    for n in (73_876_480, 36_944, 1, 2 * L2 - 1):             # b32, tiny, extremes
        c = bench.input_copies(n)
        assert c >= 2 or n * c >= 2 * L2
        assert c == bench.MAX_INPUT_COPIES or c * n >= 2 * L2
        assert c <= bench.MAX_INPUT_COPIES
        assert c == 1 or (c - 1) * n < 2 * L2 or c == bench.MAX_INPUT_COPIES
    assert bench.input_copies(73_876_480) == 4


def _sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def test_traffic_record_matches_sources_and_workload():
    src = ["speculative_decoding_verification_lse_b200/csrc/row_stats.cu",
           "speculative_decoding_verification_lse_b200/csrc/stats_device.cuh",
           "speculative_decoding_verification_lse_b200/csrc/sv_common.cuh"]
    with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
        recs = [l.split() for l in f if l.strip() and not l.startswith("#")]
    mine = [r for r in recs if r[0] == "row_stats" and r[1] == _sha(src)]
    tr = bench.traffic_record("row_stats", src, 985_006_080)
    if mine:
        assert tr == (float(mine[0][2]), int(mine[0][3]))
        # traffic is at least the algorithmic bytes and within 2% of them
        assert 985_006_080 <= tr[0] <= 1.02 * 985_006_080
    else:
        assert tr is None
    # another workload's launch never borrows the record
    assert bench.traffic_record("row_stats", src, 82_083_840) is None
