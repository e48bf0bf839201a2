"""The benchmark's algorithmic byte and flop counts (fixed formulas, whatever
the kernels do), checked against values worked out by hand from the
workload shapes: 480p ReLU 588.1 MB / 33.17 GF, 720p 60 s GDN 3.263 GB /
328.3 GF, streaming GDN 4.692 GB / 464.4 GF, D = 256 stress 17.184 GB /
2.208 TF (ReLU) and 3.573 TF (GDN)."""
import pytest

import bench
import synth


@pytest.mark.parametrize("name,mode,gbytes,gflop", [
    ("relu_480p", "relu", 0.5881, 33.17),
    ("gdn_720p_60s", "gdn", 3.263, 328.3),
    ("gdn_stream", "gdn", 4.692, 464.4),
    ("stress_d256", "relu", 17.184, 2208.0),
    ("stress_d256", "gdn", 17.184, 3573.0),
])
def test_step_counts_match_hand_worked_values(name, mode, gbytes, gflop):
    b, f = bench.step_counts(synth.workload(name), mode)
    assert abs(b / 1e9 - gbytes) / gbytes < 1e-3
    assert abs(f / 1e9 - gflop) / gflop < 1e-3


def test_frame_counts_by_hand():
    # one 2x2 frame with 3 tokens: GDN 6 S D^2 + 2 D^3, ReLU 4 S D^2 + 4 S D
    assert bench.frame_flops("gdn", 3, 2) == 6 * 3 * 4 + 2 * 8
    assert bench.frame_flops("relu", 3, 2) == 4 * 3 * 4 + 4 * 3 * 2
    # bytes: q, k, v, o of 3 x 2 bf16 per frame, 8 B of gates, a 2 x 2 fp32 state out
    assert bench.call_bytes("gdn", 1, 1, 1, 3, 2, 2, False) == 4 * 3 * 2 * 2 + 8 + 16
    # state in as well: read and written
    assert bench.call_bytes("gdn", 1, 1, 1, 3, 2, 2, True) == 4 * 3 * 2 * 2 + 8 + 32
    # ReLU: no gates, the normaliser z in/out
    assert bench.call_bytes("relu", 1, 1, 1, 3, 2, 2, False) == 4 * 3 * 2 * 2 + 16 + 8
    # the reversed scan has no state; the per-token gate reads S gates per frame
    assert bench.call_bytes("gdn_reverse", 1, 1, 1, 3, 2, 2, False) == 4 * 3 * 2 * 2 + 8
    assert bench.call_bytes("gdn_token_beta", 1, 1, 1, 3, 2, 2, False) == \
        4 * 3 * 2 * 2 + 4 + 4 * 3 + 16


def test_streaming_plan_passes_the_state_between_chunks():
    plan = bench.step_plan(synth.workload("gdn_stream"), "gdn")
    assert plan == [(8 * c, 8, c > 0) for c in range(8)]
    assert bench.step_plan(synth.workload("gdn_720p_60s"), "gdn") == [(0, 181, False)]
