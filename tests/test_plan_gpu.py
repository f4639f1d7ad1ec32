"""Key-chunk planning (host logic that queries the device's SM count, hence a GPU test): the
chunk count that `favor_partials_bytes` reports for each workload equals a restatement of the
planner's cost model, waves of key-pass CTAs times (tiles per chunk + half a tile of start-up)
plus the partial state the chunks write and the reduction reads (4 MB per key-tile time)."""
import math
import os
import sys

import pytest
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import linear_approximate_softmax_b200 as fv  # noqa: E402
from linear_approximate_softmax_b200 import workloads as wl  # noqa: E402


def planned_chunks(heads, L, d, m, sms):
    tiles = (L + 127) // 128
    nfeat = 256 if (d == 64 and m > 128) else 128
    units = heads * ((m + nfeat - 1) // nfeat)
    best, best_ct = math.inf, tiles
    for P in range(1, tiles + 1):
        ct = (tiles + P - 1) // P
        Pe = (tiles + ct - 1) // ct
        if Pe != P:
            continue
        waves = (units * Pe + sms - 1) // sms
        cost = waves * (ct + 0.5) + heads * Pe * m * (d + 1) * 4 / 4.0e6
        if cost < best - 1e-9:
            best, best_ct = cost, ct
    return (tiles + best_ct - 1) // best_ct


def partials_bytes(heads, P, d, m):
    r = lambda x: (x + 255) // 256 * 256  # noqa: E731
    return r(4 * heads * P * m * (d + 1)) + r(4 * heads * P * m)


@pytest.mark.gpu
@pytest.mark.parametrize("name", wl.WORKLOAD_ORDER)
def test_chunk_plan_matches_cost_model(name):
    w = wl.WORKLOADS[name]
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    P = planned_chunks(w.B * w.Hkv, w.L, w.d, w.m, sms)
    assert fv.favor_partials_bytes(w.B, w.Hkv, w.L, w.d, w.m) == partials_bytes(w.B * w.Hkv, P, w.d, w.m), (name, P)


@pytest.mark.gpu
def test_long_sequence_takes_one_wave_of_key_chunks():
    # B1 H8 L131072 m512 on 148 SMs: 9 chunks (one wave, 9.7 MB of partial state), not the
    # 37 (four waves, 40 MB) that the makespan term alone ties with
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("the figures are for 148 SMs")
    assert fv.favor_partials_bytes(1, 8, 131072, 64, 512) == partials_bytes(8, 9, 64, 512) == 9732096
