"""The CPU oracle against its pins (see oracle_pins.py): CPU only."""
import json
import os

import pytest

import oracle
import oracle_pins
from bi_level_routing_b200.workloads import WORKLOADS

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle.default())


def test_workloads_follow_the_stage_table():
    with open(os.path.join(HERE, "golden", "stage_table.json")) as f:
        g = json.load(f)
    dims = g["embed_dims"]["values"]
    for row, C in zip(g["stage_table"]["rows"], dims):
        w = WORKLOADS[f"stage{row['stage']}"]
        assert (w.H, w.W, w.heads, w.hd, w.C) == (row["H"], row["W"], row["heads"], row["head_dim"], C)
        topk = w.R if row["topk"] == "S^2" else row["topk"]
        assert w.topk == topk
        assert w.n_win == g["n_win"]["classification"]
    assert [WORKLOADS[f"stage{i}"].heads for i in range(1, 5)] == g["settings"]["num_heads"]
    assert [WORKLOADS[f"stage{i}"].topk for i in range(1, 4)] == g["settings"]["topks"][:3]
    assert WORKLOADS["stage4"].topk == WORKLOADS["stage4"].R  # -1: every region
    assert WORKLOADS["highres"].n_win == g["n_win"]["high_resolution"]


def test_oracle_rejects_bad_arguments():
    import numpy as np
    x = np.zeros((1, 6, 6, 4))
    with pytest.raises(oracle.OracleError):
        oracle.region_means(x, 4)  # 6 % 4 != 0
    with pytest.raises(oracle.OracleError):
        oracle.route(x, x, 3, 10)  # topk > R
    with pytest.raises(oracle.OracleError):
        oracle.attend(x, x, x, np.full((1, 9, 1), 9, np.int32), 2, 3)  # index outside [0, R)
    with pytest.raises(oracle.OracleError):
        oracle.attend(x, x, x, np.zeros((1, 9, 1), np.int32), 3, 3)  # C % heads != 0
