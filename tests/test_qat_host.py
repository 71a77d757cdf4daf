"""Host logic of the self-reconstruction QAT driver (no GPU)."""
import math

import pytest
import torch

from bcjr_sum_product_b200 import qat


def test_anneal_is_geometric_from_T0_to_T_end():
    ts = qat.anneal(0.3, 0.01, 5)
    assert ts[0] == pytest.approx(0.3) and ts[-1] == pytest.approx(0.01)
    ratios = [b / a for a, b in zip(ts, ts[1:])]
    assert all(r == pytest.approx(ratios[0]) for r in ratios)
    assert all(b < a for a, b in zip(ts, ts[1:]))
    assert qat.anneal(1.0, 0.01, 1) == [1.0]
    with pytest.raises(ValueError):
        qat.anneal(0.0, 0.01, 3)


def test_hard_mse_of_a_state_path():
    # 4 states, V = 2: codewords (s, -s); path 0, 3, 1 against a target
    c = torch.tensor([[0.0, 0.0], [1.0, -1.0], [2.0, -2.0], [3.0, -3.0]])
    states = torch.tensor([[0, 3, 1]], dtype=torch.int32)
    target = torch.tensor([[0.5, 0.0, 3.0, -2.0, 1.0, -1.5]])
    expect = 0.25 + 0.0 + 0.0 + 1.0 + 0.0 + 0.25
    assert float(qat.hard_mse(states, c, target, 2)[0]) == pytest.approx(expect)
