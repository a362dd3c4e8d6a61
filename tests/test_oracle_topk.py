"""Pins of the top-k-excluding-one oracle (oracle/topk.py): a hand-worked row
with ties, an excluded maximum and -inf entries; brute force with Python's own
sorted() on random rows; padding; invalid rows; exact bf16 widening."""
import numpy as np

from oracle import topk
from speculative_sampling_b200 import inputs


def test_hand_worked_row():
    row = np.array([[1.0, 5.0, 3.0, 5.0, -np.inf, 3.0, 7.0, 3.0]], np.float32)
    # exclude token 6 (the maximum); order by value, equal values by index
    idx, val = topk.topk_exclude(row, np.array([6]), 5)
    assert idx.tolist() == [[1, 3, 2, 5, 7]]
    assert val.tolist() == [[5.0, 5.0, 3.0, 3.0, 3.0]]
    idx, _ = topk.topk_exclude(row, np.array([-1]), 3)
    assert idx.tolist() == [[6, 1, 3]]
    # more than the row holds: padded with -1 / -inf, the -inf entry last
    idx, val = topk.topk_exclude(row, np.array([2]), 9)
    assert idx.tolist() == [[6, 1, 3, 5, 7, 0, 4, -1, -1]]
    assert val[0, 6] == -np.inf and val[0, 7] == -np.inf


def test_matches_python_sorted_on_random_rows():
    rng = np.random.default_rng(4)
    for trial in range(40):
        V = int(rng.integers(2, 300))
        k = int(rng.integers(1, 70))
        row = np.round(rng.normal(0, 2, V), 1).astype(np.float32)  # many ties
        ex = int(rng.integers(-1, V))
        idx, val = topk.topk_exclude(row[None], np.array([ex]), k)
        want = sorted((i for i in range(V) if i != ex), key=lambda i: (-float(row[i]), i))[:k]
        got = [int(i) for i in idx[0] if i >= 0]
        assert got == want
        assert all(val[0, j] == row[want[j]] for j in range(len(want)))


def test_invalid_row_and_bf16_widening():
    row = np.array([[1.0, np.nan, 2.0]], np.float32)
    idx, val = topk.topk_exclude(row, np.array([-1]), 2)
    assert np.all(idx == -1) and np.all(np.isnan(val))
    b = inputs.f32_to_bf16_bits(np.array([[0.1, 0.3, 0.2]], np.float32))
    idx, val = topk.topk_exclude(b, np.array([-1]), 3, dtype="bf16")
    assert idx.tolist() == [[1, 2, 0]]
    assert val[0, 0] == float(inputs.bf16_bits_to_f32(b)[0, 1])
