"""Pins of the oracle's projection (Y = X W^T in fp64) against things other
than itself: identity weights return X, one-hot rows select weight columns,
and a pure-Python triple loop on a tiny integer case."""
import numpy as np
import torch

import oracle


def test_identity_weights_return_the_input():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(7, 64, generator=g).to(torch.bfloat16)
    w = torch.eye(64).to(torch.bfloat16)
    y = oracle.linear_rows(x, w, range(7))
    assert np.array_equal(y, x.double().numpy())


def test_one_hot_rows_select_weight_columns():
    g = torch.Generator().manual_seed(2)
    w = torch.randn(48, 32, generator=g).to(torch.bfloat16)
    x = torch.zeros(32, 32, dtype=torch.bfloat16)
    for i in range(32):
        x[i, i] = 1.0
    y = oracle.linear_rows(x, w, range(32))
    assert np.array_equal(y, w.double().numpy().T)


def test_triple_loop_on_small_integers():
    g = torch.Generator().manual_seed(3)
    x = torch.randint(-4, 5, (5, 6), generator=g).to(torch.bfloat16)
    w = torch.randint(-4, 5, (3, 6), generator=g).to(torch.bfloat16)
    y = oracle.linear_rows(x, w, [0, 2, 4])
    for r, i in enumerate([0, 2, 4]):
        for n in range(3):
            assert y[r, n] == sum(float(x[i, k]) * float(w[n, k]) for k in range(6))
