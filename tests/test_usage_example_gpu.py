"""The usage example (tests/usage_example.py) runs as written: the forward, then a backward
through the autograd wrapper, with finite results of the documented shapes."""
import pytest
import torch

import usage_example

pytestmark = pytest.mark.gpu


def test_usage_example_runs():
    env = usage_example.run()
    torch.cuda.synchronize()
    o, S_T, q = env["o"], env["S_T"], env["q"]
    assert o.shape == (4, 4096, 16, 128) and S_T.shape == (4, 16, 128, 128)
    assert torch.isfinite(o).all() and torch.isfinite(S_T).all()
    assert q.grad is not None and q.grad.shape == q.shape and torch.isfinite(q.grad.float()).all()
