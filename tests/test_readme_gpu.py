"""The usage example in README.md runs as written (the forward, then a backward through
the autograd wrapper) and gives finite results of the documented shapes."""
import os
import re

import pytest
import torch

pytestmark = pytest.mark.gpu
README = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "README.md")


def test_readme_example_runs():
    blocks = re.findall(r"```python\n(.*?)```", open(README).read(), flags=re.S)
    assert blocks, "README.md has no python example"
    env = {}
    exec(compile(blocks[0], "README.md", "exec"), env)
    torch.cuda.synchronize()
    o, S_T, q = env["o"], env["S_T"], env["q"]
    assert o.shape == (4, 4096, 16, 128) and S_T.shape == (4, 16, 128, 128)
    assert torch.isfinite(o).all() and torch.isfinite(S_T).all()
    assert q.grad is not None and q.grad.shape == q.shape and torch.isfinite(q.grad.float()).all()
