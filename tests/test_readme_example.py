"""The Python example in README.md runs as written on the GPU."""
import os
import re

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_python_example_runs():
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```python\n(.*?)```", text, flags=re.S)
    assert blocks, "no python example in the README"
    env = {}
    exec(compile(blocks[0], "README.md", "exec"), env)   # noqa: S102 - our own documentation
    import torch
    o, lse = env["o"], env["lse"]
    assert o.shape == (4096, 16, 128) and lse.shape == (16, 4096)
    assert torch.isfinite(o.float()).all()
