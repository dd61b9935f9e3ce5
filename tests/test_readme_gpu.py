"""The README's Python example runs as written and returns the shapes it states."""
import os
import re

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_example_runs():
    import torch
    text = open(os.path.join(ROOT, "README.md")).read()
    block = re.findall(r"```python\n(.*?)```", text, re.S)[0]
    env = {}
    exec(compile(block, "README.md", "exec"), env)
    torch.cuda.synchronize()
    assert tuple(env["q4"].shape) == (1, 8192, 3584) and env["q4"].dtype == torch.uint8
    assert tuple(env["q"].shape) == (32, 2048, 2048)
    assert tuple(env["s"].shape) == (32, 16, 2048)
