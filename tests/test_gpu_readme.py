"""The Python usage example in README.md runs as written on the GPU."""
from __future__ import annotations

import os
import re

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_python_example():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    text = open(os.path.join(ROOT, "README.md")).read()
    blocks = re.findall(r"```python\n(.*?)```", text, re.S)
    assert len(blocks) == 1
    exec(compile(blocks[0], "README.md", "exec"), {})
    torch.cuda.synchronize()
