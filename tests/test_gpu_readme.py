"""The usage example README.md quotes (examples/readme_example.py) runs as written on
the GPU, and README.md quotes it unchanged."""
from __future__ import annotations

import os
import runpy

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
EXAMPLE = os.path.join(ROOT, "examples", "readme_example.py")


def _example_code() -> str:
    """The example's statements: the file without its docstring."""
    text = open(EXAMPLE).read()
    return text.split('"""', 2)[2].lstrip("\n")


def test_readme_quotes_the_example():
    readme = open(os.path.join(ROOT, "README.md")).read()
    assert _example_code() in readme, "README.md's Python block differs from examples/readme_example.py"


@pytest.mark.gpu
def test_readme_example_runs():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    runpy.run_path(EXAMPLE, run_name="__main__")
    torch.cuda.synchronize()
