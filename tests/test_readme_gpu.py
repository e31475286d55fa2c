"""The README's decode-step example runs as written (needs a B200)."""

import os
import re

import pytest
import torch

from tests.conftest import ROOT

pytestmark = pytest.mark.gpu


def test_readme_example_runs(cuda_device):
    with open(os.path.join(ROOT, "README.md")) as f:
        code = re.search(r"```python\n(.*?)```", f.read(), re.S).group(1)
    scope = {}
    exec(compile(code, "README.md", "exec"), scope)
    torch.cuda.synchronize()
    out = scope["out"]
    assert out.shape == (3, 1, 32, 128) and torch.isfinite(out.float()).all()
