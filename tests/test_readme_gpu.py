"""The README's decode-step example runs as written (needs a B200)."""

import os
import re

import pytest
import torch

from tests.conftest import ROOT

pytestmark = pytest.mark.gpu


def test_readme_examples_run(cuda_device):
    with open(os.path.join(ROOT, "README.md")) as f:
        blocks = re.findall(r"```python\n(.*?)```", f.read(), re.S)
    assert len(blocks) == 2
    scope = {}
    for i, code in enumerate(blocks):              # the second continues the first
        exec(compile(code, f"README.md block {i + 1}", "exec"), scope)
    torch.cuda.synchronize()
    out, out4 = scope["out"], scope["out4"]
    assert out.shape == (3, 1, 32, 128) and torch.isfinite(out.float()).all()
    assert out4.shape == (4, 32, 128) and torch.isfinite(out4.float()).all()
