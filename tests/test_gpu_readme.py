"""The usage example in README.md runs as written."""
import os
import re

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_example_runs():
    import torch
    with open(os.path.join(ROOT, "README.md")) as f:
        code = re.findall(r"```python\n(.*?)```", f.read(), re.S)[0]
    scope = {}
    exec(compile(code, "README.md", "exec"), scope)
    torch.cuda.synchronize()
    la2 = scope["la2"]
    assert la2.last_device_error() == 0
    for name in ("o", "dq", "dk", "dv", "dlam", "o1", "oT", "op"):
        assert bool(torch.isfinite(scope[name].float()).all()), name
