"""The usage example (examples/quickstart.py, shown in the README) runs."""
import pytest

pytestmark = pytest.mark.gpu


def test_quickstart_example_runs():
    import torch

    import causal_linear_attention_fwd_b200 as la2
    from examples import quickstart

    out = quickstart.main()
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    for name in ("o", "dq", "dk", "dv", "dlam", "o1", "oT", "op"):
        assert bool(torch.isfinite(out[name].float()).all()), name
