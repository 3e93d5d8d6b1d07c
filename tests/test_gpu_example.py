"""The one-GPU usage example (zero_partitioned_mixed_reduce_b200/example.py,
which the README quotes) runs as written and does what it says."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_one_gpu_example_runs():
    from zero_partitioned_mixed_reduce_b200.example import one_gpu_step
    plan, state, ls, out = one_gpu_step()
    assert ls["t"] == 1 and ls["last_skipped"] == 0 and ls["cur"] == 1
    lo, hi = plan.layers[1]
    assert torch.equal(out.view(torch.int16), torch.cat(state.param[1])[lo:hi].view(torch.int16))
