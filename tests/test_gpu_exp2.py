"""The softmax of the shared-prefix kernel computes half of its weights 2^x on the FMA pipe (a
fitted cubic after range reduction, see device.cuh).  Checked here against CUDA's own exp2f
(torch.exp2 on the device) within the fit's error bound over the whole range the kernel feeds it,
and for the special-function-unit form the other half uses."""
import numpy as np
import pytest

from paged_kv_cache_356_b200 import binding as pa

pytestmark = pytest.mark.gpu


def _inputs():
    import torch
    rng = np.random.default_rng(11)
    x = np.concatenate([rng.uniform(-125.0, 127.0, 1 << 20), rng.uniform(-8.0, 8.0, 1 << 20),
                        np.arange(-125, 128, dtype=np.float64),                   # integers: f = 0
                        np.arange(-125, 127, dtype=np.float64) + 0.5,             # halfway: f = +-1/2
                        [0.0, -0.0, 1e-7, -1e-7, 0.49999997, -0.49999997]]).astype(np.float32)
    return torch.from_numpy(x).cuda()


def test_fma_pipe_exp2_within_its_error_bound():
    import torch
    x = _inputs()
    got = pa.pa_eval_exp2(x, 0).double()
    ref = torch.exp2(x).double()          # CUDA's exp2f, correctly rounded to within 2 ulp
    rel = ((got - ref).abs() / ref).max().item()
    assert rel < 1e-4, rel                # the cubic's 7.6e-5 plus fp32 rounding of its evaluation
    assert torch.all(got > 0)


def test_fma_pipe_exp2_clamps_below_its_range():
    import torch
    x = torch.tensor([-126.0, -200.0, -1e30, float("-inf")], device="cuda")
    got = pa.pa_eval_exp2(x, 0)
    assert torch.all(got <= 2.0 ** -124) and torch.all(got >= 0)   # tiny: rounds to 0 as a 16-bit weight


def test_special_function_unit_exp2():
    import torch
    x = _inputs()
    x = x[x > -126]                       # the instruction flushes subnormal results to zero
    got = pa.pa_eval_exp2(x, 1).double()
    ref = torch.exp2(x).double()
    assert ((got - ref).abs() / ref).max().item() < 1e-6
    assert pa.pa_eval_exp2(torch.tensor([float("-inf")], device="cuda"), 1).item() == 0.0


def test_eval_exp2_rejects_bad_method():
    import torch
    with pytest.raises(pa.PagedAttentionError):
        pa.pa_eval_exp2(torch.zeros(4, device="cuda"), 2)
