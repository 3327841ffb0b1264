"""The attention kernel's FMA-pipe exponential against 2^x.

The kernel evaluates part of its exponentials without the MUFU unit: t = n + f
with n = round(t), 2^f by a Remez cubic on [-1/2, 1/2] (7.5e-5 maximum
relative error, free_clustered_block_b200/csrc/exp2_poly_fit.py) and n added
into the exponent. ca_check_exp2_poly runs that same device function; this
test sweeps it densely and compares with fp64 2^x and with the GPU's exp2f.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu

# the cubic's levelled error plus a few fp32 roundings of its evaluation
REL_BOUND = 8e-5


def _run(x):
    import torch
    import free_clustered_block_b200 as ca
    xd = torch.from_numpy(x.astype(np.float32)).cuda()
    yd = torch.empty_like(xd)
    ca.ca_check_exp2_poly(xd, yd)
    ref32 = torch.exp2(xd)
    torch.cuda.synchronize()
    assert ca.ca_get_device_error() == ca.CA_OK
    return yd.cpu().numpy().astype(np.float64), ref32.cpu().numpy().astype(np.float64)


def test_relative_error_over_the_normal_range():
    # every range the softmax produces: t = s - m <= 8, down to the bf16 floor
    x = np.concatenate([np.linspace(-125.0, 8.0, 4_000_001),
                        np.linspace(-0.5, 0.5, 1_000_001),          # the reduced interval itself
                        np.arange(-125, 9, dtype=np.float64)])      # the integers (f = 0)
    x = x.astype(np.float32).astype(np.float64)
    y, y32 = _run(x)
    exact = np.exp2(x)
    rel = np.abs(y / exact - 1.0)
    assert rel.max() <= REL_BOUND, f"max relative error {rel.max():.3g} at x = {x[rel.argmax()]}"
    # and against the GPU's own exp2f, which is far more accurate than the cubic
    rel32 = np.abs(y / y32 - 1.0)
    assert rel32.max() <= REL_BOUND + 1e-6


def test_underflow_and_masked_inputs_give_negligible_values():
    x = np.array([-125.5, -126.0, -130.0, -1e4, -np.inf], dtype=np.float32).astype(np.float64)
    y, _ = _run(x)
    assert np.all(np.isfinite(y))
    assert np.all(y >= 0.0)
    assert np.all(y <= 2.0 ** -124)


def test_odd_length_and_empty():
    x = np.linspace(-3.0, 3.0, 7)
    y, _ = _run(x)
    assert np.abs(y / np.exp2(x.astype(np.float32).astype(np.float64)) - 1).max() <= REL_BOUND
    import torch
    import free_clustered_block_b200 as ca
    e = torch.empty(0, device="cuda")
    ca.ca_check_exp2_poly(e, e)   # n = 0: nothing to do
