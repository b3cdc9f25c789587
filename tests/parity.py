"""Comparison helpers shared by the GPU parity tests.

Tolerances (written here once, used by every test):
* bf16 / f16 outputs: elementwise |gpu - ref| <= 2e-3 + 1e-2 * |ref|
  (max abs error 2e-3, max relative error 1e-2, in allclose form);
* fp32 outputs: |gpu - ref| <= 1e-5.
The reference is the fp64 oracle evaluated on the same stored inputs.
"""
import numpy as np

BF16_ATOL = 2e-3
BF16_RTOL = 1e-2
F32_ATOL = 1e-5


def to_numpy_f64(t):
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def assert_decode_close(gpu, ref, dtype: str, what: str = ""):
    """gpu: torch tensor (any float dtype); ref: fp64 numpy array of the same shape."""
    g = to_numpy_f64(gpu) if not isinstance(gpu, np.ndarray) else gpu.astype(np.float64)
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    err = np.abs(g - ref)
    if dtype == "f32":
        bad = err > F32_ATOL
        assert not bad.any(), f"{what}: max abs err {err.max():.3g} > {F32_ATOL}"
    else:
        bound = BF16_ATOL + BF16_RTOL * np.abs(ref)
        bad = err > bound
        assert not bad.any(), (f"{what}: {bad.sum()} elements out of tolerance; max abs err {err.max():.3g}, "
                               f"worst at {np.unravel_index(np.argmax(err - bound), err.shape)}")
    big = np.abs(ref) >= BF16_ATOL / BF16_RTOL
    return {"max_abs": float(err.max()) if err.size else 0.0,
            "max_rel": float((err[big] / np.abs(ref[big])).max()) if big.any() else 0.0}


def bits_of(t):
    """Raw bit pattern of a device tensor as a numpy array (for bit-exact checks)."""
    import torch
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.view(torch.int32).cpu().numpy().view(np.uint32)
    return t.cpu().numpy()


def host_bits(a):
    a = np.asarray(a)
    if a.dtype == np.float32:
        return a.view(np.uint32)
    return a
