"""Shared test helpers: moving synth bit patterns onto the GPU and the parity
tolerances. No attention arithmetic lives here."""
import numpy as np

# Tolerances for O and LSE: max-abs 1e-2 and mean-abs 1e-3 on O, 1e-3 on LSE
# (bf16 inputs, fp32 accumulation).
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3


def to_dev(bits, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def from_dev(t):
    """bf16 CUDA tensor -> float64 numpy."""
    import torch
    return t.detach().to(torch.float32).cpu().numpy().astype(np.float64)


def assert_close_o(got, ref, what=""):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err.max() <= O_MAX_ABS, f"{what}: O max-abs {err.max():.3e} > {O_MAX_ABS}"
    assert err.mean() <= O_MEAN_ABS, f"{what}: O mean-abs {err.mean():.3e} > {O_MEAN_ABS}"
    return float(err.max()), float(err.mean())


def assert_close_lse(got, ref, what=""):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite LSE"
    assert err.max() <= LSE_MAX_ABS, f"{what}: LSE max-abs {err.max():.3e} > {LSE_MAX_ABS}"
    return float(err.max())
