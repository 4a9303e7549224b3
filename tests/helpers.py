"""Shared test helpers: moving synth bit patterns onto the GPU and the parity
tolerances. No attention arithmetic lives here.

Every comparison records its measured error next to its bound; the session's
terminal summary (conftest.py) prints them, smallest headroom first, so that a
drift towards a bound shows before a test fails."""
import numpy as np

# Tolerances for O and LSE: max-abs 1e-2 and mean-abs 1e-3 on O, 1e-3 on LSE
# (bf16 inputs, fp32 accumulation).
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3

# (what, quantity, measured, bound) for every comparison of the session
HEADROOM = []


def record(what, quantity, measured, bound):
    HEADROOM.append((str(what), quantity, float(measured), float(bound)))


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
    record(what, "O max-abs", err.max(), O_MAX_ABS)
    record(what, "O mean-abs", err.mean(), O_MEAN_ABS)
    assert err.max() <= O_MAX_ABS, f"{what}: O max-abs {err.max():.3e} > {O_MAX_ABS}"
    assert err.mean() <= O_MEAN_ABS, f"{what}: O mean-abs {err.mean():.3e} > {O_MEAN_ABS}"
    return float(err.max()), float(err.mean())


def assert_close_lse(got, ref, what=""):
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite LSE"
    record(what, "LSE max-abs", err.max(), LSE_MAX_ABS)
    assert err.max() <= LSE_MAX_ABS, f"{what}: LSE max-abs {err.max():.3e} > {LSE_MAX_ABS}"
    return float(err.max())


def assert_close_grad(got, ref, what=""):
    """Gradient tolerance: the O bar scaled to the tensor's magnitude,
    max-abs <= 1e-2 * max(1, max|ref|) and mean-abs <= 1e-3 * max(1, mean|ref|)."""
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), f"{what}: non-finite gradient"
    bmax = O_MAX_ABS * max(1.0, float(np.abs(ref).max()))
    bmean = O_MEAN_ABS * max(1.0, float(np.abs(ref).mean()))
    record(what, "max-abs", err.max(), bmax)
    record(what, "mean-abs", err.mean(), bmean)
    assert err.max() <= bmax, f"{what}: max-abs {err.max():.3e} > {bmax:.3e}"
    assert err.mean() <= bmean, f"{what}: mean-abs {err.mean():.3e} > {bmean:.3e}"
    return float(err.max()), float(err.mean())
