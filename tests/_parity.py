"""Comparison helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch

# Attention tolerances for bf16 inputs with fp32 accumulation against the float64
# oracle: O max-abs 2e-2 and mean-abs 2e-3, LSE max-abs 1e-3.
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_attention_close(o_gpu: np.ndarray, lse_gpu: np.ndarray, o_ref: np.ndarray,
                           lse_ref: np.ndarray, what: str = ""):
    """o_*: [..., D] rows; lse_*: matching rows.  -inf LSE must match exactly."""
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    inf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), inf_ref), f"{what}: -inf LSE rows differ"
    assert np.all(o_gpu[inf_ref] == 0), f"{what}: rows without kept keys must be zero"
    d = np.abs(o_gpu - o_ref)
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    mx, mean = float(d.max()) if d.size else 0.0, float(d.mean()) if d.size else 0.0
    assert mx <= O_MAX_ABS, f"{what}: O max-abs {mx:.3e} > {O_MAX_ABS}"
    assert mean <= O_MEAN_ABS, f"{what}: O mean-abs {mean:.3e} > {O_MEAN_ABS}"
    fin = ~inf_ref
    if fin.any():
        le = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max())
        assert le <= LSE_MAX_ABS, f"{what}: LSE max-abs {le:.3e} > {LSE_MAX_ABS}"
    return mx, mean
