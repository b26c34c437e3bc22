"""Shared helpers for the GPU parity tests: tolerances and comparisons against the oracle."""
import numpy as np
import torch

# Tolerances of the attention parity contract (bf16 inputs, fp32 accumulation):
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_MAX_ABS = 1e-3
GRAD_MAX_ABS = 5e-2
GRAD_REL_L2 = 1e-2


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def check_o(o_gpu: np.ndarray, o_ref: np.ndarray, what: str = "O"):
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite values"
    err = np.abs(o_gpu - o_ref)
    assert err.max() <= O_MAX_ABS, f"{what}: max-abs {err.max():.3e} > {O_MAX_ABS}"
    assert err.mean() <= O_MEAN_ABS, f"{what}: mean-abs {err.mean():.3e} > {O_MEAN_ABS}"
    return err.max(), err.mean()


def check_lse(l_gpu: np.ndarray, l_ref: np.ndarray):
    fin = np.isfinite(l_ref)
    assert (np.isfinite(l_gpu) == fin).all(), "LSE: finiteness differs"
    err = np.abs(l_gpu[fin] - l_ref[fin])
    if err.size:
        assert err.max() <= LSE_MAX_ABS, f"LSE: max-abs {err.max():.3e} > {LSE_MAX_ABS}"
    return err.max() if err.size else 0.0


def check_grad(g_gpu: np.ndarray, g_ref: np.ndarray, what: str):
    assert np.isfinite(g_gpu).all(), f"{what}: non-finite values"
    err = np.abs(g_gpu - g_ref)
    rel = np.linalg.norm(g_gpu - g_ref) / max(np.linalg.norm(g_ref), 1e-30)
    assert err.max() <= GRAD_MAX_ABS, f"{what}: max-abs {err.max():.3e} > {GRAD_MAX_ABS}"
    assert rel <= GRAD_REL_L2, f"{what}: rel-L2 {rel:.3e} > {GRAD_REL_L2}"
    return err.max(), rel
