"""Helpers shared by the GPU parity tests."""
import numpy as np
import torch

# Float-format bar: relative L2 over all compared outputs, and a per-element
# bound relative to sum_k |w x| (the scale of the rounding any fp32 order of
# summation may add).
REL_L2 = 1e-5
ELEM = 2e-3


def dev(a: np.ndarray, device="cuda"):
    """numpy -> torch on the GPU, bit patterns preserved (uint16 -> int16)."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).to(device)


def host(t) -> np.ndarray:
    return t.detach().cpu().numpy()


def check_float(y_gpu: np.ndarray, y64: np.ndarray, absdot: np.ndarray, what: str):
    y_gpu = np.asarray(y_gpu, np.float64).ravel()
    y64 = np.asarray(y64, np.float64).ravel()
    absdot = np.asarray(absdot, np.float64).ravel()
    assert np.isfinite(y_gpu).all(), f"{what}: non-finite output"
    diff = np.abs(y_gpu - y64)
    nrm = np.linalg.norm(y64)
    rel = np.linalg.norm(y_gpu - y64) / nrm if nrm > 0 else np.linalg.norm(y_gpu)
    assert rel <= REL_L2, f"{what}: relative L2 {rel:.3e} > {REL_L2}"
    bad = diff > ELEM * absdot
    assert not bad.any(), (f"{what}: {bad.sum()} elements exceed {ELEM}*sum|wx| "
                           f"(worst {diff[bad].max():.3e})")
    return rel


def sample_pairs(M, N, count, seed):
    g = np.random.default_rng(seed)
    ms = g.integers(0, M, size=count)
    ns = g.integers(0, N, size=count)
    # always include the corners (first / last row and batch entry)
    ms[:4] = [0, M - 1, 0, M - 1]
    ns[:4] = [0, N - 1, N - 1, 0]
    return ms.astype(np.int64), ns.astype(np.int64)
