"""Helpers shared by the GPU tests: move seeded inputs to the device and
compare results with the float64 oracle."""
import numpy as np
import torch

from test_sequence_layers_head_b200 import workloads as WL


def to_dev(raw: np.ndarray) -> torch.Tensor:
    """Storage-format numpy array (uint16 bf16 bits or float32) -> CUDA tensor."""
    if raw.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(raw).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(raw)).cuda()


def to_host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def normwise(x: np.ndarray, y: np.ndarray) -> float:
    return float(np.linalg.norm((x - y).ravel()) / max(np.linalg.norm(y.ravel()), 1e-300))


def maxrel(x: np.ndarray, y: np.ndarray) -> float:
    return float(np.max(np.abs(x - y)) / max(np.max(np.abs(y)), 1e-300))


def poison_like(t: torch.Tensor) -> torch.Tensor:
    """Output buffer pre-filled with NaN so unwritten elements fail parity."""
    return torch.full_like(t, float("nan"))


# Tolerances of the problem statement.
TOL_F32_MAXREL = 1e-4      # fp32 workloads: max relative error
TOL_BF16_NORMWISE = 2e-2   # bf16-input / fp32-state workloads: normwise, Z and final state


def assert_close(name, got, ref, io_dtype):
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    if got.size == 0:
        return 0.0
    if io_dtype == WL.F32:
        err = maxrel(got, ref)
        assert np.all(np.isfinite(got)), f"{name}: non-finite values"
        assert err <= TOL_F32_MAXREL, f"{name}: max relative error {err:.3e} > {TOL_F32_MAXREL}"
    else:
        err = normwise(got, ref)
        assert np.all(np.isfinite(got)), f"{name}: non-finite values"
        assert err <= TOL_BF16_NORMWISE, f"{name}: normwise error {err:.3e} > {TOL_BF16_NORMWISE}"
    return err
