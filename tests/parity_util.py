"""Shared helpers of the GPU parity tests (no arithmetic of the method)."""
import numpy as np
import torch

# Tolerances of the acceptance bar, per output element, relative to
# A[m,n] = sum_k |x[m,k] * w'[n,k]| (the oracle's tolerance scale).
TOL_FP32 = 1e-4      # fp32-accumulate paths (GEMV)
TOL_BF16 = 8e-3      # bf16 tensor-core path (prefill GEMM)


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    return t.cpu().numpy()


def assert_close(y_gpu: np.ndarray, y_ref: np.ndarray, A: np.ndarray, tol: float,
                 what: str = ""):
    y_gpu = y_gpu.astype(np.float64)
    err = np.abs(y_gpu - y_ref)
    bound = tol * A
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} outputs outside "
            f"{tol}*A; worst at {i}: gpu={y_gpu[i]!r} ref={y_ref[i]!r} "
            f"err={err[i]:.3e} bound={bound[i]:.3e}")


def group_for(group: int, K: int) -> int:
    return K if group in (0, K) else group
