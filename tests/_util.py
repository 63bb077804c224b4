"""Shared helpers of the test suite: device transfer of generator arrays and tolerance checks."""
import numpy as np

# Tolerances (|got - ref| <= atol + rtol * |ref|, element by element):
#   fp32 I/O outputs:  rtol 1e-5, atol 1e-6
#   bf16 outputs:      rtol 1.6e-2, atol 1e-2
#   gradients (bf16):  rtol 2e-2, atol 2e-2
#   saved inv_rms / mean / rstd (fp32 from either I/O type): rtol 1e-5
TOL = {
    "f32": (1e-5, 1e-6),
    "bf16": (1.6e-2, 1e-2),
    "grad_bf16": (2e-2, 2e-2),
    "stat": (1e-5, 0.0),
}


def to_dev(a, device="cuda"):
    """numpy array from the generator (uint16 = bf16 bits, float32) -> torch tensor on device."""
    import torch

    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def to_np(t):
    """torch tensor -> float64 numpy (bf16 widened exactly)."""
    import torch

    return t.detach().to("cpu", torch.float64).numpy()


def assert_close(got, ref, tol, what=""):
    rtol, atol = TOL[tol] if isinstance(tol, str) else tol
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} vs {ref.shape}"
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance "
                             f"(rtol={rtol}, atol={atol}); worst at {i}: got {got[i]!r} ref {ref[i]!r}")


def io_tol(dtype):
    return "f32" if dtype == "f32" else "bf16"


def grad_tol(dtype):
    return "f32" if dtype == "f32" else "grad_bf16"


def wgrad_tol(dtype, ref):
    """Weight gradients are sums over every row. For fp32 I/O the element-wise bound of the
    outputs cannot hold for sums whose terms cancel, so they are checked normwise: rtol 1e-5
    plus an absolute term of 1e-5 times the largest |element| of the reference gradient. bf16
    gradients use the gradient tolerance (2e-2 relative + 2e-2 absolute)."""
    if dtype == "bf16":
        return "grad_bf16"
    return (1e-5, 1e-5 * float(np.max(np.abs(ref))))
