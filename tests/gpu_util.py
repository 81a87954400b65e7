"""Helpers for the GPU parity tests: move inputs, widen results, measure errors."""
import numpy as np
import torch

# Tolerances on the infinity-norm relative error ||got - ref||_inf / ||ref||_inf, per
# output tensor: fp32 inputs 1e-4; bf16 inputs with fp32 accumulation 2e-2.
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def dev(t):
    return None if t is None else t.contiguous().cuda()


def f64(t):
    """Exact widening of a CPU/GPU fp32 or bf16 tensor to a float64 numpy array."""
    return None if t is None else t.detach().to("cpu", torch.float32).double().numpy()


def rel_inf(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU result"
    den = max(float(np.max(np.abs(ref))), 1e-300)
    return float(np.max(np.abs(got - ref)) / den)


def wkv4_state_views(s):
    """(a, b, p) -> (a/b, log(b) + p): a representation-independent view of a non-empty state."""
    s = np.asarray(s, np.float64)
    a, b, p = s[:, 0], s[:, 1], s[:, 2]
    return a / b, np.log(b) + p
