"""Helpers for the GPU parity tests: move inputs, widen results, measure errors.

Every comparison made through rel_inf is also recorded (test id, tensor, the gating
infinity-norm relative error and the floored element-wise relative error), and the session
writes the records to the JSON file named by the WKV_PARITY_RECORD environment variable
(tests/conftest.py); tests/parity_report.py turns that file into a summary table.
"""
import os

import numpy as np
import torch

# Tolerances on the infinity-norm relative error ||got - ref||_inf / ||ref||_inf, per
# output tensor: fp32 inputs 1e-4; bf16 inputs with fp32 accumulation 2e-2.
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}

RECORDS = []


def dev(t):
    return None if t is None else t.contiguous().cuda()


def f64(t):
    """Exact widening of a CPU/GPU fp32 or bf16 tensor to a float64 numpy array."""
    return None if t is None else t.detach().to("cpu", torch.float32).double().numpy()


def floored_rel(got, ref):
    """max |got - ref| / max(|ref|, 1e-3 rms(ref)): the element-wise relative error with a
    floor, so that outputs near zero do not make it unbounded (reported, never gating)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    if ref.size == 0:
        return 0.0
    floor = max(1e-3 * float(np.sqrt(np.mean(ref * ref))), 1e-300)
    return float(np.max(np.abs(got - ref) / np.maximum(np.abs(ref), floor)))


def rel_inf(got, ref, what=None):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the GPU result"
    den = max(float(np.max(np.abs(ref))), 1e-300) if ref.size else 1.0
    e = float(np.max(np.abs(got - ref)) / den) if ref.size else 0.0
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    RECORDS.append({"test": test, "what": what, "shape": list(ref.shape), "inf_rel": e,
                    "elem_rel_floored": floored_rel(got, ref)})
    return e


def wkv4_state_views(s):
    """(a, b, p) -> (a/b, log(b) + p): a representation-independent view of a non-empty state."""
    s = np.asarray(s, np.float64)
    a, b, p = s[:, 0], s[:, 1], s[:, 2]
    return a / b, np.log(b) + p
