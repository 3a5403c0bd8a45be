"""Shared test utilities: tolerances, error norms, device checks."""
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# Floating-point bar: relative L2 error against the fp64 oracle.
TOL_BF16 = 5e-3   # bf16 inputs / activations, fp32 state and accumulation
TOL_F32 = 1e-5    # fp32 inputs / activations


def rel_l2(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want.ravel())
    return float(np.linalg.norm((got - want).ravel()) / (den if den > 0 else 1.0))


def bf16_steps(a, b):
    """Largest distance between two arrays of bf16 values, in bf16 steps (the
    spacing of bf16 numbers at the larger magnitude of each pair).  Two runs of
    the scan whose chunk carries were folded in a different order round their
    fp32 states differently in the last bits, so bf16 outputs may sit one step
    apart."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    m = np.maximum(np.abs(a), np.abs(b))
    step = 2.0 ** (np.floor(np.log2(np.where(m > 0, m, 1.0))) - 7)
    return float((np.abs(a - b) / step).max()) if a.size else 0.0


def to_np(t):
    return t.detach().to("cpu").double().numpy()


def cuda_or_skip():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    return torch.device("cuda:0")


def header_symbols():
    """Function names declared in include/jamba.h."""
    with open(os.path.join(ROOT, "include", "jamba.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|jamba_status)\s+(jamba_\w+)\s*\(", text, re.M)))
