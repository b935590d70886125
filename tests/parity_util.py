"""Shared helpers of the GPU parity tests: tolerances and comparisons."""
import numpy as np

# Bars for floating-point parity with the float64 oracle on bf16 inputs:
# max-abs error of the attention output and of the natural-log LSE.
OUT_TOL = 1e-2
LSE_TOL = 1e-3


def decode_staged(D):
    """Whether the oracle decode should round its operands to bf16 for a
    comparison with the CUDA decode: for head_dim 64 and 128 the decode
    multiplies bf16 operands on the tensor cores (the rotated query views and
    the corrected remote keys are rounded to bf16); at head_dim 256 it keeps
    its rotations and dot products in fp32 registers."""
    return D <= 128


def max_abs(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (a.shape, b.shape)
    assert np.isfinite(a).all(), "non-finite values in the CUDA result"
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def assert_close(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    eo = max_abs(out_gpu, out_ref)
    el = max_abs(lse_gpu, lse_ref)
    assert eo <= OUT_TOL and el <= LSE_TOL, f"{what}: out max-abs {eo:.3e} (<= {OUT_TOL}), lse max-abs {el:.3e} (<= {LSE_TOL})"
    return eo, el
