"""Shared helpers of the GPU parity tests: tolerances and comparisons."""
import numpy as np
import torch

# Bars for floating-point parity with the float64 oracle on bf16 inputs:
# max-abs error of the attention output and of the natural-log LSE.
OUT_TOL = 1e-2
LSE_TOL = 1e-3


# Bar of the backward: max-abs error of each gradient tensor at most GRAD_TOL
# times max(1, the largest |reference| element). The kernels multiply bf16
# operands (rotated q and k, P, dS, v, dout) with fp32 accumulation; each
# product carries a relative rounding error of at most 2^-8 from its two
# operands, so a gradient element that sums n such products of similar size
# is off by about 2^-8 sqrt(n) / n of the sum's scale and at worst by 2^-8 of
# the sum of magnitudes. 1e-2 is 2.5 x 2^-8: room for the worst case over a
# tensor's elements, still far below a structural error (a wrong sign, map or
# position moves elements by O(1) of the scale).
GRAD_TOL = 1e-2


def grad_error(got, ref):
    """(max-abs error, bar) of one gradient tensor."""
    err = max_abs(got, ref)
    ref = np.asarray(ref, dtype=np.float64)
    scale = max(1.0, float(np.abs(ref).max()) if ref.size else 0.0)
    return err, GRAD_TOL * scale


def decode_staged(D):
    """Whether the oracle decode should round its operands to bf16 for a
    comparison with the CUDA decode: at every head_dim (64, 128, 256) the
    decode multiplies bf16 operands on the tensor cores (the rotated query
    views and the corrected remote keys are rounded to bf16)."""
    return D in (64, 128, 256)


def deinterleave(x):
    """Adjacent storage order (element 2i = coordinate i, 2i+1 = coordinate
    i + D/2, as half-split key caches hold each rotated key) -> the heads'
    own order along the last axis."""
    return torch.cat([x[..., 0::2], x[..., 1::2]], dim=-1)


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
