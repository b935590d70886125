"""Backward parity at the size and in the launch configuration the benchmark
times: the 131072-token bifocal prefill backward (32/8 heads, D 128, w0 2048,
G = 4 from the 32768-token pretrained window), against the float64 oracle on
what it can compute at that length:

- dq on sampled query rows (the first and last rows, rows around w0 and
  every multiple of the pretrained window, seeded random rows) for the query
  heads of the first and the last kv head;
- dq, dk and dv on the last 128 positions for the last kv head's group:
  attention is causal, so those keys receive gradient only from the rows
  after them and the oracle's sums over the tail rows are complete.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity_util import GRAD_TOL, grad_error
from position_remapping_b200.inputs import WORKLOADS, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

P = WORKLOADS["bifocal_prefill_s131072"]
TAIL = 128


def _per_vector(name, got, ref):
    """Each (position, head) vector of D elements against GRAD_TOL times its
    own largest |reference| element. At this length a late row's softmax is
    spread over ~10^5 keys and its gradients are small, so a bar scaled by
    the largest element of the whole tensor would let a structural error in
    those rows through; the floor (10^-3 of the largest vector) keeps vectors
    that are exactly zero in the reference (row 0's dq: one key, dS = 0)
    from demanding an exact zero."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref).max(axis=-1)
    scale = np.abs(ref).max(axis=-1)
    bar = GRAD_TOL * np.maximum(scale, 1e-3 * scale.max())
    worst = np.unravel_index(np.argmax(err / bar), err.shape)
    assert (err <= bar).all(), f"{name}: at {worst} max-abs {err[worst]:.3e} > {bar[worst]:.3e}"
    e, b = grad_error(got, ref)
    assert e <= b, f"{name}: max-abs {e:.3e} > {b:.3e}"
    print(f"{name}: worst error / bar {float((err / bar)[worst]):.3f}")


def test_backward_bifocal_s131072():
    from position_remapping_b200 import ropeattn as ra
    q, k, v = make_qkv(P.B, P.S, P.Hq, P.Hkv, P.D, P.seed)
    g = torch.Generator("cpu").manual_seed(P.seed + 1)
    dout = torch.randn((P.B, P.S, P.Hq, P.D), generator=g).to(torch.bfloat16)
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, lse = ra.prefill(qd, kd, vd, P.params)
    dq, dk, dv = ra.prefill_backward(qd, kd, vd, out, lse, gd, P.params)
    torch.cuda.synchronize()
    ra.status()
    del qd, kd, vd, gd, out, lse

    grp = P.Hq // P.Hkv
    rows = sample_rows(P.S, P.params, n_random=16, edge=8)
    ridx = torch.tensor(rows, device=dq.device)
    for hk in (0, P.Hkv - 1):
        heads = list(range(hk * grp, (hk + 1) * grp))
        got = dq[:, ridx][:, :, heads].cpu().numpy()
        ref = O.prefill_backward_dq_rows(q, k, v, dout, P.params, rows, stage_bf16=True, heads=heads)
        _per_vector(f"dq rows, kv head {hk}", got, ref)

    hk = P.Hkv - 1
    heads = list(range(hk * grp, (hk + 1) * grp))
    tq, tk, tv = O.prefill_backward_tail(q, k, v, dout, P.params, TAIL, stage_bf16=True, heads=heads)
    tail = slice(P.S - TAIL, P.S)
    _per_vector("dq tail", dq[:, tail][:, :, heads].cpu().numpy(), tq)
    _per_vector("dk tail", dk[:, tail, hk:hk + 1].cpu().numpy(), tk)
    _per_vector("dv tail", dv[:, tail, hk:hk + 1].cpu().numpy(), tv)
