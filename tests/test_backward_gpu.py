"""Backward parity: dq, dk, dv of the two tensor-core backward kernels
(through the C ABI) against the float64 oracle's chain rule on the same
seeded bf16 inputs, for every kind."""
import zlib

import numpy as np
import pytest
import torch

import oracle as O
from parity_util import GRAD_TOL, grad_error
from position_remapping_b200.inputs import PAIR_HALF, MapParams, make_qkv

pytestmark = pytest.mark.gpu

CASES = [
    # (id, B, S, Hq, Hkv, D, params)
    ("standard", 1, 200, 2, 1, 128, MapParams(O.STANDARD, rope_base=1e4)),
    ("standard_d64_gqa2_ragged", 1, 333, 4, 2, 64, MapParams(O.STANDARD, rope_base=1e4)),
    ("endprompt", 1, 300, 2, 2, 128, MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=250,
                                                term_start=65000)),
    ("periodic_w100_d64", 1, 400, 2, 1, 64, MapParams(O.PERIODIC, rope_base=1e4, window=100)),
    ("nope", 1, 257, 2, 1, 128, MapParams(O.NOPE)),
    ("bifocal_g3", 1, 700, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=96, w_pretrained=256)),
    ("bifocal_w0_127_key_tile_edge", 1, 600, 2, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=127,
                                                                  w_pretrained=200)),
    ("bifocal_w0_63_query_tile_edge", 1, 513, 2, 2, 128, MapParams(O.BIFOCAL, rope_base=1e4, w0=63,
                                                                   w_pretrained=128)),
    ("bifocal_d64_gqa4", 1, 450, 8, 2, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=40, w_pretrained=100)),
    ("bifocal_half_split", 1, 380, 2, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=50, w_pretrained=128,
                                                        pairing=PAIR_HALF)),
    ("bifocal_fixed_g5", 1, 300, 2, 1, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=30, fixed_group=5)),
    ("bifocal_w0_0", 1, 260, 2, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=0, w_pretrained=100)),
    ("bifocal_inside_window", 1, 200, 2, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=30, w_pretrained=256)),
    ("batch2_periodic_half", 2, 190, 2, 1, 128, MapParams(O.PERIODIC, rope_base=1e4, window=64, pairing=PAIR_HALF)),
    ("one_token", 1, 1, 2, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=0, w_pretrained=1)),
]


def _dout(B, S, Hq, D, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn((B, S, Hq, D), generator=g, dtype=torch.float32).to(torch.bfloat16)


def _run(q, k, v, dout, params):
    from position_remapping_b200 import ropeattn as ra
    qd, kd, vd, gd = q.cuda(), k.cuda(), v.cuda(), dout.cuda()
    out, lse = ra.prefill(qd, kd, vd, params)
    dq, dk, dv = ra.prefill_backward(qd, kd, vd, out, lse, gd, params)
    torch.cuda.synchronize()
    ra.status()
    return dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy()


def _check(name, got, ref):
    for what, g, r in zip(("dq", "dk", "dv"), got, ref):
        err, bar = grad_error(g, r)
        assert err <= bar, f"{name} {what}: max-abs {err:.3e} > {bar:.3e} (GRAD_TOL x max(1, max|ref|))"


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_small(case):
    name, B, S, Hq, Hkv, D, params = case
    seed = zlib.crc32(("bwd-" + name).encode()) % 10000
    q, k, v = make_qkv(B, S, Hq, Hkv, D, seed=seed)
    dout = _dout(B, S, Hq, D, seed + 1)
    got = _run(q, k, v, dout, params)
    ref = O.prefill_backward(q, k, v, dout, params, stage_bf16=True)
    _check(name, got, ref)


def test_backward_several_tiles_bifocal_g4():
    # 16 key tiles and 32 query tiles of 64 rows, both bifocal passes
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=200, w_pretrained=512)
    q, k, v = make_qkv(1, 2048, 4, 2, 128, seed=61)
    dout = _dout(1, 2048, 4, 128, 62)
    got = _run(q, k, v, dout, params)
    ref = O.prefill_backward(q, k, v, dout, params, stage_bf16=True)
    _check("bifocal_s2048_g4", got, ref)


def test_backward_deterministic():
    from position_remapping_b200 import ropeattn as ra
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=96, w_pretrained=256)
    q, k, v = (t.cuda() for t in make_qkv(1, 1000, 4, 2, 128, seed=63))
    dout = _dout(1, 1000, 4, 128, 64).cuda()
    out, lse = ra.prefill(q, k, v, params)
    a = [t.clone() for t in ra.prefill_backward(q, k, v, out, lse, dout, params)]
    b = ra.prefill_backward(q, k, v, out, lse, dout, params)
    torch.cuda.synchronize()
    ra.status()
    assert all(torch.equal(x, y) for x, y in zip(a, b))


def test_backward_rejects_head_dim_256():
    from position_remapping_b200 import ropeattn as ra
    q, k, v = (t.cuda() for t in make_qkv(1, 64, 2, 1, 256, seed=65))
    out = torch.zeros((1, 64, 2, 256), dtype=torch.float32, device="cuda")
    lse = torch.zeros((1, 2, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(ra.RopeAttnError) as e:
        ra.prefill_backward(q, k, v, out, lse, q.clone(), MapParams(O.STANDARD),
                            workspace=torch.empty(1 << 20, dtype=torch.uint8, device="cuda"))
    assert e.value.code == ra.ERR_INVALID_ARG
