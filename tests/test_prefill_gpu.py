"""Prefill parity: the CUDA path (through the C ABI) against the float64
oracle on the same seeded bf16 inputs, element by element.

Small cases run every row (several 128-row tiles, ragged tails, GQA, both
head dims, every kind and its edge cases); the full-size workloads are checked
on sampled rows (each output row is independent, so a sampled row is an exact
check) in the launch configuration the benchmark times."""
import numpy as np
import zlib

import pytest
import torch

import oracle as O
from parity_util import assert_close
from position_remapping_b200.inputs import WORKLOADS, MapParams, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

SMALL = [
    # (id, B, S, Hq, Hkv, D, params)
    ("bifocal_fixed_g5", 1, 1000, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, fixed_group=5)),
    ("bifocal_fixed_g2_d64", 2, 700, 2, 1, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=30, fixed_group=2)),
    ("standard_s512_d64", 1, 512, 1, 1, 64, MapParams(O.STANDARD, rope_base=1e4)),
    ("standard_ragged_gqa", 2, 300, 4, 2, 128, MapParams(O.STANDARD, rope_base=1e4)),
    ("standard_s1", 1, 1, 2, 1, 64, MapParams(O.STANDARD)),
    ("standard_s129", 1, 129, 2, 1, 128, MapParams(O.STANDARD, rope_base=5e5)),
    ("standard_scale", 1, 200, 2, 2, 64, MapParams(O.STANDARD, softmax_scale=0.3)),
    ("endprompt", 1, 700, 4, 1, 128, MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=500, term_start=65000)),
    ("endprompt_n1_0", 1, 260, 2, 1, 64, MapParams(O.ENDPROMPT, rope_base=1e4, interp=2.0, seg1_len=0, term_start=9000)),
    ("periodic_w100", 1, 900, 2, 2, 64, MapParams(O.PERIODIC, window=100)),
    ("periodic_w128", 2, 520, 2, 1, 128, MapParams(O.PERIODIC, window=128)),
    ("periodic_w1", 1, 300, 2, 2, 64, MapParams(O.PERIODIC, window=1)),
    ("periodic_w300", 1, 1000, 4, 4, 64, MapParams(O.PERIODIC, window=300)),
    ("periodic_w_ge_s", 1, 200, 2, 2, 64, MapParams(O.PERIODIC, window=4096)),
    ("nope", 2, 400, 2, 1, 64, MapParams(O.NOPE)),
    ("nope_d128", 1, 333, 4, 1, 128, MapParams(O.NOPE)),
    ("bifocal_g4", 1, 1000, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=256)),
    ("bifocal_w0_0", 1, 600, 2, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=0, w_pretrained=160)),
    ("bifocal_w0_300", 2, 1100, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e4, w0=300, w_pretrained=300)),
    ("bifocal_g3_d64", 1, 700, 2, 2, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=64, w_pretrained=300)),
    ("bifocal_w0_127", 1, 640, 2, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=127, w_pretrained=100)),
    # head_dim 256: one 128-row query tile per CTA, 64-key tiles
    ("standard_d256_ragged", 1, 300, 2, 1, 256, MapParams(O.STANDARD, rope_base=1e4)),
    ("endprompt_d256", 1, 400, 2, 1, 256, MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=300,
                                                     term_start=65000)),
    ("periodic_d256_w100", 1, 500, 2, 2, 256, MapParams(O.PERIODIC, window=100)),
    ("nope_d256", 1, 333, 2, 1, 256, MapParams(O.NOPE)),
    ("bifocal_d256_g4", 1, 700, 2, 1, 256, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=200)),
    ("bifocal_d256_gqa4_w0_63", 2, 520, 4, 1, 256, MapParams(O.BIFOCAL, rope_base=1e4, w0=63, w_pretrained=150)),
    ("standard_d256_s1", 1, 1, 2, 1, 256, MapParams(O.STANDARD)),
]


def _run(q, k, v, params):
    from position_remapping_b200 import ropeattn as ra
    out, lse = ra.prefill(q.cuda(), k.cuda(), v.cuda(), params)
    torch.cuda.synchronize()
    ra.status()
    return out, lse


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_prefill_small_all_rows(case):
    name, B, S, Hq, Hkv, D, params = case
    q, k, v = make_qkv(B, S, Hq, Hkv, D, seed=zlib.crc32(name.encode()) % 10000)
    out, lse = _run(q, k, v, params)
    ref_o, ref_l = O.prefill(q, k, v, params, stage_bf16=True)
    assert_close(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, name)


@pytest.mark.parametrize("D", [128, 256])
def test_bifocal_inside_window_is_bitwise_standard(D):
    # L <= w_pretrained: the bifocal map is the base model exactly (Jet-Long §3)
    q, k, v = make_qkv(1, 700, 4, 2, D, seed=5)
    a = _run(q, k, v, MapParams(O.BIFOCAL, rope_base=1e6, w0=64, w_pretrained=700))
    b = _run(q, k, v, MapParams(O.STANDARD, rope_base=1e6))
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_prefill_deterministic():
    q, k, v = make_qkv(1, 1000, 4, 2, 128, seed=6)
    p = MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=256)
    a = _run(q, k, v, p)
    b = _run(q, k, v, p)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_prefill_workspace_errors():
    from position_remapping_b200 import ropeattn as ra
    q, k, v = (t.cuda() for t in make_qkv(1, 256, 2, 1, 64, seed=7))
    p = MapParams(O.STANDARD)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ra.RopeAttnError) as e:
        ra.prefill(q, k, v, p, workspace=small)
    assert e.value.code == ra.ERR_WORKSPACE


FULL = ["endprompt_s8192", "periodic_s32768", "nope_s32768", "bifocal_prefill_s131072"]


@pytest.mark.parametrize("name", FULL)
def test_prefill_full_size_sampled_rows(name):
    w = WORKLOADS[name]
    q, k, v = make_qkv(w.B, w.S, w.Hq, w.Hkv, w.D, w.seed)
    out, lse = _run(q, k, v, w.params)
    if name == "periodic_s32768":
        rows = list(range(w.S))          # every row: the windowed oracle is cheap here
    else:
        rows = sample_rows(w.S, w.params, n_random=512, edge=32 if w.S > 100000 else 64)
    ref_o, ref_l = O.prefill(q, k, v, w.params, rows=rows, stage_bf16=True)
    got_o = out.cpu().numpy()[:, rows]
    got_l = lse.cpu().numpy()[:, :, rows]
    assert_close(got_o, got_l, ref_o, ref_l, name)
