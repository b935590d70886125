"""Parity at the sizes the benchmark times its variants, in the same launch
configurations: the bifocal prefill at 32768 tokens (32/8 heads, G = 4)
with half-split pairing, a fixed group size and head_dim 256 (sampled rows,
every head), and the 131072-key bifocal decode at head_dim 64 and 256, GQA
groups 8 and 16 and half-split pairing (the first and the last kv head's
query heads), against the float64 oracle."""
import pytest

import oracle as O
from parity_util import assert_close, decode_staged, deinterleave
from position_remapping_b200.inputs import WORKLOADS, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

P = WORKLOADS["bifocal_prefill_s131072"]
DEC = WORKLOADS["bifocal_decode_n131072"]
BASE = P.params.replace(w_pretrained=8192)

PREFILL = [
    ("half_split", 128, BASE.replace(pairing=1)),
    ("fixed_g4", 128, BASE.replace(fixed_group=4)),
    ("d256", 256, BASE),
]


@pytest.mark.parametrize("case", PREFILL, ids=[c[0] for c in PREFILL])
def test_prefill_variant_s32768(case):
    from position_remapping_b200 import ropeattn as ra
    name, D, params = case
    S = 32768
    q, k, v = make_qkv(P.B, S, P.Hq, P.Hkv, D, P.seed + D)
    out, lse = ra.prefill(q.cuda(), k.cuda(), v.cuda(), params)
    ra.status()
    rows = sample_rows(S, params, n_random=64, edge=16)
    ref_o, ref_l = O.prefill(q, k, v, params, rows=rows, stage_bf16=True)
    assert_close(out.cpu().numpy()[:, rows], lse.cpu().numpy()[:, :, rows], ref_o, ref_l, name)


DECODE = [
    ("d128_grp8", 128, 64, DEC.params),
    ("d128_grp16", 128, 128, DEC.params),
    ("half_split", 128, 16, DEC.params.replace(pairing=1)),
    ("d64_grp2", 64, 16, DEC.params),
    ("d256_grp2", 256, 16, DEC.params),
]


@pytest.mark.parametrize("case", DECODE, ids=[c[0] for c in DECODE])
def test_decode_variant_n131072(case):
    from position_remapping_b200 import ropeattn as ra
    name, D, Hq, params = case
    q, kc, vc = make_qkv(DEC.B, DEC.S, Hq, DEC.Hkv, D, DEC.seed + D + Hq, q_len=1)
    out, lse = ra.decode(q.cuda(), kc.cuda(), vc.cuda(), params)
    ra.status()
    grp = Hq // DEC.Hkv
    for hk in (0, DEC.Hkv - 1):
        # query heads of kv head hk (contiguous GQA groups) against the oracle
        # on that kv head alone: the same arithmetic for those heads
        hs = slice(hk * grp, (hk + 1) * grp)
        # with half-split pairing the cache holds each rotated key in adjacent
        # order; the oracle takes the heads' own order
        kh = kc[:, :, hk:hk + 1]
        if params.pairing == 1:
            kh = deinterleave(kh)
        ref_o, ref_l = O.decode(q[:, hs], kh, vc[:, :, hk:hk + 1], params, stage_bf16=decode_staged(D))
        assert_close(out.cpu().numpy()[:, hs], lse.cpu().numpy()[:, hs], ref_o, ref_l, f"{name} kv head {hk}")
