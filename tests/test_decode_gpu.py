"""Decode parity: the split-KV CUDA kernel (through the C ABI) against the
float64 oracle on the same seeded bf16 query and cache."""
import zlib

import pytest
import torch

import oracle as O
from parity_util import assert_close, decode_staged
from position_remapping_b200.inputs import WORKLOADS, MapParams, make_qkv

pytestmark = pytest.mark.gpu

SMALL = [
    ("standard", 2, 1000, 4, 2, 128, MapParams(O.STANDARD, rope_base=1e4)),
    ("standard_n1", 1, 1, 2, 1, 128, MapParams(O.STANDARD, rope_base=1e4)),
    ("endprompt", 1, 777, 4, 1, 128, MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=600, term_start=65000)),
    ("periodic", 2, 3000, 2, 2, 64, MapParams(O.PERIODIC, window=1024)),
    ("periodic_w_gt_n", 1, 300, 2, 1, 64, MapParams(O.PERIODIC, window=1000)),
    ("nope_g8", 1, 2049, 8, 1, 64, MapParams(O.NOPE)),
    ("bifocal_g2", 1, 5000, 16, 8, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=300, w_pretrained=2500)),
    ("bifocal_g10", 2, 1001, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=50, w_pretrained=100)),
    ("bifocal_g3_grp4", 1, 9000, 8, 2, 128, MapParams(O.BIFOCAL, rope_base=1e4, w0=1000, w_pretrained=3001)),
    ("bifocal_w0_0_d64", 1, 4097, 4, 1, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=0, w_pretrained=1024)),
    ("bifocal_inside_window", 1, 500, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=512)),
    ("bifocal_g4_d64_grp4", 2, 4097, 8, 2, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=300, w_pretrained=1100)),
    ("bifocal_g8_d128", 1, 8000, 4, 4, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=2048, w_pretrained=1000)),
    ("bifocal_g2_edge_local", 1, 3000, 2, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=2900, w_pretrained=1500)),
    ("bifocal_fixed_g5_phasor", 1, 3000, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=200, fixed_group=5)),
    ("bifocal_fixed_g4_table", 1, 5000, 8, 4, 128, MapParams(O.BIFOCAL, rope_base=1e4, w0=300, fixed_group=4)),
    # GQA groups up to 16 (padded to a power of two on the tensor cores), group
    # sizes G that do not divide the rotation's row step, short caches
    ("standard_grp16_d128", 1, 3000, 32, 2, 128, MapParams(O.STANDARD, rope_base=1e4)),
    ("bifocal_grp8_g3", 1, 6000, 16, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=500, w_pretrained=2000)),
    ("bifocal_grp16_d128", 1, 3000, 16, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=300, w_pretrained=1000)),
    ("bifocal_grp16_d64_g3", 2, 2000, 32, 2, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=100, w_pretrained=700)),
    ("bifocal_grp3", 1, 2500, 12, 4, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=200, w_pretrained=900)),
    ("bifocal_fixed_g7_d64", 1, 3001, 4, 2, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=129, fixed_group=7)),
    ("bifocal_n130_w0_1", 1, 130, 2, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=1, w_pretrained=64)),
    ("endprompt_grp8_d64", 2, 1500, 16, 2, 64, MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=1400, term_start=65000)),
    ("d256_standard", 1, 3000, 2, 1, 256, MapParams(O.STANDARD, rope_base=1e4)),
    ("d256_bifocal_g3_grp2", 2, 5000, 4, 2, 256, MapParams(O.BIFOCAL, rope_base=1e6, w0=400, w_pretrained=2000)),
    ("d256_periodic", 1, 2500, 2, 2, 256, MapParams(O.PERIODIC, rope_base=1e4, window=512)),
    ("d256_bifocal_grp1", 1, 4097, 2, 2, 256, MapParams(O.BIFOCAL, rope_base=1e4, w0=100, w_pretrained=1024)),
    # long key ranges per split (8 kv heads: 18 splits on 148 SMs, 12-19
    # tiles each), so the K-tile ring and the V-half ring wrap many times
    # at both head dims and the phasor is re-seeded mid-split
    ("long_bifocal_d128_grp2", 1, 40000, 16, 8, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=2048, w_pretrained=12000)),
    ("long_bifocal_d64_grp8_g3", 1, 40000, 64, 8, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=500, w_pretrained=15000)),
    ("long_standard_d64_grp16", 1, 30001, 128, 8, 64, MapParams(O.STANDARD, rope_base=1e4)),
    ("long_periodic_d128_grp4", 1, 33000, 32, 8, 128, MapParams(O.PERIODIC, rope_base=1e4, window=30000)),
    ("long_bifocal_b2_d128_grp4", 2, 20000, 32, 8, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=700, w_pretrained=6000)),
    # head_dim 256 on the tensor cores: two O^T blocks, two-slot rings, GQA up to 16
    ("d256_bifocal_grp4_g3", 1, 5000, 8, 2, 256, MapParams(O.BIFOCAL, rope_base=1e6, w0=400, w_pretrained=2000)),
    ("d256_bifocal_grp8", 2, 3000, 16, 2, 256, MapParams(O.BIFOCAL, rope_base=1e4, w0=128, w_pretrained=1024)),
    ("d256_standard_grp16", 1, 2000, 32, 2, 256, MapParams(O.STANDARD, rope_base=1e4)),
    ("long_bifocal_d256_grp2", 1, 40000, 16, 8, 256, MapParams(O.BIFOCAL, rope_base=1e6, w0=2048, w_pretrained=12000)),
]


def _run(q, kc, vc, params):
    from position_remapping_b200 import ropeattn as ra
    out, lse = ra.decode(q.cuda(), kc.cuda(), vc.cuda(), params)
    torch.cuda.synchronize()
    ra.status()
    return out, lse


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_decode_small(case):
    name, B, n, Hq, Hkv, D, params = case
    q, kc, vc = make_qkv(B, n, Hq, Hkv, D, seed=zlib.crc32(name.encode()) % 10000, q_len=1)
    out, lse = _run(q, kc, vc, params)
    ref_o, ref_l = O.decode(q, kc, vc, params, stage_bf16=decode_staged(D))
    assert_close(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, name)


def test_decode_full_size():
    w = WORKLOADS["bifocal_decode_n131072"]
    q, kc, vc = make_qkv(w.B, w.S, w.Hq, w.Hkv, w.D, w.seed, q_len=1)
    out, lse = _run(q, kc, vc, w.params)
    ref_o, ref_l = O.decode(q, kc, vc, w.params, stage_bf16=decode_staged(w.D))
    assert_close(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, w.name)


def test_decode_deterministic_and_repeatable():
    w = WORKLOADS["bifocal_decode_n131072"]
    q, kc, vc = (t.cuda() for t in make_qkv(w.B, w.S, w.Hq, w.Hkv, w.D, w.seed, q_len=1))
    from position_remapping_b200 import ropeattn as ra
    ws = torch.empty(ra.decode_workspace_size(w.B, w.S, w.Hq, w.Hkv, w.D), dtype=torch.uint8, device="cuda")
    a = ra.decode(q, kc, vc, w.params, workspace=ws)
    a = (a[0].clone(), a[1].clone())
    b = ra.decode(q, kc, vc, w.params, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_decode_workspace_error():
    from position_remapping_b200 import ropeattn as ra
    q, kc, vc = (t.cuda() for t in make_qkv(1, 1000, 4, 2, 128, seed=3, q_len=1))
    with pytest.raises(ra.RopeAttnError) as e:
        ra.decode(q, kc, vc, MapParams(O.STANDARD), workspace=torch.empty(8, dtype=torch.uint8, device="cuda"))
    assert e.value.code == ra.ERR_WORKSPACE
