"""Comparator: the literal three-call bifocal prefill with a separate merge
kernel (Jet-Long §3.3 Eq. 7) through the C ABI, against the oracle's
three-call route and against the fused prefill on the same inputs."""
import zlib

import pytest
import torch

import oracle as O
from parity_util import assert_close, decode_staged
from position_remapping_b200.inputs import MapParams, make_qkv

pytestmark = pytest.mark.gpu

CASES = [
    ("g4_d128", 1, 1000, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=300)),
    ("w0_0_d64", 2, 777, 2, 1, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=0, w_pretrained=256)),
    ("g3_d256", 1, 600, 2, 1, 256, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=200)),
    ("g3_wide_window", 1, 3000, 4, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=1000, w_pretrained=1000)),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_three_call_matches_oracle_and_fused(case):
    from position_remapping_b200 import ropeattn as ra
    name, B, S, Hq, Hkv, D, params = case
    q, k, v = make_qkv(B, S, Hq, Hkv, D, seed=zlib.crc32(f"three-{name}".encode()) % 10000)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o3, l3 = ra.prefill_three_call(qd, kd, vd, params)
    of, lf = ra.prefill(qd, kd, vd, params)
    torch.cuda.synchronize()
    ra.status()
    ref_o, ref_l = O.prefill_three_call(q, k, v, params, stage_bf16=True)
    # oracle layout: out [B,S,Hq,D], lse [B,Hq,S]
    assert_close(o3.cpu().numpy(), l3.cpu().numpy(), ref_o, ref_l, name + " three-call")
    assert_close(of.cpu().numpy(), lf.cpu().numpy(), ref_o, ref_l, name + " fused")


def test_three_call_rejects_non_bifocal():
    from position_remapping_b200 import ropeattn as ra
    q, k, v = (t.cuda() for t in make_qkv(1, 256, 2, 1, 64, seed=5))
    with pytest.raises(ra.RopeAttnError) as e:
        ra.prefill_three_call(q, k, v, MapParams(O.BIFOCAL, rope_base=1e4, w0=10, w_pretrained=1000))  # G = 1
    assert e.value.code == ra.ERR_INVALID_ARG


UNFUSED = [
    ("g4_table", 1, 5000, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=300, w_pretrained=1250)),
    ("g3_phasor_d64", 2, 3001, 4, 1, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=100, w_pretrained=1001)),
    ("fixed_g7", 1, 4000, 8, 4, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=50, fixed_group=7)),
]


@pytest.mark.parametrize("case", UNFUSED, ids=[c[0] for c in UNFUSED])
def test_unfused_decode_matches_oracle_and_fused(case):
    """Comparator: the correction rotation as a separate pass over the cache
    followed by a standard-RoPE decode (Jet-Long Eq. 5-6)."""
    from position_remapping_b200 import ropeattn as ra
    name, B, n, Hq, Hkv, D, params = case
    q, kc, vc = make_qkv(B, n, Hq, Hkv, D, seed=zlib.crc32(f"unfused-{name}".encode()) % 10000, q_len=1)
    qd, kd, vd = q.cuda(), kc.cuda(), vc.cuda()
    ou, lu = ra.decode_unfused(qd, kd, vd, params)
    of, lf = ra.decode(qd, kd, vd, params)
    torch.cuda.synchronize()
    ra.status()
    ref_o, ref_l = O.decode(q, kc, vc, params, stage_bf16=decode_staged(D))
    assert_close(ou.cpu().numpy(), lu.cpu().numpy(), ref_o, ref_l, name + " unfused")
    assert_close(of.cpu().numpy(), lf.cpu().numpy(), ref_o, ref_l, name + " fused")
