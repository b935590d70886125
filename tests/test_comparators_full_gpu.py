"""Parity of the comparators at the sizes and in the launch configurations
the benchmark times them, against the float64 oracle on sampled rows: the
131072-token prefill with standard RoPE (the unmodified-model reference of
the comparison), the literal three-call bifocal route with its separate
merge (Jet-Long §3.3 Eq. 7) on the same inputs, and the unfused bifocal
decode (the correction rotation as its own pass, Eq. 5-6) over the
131072-key cache."""
import pytest
import torch

import oracle as O
from parity_util import assert_close, decode_staged
from position_remapping_b200.inputs import WORKLOADS, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

P = WORKLOADS["bifocal_prefill_s131072"]
DEC = WORKLOADS["bifocal_decode_n131072"]


def test_standard_and_three_call_prefill_s131072():
    from position_remapping_b200 import ropeattn as ra
    q, k, v = make_qkv(P.B, P.S, P.Hq, P.Hkv, P.D, P.seed)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    std = P.params.replace(kind=O.STANDARD)
    rows = sample_rows(P.S, P.params, n_random=32, edge=8)
    ridx = torch.tensor(rows, device=qd.device)
    for name, params, call in (("standard RoPE", std, ra.prefill),
                               ("three-call bifocal", P.params, ra.prefill_three_call)):
        out, lse = call(qd, kd, vd, params)
        torch.cuda.synchronize()
        ra.status()
        got_o, got_l = out[:, ridx].cpu().numpy(), lse[:, :, ridx].cpu().numpy()
        del out, lse
        ref_o, ref_l = O.prefill(q, k, v, params, rows=rows, stage_bf16=True)
        assert_close(got_o, got_l, ref_o, ref_l, name)


def test_unfused_decode_n131072():
    from position_remapping_b200 import ropeattn as ra
    q, kc, vc = make_qkv(DEC.B, DEC.S, DEC.Hq, DEC.Hkv, DEC.D, DEC.seed, q_len=1)
    out, lse = ra.decode_unfused(q.cuda(), kc.cuda(), vc.cuda(), DEC.params)
    torch.cuda.synchronize()
    ra.status()
    grp = DEC.Hq // DEC.Hkv
    for hk in (0, DEC.Hkv - 1):
        hs = slice(hk * grp, (hk + 1) * grp)
        ref_o, ref_l = O.decode(q[:, hs], kc[:, :, hk:hk + 1], vc[:, :, hk:hk + 1], DEC.params,
                                stage_bf16=decode_staged(DEC.D))
        assert_close(out.cpu().numpy()[:, hs], lse.cpu().numpy()[:, hs], ref_o, ref_l, f"unfused kv head {hk}")
