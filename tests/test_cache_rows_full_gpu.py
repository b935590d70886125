"""Parity of the decode-cache rows at the sizes and in the launch
configurations the benchmark times them, against the float64 oracle on
sampled rows:

- the cache of the 131072-token bifocal prefill (32/8 heads, D 128) written
  in one call (Jet-Long §3.2 Eq. 4);
- the last 8192 rows of that prefill computed from the cache (local keys as
  stored, remote keys through the correction rotation, Eq. 5-6), for the
  query heads of the first and the last kv head;
- a decode step over the 131072-key bifocal cache (16/8 heads) that first
  appends its own token at the last row, then attends.
"""
import numpy as np
import pytest
import torch

import oracle as O
from parity_util import assert_close, decode_staged
from position_remapping_b200.inputs import WORKLOADS, make_qkv, sample_rows

pytestmark = pytest.mark.gpu

P = WORKLOADS["bifocal_prefill_s131072"]
DEC = WORKLOADS["bifocal_decode_n131072"]
CHUNK = 8192


def _bf16_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check_cache_rows(kc, k, params, rows, name, k_start=0):
    """Sampled cache rows r against the oracle's entries for the raw keys
    k[:, r - k_start] rounded to bf16, with the fp32-rotation allowance of the
    small-size cache test (one bf16 ulp from rounding, a few fp32 ulps of
    |x0| + |x1| per pair)."""
    D = k.shape[-1]
    for r in rows:
        x = k[:, r - k_start:r - k_start + 1]
        got = _bf16_f64(kc[:, r:r + 1])
        ref = O.round_bf16(O.cache_keys(x, params, start=r))
        kin = np.abs(x.float().numpy().astype(np.float64))
        pair = kin.reshape(*kin.shape[:-1], D // 2, 2).sum(-1).repeat(2, axis=-1)
        tol = np.abs(ref) * 2.0 ** -7 + pair * 2.0 ** -21
        err = np.abs(got - ref)
        assert np.all(err <= tol), f"{name}: row {r} max err {err.max():.3e}"


def test_cache_write_and_chunk_s131072():
    from position_remapping_b200 import ropeattn as ra
    q, k, v = make_qkv(P.B, P.S, P.Hq, P.Hkv, P.D, P.seed)
    kd, vd = k.cuda(), v.cuda()
    kc, vc = torch.empty_like(kd), torch.empty_like(vd)
    ra.cache_write(kd, vd, kc, vc, P.params, 0)
    torch.cuda.synchronize()
    ra.status()
    rows = sample_rows(P.S, P.params, n_random=32, edge=8)
    _check_cache_rows(kc, k, P.params, rows, "cache write")
    assert torch.equal(vc, vd)

    start = P.S - CHUNK
    out, lse = ra.prefill_chunk(q[:, start:].contiguous().cuda(), kc, vc, P.params, start)
    torch.cuda.synchronize()
    ra.status()
    kc_h = kc.cpu()
    del kd, vd, kc, vc
    grp = P.Hq // P.Hkv
    heads = list(range(grp)) + list(range(P.Hq - grp, P.Hq))
    rnd = torch.randint(0, CHUNK, (24,), generator=torch.Generator().manual_seed(5))
    crow = sorted({start, start + 1, start + 127, start + 128, P.S - 2, P.S - 1}
                  | {r for r in rows if r >= start} | set((start + rnd).tolist()))
    ref_o, ref_l = O.prefill_from_cache(q[:, start:], kc_h, v, P.params, start, stage_bf16=True, rows=crow,
                                        heads=heads)
    idx = [r - start for r in crow]
    got_o = out[:, idx][:, :, heads].cpu().numpy()
    got_l = lse[:, heads][:, :, idx].cpu().numpy()
    assert_close(got_o, got_l, ref_o, ref_l, "chunk from the cache")


def test_decode_with_append_n131072():
    from position_remapping_b200 import ropeattn as ra
    q, kc, vc = make_qkv(DEC.B, DEC.S, DEC.Hq, DEC.Hkv, DEC.D, DEC.seed, q_len=1)
    _, kn, vn = make_qkv(DEC.B, 1, DEC.Hq, DEC.Hkv, DEC.D, DEC.seed + 7)
    kcd, vcd = kc.cuda(), vc.cuda()
    ra.cache_write(kn.cuda(), vn.cuda(), kcd, vcd, DEC.params, DEC.S - 1)
    out, lse = ra.decode(q.cuda(), kcd, vcd, DEC.params)
    torch.cuda.synchronize()
    ra.status()
    # the appended row is the new token's cache entry; every other row untouched
    _check_cache_rows(kcd, kn, DEC.params, [DEC.S - 1], "appended row", k_start=DEC.S - 1)
    kc_after, vc_after = kcd.cpu(), vcd.cpu()
    assert torch.equal(kc_after[:, :-1], kc[:, :-1]) and torch.equal(vc_after[:, :-1], vc[:, :-1])
    assert torch.equal(vc_after[:, -1:], vn)
    grp = DEC.Hq // DEC.Hkv
    for hk in (0, DEC.Hkv - 1):
        hs = slice(hk * grp, (hk + 1) * grp)
        ref_o, ref_l = O.decode(q[:, hs], kc_after[:, :, hk:hk + 1], vc_after[:, :, hk:hk + 1], DEC.params,
                                stage_bf16=decode_staged(DEC.D))
        assert_close(out.cpu().numpy()[:, hs], lse.cpu().numpy()[:, hs], ref_o, ref_l, f"decode kv head {hk}")
