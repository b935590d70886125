"""Decode-cache writer and multi-step decode (Jet-Long §3.2 Eq. 4-6).

ropeattn_cache_write (through the C ABI) against the float64 oracle's cache
entries, and a decode loop that appends one token per step to a cache
written once, across the lengths where the bifocal group size G changes,
against the oracle decode on the same cache."""
import zlib

import numpy as np
import pytest
import torch

import oracle as O
from parity_util import assert_close, decode_staged
from position_remapping_b200.inputs import MapParams, make_qkv

pytestmark = pytest.mark.gpu

KINDS = [
    ("standard", MapParams(O.STANDARD, rope_base=1e4)),
    ("endprompt", MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=1100, term_start=65000)),
    ("periodic", MapParams(O.PERIODIC, rope_base=1e4, window=512)),
    ("nope", MapParams(O.NOPE)),
    ("bifocal", MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=256)),
]


def _bf16_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("case", KINDS, ids=[c[0] for c in KINDS])
def test_cache_write_matches_oracle(case, D):
    from position_remapping_b200 import ropeattn as ra
    name, params = case
    B, count, Hkv, start, cache_len = 2, 300, 2, 1000, 1500
    _, k, v = make_qkv(B, count, 2, Hkv, D, seed=zlib.crc32(f"cache-{name}-{D}".encode()) % 10000)
    kc = torch.full((B, cache_len, Hkv, D), 3.0, dtype=torch.bfloat16, device="cuda")
    vc = torch.full((B, cache_len, Hkv, D), 3.0, dtype=torch.bfloat16, device="cuda")
    ra.cache_write(k.cuda(), v.cuda(), kc, vc, params, start)
    torch.cuda.synchronize()
    ra.status()
    got = _bf16_f64(kc[:, start:start + count])
    ref = O.round_bf16(O.cache_keys(k, params, start))
    # same rounding model (rotate, then round to bf16). The kernel rotates in
    # fp32: its result differs from the fp64 rotation by at most a few fp32
    # ulps of the inputs (|x0| + |x1| per pair), which the bf16 rounding can
    # turn into one bf16 ulp of the result
    err = np.abs(got - ref)
    kin = np.abs(k.float().numpy().astype(np.float64))
    pair = kin.reshape(*kin.shape[:-1], D // 2, 2).sum(-1).repeat(2, axis=-1)
    tol = np.abs(ref) * 2.0 ** -7 + pair * 2.0 ** -21
    assert np.all(err <= tol), f"{name}: max err {err.max():.3e}"
    assert np.mean(err == 0) > 0.99
    if params.kind == O.NOPE:
        assert torch.equal(kc[:, start:start + count].cpu(), k)
    assert torch.equal(vc[:, start:start + count].cpu(), v)
    # rows outside [start, start + count) are untouched
    assert bool((kc[:, :start] == 3.0).all()) and bool((kc[:, start + count:] == 3.0).all())
    assert bool((vc[:, :start] == 3.0).all()) and bool((vc[:, start + count:] == 3.0).all())


def test_cache_write_in_chunks_equals_one_write():
    from position_remapping_b200 import ropeattn as ra
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=256)
    _, k, v = (t.cuda() for t in make_qkv(1, 1000, 2, 2, 128, seed=41))
    a_k = torch.zeros_like(k)
    a_v = torch.zeros_like(v)
    ra.cache_write(k, v, a_k, a_v, params, 0)
    b_k = torch.zeros_like(k)
    b_v = torch.zeros_like(v)
    for s0, s1 in ((0, 1), (1, 333), (333, 999), (999, 1000)):
        ra.cache_write(k[:, s0:s1].contiguous(), v[:, s0:s1].contiguous(), b_k, b_v, params, s0)
    torch.cuda.synchronize()
    assert torch.equal(a_k, b_k) and torch.equal(a_v, b_v)


def test_multistep_decode_across_group_changes():
    """Prefill writes the cache of 500 tokens once; each decode step appends
    its token and attends over the first n rows, for n = 501..800, across
    G = ceil(n / 256) = 2 -> 3 (n = 513) -> 4 (n = 769), with no cache
    rewrite (Jet-Long §3.2)."""
    from position_remapping_b200 import ropeattn as ra
    params = MapParams(O.BIFOCAL, rope_base=1e4, w0=64, w_pretrained=256)
    N, S0, Hq, Hkv, D = 800, 500, 4, 2, 128
    q, k, v = make_qkv(1, N, Hq, Hkv, D, seed=42)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kc = torch.zeros_like(kd)
    vc = torch.zeros_like(vd)
    ra.cache_write(kd[:, :S0].contiguous(), vd[:, :S0].contiguous(), kc, vc, params, 0)
    outs, lses = [], []
    for n in range(S0 + 1, N + 1):
        ra.cache_write(kd[:, n - 1:n].contiguous(), vd[:, n - 1:n].contiguous(), kc, vc, params, n - 1)
        o, l = ra.decode(qd[:, n - 1].contiguous(), kc[:, :n], vc[:, :n], params)
        outs.append(o.clone())
        lses.append(l.clone())
    torch.cuda.synchronize()
    ra.status()
    # the cache written step by step equals one write of all N tokens
    full_k = torch.zeros_like(kd)
    full_v = torch.zeros_like(vd)
    ra.cache_write(kd, vd, full_k, full_v, params, 0)
    torch.cuda.synchronize()
    assert torch.equal(kc, full_k) and torch.equal(vc, full_v)
    cache = kc.cpu()
    seen_G = set()
    for i, n in enumerate(range(S0 + 1, N + 1)):
        seen_G.add(O.group_size(n, params.w_pretrained))
        ref_o, ref_l = O.decode(q[:, n - 1], cache[:, :n], v[:, :n], params, stage_bf16=decode_staged(D))
        assert_close(outs[i].cpu().numpy(), lses[i].cpu().numpy(), ref_o, ref_l, f"n={n}")
    assert seen_G == {2, 3, 4}


def test_batched_decode_over_caches_with_spare_rows():
    """B = 3 sequences share one [B, capacity, Hkv, D] cache allocation; each
    step appends the token of every sequence (ropeattn_cache_write) and
    decodes over the first n rows (ropeattn_decode_cache), across G = 3 -> 4
    at n = 769."""
    from position_remapping_b200 import ropeattn as ra
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=256)
    B, cap, Hq, Hkv, D = 3, 1024, 4, 2, 128
    S0, N = 740, 790
    q, k, v = make_qkv(B, N, Hq, Hkv, D, seed=43)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    kc = torch.zeros((B, cap, Hkv, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ra.cache_write(kd[:, :S0].contiguous(), vd[:, :S0].contiguous(), kc, vc, params, 0)
    outs = []
    for n in range(S0 + 1, N + 1):
        ra.cache_write(kd[:, n - 1:n].contiguous(), vd[:, n - 1:n].contiguous(), kc, vc, params, n - 1)
        o, l = ra.decode_cache(qd[:, n - 1].contiguous(), kc, vc, n, params)
        outs.append((o.clone(), l.clone()))
    torch.cuda.synchronize()
    ra.status()
    cache = kc.cpu()
    for i, n in enumerate(range(S0 + 1, N + 1)):
        if i % 7 and n not in (768, 769, 770, N):
            continue   # a sample of the steps, and every step around the G change
        ref_o, ref_l = O.decode(q[:, n - 1], cache[:, :n], v[:, :n], params, stage_bf16=decode_staged(D))
        assert_close(outs[i][0].cpu().numpy(), outs[i][1].cpu().numpy(), ref_o, ref_l, f"n={n}")
    # the same call on a dense copy of the first n rows gives the same bits
    n = N
    dense = (kc[:, :n].contiguous(), vc[:, :n].contiguous())
    a = ra.decode(qd[:, n - 1].contiguous(), dense[0], dense[1], params)
    torch.cuda.synchronize()
    assert torch.equal(a[0], outs[-1][0]) and torch.equal(a[1], outs[-1][1])
