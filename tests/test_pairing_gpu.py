"""Half-split pairing (coordinates (i, i + D/2) turned by p * theta_i) on the
CUDA path, through the C ABI, against the float64 oracle with the same
pairing.

The library runs every attention kernel in adjacent order: a half-split call
permutes the query on entry and its keys where they are rotated, and its key
caches hold each rotated key in adjacent order (element 2i = coordinate i,
2i+1 = coordinate i + D/2). The tests read such caches back to the heads'
own order with that documented permutation before handing them to the
oracle."""
import zlib

import numpy as np
import pytest
import torch

import oracle as O
from parity_util import assert_close, decode_staged
from position_remapping_b200.inputs import PAIR_HALF, MapParams, make_qkv

pytestmark = pytest.mark.gpu


def _interleave(x):
    """Half-split order -> adjacent order along the last axis."""
    P = x.shape[-1] // 2
    return torch.stack([x[..., :P], x[..., P:]], dim=-1).reshape(x.shape)


def _deinterleave(x):
    """Adjacent order -> half-split order along the last axis."""
    return torch.cat([x[..., 0::2], x[..., 1::2]], dim=-1)


def _seed(name):
    return zlib.crc32(name.encode()) % 10000


PREFILL = [
    # (id, B, S, Hq, Hkv, D, params)
    ("standard_gqa", 2, 300, 4, 2, 128, MapParams(O.STANDARD, rope_base=1e4, pairing=PAIR_HALF)),
    ("endprompt_d64", 1, 700, 2, 1, 64,
     MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=500, term_start=65000, pairing=PAIR_HALF)),
    ("periodic_w100_d64", 1, 900, 2, 2, 64, MapParams(O.PERIODIC, window=100, pairing=PAIR_HALF)),
    ("nope", 1, 333, 4, 1, 128, MapParams(O.NOPE, pairing=PAIR_HALF)),
    ("bifocal_g4", 1, 1000, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=256,
                                                 pairing=PAIR_HALF)),
    ("bifocal_g3_d64", 1, 700, 2, 2, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=64, w_pretrained=300,
                                                   pairing=PAIR_HALF)),
    ("bifocal_d256", 1, 600, 2, 1, 256, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=200,
                                                  pairing=PAIR_HALF)),
]


@pytest.mark.parametrize("case", PREFILL, ids=[c[0] for c in PREFILL])
def test_half_split_prefill_all_rows(case):
    from position_remapping_b200 import ropeattn as ra
    name, B, S, Hq, Hkv, D, params = case
    q, k, v = make_qkv(B, S, Hq, Hkv, D, seed=_seed("half-" + name))
    out, lse = ra.prefill(q.cuda(), k.cuda(), v.cuda(), params)
    torch.cuda.synchronize()
    ra.status()
    ref_o, ref_l = O.prefill(q, k, v, params, stage_bf16=True)
    assert_close(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, name)


def test_half_split_prefill_is_adjacent_on_permuted_heads_bitwise():
    # the permutation is the whole difference: same kernels, same bits
    from position_remapping_b200 import ropeattn as ra
    half = MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=256, pairing=PAIR_HALF)
    adj = half.replace(pairing=0)
    q, k, v = (t.cuda() for t in make_qkv(1, 1000, 4, 2, 128, seed=51))
    a = ra.prefill(q, k, v, half)
    b = ra.prefill(_interleave(q).contiguous(), _interleave(k).contiguous(), v, adj)
    c = ra.prefill_three_call(q, k, v, half)
    d = ra.prefill_three_call(_interleave(q).contiguous(), _interleave(k).contiguous(), v, adj)
    torch.cuda.synchronize()
    ra.status()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert torch.equal(c[0], d[0]) and torch.equal(c[1], d[1])


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("kind", ["standard", "periodic", "bifocal", "nope"])
def test_half_split_cache_write(kind, D):
    from position_remapping_b200 import ropeattn as ra
    params = {"standard": MapParams(O.STANDARD, rope_base=1e4, pairing=PAIR_HALF),
              "periodic": MapParams(O.PERIODIC, rope_base=1e4, window=512, pairing=PAIR_HALF),
              "bifocal": MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=256, pairing=PAIR_HALF),
              "nope": MapParams(O.NOPE, pairing=PAIR_HALF)}[kind]
    B, count, Hkv, start, cache_len = 2, 300, 2, 1000, 1500
    _, k, v = make_qkv(B, count, 2, Hkv, D, seed=_seed(f"half-cache-{kind}-{D}"))
    kc = torch.zeros((B, cache_len, Hkv, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ra.cache_write(k.cuda(), v.cuda(), kc, vc, params, start)
    torch.cuda.synchronize()
    ra.status()
    assert torch.equal(vc[:, start:start + count].cpu(), v)
    got = kc[:, start:start + count].cpu()
    if params.kind == O.NOPE:
        # nothing rotates, so the pairing does not apply: keys are stored as given
        assert torch.equal(got, k)
        return
    got = got.float().numpy().astype(np.float64)
    ref = O.round_bf16(O.cache_keys(k, params, start))
    ref = _interleave(torch.from_numpy(ref)).numpy()
    kin = np.abs(k.float().numpy().astype(np.float64))
    P = D // 2
    pair = (kin[..., :P] + kin[..., P:]).repeat(2, axis=-1)    # pair i's inputs, at 2i and 2i+1
    err = np.abs(got - ref)
    tol = np.abs(ref) * 2.0 ** -7 + pair * 2.0 ** -21
    assert np.all(err <= tol), f"max err {err.max():.3e}"
    assert np.mean(err == 0) > 0.99


DECODE = [
    # (id, B, n, Hq, Hkv, D, params)
    ("bifocal_table", 1, 1500, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=256,
                                                    pairing=PAIR_HALF)),
    ("bifocal_phasor_gqa4", 2, 1300, 8, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=400,
                                                          pairing=PAIR_HALF)),
    ("bifocal_d256", 1, 1100, 2, 2, 256, MapParams(O.BIFOCAL, rope_base=1e6, w0=64, w_pretrained=300,
                                                   pairing=PAIR_HALF)),
    ("standard_d64", 2, 777, 8, 1, 64, MapParams(O.STANDARD, rope_base=1e4, pairing=PAIR_HALF)),
    ("periodic_w256", 1, 1000, 2, 2, 64, MapParams(O.PERIODIC, window=256, pairing=PAIR_HALF)),
    ("endprompt", 1, 900, 4, 4, 128,
     MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=600, term_start=65000, pairing=PAIR_HALF)),
]


@pytest.mark.parametrize("case", DECODE, ids=[c[0] for c in DECODE])
def test_half_split_decode_from_written_cache(case):
    from position_remapping_b200 import ropeattn as ra
    name, B, n, Hq, Hkv, D, params = case
    q, k, v = make_qkv(B, n, Hq, Hkv, D, seed=_seed("half-dec-" + name))
    kc = torch.empty_like(k, device="cuda")
    vc = torch.empty_like(v, device="cuda")
    ra.cache_write(k.cuda(), v.cuda(), kc, vc, params, 0)
    qd = q[:, n - 1].contiguous()
    out, lse = ra.decode(qd.cuda(), kc, vc, params)
    torch.cuda.synchronize()
    ra.status()
    cache = _deinterleave(kc.cpu())          # the heads' own order, as the oracle takes it
    ref_o, ref_l = O.decode(qd, cache, v, params, stage_bf16=decode_staged(D))
    assert_close(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, name)
    if params.kind == O.BIFOCAL and Hq // Hkv <= 2 and D <= 128:
        uo, ul = ra.decode_unfused(qd.cuda(), kc, vc, params)
        torch.cuda.synchronize()
        ra.status()
        assert_close(uo.cpu().numpy(), ul.cpu().numpy(), ref_o, ref_l, name + " unfused")


@pytest.mark.parametrize("start", [0, 700, 999])
def test_half_split_prefill_chunk_from_cache(start):
    from position_remapping_b200 import ropeattn as ra
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=256, pairing=PAIR_HALF)
    L = 1000
    q, k, v = make_qkv(1, L, 4, 2, 128, seed=52)
    kc = torch.empty_like(k, device="cuda")
    vc = torch.empty_like(v, device="cuda")
    ra.cache_write(k.cuda(), v.cuda(), kc, vc, params, 0)
    qc = q[:, start:].contiguous()
    out, lse = ra.prefill_chunk(qc.cuda(), kc, vc, params, start)
    torch.cuda.synchronize()
    ra.status()
    ref_o, ref_l = O.prefill_from_cache(qc, _deinterleave(kc.cpu()), v, params, start, stage_bf16=True)
    assert_close(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, f"start={start}")
