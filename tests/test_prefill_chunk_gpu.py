"""Chunked prefill from a decode cache: ropeattn_prefill_chunk (through the
C ABI) against the oracle's prefill rows computed from the same cache
(Jet-Long §3.2 Eq. 4-6: keys read as stored, remote keys through the
correction rotation), at chunk offsets inside and across the bifocal local
window and across G changes."""
import zlib

import pytest
import torch

import oracle as O
from parity_util import assert_close
from position_remapping_b200.inputs import MapParams, make_qkv

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, L, start, Hq, Hkv, D, params
    ("standard", 2, 700, 300, 4, 2, 128, MapParams(O.STANDARD, rope_base=1e4)),
    ("endprompt", 1, 900, 500, 4, 1, 128, MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=600,
                                                     term_start=65000)),
    ("periodic", 1, 1500, 1000, 2, 2, 64, MapParams(O.PERIODIC, rope_base=1e4, window=256)),
    ("nope", 1, 800, 1, 4, 2, 64, MapParams(O.NOPE)),
    ("bifocal_g3", 1, 1700, 1200, 8, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=200, w_pretrained=600)),
    ("bifocal_whole", 1, 1000, 0, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=300)),
    ("bifocal_small_chunk", 2, 2049, 2000, 4, 1, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=64, w_pretrained=512)),
    ("bifocal_one_row", 1, 3001, 3000, 4, 4, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=1000, w_pretrained=1000)),
    ("bifocal_in_window", 1, 400, 200, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=500, w_pretrained=100)),
    ("bifocal_d256", 1, 900, 500, 2, 1, 256, MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=300)),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_prefill_chunk_matches_oracle(case):
    from position_remapping_b200 import ropeattn as ra
    name, B, L, start, Hq, Hkv, D, params = case
    q, k, v = make_qkv(B, L, Hq, Hkv, D, seed=zlib.crc32(f"chunk-{name}".encode()) % 10000)
    kc = torch.zeros((B, L, Hkv, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ra.cache_write(k.cuda(), v.cuda(), kc, vc, params, 0)
    qc = q[:, start:].contiguous().cuda()
    out, lse = ra.prefill_chunk(qc, kc, vc, params, start)
    torch.cuda.synchronize()
    ra.status()
    ref_o, ref_l = O.prefill_from_cache(q[:, start:], kc.cpu(), v, params, start, stage_bf16=True)
    assert_close(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, name)


def test_chunks_cover_a_whole_prefill():
    """Three chunks (each appended to the cache before it runs) give the rows
    of one whole prefill from the cache, bit for bit (same kernel, same keys)."""
    from position_remapping_b200 import ropeattn as ra
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=128, w_pretrained=512)
    B, L, Hq, Hkv, D = 1, 1500, 4, 2, 128
    q, k, v = (t.cuda() for t in make_qkv(B, L, Hq, Hkv, D, seed=77))
    kc = torch.zeros_like(k)
    vc = torch.zeros_like(v)
    ra.cache_write(k, v, kc, vc, params, 0)
    whole_o, whole_l = ra.prefill_chunk(q, kc, vc, params, 0)
    # G depends on L, so rows of a shorter prefix differ: compare the last chunk
    # (L rows of keys) with the whole prefill's last rows
    s0 = 1100
    last_o, last_l = ra.prefill_chunk(q[:, s0:].contiguous(), kc, vc, params, s0)
    torch.cuda.synchronize()
    assert torch.equal(last_o, whole_o[:, s0:]) and torch.equal(last_l, whole_l[:, :, s0:])


@pytest.mark.parametrize("kind", ["bifocal", "standard"])
def test_chunk_over_caches_with_spare_rows(kind):
    """B = 2 sequences in one [B, capacity, Hkv, D] allocation: a chunk over
    the first start + count rows equals the chunk over dense copies of those
    rows, bit for bit, and matches the oracle."""
    from position_remapping_b200 import ropeattn as ra
    params = (MapParams(O.BIFOCAL, rope_base=1e6, w0=150, w_pretrained=400) if kind == "bifocal"
              else MapParams(O.STANDARD, rope_base=1e4))
    B, cap, L, start, Hq, Hkv, D = 2, 1600, 1200, 900, 4, 2, 128
    q, k, v = make_qkv(B, L, Hq, Hkv, D, seed=78)
    kc = torch.zeros((B, cap, Hkv, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ra.cache_write(k.cuda(), v.cuda(), kc, vc, params, 0)
    qc = q[:, start:].contiguous().cuda()
    a_o, a_l = ra.prefill_chunk(qc, kc, vc, params, start)
    b_o, b_l = ra.prefill_chunk(qc, kc[:, :L].contiguous(), vc[:, :L].contiguous(), params, start)
    torch.cuda.synchronize()
    ra.status()
    assert torch.equal(a_o, b_o) and torch.equal(a_l, b_l)
    ref_o, ref_l = O.prefill_from_cache(q[:, start:], kc[:, :L].cpu(), v, params, start, stage_bf16=True)
    assert_close(a_o.cpu().numpy(), a_l.cpu().numpy(), ref_o, ref_l, kind)
