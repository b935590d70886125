"""Out-of-bounds writes, checked without a sanitizer: every output tensor and
every workspace is a view into a larger buffer whose guard words before and
after it hold a sentinel bit pattern. After the call each guard word must be
unchanged, and every output element must have been written (no sentinel left
inside the view). Ragged lengths, every kind, the bifocal map, chunked
prefill, decode and the backward."""
import pytest
import torch

import oracle as O
from position_remapping_b200.inputs import PAIR_HALF, MapParams, make_qkv

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FC0DEAD          # a quiet NaN with a payload no kernel produces
GUARD = 4096                   # guard words (16 KiB) on each side


class Guarded:
    """A contiguous view of `shape` inside a sentinel-filled buffer."""

    def __init__(self, shape, dtype=torch.float32):
        n = 1
        for d in shape:
            n *= d
        words = (n * torch.tensor([], dtype=dtype).element_size() + 3) // 4
        self.n, self.words = n, words
        self.raw = torch.full((GUARD + words + GUARD,), SENTINEL, dtype=torch.int32, device="cuda")
        self.t = self.raw[GUARD:GUARD + words].view(dtype)[:n].view(shape)

    def check(self, name, interior=True):
        raw = self.raw.cpu()
        assert bool((raw[:GUARD] == SENTINEL).all()), f"{name}: write before the tensor"
        assert bool((raw[GUARD + self.words:] == SENTINEL).all()), f"{name}: write after the tensor"
        if interior and self.t.dtype == torch.float32:
            assert not bool((raw[GUARD:GUARD + self.words] == SENTINEL).any()), f"{name}: element not written"


def _ws(nbytes):
    return Guarded((max(nbytes, 1),), torch.uint8)


PREFILL = [
    ("standard_d128", 333, 4, 2, 128, MapParams(O.STANDARD, rope_base=1e4)),
    ("periodic_d64", 517, 2, 1, 64, MapParams(O.PERIODIC, rope_base=1e4, window=100)),
    ("nope_d256", 201, 2, 1, 256, MapParams(O.NOPE)),
    ("endprompt_d128", 390, 2, 2, 128, MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=300,
                                                 term_start=65000)),
    ("bifocal_g3_d128", 701, 4, 2, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=96, w_pretrained=256)),
    ("bifocal_half_d64", 455, 2, 1, 64, MapParams(O.BIFOCAL, rope_base=1e4, w0=50, w_pretrained=200,
                                                  pairing=PAIR_HALF)),
    ("bifocal_g3_d256", 390, 2, 1, 256, MapParams(O.BIFOCAL, rope_base=1e6, w0=40, w_pretrained=150)),
]


@pytest.mark.parametrize("case", PREFILL, ids=[c[0] for c in PREFILL])
def test_prefill_writes_only_its_outputs(case):
    from position_remapping_b200 import ropeattn as ra
    name, S, Hq, Hkv, D, params = case
    q, k, v = (t.cuda() for t in make_qkv(1, S, Hq, Hkv, D, seed=S))
    out, lse = Guarded((1, S, Hq, D)), Guarded((1, Hq, S))
    ws = _ws(ra.prefill_workspace_size(params, 1, S, Hq, Hkv, D))
    ra.prefill(q, k, v, params, out=out.t, lse=lse.t, workspace=ws.t)
    torch.cuda.synchronize()
    ra.status()
    out.check("out")
    lse.check("lse")
    ws.check("workspace", interior=False)


def test_chunked_prefill_writes_only_its_outputs():
    from position_remapping_b200 import ropeattn as ra
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=100, w_pretrained=256)
    L, start, Hq, Hkv, D = 777, 500, 4, 2, 128
    q, k, v = (t.cuda() for t in make_qkv(1, L, Hq, Hkv, D, seed=9))
    kc, vc = torch.empty_like(k), torch.empty_like(v)
    ra.cache_write(k, v, kc, vc, params, 0)
    count = L - start
    out, lse = Guarded((1, count, Hq, D)), Guarded((1, Hq, count))
    ws = _ws(ra.prefill_chunk_workspace_size(params, 1, start, count, Hq, Hkv, D))
    ra.prefill_chunk(q[:, start:].contiguous(), kc, vc, params, start, out=out.t, lse=lse.t, workspace=ws.t)
    torch.cuda.synchronize()
    ra.status()
    out.check("out")
    lse.check("lse")
    ws.check("workspace", interior=False)


DECODE = [
    ("bifocal_d128_grp2", 2, 3001, 16, 8, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=200, w_pretrained=1000)),
    ("periodic_d64_grp4", 1, 2049, 8, 2, 64, MapParams(O.PERIODIC, rope_base=1e4, window=512)),
    ("standard_d256", 1, 1500, 2, 1, 256, MapParams(O.STANDARD, rope_base=1e4)),
    ("bifocal_n5", 1, 5, 4, 1, 128, MapParams(O.BIFOCAL, rope_base=1e6, w0=1, w_pretrained=2)),
]


@pytest.mark.parametrize("case", DECODE, ids=[c[0] for c in DECODE])
def test_decode_writes_only_its_outputs(case):
    from position_remapping_b200 import ropeattn as ra
    name, B, n, Hq, Hkv, D, params = case
    q, kc, vc = (t.cuda() for t in make_qkv(B, n, Hq, Hkv, D, seed=n, q_len=1))
    out, lse = Guarded((B, Hq, D)), Guarded((B, Hq))
    ws = _ws(ra.decode_workspace_size(B, n, Hq, Hkv, D))
    for _ in range(2):   # the second call reuses the workspace, as a serving loop does
        ra.decode(q, kc, vc, params, out=out.t, lse=lse.t, workspace=ws.t)
    torch.cuda.synchronize()
    ra.status()
    out.check("out")
    lse.check("lse")
    ws.check("workspace", interior=False)


@pytest.mark.parametrize("D,params", [
    (128, MapParams(O.BIFOCAL, rope_base=1e6, w0=96, w_pretrained=256)),
    (64, MapParams(O.PERIODIC, rope_base=1e4, window=64, pairing=PAIR_HALF)),
], ids=["bifocal_d128", "periodic_half_d64"])
def test_backward_writes_only_its_outputs(D, params):
    from position_remapping_b200 import ropeattn as ra
    S, Hq, Hkv = 459, 4, 2
    q, k, v = (t.cuda() for t in make_qkv(1, S, Hq, Hkv, D, seed=11))
    out, lse = ra.prefill(q, k, v, params)
    dout = torch.randn((1, S, Hq, D), device="cuda").to(torch.bfloat16)
    dq, dk, dv = Guarded((1, S, Hq, D)), Guarded((1, S, Hkv, D)), Guarded((1, S, Hkv, D))
    ws = _ws(ra.prefill_backward_workspace_size(params, 1, S, Hq, Hkv, D))
    ra.prefill_backward(q, k, v, out, lse, dout, params, dq=dq.t, dk=dk.t, dv=dv.t, workspace=ws.t)
    torch.cuda.synchronize()
    ra.status()
    for g, nm in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        g.check(nm)
    ws.check("workspace", interior=False)
