"""Prefill and decode with caller-provided outputs and workspace are plain
stream work (tensor maps are encoded on the host and passed by value, the
split counters are cleared by an async memset), so a serving loop can capture
them in a CUDA graph once and replay it with new inputs written in place.
The replays must equal direct calls on the same inputs, bit for bit."""
import pytest
import torch

import oracle as O
from position_remapping_b200.inputs import MapParams, make_qkv

pytestmark = pytest.mark.gpu


def _fresh(t, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(t.shape, generator=g).to(torch.bfloat16).to(t.device)


def test_decode_replays_in_a_cuda_graph():
    from position_remapping_b200 import ropeattn as ra
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=300, w_pretrained=2000)
    q, kc, vc = make_qkv(1, 6000, 8, 2, 128, seed=31, device="cuda", q_len=1)
    out = torch.empty((1, 8, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((1, 8), dtype=torch.float32, device="cuda")
    ws = torch.empty(ra.decode_workspace_size(1, 6000, 8, 2, 128), dtype=torch.uint8, device="cuda")
    ra.decode(q, kc, vc, params, out=out, lse=lse, workspace=ws)   # first launch outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ra.decode(q, kc, vc, params, out=out, lse=lse, workspace=ws)
    for seed in (1, 2, 3):
        q.copy_(_fresh(q, seed))
        g.replay()
        torch.cuda.synchronize()
        ref_o, ref_l = ra.decode(q, kc, vc, params)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l), seed
    ra.status()


def test_prefill_replays_in_a_cuda_graph():
    from position_remapping_b200 import ropeattn as ra
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=200, w_pretrained=1024)
    B, S, Hq, Hkv, D = 1, 3000, 4, 2, 128
    q, k, v = make_qkv(B, S, Hq, Hkv, D, seed=32, device="cuda")
    out = torch.empty((B, S, Hq, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device="cuda")
    ws = torch.empty(ra.prefill_workspace_size(params, B, S, Hq, Hkv, D), dtype=torch.uint8, device="cuda")
    ra.prefill(q, k, v, params, out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        ra.prefill(q, k, v, params, out=out, lse=lse, workspace=ws)
    for seed in (4, 5):
        q.copy_(_fresh(q, seed))
        k.copy_(_fresh(k, seed + 100))
        g.replay()
        torch.cuda.synchronize()
        ref_o, ref_l = ra.prefill(q, k, v, params)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_o) and torch.equal(lse, ref_l), seed
    ra.status()
