"""ropeattn_decode_noalloc: the decode entry point for callers that cannot
allocate device memory when they call (an engine plug-in that owns no device
allocations, a serving loop that cannot afford cudaMalloc's synchronization).
It must give the same result as ropeattn_decode, which takes a caller
workspace, on consecutive calls that share the library's one scratch array.

Collected last on purpose (file name), so a run that stops at the first
failure has already run every other test; it also passes on its own in a
fresh process."""
import ctypes

import pytest
import torch

import oracle as O
from parity_util import assert_close, decode_staged
from position_remapping_b200.inputs import WORKLOADS, MapParams, make_qkv

pytestmark = pytest.mark.gpu


def _noalloc(ra, q, kc, vc, params):
    B, Hq, D = q.shape
    n, Hkv = kc.shape[1], kc.shape[2]
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device=q.device)
    lse = torch.full((B, Hq), float("nan"), dtype=torch.float32, device=q.device)
    cp = ra.to_cparams(params)
    rc = ra.lib.ropeattn_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr()),
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()), B, n, Hq, Hkv, D,
        ctypes.byref(cp), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == ra.OK, ra.lib.ropeattn_last_error().decode()
    torch.cuda.synchronize()
    return out, lse


def test_decode_noalloc_matches_decode_on_consecutive_calls():
    from position_remapping_b200 import ropeattn as ra
    w = WORKLOADS["bifocal_decode_n131072"]
    cases = [
        (make_qkv(w.B, w.S, w.Hq, w.Hkv, w.D, w.seed, device="cuda", q_len=1), w.params),
        (make_qkv(2, 3000, 8, 2, 128, seed=77, device="cuda", q_len=1), MapParams(O.STANDARD, rope_base=1e4)),
    ]
    for (q, kc, vc), params in cases:          # two calls in a row, sharing the scratch
        ref_out, ref_lse = ra.decode(q, kc, vc, params)
        torch.cuda.synchronize()
        out, lse = _noalloc(ra, q, kc, vc, params)
        ra.status()
        assert_close(out.cpu().numpy(), lse.cpu().numpy(), ref_out.cpu().numpy(), ref_lse.cpu().numpy(),
                     "decode_noalloc vs decode")
        # and both against the float64 oracle (bf16 tensor-core operands at head_dim 128)
        o_ref, l_ref = O.decode(q.cpu(), kc.cpu(), vc.cpu(), params, stage_bf16=decode_staged(q.shape[-1]))
        assert_close(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, "decode_noalloc vs oracle")


def test_decode_noalloc_rejects_shapes_beyond_its_scratch():
    from position_remapping_b200 import ropeattn as ra
    # 512 x 32 heads x 128 x 4 B of partials alone is 8 MiB > the 4 MiB scratch
    assert ra.decode_workspace_size(512, 256, 32, 32, 128) > (4 << 20)
    cp = ra.to_cparams(MapParams(O.STANDARD))
    null = ctypes.c_void_p(0)
    rc = ra.lib.ropeattn_decode_noalloc(null, null, null, null, null, 512, 256, 32, 32, 128, ctypes.byref(cp), null)
    assert rc == ra.ERR_WORKSPACE
    assert "scratch" in ra.lib.ropeattn_last_error().decode()
