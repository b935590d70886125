"""Failure detection on the GPU without a fault: a kernel whose mbarrier wait
nothing completes gives up after a short limit through the library's bounded
wait, the status word reports the timeout, and the context keeps working."""
import time

import pytest
import torch

import oracle as O
from parity_util import assert_close, decode_staged
from position_remapping_b200.inputs import MapParams, make_qkv

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_survives():
    from position_remapping_b200 import ropeattn as ra
    ra.status()                                   # start from a clean status word
    t0 = time.perf_counter()
    res = ra.wait_selftest(limit_ns=2_000_000)    # 2 ms
    elapsed = time.perf_counter() - t0
    assert res == 0                               # the wait gave up
    assert elapsed < 5.0
    with pytest.raises(ra.RopeAttnError) as e:
        ra.status()
    assert e.value.code == ra.ERR_TIMEOUT
    ra.status()                                   # reading cleared it
    # the context is usable: a decode right after still matches the oracle
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=50, w_pretrained=300)
    q, kc, vc = make_qkv(1, 1000, 4, 2, 128, seed=91, q_len=1)
    out, lse = ra.decode(q.cuda(), kc.cuda(), vc.cuda(), params)
    torch.cuda.synchronize()
    ra.status()
    ref_o, ref_l = O.decode(q, kc, vc, params, stage_bf16=decode_staged(128))
    assert_close(out.cpu().numpy(), lse.cpu().numpy(), ref_o, ref_l, "after timeout")


def test_selftest_argument_checks():
    from position_remapping_b200 import ropeattn as ra
    with pytest.raises(ra.RopeAttnError) as e:
        ra.wait_selftest(limit_ns=10)
    assert e.value.code == ra.ERR_INVALID_ARG
