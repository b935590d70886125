"""The C-ABI library: it loads without a GPU, exports every symbol the header
declares, its parameter struct matches the C layout, and host-side argument
checks reject bad calls before any launch. CPU only."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ropeattn.h")


@pytest.fixture(scope="module")
def ra():
    from position_remapping_b200 import build
    build.build()
    from position_remapping_b200 import ropeattn
    return ropeattn


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ropeattn_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(ra):
    names = declared_functions()
    assert len(names) >= 8
    lib = ctypes.CDLL(ra.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(ra.EXPORTS)
    out = subprocess.run(["nm", "-D", "--defined-only", ra.LIB_PATH], capture_output=True, text=True).stdout
    for n in names:
        assert re.search(rf"\bT {n}\b", out), n


def test_library_has_no_libcuda_dependency(ra):
    out = subprocess.run(["ldd", ra.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out


def test_param_struct_layout_matches_c(ra):
    prog = r'''
#include <stdio.h>
#include <stddef.h>
#include "ropeattn.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(ropeattn_params),
    offsetof(ropeattn_params, kind), offsetof(ropeattn_params, fixed_group),
    offsetof(ropeattn_params, rope_base), offsetof(ropeattn_params, interp),
    offsetof(ropeattn_params, seg1_len), offsetof(ropeattn_params, term_start), offsetof(ropeattn_params, window),
    offsetof(ropeattn_params, w0), offsetof(ropeattn_params, w_pretrained), offsetof(ropeattn_params, softmax_scale),
    offsetof(ropeattn_params, pairing), offsetof(ropeattn_params, reserved));
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "t.c")
        exe = os.path.join(d, "t")
        open(c, "w").write(prog)
        subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        got = list(map(int, subprocess.run([exe], capture_output=True, text=True).stdout.split()))
    P = ra.CParams
    want = [ctypes.sizeof(P)] + [getattr(P, f).offset for f in
            ("kind", "fixed_group", "rope_base", "interp", "seg1_len", "term_start", "window", "w0", "w_pretrained",
             "softmax_scale", "pairing", "reserved")]
    assert got == want


def _p(**kw):
    from position_remapping_b200.inputs import MapParams
    return MapParams(**kw)


def test_host_argument_checks(ra):
    from position_remapping_b200.inputs import BIFOCAL, ENDPROMPT, NOPE, PERIODIC, STANDARD
    lib = ra.lib
    cp = ra.to_cparams
    nullp = ctypes.c_void_p(0)
    # bad head_dim, head ratio: rejected before any device work
    for D, Hq, Hkv in ((96, 4, 2), (128, 6, 4), (64, 0, 1)):
        rc = lib.ropeattn_prefill(nullp, nullp, nullp, nullp, nullp, 1, 16, Hq, Hkv, D,
                                  ctypes.byref(cp(_p(kind=STANDARD))), nullp, 0, nullp)
        assert rc == ra.ERR_INVALID_ARG
        assert lib.ropeattn_last_error().decode()
    # head_dim 256 passes the shape checks of every entry point (the prefill
    # runs it with one query tile per CTA)
    assert lib.ropeattn_prefill_workspace_size(ctypes.byref(cp(_p(kind=STANDARD))), 1, 4096, 2, 1, 256) == \
        4096 * 256 * 2 + 4096 * 128 * 8
    assert lib.ropeattn_prefill_workspace_size(ctypes.byref(cp(_p(kind=STANDARD))), 1, 4096, 2, 1, 96) == 0
    bif = ctypes.byref(cp(_p(kind=BIFOCAL, w0=64, w_pretrained=1024)))
    assert lib.ropeattn_prefill_chunk_workspace_size(bif, 1, 3000, 1096, 2, 1, 256) > 0
    assert lib.ropeattn_prefill_three_call_workspace_size(bif, 1, 4096, 2, 1, 256) > \
        lib.ropeattn_prefill_workspace_size(bif, 1, 4096, 2, 1, 256) > 0
    assert lib.ropeattn_decode_workspace_size(1, 1000, 2, 1, 256) > 0
    # the backward offers head_dim 64 and 128 only: no workspace size and a
    # rejection before any device work for 256
    std = ctypes.byref(cp(_p(kind=STANDARD)))
    assert lib.ropeattn_prefill_backward_workspace_size(std, 1, 4096, 2, 1, 128) > 0
    assert lib.ropeattn_prefill_backward_workspace_size(std, 1, 4096, 2, 1, 256) == 0
    assert lib.ropeattn_prefill_backward(nullp, nullp, nullp, nullp, nullp, nullp, nullp, nullp, nullp, 1, 4096, 2, 1,
                                         256, std, nullp, 0, nullp) == ra.ERR_INVALID_ARG
    assert "64 and 128" in lib.ropeattn_last_error().decode()
    assert lib.ropeattn_decode(nullp, nullp, nullp, nullp, nullp, 1, 1000, 32, 1, 256,
                               ctypes.byref(cp(_p(kind=STANDARD))), nullp, 0, nullp) == ra.ERR_INVALID_ARG  # GQA 32
    assert "16" in lib.ropeattn_last_error().decode()
    bad = [_p(kind=9), _p(kind=PERIODIC, window=0), _p(kind=BIFOCAL, w0=-1, w_pretrained=8),
           _p(kind=BIFOCAL, w0=4, w_pretrained=0), _p(kind=ENDPROMPT, interp=0.5),
           _p(kind=STANDARD, rope_base=1.0), _p(kind=STANDARD, softmax_scale=-1.0),
           _p(kind=STANDARD, pairing=2), _p(kind=BIFOCAL, w0=4, w_pretrained=8, pairing=-1)]
    for p in bad:
        rc = lib.ropeattn_prefill(nullp, nullp, nullp, nullp, nullp, 1, 16, 2, 1, 64,
                                  ctypes.byref(cp(p)), nullp, 0, nullp)
        assert rc == ra.ERR_INVALID_ARG, p
    c = cp(_p(kind=STANDARD))
    c.reserved[1] = 3
    assert lib.ropeattn_prefill(nullp, nullp, nullp, nullp, nullp, 1, 16, 2, 1, 64, ctypes.byref(c),
                                nullp, 0, nullp) == ra.ERR_INVALID_ARG
    # null tensors with work to do
    assert lib.ropeattn_prefill(nullp, nullp, nullp, nullp, nullp, 1, 16, 2, 1, 64,
                                ctypes.byref(cp(_p(kind=NOPE))), nullp, 0, nullp) == ra.ERR_INVALID_ARG
    # empty problems are no-ops
    assert lib.ropeattn_prefill(nullp, nullp, nullp, nullp, nullp, 0, 16, 2, 1, 64,
                                ctypes.byref(cp(_p(kind=NOPE))), nullp, 0, nullp) == ra.OK
    assert lib.ropeattn_decode(nullp, nullp, nullp, nullp, nullp, 1, 0, 2, 1, 64,
                               ctypes.byref(cp(_p(kind=NOPE))), nullp, 0, nullp) == ra.OK
    # decode group-size limit
    assert lib.ropeattn_decode(nullp, nullp, nullp, nullp, nullp, 1, 64, 16, 2, 128,
                               ctypes.byref(cp(_p(kind=NOPE))), nullp, 0, nullp) == ra.ERR_INVALID_ARG
    # posmap: BIFOCAL needs the remote output
    G = ctypes.c_int32(0)
    assert lib.ropeattn_posmap(ctypes.byref(cp(_p(kind=BIFOCAL, w0=2, w_pretrained=8))), 10, nullp, nullp,
                               ctypes.byref(G), nullp) == ra.ERR_INVALID_ARG
    assert lib.ropeattn_posmap(ctypes.byref(cp(_p(kind=BIFOCAL, w0=2, w_pretrained=8))), 0, nullp, nullp,
                               ctypes.byref(G), nullp) == ra.OK and G.value == 1


def test_cache_write_argument_checks(ra):
    from position_remapping_b200.inputs import BIFOCAL, STANDARD
    lib = ra.lib
    nullp = ctypes.c_void_p(0)
    p = ctypes.byref(ra.to_cparams(_p(kind=BIFOCAL, w0=4, w_pretrained=8)))
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: rejected before any device work
    # rows past the end of the cache
    assert lib.ropeattn_cache_write(fake, fake, fake, fake, 1, 90, 20, 100, 2, 64, p, nullp) == ra.ERR_INVALID_ARG
    # negative sizes, bad head_dim
    assert lib.ropeattn_cache_write(fake, fake, fake, fake, 1, -1, 2, 100, 2, 64, p, nullp) == ra.ERR_INVALID_ARG
    assert lib.ropeattn_cache_write(fake, fake, fake, fake, 1, 0, 2, 100, 2, 96, p, nullp) == ra.ERR_INVALID_ARG
    # v and v_cache must come together; k must be given
    assert lib.ropeattn_cache_write(fake, fake, fake, nullp, 1, 0, 2, 100, 2, 64, p, nullp) == ra.ERR_INVALID_ARG
    assert lib.ropeattn_cache_write(nullp, nullp, fake, nullp, 1, 0, 2, 100, 2, 64, p, nullp) == ra.ERR_INVALID_ARG
    # misaligned pointers (the kernel moves 16-byte groups)
    for off in (2, 4, 8):
        odd = ctypes.c_void_p((1 << 20) + off)
        assert lib.ropeattn_cache_write(odd, nullp, fake, nullp, 1, 0, 2, 100, 2, 64, p, nullp) == ra.ERR_INVALID_ARG
        assert lib.ropeattn_cache_write(fake, nullp, odd, nullp, 1, 0, 2, 100, 2, 64, p, nullp) == ra.ERR_INVALID_ARG
        assert "16-byte" in lib.ropeattn_last_error().decode()
    # nothing to write
    q = ctypes.byref(ra.to_cparams(_p(kind=STANDARD)))
    assert lib.ropeattn_cache_write(nullp, nullp, nullp, nullp, 1, 5, 0, 100, 2, 64, q, nullp) == ra.OK


def test_workspace_sizes(ra):
    from position_remapping_b200.inputs import WORKLOADS
    w = WORKLOADS["bifocal_prefill_s131072"]
    n = ra.prefill_workspace_size(w.params, w.B, w.S, w.Hq, w.Hkv, w.D)
    # two rotated key copies + two query angle tables
    assert n == 2 * (w.B * w.S * w.Hkv * w.D * 2) + 2 * (w.S * w.D // 2 * 8)
    nope = WORKLOADS["nope_s32768"]
    assert ra.prefill_workspace_size(nope.params, nope.B, nope.S, nope.Hq, nope.Hkv, nope.D) == 0
    # a bifocal map that fits the pretrained window is the standard map: one copy
    short = w.params.replace(w_pretrained=1 << 20)
    assert ra.prefill_workspace_size(short, 1, 4096, 32, 8, 128) == 4096 * 8 * 128 * 2 + 4096 * 64 * 8
    assert ra.decode_workspace_size(1, 131072, 16, 8, 128) > 0
    # half-split pairing adds a copy of q in adjacent order (not for NOPE, which rotates nothing)
    half = w.params.replace(pairing=1)
    assert ra.prefill_workspace_size(half, w.B, w.S, w.Hq, w.Hkv, w.D) == n + w.B * w.S * w.Hq * w.D * 2
    assert ra.prefill_workspace_size(nope.params.replace(pairing=1), nope.B, nope.S, nope.Hq, nope.Hkv, nope.D) == 0
    assert (ra.prefill_chunk_workspace_size(half, 1, 4096, 1000, 32, 8, 128) ==
            ra.prefill_chunk_workspace_size(w.params, 1, 4096, 1000, 32, 8, 128) + 1000 * 32 * 128 * 2)


def test_binding_checks_tensors_before_the_call(ra):
    # the C ABI sees only pointers: dtype, shape, layout and device are
    # checked by the binding, before any library call (CPU tensors here)
    import torch
    from position_remapping_b200.inputs import BIFOCAL
    p = _p(kind=BIFOCAL, w0=4, w_pretrained=8)
    q = torch.zeros((1, 16, 2, 64), dtype=torch.bfloat16)
    k = torch.zeros((1, 16, 1, 64), dtype=torch.bfloat16)
    cases = [
        lambda: ra.prefill(q.float(), k, k, p),                        # wrong dtype
        lambda: ra.prefill(q[0], k, k, p),                             # wrong rank
        lambda: ra.prefill(q, k, k[:, :8], p),                         # v does not match k
        lambda: ra.prefill(q, k[:, :8], k[:, :8], p),                  # k rows do not match q
        lambda: ra.prefill(q.transpose(1, 2), k, k, p),                # not contiguous
        lambda: ra.prefill(q, k, k, p),                                # not on a CUDA device
        lambda: ra.decode(q[:, 0], k, k.float(), p),                   # v_cache dtype
        lambda: ra.decode(q[:, 0, :, :32].contiguous(), k, k, p),      # head_dim mismatch
        lambda: ra.cache_write(k, k, k, None, p, 0),                   # v without v_cache
        lambda: ra.prefill_chunk(q, k, k, p, 4),                       # cache shorter than start + count
    ]
    for i, fn in enumerate(cases):
        with pytest.raises((ValueError, TypeError)):
            fn()


def test_binding_rejects_tensors_of_another_device(ra, monkeypatch):
    # every tensor must live on the current device (the library launches there
    # and encodes its pointers into TMA maps); the device is faked here, so no
    # kernel and no GPU are involved
    import torch
    from position_remapping_b200.inputs import BIFOCAL
    p = _p(kind=BIFOCAL, w0=4, w_pretrained=8)
    q = torch.zeros((1, 16, 2, 64), dtype=torch.bfloat16)
    k = torch.zeros((1, 16, 1, 64), dtype=torch.bfloat16)
    ws = torch.zeros(1024, dtype=torch.uint8)
    other = {id(k): 1}                                       # k claims cuda:1, the rest cuda:0
    monkeypatch.setattr(ra, "_current_device", lambda: 0)
    monkeypatch.setattr(ra, "_device_of", lambda t: ("cuda", other.get(id(t), 0)))
    called = []
    monkeypatch.setattr(ra, "_check", lambda rc: called.append(rc))
    for fn in (lambda: ra.prefill(q, k, k, p, workspace=ws),
               lambda: ra.decode(q[:, 0].contiguous(), k, k, p, workspace=ws),
               lambda: ra.cache_write(k, k, q, q, p, 0)):
        with pytest.raises(ValueError, match="cuda:1"):
            fn()
    other.clear()
    other[id(ws)] = 2                                        # only the workspace elsewhere
    with pytest.raises(ValueError, match="cuda:2"):
        ra.prefill(q, k, k, p, workspace=ws)
    assert not called                                        # no library call was made
