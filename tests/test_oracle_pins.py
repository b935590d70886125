"""Pins of the float64 oracle against facts fixed outside the oracle itself:
hand-worked values from the pages' definitions (tests/golden), closed forms,
library routines (torch SDPA in float64, complex multiplication), invariants
the pages state, and brute force on tiny inputs. CPU only."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from conftest import read_golden
from position_remapping_b200.inputs import MapParams, make_qkv


# ----------------------------------------------------------------------------
# bf16 rounding helper: against torch's float32 -> bfloat16 conversion (RNE)
# ----------------------------------------------------------------------------
def test_round_bf16_matches_torch_conversion():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(200000, generator=g) * 3.0
    # exact ties: 8 significant bits plus a half ulp
    ties = torch.tensor([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 2.0 + 2 ** -7,
                         1.5 + 2 ** -9, 0.0, 1.0, -2.5], dtype=torch.float32)
    x = torch.cat([x, ties])
    want = x.to(torch.bfloat16).double().numpy()
    got = O.round_bf16(x.double().numpy())
    assert np.array_equal(got, want)


# ----------------------------------------------------------------------------
# RoPE (Periodic RoPE §3.1 Eq. 1-2)
# ----------------------------------------------------------------------------
def test_frequencies_closed_form():
    # base 10^4: theta_i = 10^(-8i/D); for D = 8 that is 10^0 .. 10^-3
    assert np.allclose(O.rope_frequencies(8, 1e4), [1.0, 0.1, 0.01, 0.001], rtol=1e-15)
    assert np.allclose(O.rope_frequencies(4, 1e4), [1.0, 0.01], rtol=1e-15)
    # interpolation divides every frequency by s
    assert np.allclose(O.rope_frequencies(4, 1e4, 8.0), [0.125, 0.00125], rtol=1e-15)
    # base 10^6, D = 128: the slowest frequency is 10^(-6*126/128)
    f = O.rope_frequencies(128, 1e6)
    assert f.shape == (64,) and f[0] == 1.0
    assert math.isclose(f[-1], 10 ** (-6 * 126 / 128), rel_tol=1e-13)


def test_rotation_matrix_group_properties():
    f = O.rope_frequencies(16, 1e4)
    I = np.eye(16)
    assert np.allclose(O.rotation_matrix(0, f), I)
    for a, b in [(3, 5), (1000, -17), (131071, 4096)]:
        Ra, Rb = O.rotation_matrix(a, f), O.rotation_matrix(b, f)
        assert np.allclose(Ra.T @ Ra, I, atol=1e-13)
        assert math.isclose(np.linalg.det(Ra), 1.0, rel_tol=1e-12)
        # R_a R_b = R_{a+b} (Jet-Long §3.2) and R_a^T R_b = R_{b-a} (Eq. 3)
        assert np.allclose(Ra @ Rb, O.rotation_matrix(a + b, f), atol=1e-9)
        assert np.allclose(Ra.T @ Rb, O.rotation_matrix(b - a, f), atol=1e-9)


def test_rotation_sign_convention():
    # theta_0 = 1: R_t e_0 = (cos t, sin t, 0, ...), R_t e_1 = (-sin t, cos t, 0, ...)
    f = O.rope_frequencies(4, 1e4)
    for t in (1, 2, 7):
        R = O.rotation_matrix(t, f)
        assert np.allclose(R[:, 0], [math.cos(t), math.sin(t), 0, 0])
        assert np.allclose(R[:, 1], [-math.sin(t), math.cos(t), 0, 0])
        # second pair rotates at 0.01 rad per position
        assert np.allclose(R[:, 2], [0, 0, math.cos(0.01 * t), math.sin(0.01 * t)])


def test_rotate_matches_matrix_and_complex_form():
    rng = np.random.default_rng(1)
    D = 64
    f = O.rope_frequencies(D, 5e5, 2.0)
    x = rng.standard_normal((7, D))
    pos = np.array([0, 1, 5, 100, 8191, 65535, 131071])
    got = O.rotate(x, pos, f)
    for n, p in enumerate(pos):
        assert np.allclose(got[n], O.rotation_matrix(p, f) @ x[n], atol=1e-12)
    # complex form: (x_2i + i x_2i+1) * exp(i p theta_i)
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(1j * pos[:, None] * f[None, :])
    want = np.empty_like(x)
    want[:, 0::2], want[:, 1::2] = z.real, z.imag
    assert np.allclose(got, want, atol=1e-12)


def test_relative_offset_identity():
    # Eq. 3: <R_t q, R_s k> depends only on t - s
    rng = np.random.default_rng(2)
    D = 32
    f = O.rope_frequencies(D, 1e4)
    q, k = rng.standard_normal(D), rng.standard_normal(D)
    base = O.rotate(q[None], np.array([9]), f) @ O.rotate(k[None], np.array([4]), f).T
    for c in (1, 100, 77777):
        sh = O.rotate(q[None], np.array([9 + c]), f) @ O.rotate(k[None], np.array([4 + c]), f).T
        assert math.isclose(base.item(), sh.item(), rel_tol=1e-9, abs_tol=1e-9)


# ----------------------------------------------------------------------------
# position maps
# ----------------------------------------------------------------------------
def test_periodic_golden_offsets():
    for W, t, tp, pt, ptp, off, case in read_golden("periodic_offsets.txt"):
        W, t, tp = int(W), int(t), int(tp)
        assert int(O.periodic_position(t, W)) == int(pt)
        assert int(O.periodic_position(tp, W)) == int(ptp)
        assert int(O.periodic_position(t, W)) - int(O.periodic_position(tp, W)) == int(off)
        if case == "1":
            assert int(off) == t - tp
        elif case == "2":
            assert int(off) == (t - tp) - W


def test_periodic_prop1_bruteforce():
    # Proposition 1: two tokens with the same phi never share a causal window
    for W in range(1, 10):
        phi = O.periodic_position(np.arange(200), W)
        for q in range(200):
            win = phi[max(0, q - W + 1): q + 1]
            assert len(set(win.tolist())) == len(win)


def test_periodic_head_is_standard():
    # Remark 1: positions below W are unchanged
    W = 64
    t = np.arange(W)
    assert np.array_equal(O.periodic_position(t, W), t)


def test_group_size_golden_and_in_distribution():
    for L, wp, G, fmax in read_golden("jetlong_group_size.txt"):
        L, wp = int(L), int(wp)
        assert O.group_size(L, wp) == int(G)
        assert int(O.remote_position(L - 1, O.group_size(L, wp))) == int(fmax)
    # every remote position stays inside the pretrained window, and G is the
    # smallest integer with that property (§3.1)
    for wp in (1, 3, 8, 100):
        for L in range(1, 12 * wp + 3):
            G = O.group_size(L, wp)
            assert int(O.remote_position(np.arange(L), G).max()) <= wp - 1
            if G > 1:
                assert (L - 1) // (G - 1) >= wp
            if L <= wp:
                assert G == 1


def test_remote_position_is_floor_division():
    for G in (1, 2, 3, 4, 7):
        for x in range(0, 50):
            assert int(O.remote_position(x, G)) == math.floor(x / G)


def test_endprompt_golden_positions():
    for n1, ts, t, p in read_golden("endprompt_positions.txt"):
        assert int(O.endprompt_position(int(t), int(n1), int(ts))) == int(p)
    # with PI factor 8 every position of the 64K range maps inside the 8K window
    assert 65535 / 8.0 < 8192


# ----------------------------------------------------------------------------
# attention: closed forms
# ----------------------------------------------------------------------------
def _unit_qk(S, qv, kv, v):
    """q/k identical unit pairs at every position, v given: shapes [1,S,1,D]."""
    D = len(qv)
    q = np.tile(np.asarray(qv, float), (1, S, 1, 1))
    k = np.tile(np.asarray(kv, float), (1, S, 1, 1))
    return q.reshape(1, S, 1, D), k.reshape(1, S, 1, D), np.asarray(v, float).reshape(1, S, 1, D)


def _closed(scores, vals):
    w = np.exp(np.asarray(scores))
    return (w[:, None] * np.asarray(vals)).sum(0) / w.sum(), math.log(w.sum())


@pytest.mark.parametrize("fn", ["fast", "brute"])
def test_zero_query_gives_window_mean(fn):
    # q = 0 -> every allowed score is 0: out = mean of allowed v, lse = ln(count)
    S, D = 13, 8
    rng = np.random.default_rng(3)
    v = rng.standard_normal((1, S, 2, D))
    k = rng.standard_normal((1, S, 2, D))
    q = np.zeros((1, S, 4, D))
    cases = [MapParams(O.STANDARD), MapParams(O.NOPE),
             MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=9, term_start=200),
             MapParams(O.PERIODIC, window=4), MapParams(O.PERIODIC, window=1),
             MapParams(O.BIFOCAL, rope_base=1e6, w0=2, w_pretrained=4)]
    for p in cases:
        run = O.prefill if fn == "fast" else O.brute_prefill
        out, lse = run(q, k, v, p) if fn == "brute" else run(q, k, v, p, stage_bf16=False)
        for t in range(S):
            lo = max(0, t - p.window + 1) if p.kind == O.PERIODIC else 0
            for h in range(4):
                assert np.allclose(out[0, t, h], v[0, lo:t + 1, h // 2].mean(0), atol=1e-12)
                assert math.isclose(lse[0, h, t], math.log(t + 1 - lo), abs_tol=1e-12)


@pytest.mark.parametrize("fn", ["fast", "brute"])
def test_two_dim_scores_closed_form(fn):
    """D = 2 (theta_0 = 1): with q = a e_0 and k = e_1 the score of (t, s) is
    a * scale * sin(a_t - b_s), sign-sensitive, so a transposed rotation, a
    wrong offset or a wrong routing changes the result."""
    a = 1.7
    S = 8
    rng = np.random.default_rng(4)
    vals = rng.standard_normal((S, 2))
    q, k, v = _unit_qk(S, [a, 0.0], [0.0, 1.0], vals)
    sc = a / math.sqrt(2.0)
    run = (lambda *x: O.prefill(*x, stage_bf16=False)) if fn == "fast" else O.brute_prefill
    # standard: offsets t - s
    out, lse = run(q, k, v, MapParams(O.STANDARD))
    t = 7
    w_out, w_lse = _closed([sc * math.sin(t - s) for s in range(8)], vals[:8])
    assert np.allclose(out[0, t, 0], w_out, atol=1e-12) and math.isclose(lse[0, 0, t], w_lse, abs_tol=1e-12)
    # periodic, W = 4: row 6 sees keys 3..6, phi = 3,0,1,2 vs phi(6) = 2 -> Case 2 offset for key 3
    out, lse = run(q, k, v, MapParams(O.PERIODIC, window=4))
    t = 6
    w_out, w_lse = _closed([sc * math.sin((t % 4) - (s % 4)) for s in range(3, 7)], vals[3:7])
    assert np.allclose(out[0, t, 0], w_out, atol=1e-12) and math.isclose(lse[0, 0, t], w_lse, abs_tol=1e-12)
    assert [(t % 4) - (s % 4) for s in range(3, 7)] == [-1, 2, 1, 0]
    # bifocal, L = 8, w_pre = 4 -> G = 2, w0 = 2: row 7 keys 5..7 local at (7, s),
    # keys 0..4 remote at (3, floor(s/2))
    out, lse = run(q, k, v, MapParams(O.BIFOCAL, w0=2, w_pretrained=4))
    t = 7
    offs = [3 - s // 2 for s in range(5)] + [7 - s for s in range(5, 8)]
    assert offs == [3, 3, 2, 2, 1, 2, 1, 0]
    w_out, w_lse = _closed([sc * math.sin(o) for o in offs], vals)
    assert np.allclose(out[0, t, 0], w_out, atol=1e-12) and math.isclose(lse[0, 0, t], w_lse, abs_tol=1e-12)
    # endprompt, n1 = 5, terminal at 20, interp 2: positions 0..4, 20, 21, 22
    out, lse = run(q, k, v, MapParams(O.ENDPROMPT, seg1_len=5, term_start=20, interp=2.0))
    pos = [0, 1, 2, 3, 4, 20, 21, 22]
    w_out, w_lse = _closed([sc * math.sin((pos[7] - pos[s]) / 2.0) for s in range(8)], vals)
    assert np.allclose(out[0, 7, 0], w_out, atol=1e-12) and math.isclose(lse[0, 0, 7], w_lse, abs_tol=1e-12)


# ----------------------------------------------------------------------------
# attention: library routine (torch SDPA in float64)
# ----------------------------------------------------------------------------
def _sdpa(q, k, v, mask=None):
    """q [S,H,D], k/v [S,Hkv,D] float64 -> torch SDPA with GQA expansion."""
    H, Hkv = q.shape[1], k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)
    kt = torch.from_numpy(np.repeat(k, H // Hkv, axis=1)).permute(1, 0, 2)
    vt = torch.from_numpy(np.repeat(v, H // Hkv, axis=1)).permute(1, 0, 2)
    if mask is None:
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    else:
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(mask))
    return o.permute(1, 0, 2).numpy()


def _complex_rope(x, pos, base, interp=1.0):
    """Independent RoPE: complex multiply by exp(i * pos * base^(-2i/D) / s)."""
    D = x.shape[-1]
    th = np.array([base ** (-(2.0 * i) / D) for i in range(D // 2)]) / interp
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * np.asarray(pos)[:, None, None] * th[None, None, :])
    out = np.empty_like(x)
    out[..., 0::2], out[..., 1::2] = z.real, z.imag
    return out


def test_nope_and_standard_match_sdpa():
    q, k, v = make_qkv(1, 97, 4, 2, 32, seed=11)
    qf, kf, vf = (O.to_f64(x)[0] for x in (q, k, v))
    out, lse = O.prefill(q, k, v, MapParams(O.NOPE), stage_bf16=False)
    assert np.allclose(out[0], _sdpa(qf, kf, vf), atol=1e-12)
    pos = np.arange(97)
    out, _ = O.prefill(q, k, v, MapParams(O.STANDARD, rope_base=1e4), stage_bf16=False)
    ref = _sdpa(_complex_rope(qf, pos, 1e4), _complex_rope(kf, pos, 1e4), vf)
    assert np.allclose(out[0], ref, atol=1e-12)


def test_periodic_and_endprompt_match_sdpa():
    S, W = 70, 16
    q, k, v = make_qkv(1, S, 2, 1, 16, seed=12)
    qf, kf, vf = (O.to_f64(x)[0] for x in (q, k, v))
    t = np.arange(S)
    mask = (t[:, None] >= t[None, :]) & (t[:, None] - t[None, :] <= W - 1)
    out, _ = O.prefill(q, k, v, MapParams(O.PERIODIC, window=W), stage_bf16=False)
    ref = _sdpa(_complex_rope(qf, t % W, 1e4), _complex_rope(kf, t % W, 1e4), vf, mask)
    assert np.allclose(out[0], ref, atol=1e-12)
    p = MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=50, term_start=60000)
    pos = np.where(t < 50, t, 60000 + t - 50)
    out, _ = O.prefill(q, k, v, p, stage_bf16=False)
    ref = _sdpa(_complex_rope(qf, pos, 5e5, 8.0), _complex_rope(kf, pos, 5e5, 8.0), vf)
    assert np.allclose(out[0], ref, atol=1e-12)


# ----------------------------------------------------------------------------
# attention: reductions and equivalences the pages state
# ----------------------------------------------------------------------------
def test_bifocal_reduces_to_standard():
    q, k, v = make_qkv(2, 40, 4, 2, 16, seed=13)
    std = O.prefill(q, k, v, MapParams(O.STANDARD, rope_base=1e6))
    # L <= w_pretrained -> G = 1 -> f(x) = x (Jet-Long §3)
    b1 = O.prefill(q, k, v, MapParams(O.BIFOCAL, rope_base=1e6, w0=3, w_pretrained=40))
    # w0 >= L-1 -> every key local
    b2 = O.prefill(q, k, v, MapParams(O.BIFOCAL, rope_base=1e6, w0=39, w_pretrained=7))
    for b in (b1, b2):
        assert np.array_equal(b[0], std[0]) and np.array_equal(b[1], std[1])


def test_periodic_short_sequence_is_standard():
    # Remark 1: a sequence no longer than W is standard causal RoPE
    q, k, v = make_qkv(1, 32, 2, 2, 16, seed=14)
    a = O.prefill(q, k, v, MapParams(O.PERIODIC, window=32))
    b = O.prefill(q, k, v, MapParams(O.STANDARD))
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_endprompt_degenerate_is_standard_and_shift_invariant():
    q, k, v = make_qkv(1, 30, 2, 1, 16, seed=15)
    std = O.prefill(q, k, v, MapParams(O.STANDARD), stage_bf16=False)
    a = O.prefill(q, k, v, MapParams(O.ENDPROMPT, seg1_len=10, term_start=10), stage_bf16=False)
    assert np.array_equal(a[0], std[0])
    # n1 = 0: every position shifted by term_start -> same scores (Eq. 3)
    b = O.prefill(q, k, v, MapParams(O.ENDPROMPT, seg1_len=0, term_start=12345), stage_bf16=False)
    assert np.allclose(b[0], std[0], atol=1e-10) and np.allclose(b[1], std[1], atol=1e-10)


@pytest.mark.parametrize("w0,wp,pairing", [(0, 5, 0), (3, 5, 0), (6, 4, 0), (11, 8, 0), (3, 5, 1)])
def test_three_call_merge_equals_routed(w0, wp, pairing):
    q, k, v = make_qkv(1, 33, 4, 2, 16, seed=16)
    p = MapParams(O.BIFOCAL, rope_base=1e4, w0=w0, w_pretrained=wp, pairing=pairing)
    a = O.prefill(q, k, v, p)
    b = O.prefill_three_call(q, k, v, p)
    assert np.allclose(a[0], b[0], atol=1e-10) and np.allclose(a[1], b[1], atol=1e-10)


def test_w0_zero_is_self_only_local():
    # w0 = 0: only the diagonal uses exact positions (Jet-Long §4.4)
    S = 12
    q, k, v = _unit_qk(S, [1.0, 0.0], [0.0, 1.0], np.eye(S, 2))
    p = MapParams(O.BIFOCAL, w0=0, w_pretrained=3)    # G = 4
    out, lse = O.prefill(q, k, v, p, stage_bf16=False)
    t = 11
    offs = [t // 4 - s // 4 for s in range(t)] + [0]
    _, w_lse = _closed([math.sin(o) / math.sqrt(2) for o in offs], np.eye(S, 2))
    assert math.isclose(lse[0, 0, t], w_lse, abs_tol=1e-12)


@pytest.mark.parametrize("kind", [O.STANDARD, O.ENDPROMPT, O.PERIODIC, O.NOPE, O.BIFOCAL])
@pytest.mark.parametrize("stage", [False, True])
def test_fast_matches_brute(kind, stage):
    params = {O.STANDARD: MapParams(O.STANDARD, rope_base=1e4),
              O.ENDPROMPT: MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=11, term_start=65500),
              O.PERIODIC: MapParams(O.PERIODIC, window=5),
              O.NOPE: MapParams(O.NOPE),
              O.BIFOCAL: MapParams(O.BIFOCAL, rope_base=1e6, w0=3, w_pretrained=6)}[kind]
    q, k, v = make_qkv(1, 19, 4, 2, 8, seed=17)
    a = O.prefill(q, k, v, params, stage_bf16=stage)
    b = O.brute_prefill(q, k, v, params, stage_bf16=stage)
    assert np.allclose(a[0], b[0], atol=1e-12) and np.allclose(a[1], b[1], atol=1e-12)
    rows = [0, 5, 18]
    c = O.prefill(q, k, v, params, rows=rows, stage_bf16=stage)
    assert np.allclose(c[0], a[0][:, rows], atol=1e-13) and np.allclose(c[1], a[1][:, :, rows], atol=1e-13)


# ----------------------------------------------------------------------------
# decode (Jet-Long §3.2)
# ----------------------------------------------------------------------------
def _cache(k_raw, params, D):
    """Rotate raw keys to their own positions with the independent complex
    form: the cache invariant of Eq. 4."""
    n = k_raw.shape[1]
    t = np.arange(n)
    if params.kind == O.NOPE:
        return k_raw.copy()
    interp = params.interp if params.kind == O.ENDPROMPT else 1.0
    if params.kind == O.PERIODIC:
        pos = t % params.window
    elif params.kind == O.ENDPROMPT:
        pos = np.where(t < params.seg1_len, t, params.term_start + t - params.seg1_len)
    else:
        pos = t
    return np.stack([_complex_rope(k_raw[b], pos, params.rope_base, interp) for b in range(k_raw.shape[0])])


@pytest.mark.parametrize("kind", [O.STANDARD, O.ENDPROMPT, O.PERIODIC, O.NOPE, O.BIFOCAL])
def test_decode_matches_definition_on_raw_keys(kind):
    params = {O.STANDARD: MapParams(O.STANDARD, rope_base=1e4),
              O.ENDPROMPT: MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=11, term_start=65500),
              O.PERIODIC: MapParams(O.PERIODIC, window=5),
              O.NOPE: MapParams(O.NOPE),
              O.BIFOCAL: MapParams(O.BIFOCAL, rope_base=1e6, w0=3, w_pretrained=6)}[kind]
    qf, kf, vf = make_qkv(2, 23, 4, 2, 8, seed=18, q_len=1)
    qn, kn, vn = O.to_f64(qf), O.to_f64(kf), O.to_f64(vf)
    a = O.decode(qn, _cache(kn, params, 8), vn, params)
    b = O.brute_decode(qn, kn, vn, params)
    assert np.allclose(a[0], b[0], atol=1e-12) and np.allclose(a[1], b[1], atol=1e-12)


def test_decode_equals_last_prefill_row():
    # the correction rotation reaches the prefill score of row n-1 (R_a R_b = R_{a+b})
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=5, w_pretrained=8)
    q, k, v = make_qkv(1, 30, 4, 2, 16, seed=19)
    qn, kn, vn = O.to_f64(q), O.to_f64(k), O.to_f64(v)
    pre = O.prefill(qn, kn, vn, params, rows=[29], stage_bf16=False)
    dec = O.decode(qn[:, 29], _cache(kn, params, 16), vn, params)
    assert np.allclose(dec[0], pre[0][:, 0], atol=1e-12)
    assert np.allclose(dec[1], pre[1][:, :, 0], atol=1e-12)


@pytest.mark.parametrize("kind", [O.STANDARD, O.ENDPROMPT, O.PERIODIC, O.NOPE, O.BIFOCAL])
def test_staged_decode_equals_last_row_from_cache(kind):
    # bf16 operand rounding of the decode (rotated query views, corrected
    # remote keys) is the rounding the chunked prefill from a cache applies to
    # the same row: prefill_from_cache rotates the raw query straight to f(t)
    # and each key by f(s) - s, decode goes through Delta q and Delta k (Eq. 6)
    params = {O.STANDARD: MapParams(O.STANDARD, rope_base=1e4),
              O.ENDPROMPT: MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=11, term_start=65500),
              O.PERIODIC: MapParams(O.PERIODIC, window=5),
              O.NOPE: MapParams(O.NOPE),
              O.BIFOCAL: MapParams(O.BIFOCAL, rope_base=1e6, w0=3, w_pretrained=6)}[kind]
    q, k, v = make_qkv(2, 29, 4, 2, 16, seed=36)
    qn, kn, vn = O.to_f64(q), O.to_f64(k), O.to_f64(v)
    cache = O.round_bf16(O.cache_keys(kn, params))          # a bf16 cache, as stored on the device
    a = O.decode(qn[:, 28], cache, vn, params, stage_bf16=True)
    b = O.prefill_from_cache(qn[:, 28:], cache, vn, params, 28, stage_bf16=True)
    assert np.allclose(a[0], b[0][:, 0], atol=1e-12) and np.allclose(a[1], b[1][:, :, 0], atol=1e-12)
    u = O.decode(qn[:, 28], cache, vn, params, stage_bf16=False)
    d = max(np.abs(a[0] - u[0]).max(), np.abs(a[1] - u[1]).max())
    if kind == O.NOPE:
        assert d == 0.0        # bf16 inputs, no rotation: nothing to round
    else:
        assert 1e-7 < d < 0.05  # the rounding is applied, and is of bf16 size


@pytest.mark.parametrize("kind", [O.STANDARD, O.ENDPROMPT, O.PERIODIC, O.NOPE, O.BIFOCAL])
def test_cache_keys_match_complex_form_and_offsets(kind):
    # Eq. 4: the cache entry of token t is its key rotated at the kind's
    # position of t, whatever the chunk it is written in
    params = {O.STANDARD: MapParams(O.STANDARD, rope_base=1e4),
              O.ENDPROMPT: MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=11, term_start=65500),
              O.PERIODIC: MapParams(O.PERIODIC, window=5),
              O.NOPE: MapParams(O.NOPE),
              O.BIFOCAL: MapParams(O.BIFOCAL, rope_base=1e6, w0=3, w_pretrained=6)}[kind]
    _, kf, _ = make_qkv(2, 23, 2, 2, 8, seed=31)
    kn = O.to_f64(kf)
    whole = O.cache_keys(kn, params)
    assert np.allclose(whole, _cache(kn, params, 8), atol=1e-12)
    parts = np.concatenate([O.cache_keys(kn[:, :7], params, 0), O.cache_keys(kn[:, 7:16], params, 7),
                            O.cache_keys(kn[:, 16:], params, 16)], axis=1)
    assert np.allclose(parts, whole, atol=1e-12)


def test_decode_over_growing_cache_crosses_group_changes():
    # Jet-Long §3.2: the cache written once (Eq. 4) serves every later step,
    # including the lengths where G = ceil(L / w_pre) changes; each step's
    # decode equals the last row of a prefill of that length (L = n)
    params = MapParams(O.BIFOCAL, rope_base=1e4, w0=3, w_pretrained=8)
    q, k, v = make_qkv(1, 26, 4, 2, 8, seed=32)
    qn, kn, vn = O.to_f64(q), O.to_f64(k), O.to_f64(v)
    cache = O.cache_keys(kn, params)
    Gs = set()
    for n in (8, 9, 16, 17, 24, 25, 26):
        Gs.add(O.group_size(n, params.w_pretrained))
        dec = O.decode(qn[:, n - 1], cache[:, :n], vn[:, :n], params)
        pre = O.prefill(qn[:, :n], kn[:, :n], vn[:, :n], params, rows=[n - 1], stage_bf16=False)
        assert np.allclose(dec[0], pre[0][:, 0], atol=1e-12)
        assert np.allclose(dec[1], pre[1][:, :, 0], atol=1e-12)
    assert Gs == {1, 2, 3, 4}


@pytest.mark.parametrize("kind", [O.STANDARD, O.ENDPROMPT, O.PERIODIC, O.NOPE, O.BIFOCAL])
def test_prefill_from_cache_equals_prefill_rows(kind):
    # a chunk of rows computed from the Eq. 4 cache (remote keys through the
    # correction rotation of Eq. 6) equals the same rows of the plain prefill
    params = {O.STANDARD: MapParams(O.STANDARD, rope_base=1e4),
              O.ENDPROMPT: MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=11, term_start=65500),
              O.PERIODIC: MapParams(O.PERIODIC, window=5),
              O.NOPE: MapParams(O.NOPE),
              O.BIFOCAL: MapParams(O.BIFOCAL, rope_base=1e6, w0=3, w_pretrained=6)}[kind]
    q, k, v = make_qkv(2, 27, 4, 2, 8, seed=33)
    qn, kn, vn = O.to_f64(q), O.to_f64(k), O.to_f64(v)
    cache = O.cache_keys(kn, params)
    for start in (0, 1, 13, 26):
        a = O.prefill_from_cache(qn[:, start:], cache, vn, params, start, stage_bf16=False)
        b = O.prefill(qn, kn, vn, params, rows=list(range(start, 27)), stage_bf16=False)
        assert np.allclose(a[0], b[0], atol=1e-12) and np.allclose(a[1], b[1], atol=1e-12)
        # the row and head selection (used at full size) picks the same values
        rows, heads = [r for r in (start, 20, 26) if r >= start], [3, 0]
        for staged in (False, True):
            full = O.prefill_from_cache(qn[:, start:], cache, vn, params, start, stage_bf16=staged)
            sel = O.prefill_from_cache(q[:, start:], cache, v, params, start, stage_bf16=staged, rows=rows,
                                       heads=heads)
            idx = [r - start for r in rows]
            assert np.allclose(sel[0], full[0][:, idx][:, :, heads], rtol=0, atol=1e-12)
            assert np.allclose(sel[1], full[1][:, heads][:, :, idx], rtol=0, atol=1e-12)


def test_fixed_group_positions_and_brute_force():
    # a single group size fixed up front: G does not follow L (Jet-Long §2.2
    # contrasts its dynamic G with this); f(t) = floor(t / G) as in Eq. 3
    for L in (5, 100, 10000):
        p = MapParams(O.BIFOCAL, rope_base=1e4, w0=3, fixed_group=3)
        loc, rem, G = O.position_maps(p, L)
        assert G == 3 and np.array_equal(rem, np.arange(L) // 3) and np.array_equal(loc, np.arange(L))
    assert O.bifocal_group(MapParams(O.BIFOCAL, w_pretrained=8), 20) == O.group_size(20, 8) == 3
    params = MapParams(O.BIFOCAL, rope_base=1e4, w0=2, fixed_group=5)
    q, k, v = make_qkv(1, 17, 2, 1, 8, seed=34)
    a = O.prefill(q, k, v, params, stage_bf16=False)
    b = O.brute_prefill(q, k, v, params)
    assert np.allclose(a[0], b[0], atol=1e-12) and np.allclose(a[1], b[1], atol=1e-12)
    qd, kd, vd = make_qkv(1, 17, 2, 1, 8, seed=35, q_len=1)
    qn, kn, vn = O.to_f64(qd), O.to_f64(kd), O.to_f64(vd)
    c = O.decode(qn, _cache(kn, params, 8), vn, params)
    d = O.brute_decode(qn, kn, vn, params)
    assert np.allclose(c[0], d[0], atol=1e-12) and np.allclose(c[1], d[1], atol=1e-12)


# ----------------------------------------------------------------------------
# half-split pairing: coordinates (i, i + D/2) turned by p * theta_i
# ----------------------------------------------------------------------------
def _complex_rope_half(x, pos, base, interp=1.0):
    """Independent half-split RoPE: the first and second halves of the head
    are the real and imaginary parts, multiplied by exp(i * pos * theta_i)."""
    D = x.shape[-1]
    P = D // 2
    th = np.array([base ** (-(2.0 * i) / D) for i in range(P)]) / interp
    z = (x[..., :P] + 1j * x[..., P:]) * np.exp(1j * np.asarray(pos)[:, None, None] * th[None, None, :])
    return np.concatenate([z.real, z.imag], axis=-1)


def _interleave(x):
    """(x_0, x_{D/2}, x_1, x_{D/2+1}, ...): half-split order to adjacent order."""
    P = x.shape[-1] // 2
    out = np.empty_like(x)
    out[..., 0::2], out[..., 1::2] = x[..., :P], x[..., P:]
    return out


def test_half_split_rotation_basis_vectors():
    # D = 8, theta = (1, 0.1, 0.01, 0.001): R e_i = cos e_i + sin e_{i+4},
    # R e_{i+4} = -sin e_i + cos e_{i+4}
    f = O.rope_frequencies(8, 1e4)
    for t in (1, 3, 1000):
        R = O.rotation_matrix(t, f, O.PAIR_HALF)
        for i, th in enumerate((1.0, 0.1, 0.01, 0.001)):
            c, s = math.cos(t * th), math.sin(t * th)
            col_i = np.zeros(8)
            col_i[i], col_i[i + 4] = c, s
            col_j = np.zeros(8)
            col_j[i], col_j[i + 4] = -s, c
            assert np.allclose(R[:, i], col_i, atol=1e-13)
            assert np.allclose(R[:, i + 4], col_j, atol=1e-13)
    assert O.pair_index(3, 16, O.PAIR_HALF) == (3, 11) and O.pair_index(3, 16) == (6, 7)


def test_half_split_group_properties_and_complex_form():
    D = 32
    f = O.rope_frequencies(D, 5e5, 4.0)
    I = np.eye(D)
    for a, b in [(3, 5), (70000, -17)]:
        Ra, Rb = O.rotation_matrix(a, f, O.PAIR_HALF), O.rotation_matrix(b, f, O.PAIR_HALF)
        assert np.allclose(Ra.T @ Ra, I, atol=1e-13)
        assert np.allclose(Ra @ Rb, O.rotation_matrix(a + b, f, O.PAIR_HALF), atol=1e-9)
        # the same rotation seen through the interleaving permutation
        Pi = _interleave(I).T        # Pi @ x = interleave(x)
        assert np.allclose(Ra, Pi.T @ O.rotation_matrix(a, f) @ Pi, atol=1e-13)
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 1, D))
    pos = np.array([0, 1, 9, 4096, 65535, 131071])
    got = O.rotate(x[:, 0], pos, f, O.PAIR_HALF)
    assert np.allclose(got, _complex_rope_half(x, pos, 5e5, 4.0)[:, 0], atol=1e-12)


_HALF_PARAMS = {
    O.STANDARD: MapParams(O.STANDARD, rope_base=1e4, pairing=1),
    O.ENDPROMPT: MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=11, term_start=65500, pairing=1),
    O.PERIODIC: MapParams(O.PERIODIC, window=5, pairing=1),
    O.BIFOCAL: MapParams(O.BIFOCAL, rope_base=1e6, w0=3, w_pretrained=6, pairing=1),
}


@pytest.mark.parametrize("kind", [O.STANDARD, O.ENDPROMPT, O.PERIODIC, O.BIFOCAL])
def test_half_split_prefill_brute_and_permutation(kind):
    params = _HALF_PARAMS[kind]
    q, k, v = make_qkv(1, 19, 4, 2, 8, seed=41)
    a = O.prefill(q, k, v, params, stage_bf16=False)
    b = O.brute_prefill(q, k, v, params)
    assert np.allclose(a[0], b[0], atol=1e-12) and np.allclose(a[1], b[1], atol=1e-12)
    # scores are unchanged when q and k are permuted alike: half-split on
    # (q, k) is adjacent pairing on the interleaved (q, k)
    adj = params.replace(pairing=0)
    qn, kn, vn = O.to_f64(q), O.to_f64(k), O.to_f64(v)
    c = O.prefill(_interleave(qn), _interleave(kn), vn, adj, stage_bf16=False)
    assert np.allclose(a[0], c[0], atol=1e-12) and np.allclose(a[1], c[1], atol=1e-12)
    # and it is a different map from adjacent pairing on the same inputs
    d = O.prefill(q, k, v, adj, stage_bf16=False)
    assert not np.allclose(a[0], d[0], atol=1e-6)


@pytest.mark.parametrize("kind", [O.STANDARD, O.PERIODIC, O.BIFOCAL])
def test_half_split_cache_and_decode(kind):
    params = _HALF_PARAMS[kind]
    qf, kf, vf = make_qkv(2, 23, 4, 2, 8, seed=42, q_len=1)
    qn, kn, vn = O.to_f64(qf), O.to_f64(kf), O.to_f64(vf)
    t = np.arange(23)
    pos = t % params.window if kind == O.PERIODIC else t
    cache = O.cache_keys(kn, params)
    want = np.stack([_complex_rope_half(kn[b], pos, params.rope_base) for b in range(2)])
    assert np.allclose(cache, want, atol=1e-12)
    a = O.decode(qn, cache, vn, params)
    b = O.brute_decode(qn, kn, vn, params)
    assert np.allclose(a[0], b[0], atol=1e-12) and np.allclose(a[1], b[1], atol=1e-12)


# ----------------------------------------------------------------------------
# backward of the prefill
# ----------------------------------------------------------------------------
_BWD_PARAMS = [
    ("standard", MapParams(O.STANDARD, rope_base=1e2)),
    ("endprompt", MapParams(O.ENDPROMPT, rope_base=1e3, interp=2.0, seg1_len=4, term_start=40)),
    ("periodic", MapParams(O.PERIODIC, rope_base=1e2, window=4)),
    ("nope", MapParams(O.NOPE)),
    ("bifocal", MapParams(O.BIFOCAL, rope_base=1e2, w0=2, w_pretrained=4)),
    ("bifocal_half", MapParams(O.BIFOCAL, rope_base=1e2, w0=1, w_pretrained=3, pairing=1)),
    ("bifocal_fixed", MapParams(O.BIFOCAL, rope_base=1e2, w0=3, fixed_group=2)),
]


@pytest.mark.parametrize("case", _BWD_PARAMS, ids=[c[0] for c in _BWD_PARAMS])
def test_backward_matches_finite_differences(case):
    # d/dx of sum(dout * out) by central differences of the forward oracle,
    # every element of q, k and v (GQA group of 2 so dk, dv collect heads)
    _, params = case
    rng = np.random.default_rng(61)
    B, S, Hq, Hkv, D = 1, 9, 2, 1, 4
    q, k, v = (rng.standard_normal(s) for s in ((B, S, Hq, D), (B, S, Hkv, D), (B, S, Hkv, D)))
    dout = rng.standard_normal((B, S, Hq, D))
    dq, dk, dv = O.prefill_backward(q, k, v, dout, params)

    def loss(qq, kk, vv):
        return float((O.prefill(qq, kk, vv, params, stage_bf16=False)[0] * dout).sum())

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": (q, k, v), "k": (q, k, v), "v": (q, k, v)}[name]
            ap = [xp if a is x else a for a in args]
            am = [xm if a is x else a for a in args]
            fd[idx] = (loss(*ap) - loss(*am)) / (2 * h)
        assert np.allclose(g, fd, rtol=1e-6, atol=1e-8), (name, np.abs(g - fd).max())


def test_backward_closed_forms():
    rng = np.random.default_rng(62)
    params = MapParams(O.BIFOCAL, rope_base=1e4, w0=2, w_pretrained=4)
    # one token: out = v_0, so dv = dout summed over the group, dq = dk = 0
    q, k, v = rng.standard_normal((1, 1, 4, 8)), rng.standard_normal((1, 1, 2, 8)), rng.standard_normal((1, 1, 2, 8))
    dout = rng.standard_normal((1, 1, 4, 8))
    dq, dk, dv = O.prefill_backward(q, k, v, dout, params)
    assert np.array_equal(dq, np.zeros_like(dq)) and np.array_equal(dk, np.zeros_like(dk))
    assert np.allclose(dv[0, 0, 0], dout[0, 0, 0] + dout[0, 0, 1]) and np.allclose(dv[0, 0, 1], dout[0, 0, 2] + dout[0, 0, 3])
    # zero queries: uniform attention over the allowed keys, so dk = 0 and
    # dv_s = sum over rows t that allow s of dout_t / (number of keys of t)
    S = 11
    for p in (params, MapParams(O.PERIODIC, window=3)):
        q = np.zeros((1, S, 1, 8))
        k, v = rng.standard_normal((1, S, 1, 8)), rng.standard_normal((1, S, 1, 8))
        dout = rng.standard_normal((1, S, 1, 8))
        _, dk, dv = O.prefill_backward(q, k, v, dout, p)
        assert np.allclose(dk, 0.0, atol=1e-15)
        want = np.zeros((S, 8))
        for t in range(S):
            keys = [s for s in range(S) if s <= t and (p.kind != O.PERIODIC or s > t - p.window)]
            for s in keys:
                want[s] += dout[0, t, 0] / len(keys)
        assert np.allclose(dv[0, :, 0], want, atol=1e-13)


@pytest.mark.parametrize("kind", [O.STANDARD, O.PERIODIC, O.ENDPROMPT, O.NOPE])
def test_staged_backward_is_the_backward_at_rounded_operands(kind):
    # for one position map, rounding R_p q to bf16 is the same as feeding the
    # unstaged backward q' = R_p^T round(R_p q): its rotated operand is then
    # exactly the rounded one (and likewise for k), so the two gradients of
    # the rotated operands agree, and dq, dk differ only by R_p^T
    params = {O.STANDARD: MapParams(O.STANDARD, rope_base=1e4),
              O.PERIODIC: MapParams(O.PERIODIC, rope_base=1e4, window=5),
              O.ENDPROMPT: MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=7, term_start=60000),
              O.NOPE: MapParams(O.NOPE)}[kind]
    q, k, v = make_qkv(1, 17, 4, 2, 8, seed=37)
    qn, kn, vn = O.to_f64(q), O.to_f64(k), O.to_f64(v)
    dout = np.random.default_rng(5).standard_normal(qn.shape)
    pos = O.position_maps(params, 17)[0]
    fr = O.rope_frequencies(8, params.rope_base, params.interp if kind == O.ENDPROMPT else 1.0)

    def requant(x):
        if kind == O.NOPE:
            return O.round_bf16(x)
        return np.stack([O.rotate(O.round_bf16(O.rotate(x[0, :, h], pos, fr)), -pos, fr)
                         for h in range(x.shape[2])], axis=1)[None]
    a = O.prefill_backward(qn, kn, vn, dout, params, stage_bf16=True)
    b = O.prefill_backward(requant(qn), requant(kn), vn, dout, params, stage_bf16=False)
    for x, y in zip(a, b):
        assert np.allclose(x, y, atol=1e-10)
    u = O.prefill_backward(qn, kn, vn, dout, params, stage_bf16=False)
    d = max(np.abs(x - y).max() for x, y in zip(a, u))
    assert (d == 0.0) if kind == O.NOPE else (1e-8 < d < 0.1)


def test_staged_bifocal_backward_is_close_to_unstaged():
    params = MapParams(O.BIFOCAL, rope_base=1e6, w0=3, w_pretrained=6)
    q, k, v = make_qkv(1, 19, 2, 1, 8, seed=38)
    dout = np.random.default_rng(6).standard_normal((1, 19, 2, 8))
    a = O.prefill_backward(q, k, v, dout, params, stage_bf16=True)
    u = O.prefill_backward(q, k, v, dout, params, stage_bf16=False)
    d = max(np.abs(x - y).max() / max(1.0, np.abs(y).max()) for x, y in zip(a, u))
    assert 1e-8 < d < 0.05


@pytest.mark.parametrize("params", [
    MapParams(O.STANDARD, rope_base=1e4),
    MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=25, term_start=60000),
    MapParams(O.PERIODIC, rope_base=1e4, window=9),
    MapParams(O.NOPE),
    MapParams(O.BIFOCAL, rope_base=1e6, w0=6, w_pretrained=12),
    MapParams(O.BIFOCAL, rope_base=1e4, w0=3, fixed_group=3, pairing=1),
], ids=["standard", "endprompt", "periodic", "nope", "bifocal", "bifocal_fixed_half"])
@pytest.mark.parametrize("staged", [False, True])
def test_backward_dq_rows_is_the_backward_on_those_rows(params, staged):
    # the row-block dq (used at full size) against the whole-prefill backward
    # that the finite-difference and closed-form pins above fix
    q, k, v = make_qkv(2, 40, 4, 2, 16, seed=51)
    g = torch.Generator("cpu").manual_seed(52)
    dout = torch.randn((2, 40, 4, 16), generator=g).to(torch.bfloat16)
    rows, heads = [0, 5, 17, 30, 39], [1, 3]
    dq, _, _ = O.prefill_backward(q, k, v, dout, params, stage_bf16=staged)
    dq_rows = O.prefill_backward_dq_rows(q, k, v, dout, params, rows, stage_bf16=staged, heads=heads)
    ref = dq[:, rows][:, :, heads]
    assert np.max(np.abs(dq_rows - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


@pytest.mark.parametrize("params", [
    MapParams(O.STANDARD, rope_base=1e4),
    MapParams(O.ENDPROMPT, rope_base=5e5, interp=8.0, seg1_len=25, term_start=60000),
    MapParams(O.PERIODIC, rope_base=1e4, window=9),
    MapParams(O.NOPE),
    MapParams(O.BIFOCAL, rope_base=1e6, w0=6, w_pretrained=12),
    MapParams(O.BIFOCAL, rope_base=1e4, w0=3, fixed_group=3, pairing=1),
], ids=["standard", "endprompt", "periodic", "nope", "bifocal", "bifocal_fixed_half"])
@pytest.mark.parametrize("staged", [False, True])
def test_backward_tail_is_the_backward_on_the_last_positions(params, staged):
    # causal attention: the last n keys get dk, dv only from the last n rows,
    # so the tail function's sums are complete and equal the whole-prefill
    # backward there (n = 0, a ragged n and the whole sequence)
    q, k, v = make_qkv(2, 40, 4, 2, 16, seed=53)
    g = torch.Generator("cpu").manual_seed(54)
    dout = torch.randn((2, 40, 4, 16), generator=g).to(torch.bfloat16)
    dq, dk, dv = O.prefill_backward(q, k, v, dout, params, stage_bf16=staged)
    heads = [2, 3]                                    # the GQA group of kv head 1
    for n in (0, 7, 40):
        tq, tk, tv = O.prefill_backward_tail(q, k, v, dout, params, n, stage_bf16=staged, heads=heads)
        assert tq.shape == (2, n, 2, 16) and tk.shape == tv.shape == (2, n, 1, 16)
        for got, ref in ((tq, dq[:, 40 - n:][:, :, heads]), (tk, dk[:, 40 - n:, 1:2]), (tv, dv[:, 40 - n:, 1:2])):
            assert np.max(np.abs(got - ref), initial=0.0) <= 1e-12 * max(1.0, np.max(np.abs(ref), initial=0.0))


def test_backward_tail_needs_whole_groups():
    q, k, v = make_qkv(1, 10, 4, 2, 16, seed=55)
    with pytest.raises(ValueError):
        O.prefill_backward_tail(q, k, v, q, MapParams(O.NOPE), 3, heads=[0, 2, 3])
