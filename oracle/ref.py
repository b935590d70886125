"""Plain float64 CPU oracle of causal attention with RoPE at remapped positions.

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; never by the product path. It
shares no code, table or constant generator with the CUDA library.

What it computes, and where each step is defined:

* RoPE frequencies theta_i = base^(-2i/d), i = 0..d/2-1, and the
  block-diagonal 2x2 rotation R_t acting on coordinate pairs (2i, 2i+1):
  "Periodic RoPE for Infinite Context LLMs", §3.1 Eq. 1-2. The half-split
  variant (``pairing`` = 1) turns the pairs (i, i + d/2) by the same angles.
* Position interpolation divides every position by the factor s, a linear
  squeeze of the positions into the range seen in pre-training: "Jet-Long:
  Efficient Long-Context Extension with Dynamic Bifocal RoPE", §2.2; EndPrompt
  pairs its positions with it: "EndPrompt: Efficient Long-Context Extension
  via Terminal Anchoring", abstract and summary.
* Periodic position phi(t) = t mod W inside causal sliding-window attention
  over the W keys {t-W+1 .. t}: Periodic RoPE, §3.2 Eq. 4-5.
* NoPE causal attention A_ts = q.k / sqrt(d_h), s <= t: Periodic RoPE, §3.3
  Eq. 6 (this also fixes the softmax scale 1/sqrt(d) for every kind).
* EndPrompt two-segment positions: an intact first segment at 0..n1-1, then
  a terminal segment whose positions start near the target length
  (EndPrompt, abstract).
* Bifocal score: RoPE at (q, k) when q - k <= w0, else RoPE at (f(q), f(k)),
  with G = max(1, ceil(L / w_pretrained)) and f(x) = floor(x / G): Jet-Long,
  §3 Eq. 1, §3.1 Eq. 2-3.
* Decode with an untouched cache k_cache[k] = RoPE(x_k, k) (``cache_keys``)
  and the correction rotation by Delta = f(x) - x on the query and on each
  cached key: Jet-Long, §3.2 Eq. 4-6.
* The literal three-call inclusion-exclusion merge: Jet-Long, §3.3 Eq. 7
  (kept as a self-check; the routed softmax is the definition it reaches).

Readings where the pages leave a step open:
adjacent pairing (2i, 2i+1); natural-log LSE of the scaled scores; the local
set of the bifocal score is 0 <= q-k <= w0 inclusive; for prefill L = S; for
decode L = n, the cache length including the current token at n-1.

Floating point: everything is float64. ``stage_bf16=True`` rounds the rotated
q and k to bfloat16 (round to nearest even) before the dot products, because
the tensor-core prefill multiplies bf16 operands; this is a modelled input
rounding, not a change of the method.
"""
from __future__ import annotations

import math

import numpy as np

STANDARD, ENDPROMPT, PERIODIC, NOPE, BIFOCAL = 0, 1, 2, 3, 4
PAIR_ADJACENT, PAIR_HALF = 0, 1

__all__ = [
    "STANDARD", "ENDPROMPT", "PERIODIC", "NOPE", "BIFOCAL", "PAIR_ADJACENT", "PAIR_HALF",
    "round_bf16", "rope_frequencies", "pair_index", "rotation_matrix", "rotate",
    "periodic_position", "endprompt_position", "group_size", "bifocal_group", "remote_position",
    "position_maps", "softmax_scale", "prefill", "prefill_three_call", "prefill_backward",
    "prefill_backward_dq_rows", "prefill_backward_tail",
    "decode", "cache_keys", "prefill_from_cache", "brute_prefill", "brute_decode", "to_f64",
]


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------
def to_f64(x) -> np.ndarray:
    """torch tensor (any dtype, any device) or array -> float64 numpy."""
    if hasattr(x, "detach"):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (8 significant bits), ties
    to even. Written out with frexp so no library conversion is involved.
    Valid for normal-range values (|x| >= 2^-126 or x == 0), which is all the
    oracle ever rounds."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                   # x = m * 2^e, 0.5 <= |m| < 1
    r = np.round(m * 256.0)              # 8 significant bits; np.round is half-to-even
    return np.ldexp(r, e - 8)


def softmax_scale(D: int, params) -> float:
    """Periodic RoPE, §3.3 Eq. 6: scores are divided by sqrt(d_h)."""
    s = float(getattr(params, "softmax_scale", 0.0) or 0.0)
    return s if s > 0.0 else 1.0 / math.sqrt(D)


# ----------------------------------------------------------------------------
# RoPE (Periodic RoPE §3.1 Eq. 1-2; interpolation: Jet-Long §2.2)
# ----------------------------------------------------------------------------
def rope_frequencies(D: int, base: float, interp: float = 1.0) -> np.ndarray:
    """theta_i = 1 / base^(2i/D) for i = 0..D/2-1, divided by the
    interpolation factor s (angle = (p / s) * theta_i)."""
    i = np.arange(D // 2, dtype=np.float64)
    return (1.0 / np.power(float(base), 2.0 * i / D)) / float(interp)


def pair_index(i: int, D: int, pairing: int = PAIR_ADJACENT):
    """The coordinates (a, b) that rotation pair i turns: (2i, 2i+1) as in
    the block-diagonal Eq. 2, or (i, i + D/2) for half-split pairing."""
    return (i, i + D // 2) if pairing == PAIR_HALF else (2 * i, 2 * i + 1)


def rotation_matrix(p: float, freqs: np.ndarray, pairing: int = PAIR_ADJACENT) -> np.ndarray:
    """The D x D rotation R_p of Eq. 2: pair i = (a, b) gets the block
    [[cos(p th_i), -sin(p th_i)], [sin(p th_i), cos(p th_i)]] on rows/cols
    (a, b) (block-diagonal for adjacent pairing)."""
    D = 2 * len(freqs)
    R = np.zeros((D, D), dtype=np.float64)
    for i, th in enumerate(freqs):
        a, b = pair_index(i, D, pairing)
        c, s = math.cos(p * th), math.sin(p * th)
        R[a, a] = c
        R[a, b] = -s
        R[b, a] = s
        R[b, b] = c
    return R


def rotate(x: np.ndarray, pos: np.ndarray, freqs: np.ndarray, pairing: int = PAIR_ADJACENT) -> np.ndarray:
    """Apply R_{pos[n]} to x[..., n, :] (the action of Eq. 2 without forming
    the matrix). x: [..., N, D]; pos: [N] (integer-valued)."""
    x = np.asarray(x, dtype=np.float64)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * freqs[None, :]   # [N, D/2]
    c, s = np.cos(ang), np.sin(ang)
    P = len(freqs)
    first = slice(0, P) if pairing == PAIR_HALF else slice(0, None, 2)
    second = slice(P, None) if pairing == PAIR_HALF else slice(1, None, 2)
    x0, x1 = x[..., first], x[..., second]
    out = np.empty_like(x)
    out[..., first] = x0 * c - x1 * s
    out[..., second] = x0 * s + x1 * c
    return out


# ----------------------------------------------------------------------------
# position maps
# ----------------------------------------------------------------------------
def periodic_position(t, W: int):
    """Periodic RoPE §3.2 Eq. 4: phi(t) = t mod W."""
    return np.asarray(t, dtype=np.int64) % int(W)


def endprompt_position(t, n1: int, term_start: int):
    """EndPrompt two-segment positions: the first segment keeps 0..n1-1, the
    terminal segment continues from ``term_start`` (placed near the target
    length)."""
    t = np.asarray(t, dtype=np.int64)
    return np.where(t < n1, t, term_start + (t - n1))


def group_size(L: int, w_pretrained: int) -> int:
    """Jet-Long §3.1 Eq. 2: G = max(1, ceil(L / w_pretrained))."""
    return max(1, -(-int(L) // int(w_pretrained)))


def bifocal_group(params, L: int) -> int:
    """G of a BIFOCAL map for length L: the dynamic schedule of Eq. 2, or a
    single group size fixed up front (``fixed_group`` > 0), the grouping the
    baselines Jet-Long compares against use (Jet-Long §2.2)."""
    fixed = int(getattr(params, "fixed_group", 0) or 0)
    return fixed if fixed > 0 else group_size(L, params.w_pretrained)


def remote_position(t, G: int):
    """Jet-Long §3.1 Eq. 3: f(x) = floor(x / G)."""
    return np.asarray(t, dtype=np.int64) // int(G)


def position_maps(params, L: int):
    """(pos_local, pos_remote or None, G) for token indices 0..L-1.

    pos_local is the position RoPE uses for the kind (for BIFOCAL the exact
    position of the local window); pos_remote is f(t) for BIFOCAL only. NOPE
    returns zeros (unused). G is 1 unless the kind is BIFOCAL."""
    t = np.arange(int(L), dtype=np.int64)
    k = int(params.kind)
    if k == STANDARD:
        return t, None, 1
    if k == ENDPROMPT:
        return endprompt_position(t, params.seg1_len, params.term_start), None, 1
    if k == PERIODIC:
        return periodic_position(t, params.window), None, 1
    if k == NOPE:
        return np.zeros_like(t), None, 1
    if k == BIFOCAL:
        G = bifocal_group(params, L)
        return t, remote_position(t, G), G
    raise ValueError(f"unknown kind {k}")


def _pairing(params) -> int:
    return int(getattr(params, "pairing", 0) or 0)


def _freqs(params, D):
    interp = float(getattr(params, "interp", 1.0) or 1.0) if int(params.kind) == ENDPROMPT else 1.0
    return rope_frequencies(D, params.rope_base, interp)


# ----------------------------------------------------------------------------
# prefill: the routed softmax, written as its plain definition
# ----------------------------------------------------------------------------
def _allowed(params, t: int, s: np.ndarray) -> np.ndarray:
    """Keys s a query at t attends to: causal s <= t; Periodic RoPE adds the
    window {t-W+1 .. t} (§3.2)."""
    ok = s <= t
    if int(params.kind) == PERIODIC:
        ok &= s >= t - int(params.window) + 1
    return ok


def _softmax_rows(scores: np.ndarray, ok: np.ndarray, v: np.ndarray):
    """out = sum softmax(scores) v over the allowed keys; lse = ln sum exp."""
    sc = np.where(ok, scores, -np.inf)
    m = sc.max(axis=-1, keepdims=True)
    e = np.where(ok, np.exp(sc - m), 0.0)
    l = e.sum(axis=-1, keepdims=True)
    out = (e @ v) / l
    lse = (m + np.log(l))[..., 0]
    return out, lse


def prefill(q, k, v, params, rows=None, stage_bf16: bool = True):
    """Causal attention with RoPE at remapped positions (every kind).

    q [B,S,Hq,D], k/v [B,S,Hkv,D] (torch or numpy). Returns (out, lse):
    out [B,R,Hq,D], lse [B,Hq,R] for the R = len(rows) query rows (all rows
    when ``rows`` is None). GQA: q head h reads kv head h // (Hq // Hkv).

    score(t,s) = scale * <R_a q_t, R_b k_s>, with (a, b) the positions the kind
    assigns; for BIFOCAL (a,b) = (t,s) if t-s <= w0 else (f(t), f(s)) with L = S.
    """
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    grp = Hq // Hkv
    rows = np.arange(S) if rows is None else np.asarray(rows, dtype=np.int64)
    scale = softmax_scale(D, params)
    kind = int(params.kind)
    freqs = _freqs(params, D)
    pr = _pairing(params)
    p_loc, p_rem, _G = position_maps(params, S)
    stage = round_bf16 if stage_bf16 else (lambda a: a)

    out = np.zeros((B, len(rows), Hq, D))
    lse = np.zeros((B, Hq, len(rows)))
    keys = np.arange(S)
    for b in range(B):
        for hk in range(Hkv):
            kk = k[b, :, hk, :]
            kl = kk if kind == NOPE else stage(rotate(kk, p_loc, freqs, pr))
            kr = stage(rotate(kk, p_rem, freqs, pr)) if kind == BIFOCAL else None
            for h in range(hk * grp, (hk + 1) * grp):
                # rows in chunks only to bound memory; each row is independent
                for c0 in range(0, len(rows), 64):
                    rr = rows[c0:c0 + 64]
                    nk = int(rr.max()) + 1            # keys beyond the last row are masked
                    # Periodic RoPE: keys before the window of the chunk's first
                    # row are outside every row's window {t-W+1..t}: skipped
                    k0 = max(0, int(rr.min()) - int(params.window) + 1) if kind == PERIODIC else 0
                    ks = keys[k0:nk]
                    ok = np.stack([_allowed(params, int(t), ks) for t in rr])
                    qq = q[b, rr, h, :]
                    ql = qq if kind == NOPE else stage(rotate(qq, p_loc[rr], freqs, pr))
                    sc = (ql @ kl[k0:nk].T) * scale                       # [r, nk - k0]
                    if kind == BIFOCAL:
                        qr = stage(rotate(qq, p_rem[rr], freqs, pr))
                        sr = (qr @ kr[k0:nk].T) * scale
                        local = (rr[:, None] - ks[None, :]) <= int(params.w0)
                        sc = np.where(local, sc, sr)
                    o, l = _softmax_rows(sc, ok, v[b, k0:nk, hk, :])
                    out[b, c0:c0 + 64, h, :] = o
                    lse[b, h, c0:c0 + 64] = l
    return out, lse


def prefill_three_call(q, k, v, params, stage_bf16: bool = True):
    """BIFOCAL prefill by the literal route of Jet-Long §3.3: (A) sliding
    window w0 with exact positions, (B) full causal with remote positions,
    (C) sliding window w0 with remote positions, each giving (O_X, l_X), then
    Eq. 7: O = (W_A O_A + W_B O_B - W_C O_C) / (W_A + W_B - W_C), with
    M = max(l_A, l_B, l_C) and W_X = exp(l_X - M). The merged LSE is
    M + ln(W_A + W_B - W_C). Self-check only: ``prefill`` is the definition."""
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    grp = Hq // Hkv
    scale = softmax_scale(D, params)
    freqs = _freqs(params, D)
    pr = _pairing(params)
    G = bifocal_group(params, S)
    t = np.arange(S)
    f = remote_position(t, G)
    stage = round_bf16 if stage_bf16 else (lambda a: a)
    causal = t[:, None] >= t[None, :]
    swa = causal & ((t[:, None] - t[None, :]) <= int(params.w0))
    out = np.zeros((B, S, Hq, D))
    lse = np.zeros((B, Hq, S))
    for b in range(B):
        for h in range(Hq):
            hk = h // grp
            qb, qr = stage(rotate(q[b, :, h], t, freqs, pr)), stage(rotate(q[b, :, h], f, freqs, pr))
            kb, kr = stage(rotate(k[b, :, hk], t, freqs, pr)), stage(rotate(k[b, :, hk], f, freqs, pr))
            vv = v[b, :, hk]
            OA, lA = _softmax_rows((qb @ kb.T) * scale, swa, vv)
            OB, lB = _softmax_rows((qr @ kr.T) * scale, causal, vv)
            OC, lC = _softmax_rows((qr @ kr.T) * scale, swa, vv)
            M = np.maximum(np.maximum(lA, lB), lC)
            WA, WB, WC = np.exp(lA - M), np.exp(lB - M), np.exp(lC - M)
            den = WA + WB - WC
            out[b, :, h] = (WA[:, None] * OA + WB[:, None] * OB - WC[:, None] * OC) / den[:, None]
            lse[b, h] = M + np.log(den)
    return out, lse


# ----------------------------------------------------------------------------
# backward of the prefill: gradients of a scalar loss through the routed
# softmax (the fine-tuning pass EndPrompt's method needs)
# ----------------------------------------------------------------------------
def prefill_backward(q, k, v, dout, params, stage_bf16: bool = False):
    """(dq, dk, dv) of the prefill (float64) for an upstream gradient ``dout``
    of ``out`` [B,S,Hq,D]; shapes of q, k, v. ``stage_bf16`` rounds the
    rotated queries and keys to bf16 wherever they are used (the scores and
    the products R_a q_t, R_b k_s of the chain rule), the operand rounding of
    the forward's ``stage_bf16``; the rounding itself is not differentiated.

    With P the row softmax of scale * score(t,s) over the allowed keys and
    score(t,s) = <R_a q_t, R_b k_s> ((a, b) the positions the kind assigns
    to the pair; for BIFOCAL (t, s) inside the local window, (f(t), f(s))
    outside it), the chain rule gives
      dv_s  = sum_t P(t,s) dout_t
      dP    = dout_t . v_s,     dS(t,s) = P(t,s) (dP(t,s) - sum_s' P(t,s') dP(t,s'))
      dq_t  = scale * sum_s dS(t,s) R_a^T R_b k_s
      dk_s  = scale * sum_t dS(t,s) R_b^T R_a q_t
    (R^T = R of the negated position). For BIFOCAL the sums split by the
    window into a local part (map t) and a remote part (map f). dk and dv of
    a KV head collect the heads of its GQA group."""
    q, k, v, dout = to_f64(q), to_f64(k), to_f64(v), to_f64(dout)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    grp = Hq // Hkv
    scale = softmax_scale(D, params)
    kind = int(params.kind)
    freqs = _freqs(params, D)
    pr = _pairing(params)
    p_loc, p_rem, _G = position_maps(params, S)
    t = np.arange(S)
    ok = np.stack([_allowed(params, int(r), t) for r in t])          # [S, S]
    local = (t[:, None] - t[None, :]) <= int(params.w0)
    stage = round_bf16 if stage_bf16 else (lambda a: a)

    def rot(x, pos):
        return x if kind == NOPE else rotate(x, pos, freqs, pr)

    def srot(x, pos):
        return x if kind == NOPE else stage(rotate(x, pos, freqs, pr))

    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(Hq):
            hk = h // grp
            ql, kl = srot(q[b, :, h], p_loc), srot(k[b, :, hk], p_loc)
            sc = ql @ kl.T
            if kind == BIFOCAL:
                qr, kr = srot(q[b, :, h], p_rem), srot(k[b, :, hk], p_rem)
                sc = np.where(local, sc, qr @ kr.T)
            sc = np.where(ok, sc * scale, -np.inf)
            m = sc.max(axis=1, keepdims=True)
            e = np.where(ok, np.exp(sc - m), 0.0)
            P = e / e.sum(axis=1, keepdims=True)
            do = dout[b, :, h]
            dv[b, :, hk] += P.T @ do
            dP = do @ v[b, :, hk].T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            if kind == BIFOCAL:
                dSl, dSr = np.where(local, dS, 0.0), np.where(local, 0.0, dS)
                dq[b, :, h] += scale * (rot(dSl @ kl, -p_loc) + rot(dSr @ kr, -p_rem))
                dk[b, :, hk] += scale * (rot(dSl.T @ ql, -p_loc) + rot(dSr.T @ qr, -p_rem))
            else:
                dq[b, :, h] += scale * rot(dS @ kl, -p_loc)
                dk[b, :, hk] += scale * rot(dS.T @ ql, -p_loc)
    return dq, dk, dv


def _backward_rows(q, k, v, dout, params, rows, stage_bf16, heads):
    """The chain rule of ``prefill_backward`` restricted to the query rows
    ``rows`` and the query heads ``heads``: yields, per (batch b, head h),
    the row softmax P and dS of those rows over all S keys with the operands
    the sums need. Only the slices these rows and heads touch are taken to
    float64, so a row costs O(S D) instead of the O(S^2) of the whole
    prefill."""
    rows = np.asarray(rows, dtype=np.int64)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    grp = Hq // Hkv
    scale = softmax_scale(D, params)
    kind = int(params.kind)
    freqs = _freqs(params, D)
    pr = _pairing(params)
    p_loc, p_rem, _G = position_maps(params, S)
    t_all = np.arange(S)
    ok = np.stack([_allowed(params, int(r), t_all) for r in rows])            # [R, S]
    local = (rows[:, None] - t_all[None, :]) <= int(params.w0)
    stage = round_bf16 if stage_bf16 else (lambda a: a)

    def srot(x, pos):
        return x if kind == NOPE else stage(rotate(x, pos, freqs, pr))

    for b in range(B):
        keys = {}
        for j, h in enumerate(heads):
            hk = h // grp
            if hk not in keys:
                kk = to_f64(k[b, :, hk])
                keys[hk] = (srot(kk, p_loc), srot(kk, p_rem) if kind == BIFOCAL else None, to_f64(v[b, :, hk]))
            kl, kr, vv = keys[hk]
            qq = to_f64(q[b, rows, h])
            ql = srot(qq, p_loc[rows])
            qr = srot(qq, p_rem[rows]) if kind == BIFOCAL else None
            sc = ql @ kl.T
            if kind == BIFOCAL:
                sc = np.where(local, sc, qr @ kr.T)
            sc = np.where(ok, sc * scale, -np.inf)
            m = sc.max(axis=1, keepdims=True)
            e = np.where(ok, np.exp(sc - m), 0.0)
            P = e / e.sum(axis=1, keepdims=True)
            do = to_f64(dout[b, rows, h])
            dP = do @ vv.T
            dS = P * (dP - (P * dP).sum(axis=1, keepdims=True))
            yield dict(b=b, j=j, h=h, hk=hk, P=P, dS=dS, do=do, ql=ql, qr=qr, kl=kl, kr=kr, local=local,
                       scale=scale, kind=kind, freqs=freqs, pr=pr, p_loc=p_loc, p_rem=p_rem)


def _unrot(c, x, pos):
    return x if c["kind"] == NOPE else rotate(x, pos, c["freqs"], c["pr"])


def prefill_backward_dq_rows(q, k, v, dout, params, rows, stage_bf16: bool = False, heads=None):
    """dq of ``prefill_backward`` for the query rows ``rows`` only (and the
    query heads ``heads``, default all), [B, len(rows), len(heads), D]: the
    same chain rule, one block of rows at a time,
      dq_t = scale * sum_s dS(t,s) R_a^T R_b k_s,
      dS(t,s) = P(t,s) (dout_t . v_s - sum_s' P(t,s') dout_t . v_s'),
    with P the row softmax of scale * score(t,s) over the allowed keys
    (Periodic RoPE §3.1 Eq. 2, §3.2 Eq. 4; Jet-Long §3 Eq. 1, §3.1 Eq. 2-3),
    split by the window into a local and a remote part for BIFOCAL."""
    B, S, Hq, D = q.shape
    heads = list(range(Hq)) if heads is None else list(heads)
    rows = np.asarray(rows, dtype=np.int64)
    dq = np.zeros((B, len(rows), len(heads), D))
    for c in _backward_rows(q, k, v, dout, params, rows, stage_bf16, heads):
        dS, scale = c["dS"], c["scale"]
        if c["kind"] == BIFOCAL:
            dSl, dSr = np.where(c["local"], dS, 0.0), np.where(c["local"], 0.0, dS)
            g = _unrot(c, dSl @ c["kl"], -c["p_loc"][rows]) + _unrot(c, dSr @ c["kr"], -c["p_rem"][rows])
        else:
            g = _unrot(c, dS @ c["kl"], -c["p_loc"][rows])
        dq[c["b"], :, c["j"]] = scale * g
    return dq


def prefill_backward_tail(q, k, v, dout, params, n: int, stage_bf16: bool = False, heads=None):
    """(dq, dk, dv) of ``prefill_backward`` on the last ``n`` positions: dq of
    the query rows [S-n, S) for the query heads ``heads`` ([B, n, len(heads),
    D]) and dk, dv of the keys [S-n, S) for the KV heads those query heads
    belong to ([B, n, len(kv heads), D], kv heads in increasing order).
    Attention is causal for every kind, so a key s receives dk and dv only
    from the rows t >= s; for the tail keys those rows are the tail rows,
    and the sums
      dv_s = sum_t P(t,s) dout_t,   dk_s = scale * sum_t dS(t,s) R_b^T R_a q_t
    over them are complete. ``heads`` must hold whole GQA groups (dk and dv
    of a KV head collect all the heads of its group)."""
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    grp = Hq // Hkv
    heads = list(range(Hq)) if heads is None else list(heads)
    kvh = sorted({h // grp for h in heads})
    for hk in kvh:
        if not set(range(hk * grp, (hk + 1) * grp)) <= set(heads):
            raise ValueError(f"heads must hold the whole GQA group of kv head {hk}")
    n = int(n)
    if not 0 <= n <= S:
        raise ValueError("n must lie in [0, S]")
    rows = np.arange(S - n, S, dtype=np.int64)
    dq = np.zeros((B, n, len(heads), D))
    dk = np.zeros((B, n, len(kvh), D))
    dv = np.zeros((B, n, len(kvh), D))
    if n == 0:
        return dq, dk, dv
    for c in _backward_rows(q, k, v, dout, params, rows, stage_bf16, heads):
        b, x, scale = c["b"], kvh.index(c["hk"]), c["scale"]
        P, dS = c["P"][:, rows], c["dS"]
        dv[b, :, x] += P.T @ c["do"]
        if c["kind"] == BIFOCAL:
            dSl, dSr = np.where(c["local"], dS, 0.0), np.where(c["local"], 0.0, dS)
            dq[b, :, c["j"]] = scale * (_unrot(c, dSl @ c["kl"], -c["p_loc"][rows])
                                        + _unrot(c, dSr @ c["kr"], -c["p_rem"][rows]))
            dk[b, :, x] += scale * (_unrot(c, dSl[:, rows].T @ c["ql"], -c["p_loc"][rows])
                                    + _unrot(c, dSr[:, rows].T @ c["qr"], -c["p_rem"][rows]))
        else:
            dq[b, :, c["j"]] = scale * _unrot(c, dS @ c["kl"], -c["p_loc"][rows])
            dk[b, :, x] += scale * _unrot(c, dS[:, rows].T @ c["ql"], -c["p_loc"][rows])
    return dq, dk, dv


# ----------------------------------------------------------------------------
# decode (Jet-Long §3.2): untouched cache + correction rotation
# ----------------------------------------------------------------------------
def cache_keys(k, params, start: int = 0):
    """The decode cache entries of keys k [B,count,Hkv,D] at absolute token
    indices start..start+count-1: each key rotated at the kind's own position
    of its index (Jet-Long §3.2 Eq. 4, k_cache[k] = RoPE(x_k, k); the other
    kinds store keys at their own positions: EndPrompt's two segments, t mod W
    for Periodic RoPE; NoPE stores keys unrotated). The result does not depend
    on the sequence length, so the cache is never rewritten as L (and G)
    grows. Float64, not rounded."""
    k = to_f64(k)
    count, D = k.shape[1], k.shape[3]
    if int(params.kind) == NOPE:
        return k.copy()
    p_loc = position_maps(params, int(start) + count)[0][int(start):]
    freqs = _freqs(params, D)
    pr = _pairing(params)
    out = np.empty_like(k)
    for b in range(k.shape[0]):
        for h in range(k.shape[2]):
            out[b, :, h] = rotate(k[b, :, h], p_loc, freqs, pr)
    return out


def prefill_from_cache(q, k_cache, v_cache, params, start: int, stage_bf16: bool = True, rows=None, heads=None):
    """Rows start..L-1 of a prefill of length L = k_cache.shape[1] whose keys
    come from a decode cache (Eq. 4: k_cache[s] = RoPE(x_s, p(s))) instead of
    raw keys: q [B,count,Hq,D] holds the unrotated queries of tokens
    start..L-1 (count = L - start). Local scores read the cache as stored;
    for BIFOCAL, remote scores read each cached key through the correction
    rotation by Delta s = f(s) - s (Eq. 5-6, as in decode) against the query
    rotated to f(t). ``stage_bf16`` rounds the rotated queries and the
    corrected remote keys to bf16 (the cache itself is taken as given).
    ``rows`` (token indices in [start, L)) and ``heads`` (query heads)
    restrict the result to those rows and heads, for checks at lengths where
    every row is out of reach; only the slices they need are taken to
    float64. Returns out [B,R,H,D], lse [B,H,R] (R rows, H heads; by default
    every row start..L-1 and every head)."""
    B, count, Hq, D = q.shape
    L, Hkv = k_cache.shape[1], k_cache.shape[2]
    assert count == L - int(start)
    rows = np.arange(int(start), L) if rows is None else np.asarray(rows, dtype=np.int64)
    assert rows.size == 0 or (rows.min() >= int(start) and rows.max() < L)
    heads = list(range(Hq)) if heads is None else list(heads)
    grp = Hq // Hkv
    scale = softmax_scale(D, params)
    kind = int(params.kind)
    freqs = _freqs(params, D)
    pr = _pairing(params)
    p_loc, p_rem, G = position_maps(params, L)
    stage = round_bf16 if stage_bf16 else (lambda a: a)
    keys = np.arange(L)
    out = np.zeros((B, rows.size, len(heads), D))
    lse = np.zeros((B, len(heads), rows.size))
    for b in range(B):
        for hk in sorted({h // grp for h in heads}):
            kl = to_f64(k_cache[b, :, hk])
            vv = to_f64(v_cache[b, :, hk])
            kr = stage(rotate(kl, p_rem - keys, freqs, pr)) if kind == BIFOCAL else None   # Eq. 6, keys
            for j, h in enumerate(heads):
                if h // grp != hk:
                    continue
                for c0 in range(0, rows.size, 64):
                    rr = rows[c0:c0 + 64]
                    nk = int(rr.max()) + 1
                    ok = np.stack([_allowed(params, int(t), keys[:nk]) for t in rr])
                    qq = to_f64(q[b, rr - int(start), h, :])
                    ql = qq if kind == NOPE else stage(rotate(qq, p_loc[rr], freqs, pr))
                    sc = (ql @ kl[:nk].T) * scale
                    if kind == BIFOCAL:
                        qr = stage(rotate(qq, p_rem[rr], freqs, pr))
                        sr = (qr @ kr[:nk].T) * scale
                        local = (rr[:, None] - keys[None, :nk]) <= int(params.w0)
                        sc = np.where(local, sc, sr)
                    o, l = _softmax_rows(sc, ok, vv[:nk])
                    out[b, c0:c0 + 64, j, :] = o
                    lse[b, j, c0:c0 + 64] = l
    return out, lse


def decode(q, k_cache, v_cache, params, stage_bf16: bool = False):
    """One query token at position n-1 against a cache of n keys.

    q [B,Hq,D] unrotated; k_cache [B,n,Hkv,D] holds keys already rotated at
    their own positions (Eq. 4: k_cache[k] = RoPE(x_k, k)); v_cache likewise.
    L = n. The query is rotated to its position; for BIFOCAL, keys with
    (n-1) - k > w0 are read through the correction rotation
    k_remote = RoPE(k_cache[k], Delta k), Delta k = f(k) - k, and the query
    through q_remote = RoPE(q_local, Delta q) (Eq. 5-6). Rotations are in
    float64. ``stage_bf16`` rounds the rotated query views and the corrected
    remote keys to bf16 (round to nearest even) before the dot products: the
    operand rounding of a decode on bf16 tensor cores, the same modelled input
    rounding as the prefill's; the cache itself is taken as given.
    Returns out [B,Hq,D], lse [B,Hq]."""
    q, kc, vc = to_f64(q), to_f64(k_cache), to_f64(v_cache)
    B, Hq, D = q.shape
    n, Hkv = kc.shape[1], kc.shape[2]
    grp = Hq // Hkv
    scale = softmax_scale(D, params)
    kind = int(params.kind)
    freqs = _freqs(params, D)
    pr = _pairing(params)
    p_loc, _, G = position_maps(params, n)
    stage = round_bf16 if stage_bf16 else (lambda a: a)
    t = n - 1
    keys = np.arange(n)
    ok = _allowed(params, t, keys)[None, :]
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            hk = h // grp
            qq = q[b, h][None, :]
            ql = qq if kind == NOPE else rotate(qq, np.array([p_loc[t]]), freqs, pr)
            sc = (stage(ql) @ kc[b, :, hk].T) * scale              # [1, n]
            if kind == BIFOCAL:
                dq = int(remote_position(t, G)) - t                # Eq. 5
                qr = stage(rotate(ql, np.array([dq]), freqs, pr))      # Eq. 6, query
                dk = remote_position(keys, G) - keys               # Eq. 5
                kr = stage(rotate(kc[b, :, hk], dk, freqs, pr))        # Eq. 6, keys
                sr = (qr @ kr.T) * scale
                local = (t - keys) <= int(params.w0)
                sc = np.where(local[None, :], sc, sr)
            o, l = _softmax_rows(sc, ok, vc[b, :, hk])
            out[b, h] = o[0]
            lse[b, h] = l[0]
    return out, lse


# ----------------------------------------------------------------------------
# brute force: explicit matrices and loops, tiny inputs only
# ----------------------------------------------------------------------------
def _brute_positions(params, t: int, s: int, L: int, D: int):
    """(a, b) positions for the pair (t, s), or None for NoPE."""
    kind = int(params.kind)
    if kind == NOPE:
        return None
    if kind == STANDARD:
        return t, s
    if kind == ENDPROMPT:
        pos = lambda x: x if x < params.seg1_len else params.term_start + x - params.seg1_len
        return pos(t), pos(s)
    if kind == PERIODIC:
        return t % params.window, s % params.window
    fixed = int(getattr(params, "fixed_group", 0) or 0)
    G = fixed if fixed > 0 else max(1, math.ceil(L / params.w_pretrained))
    if t - s <= params.w0:
        return t, s
    return t // G, s // G


def brute_prefill(q, k, v, params, stage_bf16: bool = False):
    """Every score from explicit D x D rotation matrices, every softmax by a
    Python loop over the allowed keys. For S <= ~64."""
    q, k, v = to_f64(q), to_f64(k), to_f64(v)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    grp = Hq // Hkv
    scale = softmax_scale(D, params)
    freqs = _freqs(params, D)
    pr = _pairing(params)
    stage = round_bf16 if stage_bf16 else (lambda a: a)
    out = np.zeros((B, S, Hq, D))
    lse = np.zeros((B, Hq, S))
    for b in range(B):
        for h in range(Hq):
            hk = h // grp
            for t in range(S):
                keys = [s for s in range(S) if s <= t and
                        (int(params.kind) != PERIODIC or s >= t - params.window + 1)]
                scores = []
                for s in keys:
                    ab = _brute_positions(params, t, s, S, D)
                    if ab is None:
                        qa, kb = q[b, t, h], k[b, s, hk]
                    else:
                        qa = stage(rotation_matrix(ab[0], freqs, pr) @ q[b, t, h])
                        kb = stage(rotation_matrix(ab[1], freqs, pr) @ k[b, s, hk])
                    scores.append(scale * float(qa @ kb))
                m = max(scores)
                w = [math.exp(x - m) for x in scores]
                z = sum(w)
                out[b, t, h] = sum(wi * v[b, s, hk] for wi, s in zip(w, keys)) / z
                lse[b, h, t] = m + math.log(z)
    return out, lse


def brute_decode(q, k_raw, v, params):
    """Decode by its definition on RAW keys: the score of key s is the
    prefill score of the last row (t = n-1) computed from unrotated k_s, so
    this pins the cache-plus-correction route of ``decode`` (R_a R_b = R_{a+b})."""
    q, k_raw, v = to_f64(q), to_f64(k_raw), to_f64(v)
    B, Hq, D = q.shape
    n, Hkv = k_raw.shape[1], k_raw.shape[2]
    grp = Hq // Hkv
    scale = softmax_scale(D, params)
    freqs = _freqs(params, D)
    pr = _pairing(params)
    t = n - 1
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hq):
            hk = h // grp
            keys = [s for s in range(n) if int(params.kind) != PERIODIC or s >= t - params.window + 1]
            scores = []
            for s in keys:
                ab = _brute_positions(params, t, s, n, D)
                if ab is None:
                    sc = q[b, h] @ k_raw[b, s, hk]
                else:
                    sc = (rotation_matrix(ab[0], freqs, pr) @ q[b, h]) @ (rotation_matrix(ab[1], freqs, pr) @ k_raw[b, s, hk])
                scores.append(scale * float(sc))
            m = max(scores)
            w = [math.exp(x - m) for x in scores]
            z = sum(w)
            out[b, h] = sum(wi * v[b, s, hk] for wi, s in zip(w, keys)) / z
            lse[b, h] = m + math.log(z)
    return out, lse
