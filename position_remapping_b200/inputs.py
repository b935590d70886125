"""Seeded synthetic inputs and the named workloads.

This module is shared by the CUDA path, the tests and the benchmark. It holds
no arithmetic of the method: no positions, no rotations, no softmax. It only
fixes shapes, parameter values and random draws, so that every consumer sees
the same bits.

Draw recipe (all workloads): ``torch.Generator('cpu').manual_seed(seed)``, then
q, k, v in that order, each ``randn(float32)`` rounded to bfloat16. Values are
iid N(0, 1), which makes the logits roughly N(0, 1) at scale 1/sqrt(D).

The pages measure on Qwen3-8B prefill/generation (Jet-Long, §4.6 Table 7),
MiniWin (Periodic RoPE, Table 1) and LLaMA 8K->64K fine-tuning (EndPrompt,
abstract). None of their data or weights are used: the kernels do no
data-dependent work, so iid normal tensors of the same shapes stand in.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

# kind codes, identical to the C header's enum
STANDARD, ENDPROMPT, PERIODIC, NOPE, BIFOCAL = 0, 1, 2, 3, 4
KIND_NAMES = {STANDARD: "standard", ENDPROMPT: "endprompt", PERIODIC: "periodic",
              NOPE: "nope", BIFOCAL: "bifocal"}
# coordinate pairing codes, identical to the C header's enum
PAIR_ADJACENT, PAIR_HALF = 0, 1


@dataclasses.dataclass(frozen=True)
class MapParams:
    """Position-map kind and its parameters (plain values, no arithmetic)."""
    kind: int
    rope_base: float = 10000.0
    interp: float = 1.0          # position-interpolation factor s (EndPrompt)
    seg1_len: int = 0            # EndPrompt: length n1 of the intact first segment
    term_start: int = 0          # EndPrompt: first position of the terminal segment
    window: int = 0              # Periodic RoPE: window W (= period)
    w0: int = 0                  # Jet-Long: local window
    w_pretrained: int = 0        # Jet-Long: pretrained context window
    fixed_group: int = 0         # bifocal with one fixed group size G (0: G from L, Eq. 2)
    softmax_scale: float = 0.0   # 0 -> 1/sqrt(D)
    pairing: int = 0             # PAIR_ADJACENT (2i, 2i+1) or PAIR_HALF (i, i + D/2)

    def replace(self, **kw) -> "MapParams":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    S: int                 # prefill: sequence length; decode: cache length n
    Hq: int
    Hkv: int
    D: int
    params: MapParams
    decode: bool = False
    seed: int = 1000


# The five workloads. Sizes follow the pages' settings: Jet-Long's 32K
# pretrained window, w0 = 2048 and 128K target (§4.1, §4.6); MiniWin-style
# periodic windows (Table 1) scaled up; EndPrompt's 8K -> 64K extension with
# the terminal segment at the end of the 64K range (abstract).
WORKLOADS = {
    "standard_s512": Workload("standard_s512", 1, 512, 1, 1, 64,
                              MapParams(STANDARD, rope_base=10000.0), seed=1001),
    "endprompt_s8192": Workload("endprompt_s8192", 4, 8192, 32, 8, 128,
                                MapParams(ENDPROMPT, rope_base=500000.0, interp=8.0,
                                          seg1_len=8000, term_start=65344), seed=1002),
    "periodic_s32768": Workload("periodic_s32768", 2, 32768, 16, 16, 64,
                                MapParams(PERIODIC, rope_base=10000.0, window=1024), seed=1003),
    "nope_s32768": Workload("nope_s32768", 2, 32768, 16, 16, 64,
                            MapParams(NOPE), seed=1003),
    "bifocal_prefill_s131072": Workload("bifocal_prefill_s131072", 1, 131072, 32, 8, 128,
                                        MapParams(BIFOCAL, rope_base=1e6, w0=2048,
                                                  w_pretrained=32768), seed=1004),
    "bifocal_decode_n131072": Workload("bifocal_decode_n131072", 1, 131072, 16, 8, 128,
                                       MapParams(BIFOCAL, rope_base=1e6, w0=2048,
                                                 w_pretrained=32768), decode=True, seed=1005),
}


def make_qkv(B: int, S: int, Hq: int, Hkv: int, D: int, seed: int,
             device: Optional[str] = None, q_len: Optional[int] = None):
    """q [B, q_len or S, Hq, D], k/v [B, S, Hkv, D], bf16, iid N(0,1).

    For decode pass ``q_len=1`` and the q tensor is returned as [B, Hq, D].
    Draws happen on the CPU generator so the bits do not depend on the device.
    """
    g = torch.Generator("cpu").manual_seed(int(seed))
    ql = S if q_len is None else q_len
    q = torch.randn((B, ql, Hq, D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    k = torch.randn((B, S, Hkv, D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn((B, S, Hkv, D), generator=g, dtype=torch.float32).to(torch.bfloat16)
    if q_len == 1:
        q = q[:, 0].contiguous()
    if device is not None:
        q, k, v = q.to(device), k.to(device), v.to(device)
    return q, k, v


def workload_inputs(w: Workload, device: Optional[str] = None):
    return make_qkv(w.B, w.S, w.Hq, w.Hkv, w.D, w.seed, device=device,
                    q_len=1 if w.decode else None)


def sample_rows(S: int, params: MapParams, n_random: int = 512, seed: int = 7,
                edge: int = 64) -> list:
    """Rows to check on large prefill runs (each output row is independent).

    First and last ``edge`` rows, rows around every boundary the kind has
    (w0, window multiples, segment start, group-size multiples of the
    pretrained window) and ``n_random`` seeded random rows.
    """
    rows = set(range(min(edge, S))) | set(range(max(0, S - edge), S))
    marks = []
    if params.kind == ENDPROMPT:
        marks.append(params.seg1_len)
    if params.kind == PERIODIC and params.window > 0:
        marks += list(range(params.window, S, params.window))[:16]
    if params.kind == BIFOCAL:
        marks += [params.w0, params.w0 + 1]
        if params.w_pretrained > 0:
            marks += list(range(params.w_pretrained, S, params.w_pretrained))
    for m in marks:
        for d in (-2, -1, 0, 1, 2, 127, 128, 129):
            if 0 <= m + d < S:
                rows.add(m + d)
    g = torch.Generator("cpu").manual_seed(seed)
    if n_random > 0 and S > 0:
        rows |= set(torch.randint(0, S, (n_random,), generator=g).tolist())
    return sorted(rows)
