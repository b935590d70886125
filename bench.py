"""Benchmark of the remapped-RoPE attention hot path on B200.

One step = one Jet-Long bifocal prefill of 131072 tokens (32 q / 8 kv heads,
head_dim 128, w_pretrained 32768 -> G = 4, w0 = 2048, base 1e6: the key
rotation pre-pass and the attention kernel) followed by one bifocal decode
step over a 131072-token cache (16 q / 8 kv heads, head_dim 128). Inputs are
seeded iid N(0,1) bf16 tensors resident in HBM; every input is larger than
the 126 MB L2, so no explicit flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). ``value`` is prefill TFLOP/s over all ranks
(4*D FLOPs per attended (query, key) pair per query head, each pair once);
decode microseconds per token ride along. Multi-GPU runs are weak scaling:
each rank runs its own independent problem, no collective on the data path;
times are the max over ranks. ``--impl reference`` times the float64 CPU
oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)

from position_remapping_b200.inputs import WORKLOADS, make_qkv  # noqa: E402

METRIC = "128K bifocal-RoPE prefill TFLOP/s + decode µs/token; % of B200 roofline"
PREFILL = WORKLOADS["bifocal_prefill_s131072"]
DECODE = WORKLOADS["bifocal_decode_n131072"]
PEAK_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# oracle samples (query rows, kv heads): the reference arm's step (~4 s on 8
# host cores) and the GPU arm's cpu_baseline (~10-15 s)
REF_ROWS, REF_KV = 2, 1
CPU_ROWS, CPU_KV = 16, 3


def prefill_flops(w) -> float:
    pairs = w.S * (w.S + 1) // 2          # causal pairs per (batch, head)
    return 4.0 * w.D * pairs * w.Hq * w.B


def attended_pairs(w) -> int:
    """(query, key) pairs per (batch, query head) of a whole prefill: causal,
    or the W-key window of Periodic RoPE."""
    S = w.S
    if w.params.kind == 2 and 0 < w.params.window < S:   # PERIODIC
        W = w.params.window
        return W * (W + 1) // 2 + (S - W) * W
    return S * (S + 1) // 2


def prefill_io_bytes(w) -> int:
    """Algorithmic HBM bytes of a prefill: q, k, v read once (bf16), out (fp32)
    and lse (fp32) written once."""
    return 2 * w.B * w.S * (w.Hq + 2 * w.Hkv) * w.D + 4 * w.B * w.S * w.Hq * (w.D + 1)


def decode_bytes(w) -> int:
    kv = 2 * w.B * w.S * w.Hkv * w.D * 2
    return kv + w.B * w.Hq * w.D * 2 + w.B * w.Hq * (w.D + 1) * 4


def rank_seed(seed: int, rank: int) -> int:
    """Weak scaling: every rank runs its own independent draw of the workload."""
    return seed + 17 * rank


def max_over_ranks(values, world: int, device) -> list:
    """Element-wise max of per-rank timings (the job is as slow as its
    slowest rank). One all_reduce, taken by every rank in the same order."""
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tflops(world: int, flops_per_step: float, steps: int, ms: float) -> float:
    """Whole-job throughput: every rank's FLOPs over the slowest rank's time."""
    return world * flops_per_step * steps / (ms / 1e3) / 1e12


def load_peaks():
    path = os.path.join(HERE, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return dict(PEAK_FALLBACK), "fallback"


def source_hash(*names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(HERE, "position_remapping_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record(kernel: str, src_hash: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source; else None."""
    try:
        with open(os.path.join(HERE, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(kernel)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_hash") != src_hash:
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        mhz, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8 or (self.uuid and self.uuid not in parts[0]):
                continue
            try:
                mhz.append(float(parts[1]))
                maxes.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(n)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxes), "reasons": sorted(reasons),
                "samples": len(mhz)}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads", 0) for p in threadpool_info() if p.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ----------------------------------------------------------------------------
# CPU oracle (baseline / reference arm): bounded samples of the same workload
# ----------------------------------------------------------------------------
def oracle_rows(n_rows: int):
    S = PREFILL.S
    step = S // n_rows
    return [min(S - 1, i * step + step // 2) for i in range(n_rows)]


def oracle_step(n_rows: int, n_kv: int, q, k, v, qd, kd, vd):
    """Times the oracle on a bounded sample of one step: `n_rows` evenly
    spaced query rows of the prefill for the query heads of the first `n_kv`
    kv heads (the oracle rotates every key of each kv head it is given, the
    full 131072-token sequence, so L and G are those of the workload), and
    one decode over the full cache for the query heads of the first `n_kv`
    kv heads. Returns (prefill TFLOP/s, decode us per token of the sampled
    heads scaled to all heads, seconds, sample description)."""
    import oracle as O
    P, Dd = PREFILL, DECODE
    hq_p = n_kv * (P.Hq // P.Hkv)
    hq_d = n_kv * (Dd.Hq // Dd.Hkv)
    rows = oracle_rows(n_rows)
    flops = sum(4.0 * P.D * (t + 1) * hq_p for t in rows)
    qs, ks, vs = q[:, :, :hq_p], k[:, :, :n_kv], v[:, :, :n_kv]
    qds, kds, vds = qd[:, :hq_d], kd[:, :, :n_kv], vd[:, :, :n_kv]
    t0 = time.perf_counter()
    O.prefill(qs, ks, vs, P.params, rows=rows, stage_bf16=True)
    t1 = time.perf_counter()
    O.decode(qds, kds, vds, Dd.params)
    t2 = time.perf_counter()
    sample = (f"{n_rows} query rows (evenly spaced) x {hq_p} of {P.Hq} query heads ({n_kv} of {P.Hkv} kv heads) "
              f"of the {P.S}-token bifocal prefill, plus a {Dd.S}-key bifocal decode of {hq_d} of {Dd.Hq} "
              f"query heads (decode time scaled by {Dd.Hkv}/{n_kv})")
    return flops / (t1 - t0) / 1e12, (t2 - t1) * 1e6 * Dd.Hkv / n_kv, t2 - t0, sample


def run_reference(args):
    q, k, v = make_qkv(PREFILL.B, PREFILL.S, PREFILL.Hq, PREFILL.Hkv, PREFILL.D, PREFILL.seed)
    qd, kd, vd = make_qkv(DECODE.B, DECODE.S, DECODE.Hq, DECODE.Hkv, DECODE.D, DECODE.seed, q_len=1)
    vals, decs, secs = [], [], []
    sample = ""
    for i in range(args.warmup + args.steps):
        tf, dus, s, sample = oracle_step(REF_ROWS, REF_KV, q, k, v, qd, kd, vd)
        if i >= args.warmup:
            vals.append(tf)
            decs.append(dus)
            secs.append(s)
    value = statistics.median(vals)
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded iid N(0,1) bf16)",
        "config": config_dict(args.gpus),
        "decode_us_per_token": statistics.median(decs),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


CHUNK = 8192   # tokens of the chunked-prefill measurement (the last rows of the 131072 prefill)
CONFIGS = ("standard_s512", "endprompt_s8192", "periodic_s32768", "nope_s32768")
SWEEP = (4096, 8192, 16384, 32768, 65536, 98304, 131072)   # Jet-Long §4.6 Table 7 lengths


def _event_ms(fn, reps, stream):
    fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


def measure_cache_rows(ra, q, k, v, kd, vd, qd, stream):
    """The decode-cache rows, timed with CUDA events after the main timed
    region: writing the 131072-token prefill's cache (Eq. 4), the last 8192
    rows of the same prefill computed from that cache, and one decode step
    that appends its token to the cache before attending."""
    P, Dd = PREFILL, DECODE
    kc = torch.empty_like(k)
    vc = torch.empty_like(v)
    w_ms = _event_ms(lambda: ra.cache_write(k, v, kc, vc, P.params, 0, stream=stream), 5, stream)
    w_bytes = 4 * k.numel() * k.element_size()            # read k, v; write both caches
    start = P.S - CHUNK
    qc = q[:, start:].contiguous()
    ws = torch.empty(ra.prefill_chunk_workspace_size(P.params, P.B, start, CHUNK, P.Hq, P.Hkv, P.D),
                     dtype=torch.uint8, device=q.device)
    oc = torch.empty((P.B, CHUNK, P.Hq, P.D), dtype=torch.float32, device=q.device)
    lc = torch.empty((P.B, P.Hq, CHUNK), dtype=torch.float32, device=q.device)
    c_ms = _event_ms(lambda: ra.prefill_chunk(qc, kc, vc, P.params, start, out=oc, lse=lc, workspace=ws,
                                              stream=stream), 3, stream)
    c_flops = 4.0 * P.D * P.Hq * P.B * sum(range(start + 1, P.S + 1))
    # decode step with append: the last cached token is rewritten, then attended
    kn, vn = kd[:, -1:].contiguous(), vd[:, -1:].contiguous()
    od = torch.empty((Dd.B, Dd.Hq, Dd.D), dtype=torch.float32, device=q.device)
    ld = torch.empty((Dd.B, Dd.Hq), dtype=torch.float32, device=q.device)
    wsd = torch.empty(ra.decode_workspace_size(Dd.B, Dd.S, Dd.Hq, Dd.Hkv, Dd.D), dtype=torch.uint8, device=q.device)

    def step():
        ra.cache_write(kn, vn, kd, vd, Dd.params, Dd.S - 1, stream=stream)
        ra.decode(qd, kd, vd, Dd.params, out=od, lse=ld, workspace=wsd, stream=stream)
    s_ms = _event_ms(step, 20, stream)
    ra.status()
    return {"cache_write_gbs": w_bytes / (w_ms / 1e3) / 1e9, "cache_write_ms": w_ms,
            "cache_write_bytes": w_bytes,
            "prefill_chunk_tflops": c_flops / (c_ms / 1e3) / 1e12, "prefill_chunk_ms": c_ms,
            "prefill_chunk": f"rows {start}..{P.S - 1} of the {P.S}-token bifocal prefill from its cache",
            "decode_append_us_per_token": s_ms * 1e3}


def measure_comparators(ra, q, k, v, out, lse, ws, stream):
    """Same-box comparators of the fused bifocal prefill (CUDA events, after
    the timed regions): the same attention kernel with standard RoPE on the
    same shapes (the unmodified-model reference), and the literal three-call
    bifocal route with a separate merge kernel. Ratios are throughput
    relative to standard RoPE, as the pages report against their baseline."""
    P = PREFILL
    std = P.params.replace(kind=0)
    std_ms = _event_ms(lambda: ra.prefill(q, k, v, std, out=out, lse=lse, workspace=ws, stream=stream), 2, stream)
    fused_ms = _event_ms(lambda: ra.prefill(q, k, v, P.params, out=out, lse=lse, workspace=ws, stream=stream), 2,
                         stream)
    ws3 = torch.empty(int(ra.lib.ropeattn_prefill_three_call_workspace_size(
        ctypes.byref(ra.to_cparams(P.params)), P.B, P.S, P.Hq, P.Hkv, P.D)), dtype=torch.uint8, device=q.device)
    three_ms = _event_ms(lambda: ra.prefill_three_call(q, k, v, P.params, out=out, lse=lse, workspace=ws3,
                                                       stream=stream), 2, stream)
    del ws3
    ra.status()
    return {"standard_rope_prefill_ms": std_ms, "fused_bifocal_prefill_ms": fused_ms,
            "three_call_bifocal_prefill_ms": three_ms,
            "fused_vs_standard": std_ms / fused_ms, "three_call_vs_standard": std_ms / three_ms,
            "note": "prepare + attend, 131072 tokens, 32/8 heads, D 128; ratio = standard time / time"}


def measure_decode_comparators(ra, qd, kd, vd, stream):
    """Decode comparators on the 131072-key cache (CUDA events, after the
    timed regions): the fused bifocal decode, the same decode with the
    correction rotation as a separate pass over the cache, and standard RoPE
    on the same cache (the unmodified-model reference)."""
    Dd = DECODE
    od = torch.empty((Dd.B, Dd.Hq, Dd.D), dtype=torch.float32, device=qd.device)
    ld = torch.empty((Dd.B, Dd.Hq), dtype=torch.float32, device=qd.device)
    wsd = torch.empty(ra.decode_workspace_size(Dd.B, Dd.S, Dd.Hq, Dd.Hkv, Dd.D), dtype=torch.uint8, device=qd.device)
    wsu = torch.empty(int(ra.lib.ropeattn_decode_unfused_workspace_size(Dd.B, Dd.S, Dd.Hq, Dd.Hkv, Dd.D)),
                      dtype=torch.uint8, device=qd.device)
    std = Dd.params.replace(kind=0)
    # the decode alone, 200 calls back to back (no prefill output draining
    # from L2 underneath), and the host time of one call through the binding
    alone_us = 1e3 * _event_ms(lambda: ra.decode(qd, kd, vd, Dd.params, out=od, lse=ld, workspace=wsd,
                                                 stream=stream), 200, stream)
    torch.cuda.synchronize()
    h0 = time.perf_counter()
    for _ in range(200):
        ra.decode(qd, kd, vd, Dd.params, out=od, lse=ld, workspace=wsd, stream=stream)
    host_us = (time.perf_counter() - h0) / 200 * 1e6
    torch.cuda.synchronize()
    fused_us = 1e3 * _event_ms(lambda: ra.decode(qd, kd, vd, Dd.params, out=od, lse=ld, workspace=wsd,
                                                 stream=stream), 20, stream)
    unfused_us = 1e3 * _event_ms(lambda: ra.decode_unfused(qd, kd, vd, Dd.params, out=od, lse=ld, workspace=wsu,
                                                           stream=stream), 20, stream)
    std_us = 1e3 * _event_ms(lambda: ra.decode(qd, kd, vd, std, out=od, lse=ld, workspace=wsd, stream=stream), 20,
                             stream)
    ra.status()
    return {"decode_alone_us": alone_us, "decode_alone_gbs": decode_bytes(Dd) / (alone_us / 1e6) / 1e9,
            "decode_host_us_per_call": host_us,
            "standard_rope_decode_us": std_us, "fused_bifocal_decode_us": fused_us,
            "unfused_bifocal_decode_us": unfused_us,
            "decode_fused_vs_standard": std_us / fused_us, "decode_unfused_vs_standard": std_us / unfused_us}


def oracle_config_sample(w, q, k, v, n_rows: int):
    """The oracle on `n_rows` evenly spaced query rows of every query head
    of batch entry 0 (all rows when n_rows >= S). Returns (TFLOP/s, seconds,
    sample description)."""
    import oracle as O
    S = w.S
    rows = list(range(S)) if n_rows >= S else [min(S - 1, i * (S // n_rows) + S // (2 * n_rows))
                                               for i in range(n_rows)]
    if w.params.kind == 2 and w.params.window > 0:
        per_row = [min(t + 1, w.params.window) for t in rows]
    else:
        per_row = [t + 1 for t in rows]
    flops = 4.0 * w.D * w.Hq * sum(per_row)
    t0 = time.perf_counter()
    O.prefill(q[:1], k[:1], v[:1], w.params, rows=rows, stage_bf16=True)
    dt = time.perf_counter() - t0
    what = "all rows" if n_rows >= S else f"{len(rows)} evenly spaced query rows"
    return flops / dt / 1e12, dt, f"{what} x {w.Hq} query heads of batch entry 0"


def measure_configs(ra, peaks, stream, with_oracle: bool):
    """Every prefill workload (standard 512, EndPrompt 8192, Periodic RoPE
    SWA and NoPE 32768; the 131072 bifocal prefill and decode are the main
    timed region) timed alone with CUDA events after the timed region:
    absolute time, tokens/s, TFLOP/s against the burst bf16 peak (short
    back-to-back launches), HBM GB/s against the measured copy bandwidth,
    and the oracle on a bounded sample on the host cores."""
    res = {}
    dev = torch.device("cuda", torch.cuda.current_device())
    tpeak = float(peaks.get("bf16_tflops", 1590.0))
    hpeak = float(peaks.get("hbm_gbs", 6650.0))
    for name in CONFIGS:
        w = WORKLOADS[name]
        q, k, v = make_qkv(w.B, w.S, w.Hq, w.Hkv, w.D, w.seed, device=dev)
        out = torch.empty((w.B, w.S, w.Hq, w.D), dtype=torch.float32, device=dev)
        lse = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device=dev)
        ws = torch.empty(max(1, ra.prefill_workspace_size(w.params, w.B, w.S, w.Hq, w.Hkv, w.D)),
                         dtype=torch.uint8, device=dev)
        reps = 200 if w.S <= 1024 else 10
        ms = _event_ms(lambda: ra.prefill(q, k, v, w.params, out=out, lse=lse, workspace=ws, stream=stream),
                       reps, stream)
        flops = 4.0 * w.D * attended_pairs(w) * w.B * w.Hq
        byts = prefill_io_bytes(w)
        tf = flops / (ms / 1e3) / 1e12
        gbs = byts / (ms / 1e3) / 1e9
        bound = {"standard_s512": "latency", "periodic_s32768": "balanced"}.get(name, "tensor")
        r = {"ms": ms, "us": ms * 1e3, "tokens_per_s": w.B * w.S / (ms / 1e3), "tflops": tf,
             "tensor_frac": tf / tpeak, "hbm_gbs": gbs, "hbm_frac": gbs / hpeak, "bound": bound,
             "flop": flops, "io_bytes": byts,
             "shape": {"B": w.B, "S": w.S, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D}}
        if with_oracle:
            n_rows = w.S if w.S <= 512 else (4 if w.S <= 8192 else 2)
            otf, osec, sample = oracle_config_sample(w, q.cpu(), k.cpu(), v.cpu(), n_rows)
            r["cpu_baseline"] = {"tflops": otf, "seconds": osec, "sample": sample, "cores": blas_threads(),
                                 "extrapolated_full_s": flops / (otf * 1e12) if otf > 0 else None}
        res[name] = r
        del q, k, v, out, lse, ws
    ra.status()
    return {"note": "each workload alone, CUDA events, prepare + attend; tensor_frac vs the burst bf16 peak, "
                    "hbm_frac vs the measured copy bandwidth (io_bytes = q, k, v read, out and lse written once)",
            **res}


def measure_variants(ra, peaks, q, k, v, kd, vd, stream):
    """The variants of the method beside the main path, each alone with CUDA
    events: prefill at 32768 tokens (bifocal, 32/8 heads, G = 4 via
    w_pretrained 8192) with adjacent and half-split pairing, a fixed group
    size and head_dim 256; decode of the 131072-key bifocal cache at
    head_dim 64 and 256, GQA groups 8 and 16, and half-split pairing.
    Inputs are leading slices of the resident tensors, or seeded N(0, 1)
    draws on the device where a shape differs (the kernels do no
    data-dependent work)."""
    dev = q.device
    tpeak = float(peaks.get("bf16_tflops", 1590.0))
    hpeak = float(peaks.get("hbm_gbs", 6650.0))
    P, Dd = PREFILL, DECODE
    gen = torch.Generator(device=dev).manual_seed(20261)

    def draw(*shape):
        return torch.randn(*shape, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)

    S = 32768
    base = P.params.replace(w_pretrained=8192)
    pre = {}
    pairs = S * (S + 1) // 2
    cases = [("bifocal_s32768_d128", 128, base), ("bifocal_s32768_half_split", 128, base.replace(pairing=1)),
             ("bifocal_s32768_fixed_g4", 128, base.replace(fixed_group=4)), ("bifocal_s32768_d256", 256, base)]
    for name, D, prm in cases:
        if D == P.D:
            qs, ks, vs = q[:, :S], k[:, :S], v[:, :S]
        else:
            qs, ks, vs = draw(P.B, S, P.Hq, D), draw(P.B, S, P.Hkv, D), draw(P.B, S, P.Hkv, D)
        out = torch.empty((P.B, S, P.Hq, D), dtype=torch.float32, device=dev)
        lse = torch.empty((P.B, P.Hq, S), dtype=torch.float32, device=dev)
        ws = torch.empty(ra.prefill_workspace_size(prm, P.B, S, P.Hq, P.Hkv, D), dtype=torch.uint8, device=dev)
        # two rounds, the faster kept: the first launches after other work
        # run at whatever clock that work left
        ms = min(_event_ms(lambda: ra.prefill(qs, ks, vs, prm, out=out, lse=lse, workspace=ws, stream=stream), 5,
                           stream) for _ in range(2))
        tf = 4.0 * D * pairs * P.B * P.Hq / (ms / 1e3) / 1e12
        pre[name] = {"ms": ms, "tflops": tf, "tensor_frac": tf / tpeak, "D": D, "pairing": prm.pairing,
                     "fixed_group": prm.fixed_group}
        del qs, ks, vs, out, lse, ws
    for name in pre:
        pre[name]["time_vs_d128_adjacent"] = pre[name]["ms"] / pre["bifocal_s32768_d128"]["ms"]
    dec = {}
    n = Dd.S
    dcases = [("bifocal_n131072_d128_grp2", 128, 16, Dd.params), ("bifocal_n131072_half_split", 128, 16,
                                                                     Dd.params.replace(pairing=1)),
              ("bifocal_n131072_d128_grp8", 128, 64, Dd.params), ("bifocal_n131072_d128_grp16", 128, 128, Dd.params),
              ("bifocal_n131072_d64_grp2", 64, 16, Dd.params), ("bifocal_n131072_d256_grp2", 256, 16, Dd.params)]
    for name, D, Hq, prm in dcases:
        if D == Dd.D:
            kc, vc = kd, vd
        else:
            kc, vc = draw(Dd.B, n, Dd.Hkv, D), draw(Dd.B, n, Dd.Hkv, D)
        qq = draw(Dd.B, Hq, D)
        od = torch.empty((Dd.B, Hq, D), dtype=torch.float32, device=dev)
        ld = torch.empty((Dd.B, Hq), dtype=torch.float32, device=dev)
        wsd = torch.empty(ra.decode_workspace_size(Dd.B, n, Hq, Dd.Hkv, D), dtype=torch.uint8, device=dev)
        us = 1e3 * _event_ms(lambda: ra.decode(qq, kc, vc, prm, out=od, lse=ld, workspace=wsd, stream=stream),
                             100, stream)
        byts = 2 * Dd.B * n * Dd.Hkv * D * 2
        dec[name] = {"us": us, "gbs": byts / (us / 1e6) / 1e9, "hbm_frac": byts / (us / 1e6) / 1e9 / hpeak,
                     "kv_bytes": byts, "D": D, "Hq": Hq, "Hkv": Dd.Hkv, "pairing": prm.pairing,
                     "kernel": "decode_tc_kernel"}
        del qq, od, ld, wsd
        if D != Dd.D:
            del kc, vc
    ra.status()
    return {"note": "each alone, CUDA events (prefill: pre-pass + attention, the faster of two rounds of 5 calls; "
                    "decode: 100 calls back to "
                    "back, host cost included where it exceeds the kernel); tensor_frac vs the burst bf16 peak, "
                    "hbm_frac vs the measured copy bandwidth", "prefill": pre, "decode": dec}


def measure_sweep(ra, q, k, v, qd, kd, vd, ws, wsd, stream):
    """Bifocal against standard RoPE over the Jet-Long Table 7 lengths (4K to
    128K; w_pretrained 32768, so G = 1 up to 32K and the bifocal map is the
    standard one there), prefill (32/8 heads) and decode (16/8 heads), on
    leading slices of the 131072-token inputs, CUDA events."""
    P, Dd = PREFILL, DECODE
    rows = []
    od = torch.empty((Dd.B, Dd.Hq, Dd.D), dtype=torch.float32, device=q.device)
    ld = torch.empty((Dd.B, Dd.Hq), dtype=torch.float32, device=q.device)
    for S in SWEEP:
        qs, ks, vs = q[:, :S], k[:, :S], v[:, :S]
        out = torch.empty((P.B, S, P.Hq, P.D), dtype=torch.float32, device=q.device)
        lse = torch.empty((P.B, P.Hq, S), dtype=torch.float32, device=q.device)
        flops = 4.0 * P.D * P.Hq * P.B * S * (S + 1) // 2
        reps = 2 if S >= 65536 else 5
        f_ms = _event_ms(lambda: ra.prefill(qs, ks, vs, P.params, out=out, lse=lse, workspace=ws, stream=stream),
                         reps, stream)
        s_ms = _event_ms(lambda: ra.prefill(qs, ks, vs, P.params.replace(kind=0), out=out, lse=lse, workspace=ws,
                                            stream=stream), reps, stream)
        kds, vds = kd[:, :S], vd[:, :S]
        f_us = 1e3 * _event_ms(lambda: ra.decode(qd, kds, vds, Dd.params, out=od, lse=ld, workspace=wsd,
                                                 stream=stream), 50, stream)
        s_us = 1e3 * _event_ms(lambda: ra.decode(qd, kds, vds, Dd.params.replace(kind=0), out=od, lse=ld,
                                                 workspace=wsd, stream=stream), 50, stream)
        dbytes = 2 * Dd.B * S * Dd.Hkv * Dd.D * 2
        rows.append({"S": S, "G": max(1, -(-S // P.params.w_pretrained)),
                     "prefill_bifocal_ms": f_ms, "prefill_standard_ms": s_ms,
                     "prefill_bifocal_tflops": flops / (f_ms / 1e3) / 1e12,
                     "prefill_bifocal_tokens_per_s": S / (f_ms / 1e3),
                     "prefill_ratio_vs_standard": s_ms / f_ms,
                     "decode_bifocal_us": f_us, "decode_standard_us": s_us,
                     "decode_bifocal_gbs": dbytes / (f_us / 1e6) / 1e9,
                     "decode_ratio_vs_standard": s_us / f_us})
        del out, lse
    ra.status()
    return {"note": "ratio = standard-RoPE time / bifocal time (the pages' Table 7 reports throughput relative "
                    "to their baseline); each length alone after the timed region", "rows": rows}


def measure_backward(ra, q, k, v, out, lse, peaks, stream):
    """The backward of the 131072-token bifocal prefill (dq, dk, dv from the
    forward's out and lse and a seeded upstream gradient), CUDA events after
    the timed region. The algorithmic work is 2.5x the forward's FLOPs (five
    contractions per attended pair against the forward's two); the kernels
    execute 3.5x (S and dP are recomputed by the dq kernel)."""
    P = PREFILL
    g = torch.Generator("cpu").manual_seed(P.seed + 1)
    dout = torch.randn((P.B, P.S, P.Hq, P.D), generator=g).to(torch.bfloat16).to(q.device)
    dq = torch.empty((P.B, P.S, P.Hq, P.D), dtype=torch.float32, device=q.device)
    dk = torch.empty((P.B, P.S, P.Hkv, P.D), dtype=torch.float32, device=q.device)
    dv = torch.empty_like(dk)
    ws = torch.empty(ra.prefill_backward_workspace_size(P.params, P.B, P.S, P.Hq, P.Hkv, P.D), dtype=torch.uint8,
                     device=q.device)
    ra.prefill(q, k, v, P.params, out=out, lse=lse, stream=stream)
    ms = _event_ms(lambda: ra.prefill_backward(q, k, v, out, lse, dout, P.params, dq=dq, dk=dk, dv=dv, workspace=ws,
                                               stream=stream), 3, stream)
    ra.status()
    flops = 2.5 * prefill_flops(P)
    tf = flops / (ms / 1e3) / 1e12
    tpeak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    del dout, dq, dk, dv, ws
    return {"ms": ms, "tflops": tf, "tokens_per_s": P.B * P.S / (ms / 1e3), "peak": tpeak, "frac": tf / tpeak,
            "algorithmic": f"{flops:.6g} FLOP per call (2.5x the forward)",
            "kernels": "rope_prep_kernel x2, bwd_prep_kernel, bwd_dkdv_kernel<128>, bwd_dq_kernel<128>",
            "note": "prefill backward, 131072 tokens, 32/8 heads, D 128, G = 4; frac vs the measured sustained "
                    "bf16 peak"}


def config_dict(n_gpus):
    return {"workload": f"{PREFILL.name} + {DECODE.name}",
            "prefill": {"B": PREFILL.B, "S": PREFILL.S, "Hq": PREFILL.Hq, "Hkv": PREFILL.Hkv, "D": PREFILL.D,
                        "w0": PREFILL.params.w0, "w_pretrained": PREFILL.params.w_pretrained,
                        "rope_base": PREFILL.params.rope_base},
            "decode": {"B": DECODE.B, "n": DECODE.S, "Hq": DECODE.Hq, "Hkv": DECODE.Hkv, "D": DECODE.D},
            "l2": "inputs larger than L2 (no flush)",
            "parallelism": f"independent problem per GPU x{n_gpus}"}


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------
CONFIG_PROFILES = ("standard_s512", "endprompt_s8192", "periodic_s32768", "nope_s32768")
DECODE_PROFILES = {"decode256": 256, "decode64": 64}


def run_profile_case(which: str):
    """Capture-sized cases for ncu (a few GB on the device at most, inputs
    still larger than L2). prefill: the 131072-token workload's kernel on a
    32768-token sequence with w_pretrained 8192, so G = 4 as in the full run;
    prefill256: the same case at head_dim 256; decode: the full 131072-key
    decode (512 MiB of cache); backward: the backward of the 32768-token
    case (G = 4); prefill131072: the full-size attention, for one-pass
    counters only; standard_s512, endprompt_s8192, periodic_s32768,
    nope_s32768: those workloads at full size (under 2 GB each); decode256,
    decode64: the 131072-key bifocal decode at head_dim 256 (1 GiB of cache)
    and 64."""
    from position_remapping_b200 import ropeattn as ra
    dev = torch.device("cuda", 0)
    if which == "prefill131072":
        # the full-size attention, for one-pass counters (DRAM bytes) only
        P = PREFILL
        q, k, v = make_qkv(P.B, P.S, P.Hq, P.Hkv, P.D, P.seed, device=dev)
        out = torch.empty((P.B, P.S, P.Hq, P.D), dtype=torch.float32, device=dev)
        lse = torch.empty((P.B, P.Hq, P.S), dtype=torch.float32, device=dev)
        ws = torch.empty(ra.prefill_workspace_size(P.params, P.B, P.S, P.Hq, P.Hkv, P.D), dtype=torch.uint8,
                         device=dev)
        for _ in range(2):
            ra.prefill(q, k, v, P.params, out=out, lse=lse, workspace=ws)
    elif which == "backward":
        P = PREFILL
        S = 32768
        params = P.params.replace(w_pretrained=8192)
        q, k, v = make_qkv(P.B, S, P.Hq, P.Hkv, P.D, P.seed, device=dev)
        g = torch.Generator("cpu").manual_seed(P.seed + 1)
        dout = torch.randn((P.B, S, P.Hq, P.D), generator=g).to(torch.bfloat16).to(dev)
        out, lse = ra.prefill(q, k, v, params)
        ws = torch.empty(ra.prefill_backward_workspace_size(params, P.B, S, P.Hq, P.Hkv, P.D), dtype=torch.uint8,
                         device=dev)
        for _ in range(3):
            ra.prefill_backward(q, k, v, out, lse, dout, params, workspace=ws)
    elif which in CONFIG_PROFILES:
        w = WORKLOADS[which]
        q, k, v = make_qkv(w.B, w.S, w.Hq, w.Hkv, w.D, w.seed, device=dev)
        out = torch.empty((w.B, w.S, w.Hq, w.D), dtype=torch.float32, device=dev)
        lse = torch.empty((w.B, w.Hq, w.S), dtype=torch.float32, device=dev)
        ws = torch.empty(max(1, ra.prefill_workspace_size(w.params, w.B, w.S, w.Hq, w.Hkv, w.D)), dtype=torch.uint8,
                         device=dev)
        for _ in range(3):
            ra.prefill(q, k, v, w.params, out=out, lse=lse, workspace=ws)
    elif which in ("prefill", "prefill256"):
        P = PREFILL
        S = 32768
        D = 256 if which == "prefill256" else P.D
        params = P.params.replace(w_pretrained=8192)
        q, k, v = make_qkv(P.B, S, P.Hq, P.Hkv, D, P.seed, device=dev)
        ws = torch.empty(ra.prefill_workspace_size(params, P.B, S, P.Hq, P.Hkv, D), dtype=torch.uint8, device=dev)
        out = torch.empty((P.B, S, P.Hq, D), dtype=torch.float32, device=dev)
        lse = torch.empty((P.B, P.Hq, S), dtype=torch.float32, device=dev)
        for _ in range(3):
            ra.prefill(q, k, v, params, out=out, lse=lse, workspace=ws)
    else:
        Dd = DECODE
        D = DECODE_PROFILES.get(which, Dd.D)
        qd, kd, vd = make_qkv(Dd.B, Dd.S, Dd.Hq, Dd.Hkv, D, Dd.seed, device=dev, q_len=1)
        for _ in range(3):
            ra.decode(qd, kd, vd, Dd.params)
    torch.cuda.synchronize()
    ra.status()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["prefill", "prefill131072", "prefill256", "decode", "backward",
                                          *CONFIG_PROFILES, *DECODE_PROFILES], default=None,
                    help="run a capture-sized case of one kernel three times (for ncu); no timing, no JSON")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args)
        return
    if args.profile:
        run_profile_case(args.profile)
        return

    import datetime
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from position_remapping_b200 import ropeattn as ra

    # inputs resident in HBM (each rank its own seeded problem)
    P, Dd = PREFILL, DECODE
    q, k, v = make_qkv(P.B, P.S, P.Hq, P.Hkv, P.D, rank_seed(P.seed, rank), device=dev)
    qd, kd, vd = make_qkv(Dd.B, Dd.S, Dd.Hq, Dd.Hkv, Dd.D, rank_seed(Dd.seed, rank), device=dev, q_len=1)
    out = torch.empty((P.B, P.S, P.Hq, P.D), dtype=torch.float32, device=dev)
    lse = torch.empty((P.B, P.Hq, P.S), dtype=torch.float32, device=dev)
    ws = torch.empty(ra.prefill_workspace_size(P.params, P.B, P.S, P.Hq, P.Hkv, P.D), dtype=torch.uint8, device=dev)
    outd = torch.empty((Dd.B, Dd.Hq, Dd.D), dtype=torch.float32, device=dev)
    lsed = torch.empty((Dd.B, Dd.Hq), dtype=torch.float32, device=dev)
    wsd = torch.empty(ra.decode_workspace_size(Dd.B, Dd.S, Dd.Hq, Dd.Hkv, Dd.D), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        ra.prefill_prepare(k, P.Hq, P.params, ws, stream)
        if ev is not None:
            ev[1].record(stream)
        ra.prefill_attend(q, k, v, P.params, out, lse, ws, stream)
        if ev is not None:
            ev[2].record(stream)
        ra.decode(qd, kd, vd, Dd.params, out=outd, lse=lsed, workspace=wsd, stream=stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ra.status()

    uuid = ""
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ra.status()

    total_ms = t_start.elapsed_time(t_end)
    prep_ms = sum(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = sum(e[1].elapsed_time(e[2]) for e in evs)
    dec_ms = sum(e[2].elapsed_time(e[3]) for e in evs)

    # ---- end to end through the public API with host buffers: every step
    # uploads its inputs from pinned host memory and downloads its results.
    # The steps are pipelined the way a serving loop runs them: uploads on one
    # stream, compute on another, downloads on a third, with two device
    # buffer sets, so step i+1's upload and step i-1's download overlap step
    # i's compute (the library calls take the caller's stream).
    qh = q.cpu().pin_memory(); kh = k.cpu().pin_memory(); vh = v.cpu().pin_memory()
    qdh = qd.cpu().pin_memory()
    outh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lseh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    outdh = torch.empty(outd.shape, dtype=outd.dtype).pin_memory()
    lsedh = torch.empty(lsed.shape, dtype=lsed.dtype).pin_memory()
    h2d = (qh.numel() + kh.numel() + vh.numel() + qdh.numel()) * 2
    d2h = (outh.numel() + lseh.numel() + outdh.numel() + lsedh.numel()) * 4
    sets = [dict(q=q, k=k, v=v, out=out, lse=lse, qd=qd, outd=outd, lsed=lsed),
            dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v), out=torch.empty_like(out),
                 lse=torch.empty_like(lse), qd=torch.empty_like(qd), outd=torch.empty_like(outd),
                 lsed=torch.empty_like(lsed))]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(nsteps):
        ev_in = [torch.cuda.Event() for _ in range(nsteps)]
        ev_c = [torch.cuda.Event() for _ in range(nsteps)]
        ev_out = [torch.cuda.Event() for _ in range(nsteps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(nsteps):
            b = sets[i % 2]
            if i >= 2:
                s_in.wait_event(ev_c[i - 2])          # set b's inputs no longer read
            with torch.cuda.stream(s_in):
                b["q"].copy_(qh, non_blocking=True); b["k"].copy_(kh, non_blocking=True)
                b["v"].copy_(vh, non_blocking=True); b["qd"].copy_(qdh, non_blocking=True)
            ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])      # set b's outputs downloaded
            ra.prefill(b["q"], b["k"], b["v"], P.params, out=b["out"], lse=b["lse"], workspace=ws, stream=stream)
            ra.decode(b["qd"], kd, vd, Dd.params, out=b["outd"], lse=b["lsed"], workspace=wsd, stream=stream)
            ev_c[i].record(stream)
            s_out.wait_event(ev_c[i])
            with torch.cuda.stream(s_out):
                outh.copy_(b["out"], non_blocking=True); lseh.copy_(b["lse"], non_blocking=True)
                outdh.copy_(b["outd"], non_blocking=True); lsedh.copy_(b["lsed"], non_blocking=True)
            ev_out[i].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    e2e_run(2)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e2e_ms = e2e_run(args.steps)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    # the decode alone, end to end (its upload and download are a few KiB)
    e2e_dec_ms = _event_ms(lambda: (qd.copy_(qdh, non_blocking=True),
                                    ra.decode(qd, kd, vd, Dd.params, out=outd, lse=lsed, workspace=wsd, stream=stream),
                                    outdh.copy_(outd, non_blocking=True), lsedh.copy_(lsed, non_blocking=True)),
                           args.steps, stream) * args.steps
    ra.status()
    del sets[1]
    cache_rows = measure_cache_rows(ra, q, k, v, kd, vd, qd, stream)
    comparators = measure_comparators(ra, q, k, v, out, lse, ws, stream)
    comparators.update(measure_decode_comparators(ra, qd, kd, vd, stream))
    sweep = measure_sweep(ra, q, k, v, qd, kd, vd, ws, wsd, stream)
    peaks0, _ = load_peaks()
    variants = measure_variants(ra, peaks0, q, k, v, kd, vd, stream)
    backward = measure_backward(ra, q, k, v, out, lse, peaks0, stream)
    configs = measure_configs(ra, peaks0, stream, with_oracle=(world == 1 and not args.no_cpu_baseline))

    total_ms, prep_ms, attn_ms, dec_ms, e2e_ms, e2e_dec_ms = max_over_ranks(
        [total_ms, prep_ms, attn_ms, dec_ms, e2e_ms, e2e_dec_ms], world, dev)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    K = args.steps
    flops = prefill_flops(P)
    value = job_tflops(world, flops, K, prep_ms + attn_ms)
    attn_tflops = flops * K / (attn_ms / 1e3) / 1e12
    dec_us = dec_ms * 1e3 / K
    dec_gbs = decode_bytes(Dd) * K / (dec_ms / 1e3) / 1e9
    peaks, peak_src = load_peaks()
    # the attention kernel runs for ~0.1 s per launch inside a long step: sustained peak
    tpeak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    hpeak = float(peaks.get("hbm_gbs"))
    src_p = source_hash("prefill_sm100.cuh", "common.cuh")
    src_d = source_hash("decode_tc_sm100.cuh", "common.cuh")
    tr_p = traffic_record("prefill_kernel", src_p)
    tr_d = traffic_record("decode_kernel", src_d)

    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": total_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded iid N(0,1) bf16, no weights)",
        "config": config_dict(world),
        "prefill_ms": (prep_ms + attn_ms) / K,
        "prefill_prepare_ms": prep_ms / K,
        "prefill_attend_ms": attn_ms / K,
        "prefill_tokens_per_s": world * P.S * P.B * K / ((prep_ms + attn_ms) / 1e3),
        "decode_us_per_token": dec_us,
        "decode_kcycles_per_token": (dec_us * clocks["sm_mhz"] / 1e3) if clocks else None,
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": tpeak, "unit": "TFLOP/s",
                     "frac": attn_tflops / tpeak, "traffic": tr_p,
                     "kernel": "prefill_kernel<128,4> (attention; D=128, 4 ring slots)",
                     "peak_source": f"{peak_src} bf16_tflops_sustained",
                     "algorithmic": f"{flops:.6g} FLOP per launch"},
        "roofline_decode": {"bound": "hbm", "achieved": dec_gbs, "peak": hpeak, "unit": "GB/s",
                            "frac": dec_gbs / hpeak, "traffic": tr_d,
                            "frac_of_nominal_8tbs": dec_gbs / 8000.0,
                            "kernel": "decode_tc_kernel<128,2,1> (tcgen05 QK/PV, D=128, GQA 2 padded to 2, "
                                      "remote keys rotated in shared memory; + counter memset)",
                            "peak_source": f"{peak_src} hbm_gbs",
                            "algorithmic": f"{decode_bytes(Dd)} B per launch"},
        "clocks": clocks,
        "gpu_launches": 3 * K,
        "cache_rows": cache_rows,
        "comparators": comparators,
        "backward": backward,
        "length_sweep": sweep,
        "variants": variants,
        "configs": configs,
        "e2e": {"value": job_tflops(world, flops, K, e2e_ms), "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms / K,
                "note": "whole step (prefill and decode) per step time, uploads and downloads on their own "
                        "streams overlapping the previous and next steps' compute",
                "decode_us_per_token": e2e_dec_ms * 1e3 / K},
    }

    if world == 1 and not args.no_cpu_baseline:
        torch.cuda.synchronize()
        qc, kc, vc = make_qkv(P.B, P.S, P.Hq, P.Hkv, P.D, P.seed)
        qdc, kdc, vdc = make_qkv(Dd.B, Dd.S, Dd.Hq, Dd.Hkv, Dd.D, Dd.seed, q_len=1)
        tf, dus, secs, sample = oracle_step(CPU_ROWS, CPU_KV, qc, kc, vc, qdc, kdc, vdc)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": sample, "decode_us_per_token": dus, "seconds": secs}
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
