#!/usr/bin/env python
"""Benchmark of the compressed-KV hot path (one JSON line on rank 0).

Default (``--config headline``): the largest decode workload, Gemma-2-9B-shaped
(42 layers, 16 query / 8 KV heads, head_dim 256, bf16, batch 64 at context
4096, 3 bits per coordinate for keys and values, QJL on): a step is one decode
step of every layer -- the new token's keys and values compressed into the
packed cache (append) and decode attention of every query head over the
whole packed context. ``value`` is decode tokens per second (batch rows per
step / step time). In the same run and line, the prompt compress of the
Llama-3.1-8B-shaped prefill (32 layers x 8 KV heads, head_dim 128, fp16, 2048
tokens, 3 bits) is measured as the compression half of the metric
(``compress`` object and ``roofline_compress``).

``--config NAME`` runs one workload of synthetic/workloads.py instead: a
prefill workload (tiny, llama8b) times compress-prompt + append + attention
per step; a decode workload (qwen14b, qwen1_5b_long, gemma9b_sweep, with
``--bits`` for the Gemma sweep and ``--no-qjl``) times append + attention.

Decode caches: filling a context of millions of tokens through the float64
compress of a bf16 head_dim-256 cache would take minutes, so the packed
records of one layer's KV heads for a few batch rows are compressed from
synthetic draws and repeated over the layers and the batch (distinct buffers:
every step reads the whole cache from HBM); the calibration records repeat
with them. Layers are folded into the head index, so each kernel covers all
layers in one launch.

End to end (the ``e2e`` key): the same step with every input in pinned host
memory, through the C ABI: the prompt through sq_compress_kv_host (prefill),
the decode tokens and queries copied in, the output copied back, all inside
the timed region.

Multi-GPU: ``torchrun --nproc-per-node N bench.py --gpus N``. Each rank runs
its own independent replica (weak scaling; the path has no exchange step).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "compressed-KV decode tokens/s & compress GB/s, % of B200 HBM roofline"
HBM_FALLBACK_GBS = 6650.0
HEADLINE_DECODE = "gemma9b_sweep"
HEADLINE_COMPRESS = "llama8b"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return HBM_FALLBACK_GBS, "fallback"


# --------------------------------------------------------------------------- workload
def workload_cfg(name: str, layers: int | None = None, bits: float | None = None, qjl: bool = True):
    from synthetic.workloads import CONFIGS

    cfg = dict(CONFIGS[name])
    cfg["name"] = name
    if layers:
        cfg["layers"] = layers
    if bits is not None:
        cfg["bits_k"] = cfg["bits_v"] = float(bits)
    cfg["qjl"] = bool(qjl)
    return cfg


def build_prefill(cfg, device: str):
    """All layers of one replica, layers folded into the head index, every layer
    drawn on its own (the prompt is compressed inside the timed step)."""
    import torch

    from synthetic.workloads import TORCH_DTYPE, make_workload

    L, nkv, nq, d = cfg["layers"], cfg["n_kv"], cfg["n_q"], cfg["d"]
    T, B, ncal = cfg["ctx"], cfg["batch"], cfg["n_cal"]
    dt = TORCH_DTYPE[cfg["dtype"]]
    H, HQ = L * nkv, L * nq
    k = torch.empty(B, H, T, d, dtype=dt, device=device)
    v = torch.empty_like(k)
    k_cal = torch.empty(H, ncal, d, dtype=dt, device=device)
    v_cal = torch.empty_like(k_cal)
    q = torch.empty(B, HQ, d, dtype=dt, device=device)
    k_new = torch.empty(B, H, 1, d, dtype=dt, device=device)
    v_new = torch.empty_like(k_new)
    for layer in range(L):
        w = make_workload(cfg, layer, device=device, batch=B, tokens=T)
        nxt = make_workload(cfg, layer, device=device, batch=B, tokens=1, data_stream=1, with_calibration=False)
        hs = slice(layer * nkv, (layer + 1) * nkv)
        k[:, hs] = w.k
        v[:, hs] = w.v
        k_cal[hs] = w.k_cal
        v_cal[hs] = w.v_cal
        q[:, layer * nq:(layer + 1) * nq] = nxt.q
        k_new[:, hs] = nxt.k
        v_new[:, hs] = nxt.v
        del w, nxt
    return dict(cfg=cfg, H=H, HQ=HQ, d=d, T=T, batch=B, k=k, v=v, k_cal=k_cal, v_cal=v_cal, q=q,
                k_new=k_new, v_new=v_new)


def record_bytes(words: int, qjl: bool) -> int:
    """Bytes of one stored vector in the packed cache: record + norm (+ rho)."""
    return 4 * words + 4 + (4 if qjl else 0)


def rep_divisor(n: int, want: int) -> int:
    """The largest divisor of n that is at most want."""
    for k in range(min(n, want), 0, -1):
        if n % k == 0:
            return k
    return 1


# Source files each profiled kernel is built from (its DRAM traffic in
# profiles/traffic.json is used only while these files are unchanged).
KERNEL_SOURCES = {
    "k_compress_tc": ["tc_compress.cuh", "sm100.cuh", "sq_common.cuh"],
    "k_attn_partial_tc": ["fast_attn.cuh", "attention.cuh", "sq_common.cuh"],
    "k_decode_tc": ["tc_decode.cuh", "attention.cuh", "sm100.cuh", "sq_common.cuh"],
    "k_compress_blk": ["blk_compress.cuh", "codec.cuh", "sq_common.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the sources of `kernel`; profile counters are reported only for the
    kernel sources they were captured from."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "compressed_attention_head_b200", "csrc")
    for fn in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, algorithmic_bytes: float):
    """DRAM bytes per launch of `kernel` from profiles/traffic.json (written from an ncu
    capture of the same sources), scaled by this launch's algorithmic bytes over the
    captured launch's (DRAM traffic grows with the records read); None if stale or absent."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            ent = json.load(f)["kernels"][kernel]
        if ent["source_hash"] != kernel_source_hash(kernel):
            return None
        return ent["dram_bytes"] * algorithmic_bytes / ent["algorithmic_bytes"]
    except Exception:
        return None


def max_over_ranks(value: float, device) -> float:
    """The largest per-rank value (elapsed time) across the process group."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            # the sampler is running before the timed region starts (first line written)
            t0 = time.time()
            while time.time() - t0 < 5.0 and os.path.getsize(self.path) == 0:
                time.sleep(0.01)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        # one more sample at the end of the timed region (short regions see few)
        try:
            with open(self.path, "a") as f:
                subprocess.run(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                "--format=csv,noheader,nounits"], stdout=f, stderr=subprocess.DEVNULL, timeout=10)
        except Exception:
            pass
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for n, flag in zip(names, parts[5:9]):
                    if flag.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------- CPU oracle
def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _oracle_head(cfg, n_heads: int, tokens: int):
    """Oracle calibrations and a seeded draw of ``tokens`` tokens for the first
    ``n_heads`` KV heads of layer 0 (CPU, float64)."""
    from oracle import calibration as ocal
    from synthetic import make_workload

    g = cfg["n_q"] // cfg["n_kv"]
    w = make_workload(dict(cfg, n_kv=n_heads, n_q=n_heads * g), 0, batch=1, tokens=tokens)
    ck = [ocal.calibrate(w.k_cal[h].double().numpy(), avg_bits=cfg["bits_k"], is_key=True,
                         qjl=cfg.get("qjl", True), stream=h) for h in range(n_heads)]
    cv = [ocal.calibrate(w.v_cal[h].double().numpy(), avg_bits=cfg["bits_v"], is_key=False, stream=h)
          for h in range(n_heads)]
    return w, ck, cv


def oracle_prefill_sample(cfg, tokens: int, ctx: int):
    """Oracle seconds of one full prefill step (compress the prompt of every
    layer, append, attention of every query head over the context), from a
    timed sample of one layer: compress ``tokens`` tokens of its KV heads (K and
    V) and decode attention of its query heads over ``ctx`` packed tokens,
    extrapolated linearly in vectors and in attended token-heads."""
    import numpy as np

    from oracle import attention as oattn
    from oracle import codec as ocodec

    n_kv, g = cfg["n_kv"], cfg["n_q"] // cfg["n_kv"]
    w, ck, cv = _oracle_head(cfg, n_kv, max(tokens, ctx))
    t0 = time.perf_counter()
    packed = []
    for h in range(n_kv):
        packed.append((ocodec.compress(w.k[0, h, :tokens].double().numpy(), ck[h]),
                       ocodec.compress(w.v[0, h, :tokens].double().numpy(), cv[h])))
    t_c = time.perf_counter() - t0
    reps = max(1, math.ceil(ctx / tokens))
    tile = lambda a: np.tile(a, (reps,) + (1,) * (a.ndim - 1))[:ctx]      # noqa: E731
    kw = np.stack([tile(p[0]["words"]) for p in packed])[None]
    kn = np.stack([tile(p[0]["norm"]) for p in packed])[None]
    kr = np.stack([tile(p[0]["rnorm"]) for p in packed])[None]
    vw = np.stack([tile(p[1]["words"]) for p in packed])[None]
    vn = np.stack([tile(p[1]["norm"]) for p in packed])[None]
    q = w.q.double().numpy()
    t0 = time.perf_counter()
    oattn.attn_decode(q, kw, kn, kr, vw, vn, ck, cv, [ctx], None)
    t_a = time.perf_counter() - t0
    H, HQ, B, T = cfg["layers"] * n_kv, cfg["layers"] * cfg["n_q"], cfg["batch"], cfg["ctx"]
    step = B * H * (T + 1) * t_c / (n_kv * tokens) + B * HQ * (T + 1) * t_a / (n_kv * g * ctx)
    desc = (f"one layer ({n_kv} KV heads): compress of {tokens} tokens K+V and decode attention of "
            f"{n_kv * g} query heads over {ctx} tokens, {t_c + t_a:.1f} s of CPU work, extrapolated linearly "
            f"to the full step")
    return step, t_c + t_a, desc


def oracle_decode_sample(cfg, pairs: int):
    """Oracle seconds of one full decode step (append one token K+V and attend
    G query heads over the context + 1 tokens, for every (batch row, KV head)),
    from a timed sample of ``pairs`` (batch row, KV head) pairs at the full
    context; the packed context is built outside the timing by compressing
    4096 tokens and repeating them."""
    import numpy as np

    from oracle import attention as oattn
    from oracle import codec as ocodec

    g, T = cfg["n_q"] // cfg["n_kv"], cfg["ctx"]
    base = min(T, 4096)
    w, ck, cv = _oracle_head(cfg, 1, base + 1)
    pk = ocodec.compress(w.k[0, 0, :base].double().numpy(), ck[0])
    pv = ocodec.compress(w.v[0, 0, :base].double().numpy(), cv[0])
    reps = math.ceil((T + 1) / base)
    tile = lambda a: np.tile(a, (reps,) + (1,) * (a.ndim - 1))[:T + 1]    # noqa: E731
    kw, kn, kr = tile(pk["words"]), tile(pk["norm"]), tile(pk["rnorm"])
    vw, vn = tile(pv["words"]), tile(pv["norm"])
    xk = w.k[0, 0, base:base + 1].double().numpy()
    xv = w.v[0, 0, base:base + 1].double().numpy()
    q = w.q.double().numpy()
    t0 = time.perf_counter()
    for _ in range(pairs):
        ok_ = ocodec.compress(xk, ck[0])
        ov_ = ocodec.compress(xv, cv[0])
        kw[T], kn[T], kr[T] = ok_["words"][0], ok_["norm"][0], ok_["rnorm"][0]
        vw[T], vn[T] = ov_["words"][0], ov_["norm"][0]
        oattn.attn_decode(q, kw[None, None], kn[None, None], kr[None, None], vw[None, None], vn[None, None],
                          ck, cv, [T + 1], None)
    t = time.perf_counter() - t0
    B, H = cfg["batch"], cfg["layers"] * cfg["n_kv"]
    step = B * H * t / pairs
    desc = (f"{pairs} (batch row, KV head) pairs of one decode step: append of the new token (K and V) and "
            f"decode attention of {g} query heads over {T + 1} packed tokens, {t:.1f} s of CPU work, "
            f"extrapolated linearly to the {B} x {H} pairs of the step")
    return step, t, desc


def step_tokens(cfg) -> int:
    """Tokens one step processes: prompt + decode token for prefill, one decode token per row otherwise."""
    return cfg["batch"] * ((cfg["ctx"] + 1) if cfg["mode"] == "prefill" else 1)


def workload_config(cfg, world):
    qjl = cfg.get("qjl", True)
    return {"workload": f"{cfg['name']}: {cfg['layers']} layers x {cfg['n_kv']} KV / {cfg['n_q']} query heads, "
                        f"head_dim {cfg['d']}, {cfg['dtype']} KV, "
                        + (f"prompt {cfg['ctx']} tokens + 1 decode token" if cfg["mode"] == "prefill"
                           else f"1 decode token over a {cfg['ctx']}-token packed cache")
                        + f", batch {cfg['batch']} per GPU, K {cfg['bits_k']} / V {cfg['bits_v']} bits per "
                        f"coordinate, QJL {'on' if qjl else 'off'}",
            "global_batch": cfg["batch"] * world, "layers": cfg["layers"], "head_dim": cfg["d"],
            "context": cfg["ctx"], "l2": "inputs larger than L2 every step (no flush needed)"}


# --------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The oracle (NumPy float64, as it stands) on the host cores, on a bounded
    sample of the same workload each step, extrapolated to the full step."""
    if rank != 0:
        return
    name = HEADLINE_DECODE if args.config == "headline" else args.config
    cfg = workload_cfg(name, args.layers, args.bits, not args.no_qjl)
    times, samples = [], []
    desc = ""
    for i in range(args.warmup + args.steps):
        if cfg["mode"] == "decode":
            t, secs, desc = oracle_decode_sample(cfg, pairs=args.ref_pairs)
        else:
            t, secs, desc = oracle_prefill_sample(cfg, tokens=args.ref_tokens, ctx=args.ref_ctx)
        if i >= args.warmup:
            times.append(t)
            samples.append(secs)
    t = statistics.mean(times)
    value = step_tokens(cfg) / t
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t,
            "ms_per_step_kind": "extrapolated from the timed sample of each step (see cpu_baseline.sample)",
            "sample_ms_per_step": 1e3 * statistics.mean(samples),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- GPU arm
def _events(n):
    import torch
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


def _time_loop(step, steps, warmup, world, dev, n_marks):
    """Eager timing of ``steps`` steps (after ``warmup``), barrier + synchronize on
    both sides; per-step marks for the per-launch breakdown. Returns
    (seconds per step, max over ranks; list of per-step mark lists)."""
    import torch
    import torch.distributed as dist

    for _ in range(warmup):
        step(None)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    marks = [_events(n_marks) for _ in range(steps)]
    a, b = _events(2)
    a.record()
    for i in range(steps):
        step(marks[i])
    b.record()
    torch.cuda.synchronize()
    return max_over_ranks(a.elapsed_time(b) / 1e3, dev) / steps, marks


def _time_graph(step, steps, warmup, world, dev):
    """The same step captured once as a CUDA graph and replayed (every call is
    asynchronous and allocates nothing; the per-device tables were uploaded by
    sq_init before capture). Seconds per step (max over ranks), or None."""
    import torch
    import torch.distributed as dist

    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step(None)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            step(None)
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a, b = _events(2)
        a.record()
        for _ in range(steps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        t = max_over_ranks(a.elapsed_time(b) / 1e3, dev) / steps
        del g
        return t
    except Exception as exc:       # report, keep the eager number
        print(f"graph capture failed: {exc}", file=sys.stderr)
        return None


def _mean_ms(marks, i, j):
    return statistics.mean(m[i].elapsed_time(m[j]) for m in marks)


def _calibrate(sq, cfg, H, k_cal, v_cal, dev):
    """Records of H heads (GPU calibration); returns (rk, rv, words_k, words_v, ms, bad)."""
    import torch

    d, ncal = cfg["d"], k_cal.shape[1]
    pk = sq.calib_params(d, H, cfg["bits_k"], True, qjl=cfg.get("qjl", True))
    pv = sq.calib_params(d, H, cfg["bits_v"], False)
    rk, rv = sq.alloc_records(H, d, dev), sq.alloc_records(H, d, dev)
    ws = torch.empty(sq.sq_calibrate_workspace(pk, ncal), dtype=torch.uint8, device=dev)
    st_k = torch.zeros(H, dtype=torch.int32, device=dev)      # separate tensors: 16-byte aligned
    st_v = torch.zeros(H, dtype=torch.int32, device=dev)
    a, b = _events(2)
    torch.cuda.synchronize()
    a.record()
    sq.sq_calibrate(pk, k_cal, ncal, ncal * d, d, rk, ws, st_k)
    sq.sq_calibrate(pv, v_cal, ncal, ncal * d, d, rv, ws, st_v)
    b.record()
    torch.cuda.synchronize()
    n_bad = int((st_k != 0).sum().item()) + int((st_v != 0).sum().item())
    return rk, rv, sq.sq_record_words(pk), sq.sq_record_words(pv), a.elapsed_time(b), n_bad


def measure_prefill(cfg, args, world, dev):
    """Prompt compress of every layer + append + attention per step."""
    import torch

    from compressed_attention_head_b200 import sq

    wl = build_prefill(cfg, dev)
    H, HQ, d, T, B = wl["H"], wl["HQ"], wl["d"], wl["T"], wl["batch"]
    qjl = cfg.get("qjl", True)
    rk, rv, words_k, words_v, calib_ms, n_bad = _calibrate(sq, cfg, H, wl["k_cal"], wl["v_cal"], dev)
    cap = ((T + 1 + 31) // 32) * 32
    kc = sq.alloc_cache(B, H, cap, words_k, qjl, dev)
    vc = sq.alloc_cache(B, H, cap, words_v, False, dev)
    pos0 = torch.zeros(B, dtype=torch.int32, device=dev)
    posT = torch.full((B,), T, dtype=torch.int32, device=dev)
    lens = torch.full((B,), T + 1, dtype=torch.int32, device=dev)
    max_ctx = T + 1
    aws = torch.empty(sq.sq_attn_workspace(B, HQ, H, d, max_ctx), dtype=torch.uint8, device=dev)
    out = torch.empty(B, HQ, d, dtype=torch.float32, device=dev)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(ev):
        if ev: ev[0].record()
        sq.sq_compress_kv(rk, None, wl["k"], None, B, H, d, T, pos0, kc, None, flags)
        if ev: ev[1].record()
        sq.sq_compress_kv(None, rv, None, wl["v"], B, H, d, T, pos0, None, vc, flags)
        if ev: ev[2].record()
        sq.sq_compress_kv(rk, rv, wl["k_new"], wl["v_new"], B, H, d, 1, posT, kc, vc, flags)
        if ev: ev[3].record()
        sq.sq_attn_decode(rk, rv, kc, vc, lens, B, HQ, H, d, max_ctx, wl["q"], 0.0, out, None, aws, flags)
        if ev: ev[4].record()

    eager, marks = _time_loop(step, args.steps, args.warmup, world, dev, 5)
    graph = None if args.no_graph else _time_graph(step, args.steps, args.warmup, world, dev)
    ck_ms, cv_ms = _mean_ms(marks, 0, 1), _mean_ms(marks, 1, 2)
    app_ms, att_ms = _mean_ms(marks, 2, 3), _mean_ms(marks, 3, 4)
    esz = wl["k"].element_size()
    rec_k, rec_v = record_bytes(words_k, qjl), record_bytes(words_v, False)
    comp_k = B * H * T * (d * esz + rec_k)
    comp_v = B * H * T * (d * esz + rec_v)
    attn_bytes = B * H * (T + 1) * (rec_k + rec_v)
    res = dict(cfg=cfg, step_s=graph or eager, eager_s=eager, graph_s=graph, calib_ms=calib_ms, n_bad=n_bad,
               calib_heads=2 * H, ck_ms=ck_ms, cv_ms=cv_ms, app_ms=app_ms, att_ms=att_ms,
               comp_bytes=(comp_k + comp_v) / 2, comp_ms=(ck_ms + cv_ms) / 2, comp_k=comp_k, comp_v=comp_v,
               attn_bytes=attn_bytes, rec_k=rec_k, rec_v=rec_v, tokens=step_tokens(cfg),
               launches=4 + 2 + 3, flags=flags)
    if not args.no_e2e:
        hk, hv = wl["k"].cpu().pin_memory(), wl["v"].cpu().pin_memory()
        hkn, hvn, hq = wl["k_new"].cpu().pin_memory(), wl["v_new"].cpu().pin_memory(), wl["q"].cpu().pin_memory()
        hout = torch.empty_like(out, device="cpu").pin_memory()
        staging = torch.empty(sq.sq_compress_host_staging(B, H, d, wl["k"].dtype, T), dtype=torch.uint8,
                              device=dev)

        def e2e_step(ev):
            wl["k_new"].copy_(hkn, non_blocking=True)
            wl["v_new"].copy_(hvn, non_blocking=True)
            wl["q"].copy_(hq, non_blocking=True)
            sq.sq_compress_kv_host(rk, rv, hk, hv, B, H, d, T, pos0, kc, vc, staging, flags)
            sq.sq_compress_kv(rk, rv, wl["k_new"], wl["v_new"], B, H, d, 1, posT, kc, vc, flags)
            sq.sq_attn_decode(rk, rv, kc, vc, lens, B, HQ, H, d, max_ctx, wl["q"], 0.0, out, None, aws, flags)
            hout.copy_(out, non_blocking=True)

        t_e2e, _ = _time_loop(e2e_step, args.steps, args.warmup, world, dev, 1)
        h2d = sum(t.numel() * t.element_size() for t in (hk, hv, hkn, hvn, hq))
        res["e2e"] = {"value": step_tokens(cfg) * world / t_e2e, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": hout.numel() * hout.element_size()}
    if not args.no_prefill_attn:
        # causal attention of the whole prompt over its packed cache (every query
        # position of every head attends to the positions up to its own): queries
        # drawn like the keys of their KV head, scaled to the decode queries' norm
        del wl["k_new"], wl["v_new"]
        G = HQ // H
        kq = wl["k"].repeat_interleave(G, dim=1)
        scale_q = (wl["q"].float().norm(dim=-1).mean() / wl["k"][:, :, :64].float().norm(dim=-1).mean()).item()
        qp = (kq.float() * scale_q).to(wl["k"].dtype).contiguous()
        del kq
        outp = torch.empty(B, HQ, T, d, dtype=torch.float16, device=dev)
        pws = torch.empty(sq.sq_attn_prefill_workspace(B, HQ, H, d, T, max_ctx), dtype=torch.uint8, device=dev)

        def pf_step(ev):
            sq.sq_attn_prefill(rk, rv, kc, vc, pos0, B, HQ, H, d, T, max_ctx, qp, 0.0, outp, pws, flags)

        t_pf, _ = _time_loop(pf_step, max(2, args.steps // 4), 3, world, dev, 1)
        res["prefill_attn"] = {
            "workload": f"causal attention of the {T}-token prompt over its packed cache: {B} x {HQ} query heads "
                        f"({cfg['layers']} layers x {cfg['n_q']}) x {T} positions, fp16 queries and outputs",
            "ms": 1e3 * t_pf, "query_tokens_per_s": B * T * world / t_pf,
            "query_head_positions_per_s": B * HQ * T * world / t_pf, "launches": 3}
        del qp, outp, pws
    return res


def measure_decode(cfg, args, world, dev):
    """Append one token per (row, KV head) + attention over the packed context."""
    import torch

    from compressed_attention_head_b200 import sq
    from synthetic.workloads import make_workload

    L, nkv, nq, d, T, B = cfg["layers"], cfg["n_kv"], cfg["n_q"], cfg["d"], cfg["ctx"], cfg["batch"]
    H, HQ = L * nkv, L * nq
    qjl = cfg.get("qjl", True)
    b0 = rep_divisor(B, args.base_rows)
    w = make_workload(cfg, 0, device=dev, batch=b0, tokens=T)
    nxt = make_workload(cfg, 0, device=dev, batch=b0, tokens=1, data_stream=1, with_calibration=False)
    rk0, rv0, words_k, words_v, calib_ms, n_bad = _calibrate(sq, cfg, nkv, w.k_cal, w.v_cal, dev)
    size = sq.sq_calib_bytes(d)
    rk = rk0.view(nkv, size).repeat(L, 1).reshape(-1).contiguous()
    rv = rv0.view(nkv, size).repeat(L, 1).reshape(-1).contiguous()
    cap = ((T + 1 + 31) // 32) * 32
    k1 = sq.alloc_cache(b0, nkv, cap, words_k, qjl, dev)
    v1 = sq.alloc_cache(b0, nkv, cap, words_v, False, dev)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    sq.sq_compress_kv(rk0, rv0, w.k, w.v, b0, nkv, d, T, None, k1, v1, flags)
    torch.cuda.synchronize()
    comp = None
    if not args.no_cache_compress:
        # the prompt compress of this shape (one layer's heads, the base rows),
        # keys and values timed apart; it rewrites the same records. Its inputs
        # may fit in L2: a 256 MB write before each step evicts them.
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

        def comp_step(ev):
            flush.fill_(1)
            if ev: ev[0].record()
            sq.sq_compress_kv(rk0, None, w.k, None, b0, nkv, d, T, None, k1, None, flags)
            if ev: ev[1].record()
            sq.sq_compress_kv(None, rv0, None, w.v, b0, nkv, d, T, None, None, v1, flags)
            if ev: ev[2].record()

        _, cmarks = _time_loop(comp_step, max(2, args.steps // 4), 3, world, dev, 3)
        n_vec, esz = b0 * nkv * T, w.k.element_size()
        comp = dict(n=n_vec, rows=b0, k_ms=_mean_ms(cmarks, 0, 1), v_ms=_mean_ms(cmarks, 1, 2),
                    k_bytes=n_vec * (d * esz + record_bytes(words_k, qjl)),
                    v_bytes=n_vec * (d * esz + record_bytes(words_v, False)),
                    tensor_core=w.k.dtype == torch.float16 and d == 128 and T >= 64)
        del flush
    del w
    rb = B // b0

    kc, vc = k1.tiled(rb, L), v1.tiled(rb, L)
    del k1, v1
    q = nxt.q.repeat(rb, L, 1).contiguous()
    k_new = nxt.k.repeat(rb, L, 1, 1).contiguous()
    v_new = nxt.v.repeat(rb, L, 1, 1).contiguous()
    del nxt
    torch.cuda.empty_cache()
    posT = torch.full((B,), T, dtype=torch.int32, device=dev)
    lens = torch.full((B,), T + 1, dtype=torch.int32, device=dev)
    max_ctx = T + 1
    aws = torch.empty(sq.sq_attn_workspace(B, HQ, H, d, max_ctx), dtype=torch.uint8, device=dev)
    out = torch.empty(B, HQ, d, dtype=torch.float32, device=dev)

    def step(ev):
        if ev: ev[0].record()
        if args.separate:
            sq.sq_compress_kv(rk, rv, k_new, v_new, B, H, d, 1, posT, kc, vc, flags)
            if ev: ev[1].record()
            sq.sq_attn_decode(rk, rv, kc, vc, lens, B, HQ, H, d, max_ctx, q, 0.0, out, None, aws, flags)
        else:
            # the fused step: appends + query preparation in one launch, partials with the
            # last-block merge in the next, the rotation back in the last (three on the
            # tcgen05 path)
            sq.sq_decode_step(rk, rv, kc, vc, k_new, v_new, q, posT, B, HQ, H, d, max_ctx, 0.0, out, None, aws, flags)
            if ev: ev[1].record()
        if ev: ev[2].record()

    eager, marks = _time_loop(step, args.steps, args.warmup, world, dev, 3)
    graph = None if args.no_graph else _time_graph(step, args.steps, args.warmup, world, dev)
    rec_k, rec_v = record_bytes(words_k, qjl), record_bytes(words_v, False)
    attn_bytes = B * H * (T + 1) * (rec_k + rec_v)
    td = args.attn_path == 0 and cfg["d"] in (64, 128, 256) and cfg["n_q"] // cfg["n_kv"] <= 16
    if args.separate:
        app_ms, att_ms = _mean_ms(marks, 0, 1), _mean_ms(marks, 1, 2)
        launches = 2 + 3
        kernel = "sq_attn_decode (prepare + partials" + (" merging their splits + rotation)" if td else " + combine)")
    else:
        # one call: its launches are timed together (the step's whole time)
        app_ms, att_ms = 0.0, _mean_ms(marks, 0, 1)
        launches = 3 if td else 5
        kernel = ("sq_decode_step (append + prepare launch, partials launch merging their splits, rotation "
                  "launch)" if td else "sq_decode_step (appends, prepare, partials, combine)")
    res = dict(cfg=cfg, step_s=graph or eager, eager_s=eager, graph_s=graph, calib_ms=calib_ms, n_bad=n_bad,
               calib_heads=2 * nkv, app_ms=app_ms, att_ms=att_ms, attn_bytes=attn_bytes, rec_k=rec_k,
               rec_v=rec_v, tokens=step_tokens(cfg), launches=launches, kernel=kernel, flags=flags, base_rows=b0,
               cache_compress=comp,
               cache_bytes=sum(t.numel() * t.element_size() for t in (kc.codes, kc.norm, vc.codes, vc.norm)
                               + ((kc.rnorm,) if kc.rnorm is not None else ())))
    if not args.no_e2e:
        hkn, hvn, hq = k_new.cpu().pin_memory(), v_new.cpu().pin_memory(), q.cpu().pin_memory()
        hout = torch.empty_like(out, device="cpu").pin_memory()
        # The step in chunks of batch rows: the inputs of chunk i + 1 are copied in
        # (pinned host -> device, a copy stream) while chunk i computes, and the
        # outputs of chunk i are copied out while chunk i + 1 computes. Each chunk
        # pays a split setup and combine of its own: worth it only for long copies.
        copy_bytes = sum(t.numel() * t.element_size() for t in (hkn, hvn, hq, hout))
        want = args.e2e_chunks or (4 if copy_bytes >= (16 << 20) else 1)
        nch = want if (not args.separate and want > 1 and B % want == 0) else 1
        rows = B // nch
        c_in, c_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(nch)]
        ev_done = [torch.cuda.Event() for _ in range(nch)]
        ev_out = torch.cuda.Event()

        def sub(cache, r0, r1):
            return sq.PackedCache(cache.codes[r0:r1], cache.norm[r0:r1],
                                  cache.rnorm[r0:r1] if cache.rnorm is not None else None, r1 - r0, cache.n_heads,
                                  cache.cap, cache.words)

        parts = [(i * rows, (i + 1) * rows, sub(kc, i * rows, (i + 1) * rows), sub(vc, i * rows, (i + 1) * rows))
                 for i in range(nch)]
        # the library wants 16-byte aligned position arrays: one buffer per chunk
        pos_parts = [posT[r0:r1].clone() for r0, r1, _, _ in parts]
        # fewer rows per call can take more context splits per row: size the
        # workspace for the chunk too
        ws_e2e = max(aws.numel(), sq.sq_attn_workspace(rows, HQ, H, d, max_ctx))
        aws_e2e = aws if ws_e2e == aws.numel() else torch.empty(ws_e2e, dtype=torch.uint8, device=dev)

        def e2e_step(ev):
            if args.separate:
                k_new.copy_(hkn, non_blocking=True)
                v_new.copy_(hvn, non_blocking=True)
                q.copy_(hq, non_blocking=True)
                sq.sq_compress_kv(rk, rv, k_new, v_new, B, H, d, 1, posT, kc, vc, flags)
                sq.sq_attn_decode(rk, rv, kc, vc, lens, B, HQ, H, d, max_ctx, q, 0.0, out, None, aws, flags)
                hout.copy_(out, non_blocking=True)
                return
            cur = torch.cuda.current_stream()
            c_in.wait_stream(cur)
            for i, (r0, r1, kci, vci) in enumerate(parts):
                with torch.cuda.stream(c_in):
                    k_new[r0:r1].copy_(hkn[r0:r1], non_blocking=True)
                    v_new[r0:r1].copy_(hvn[r0:r1], non_blocking=True)
                    q[r0:r1].copy_(hq[r0:r1], non_blocking=True)
                    ev_in[i].record(c_in)
            for i, (r0, r1, kci, vci) in enumerate(parts):
                cur.wait_event(ev_in[i])
                sq.sq_decode_step(rk, rv, kci, vci, k_new[r0:r1], v_new[r0:r1], q[r0:r1], pos_parts[i], r1 - r0,
                                  HQ, H, d, max_ctx, 0.0, out[r0:r1], None, aws_e2e, flags)
                ev_done[i].record(cur)
                with torch.cuda.stream(c_out):
                    c_out.wait_event(ev_done[i])
                    hout[r0:r1].copy_(out[r0:r1], non_blocking=True)
            ev_out.record(c_out)
            cur.wait_event(ev_out)

        t_e2e, _ = _time_loop(e2e_step, args.steps, args.warmup, world, dev, 1)
        res["e2e"] = {"value": B * world / t_e2e, "unit": "tokens/s",
                      "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (hkn, hvn, hq)),
                      "d2h_bytes_per_step": hout.numel() * hout.element_size(), "chunks": nch}
    return res


def _roofline(kernel, ncu_name, nbytes, ms, tokens, peak, peak_kind):
    achieved = nbytes / (ms / 1e3) / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
            "unit": "GB/s", "frac": achieved / peak, "traffic": profiled_traffic(ncu_name, nbytes),
            "bytes_per_launch": nbytes, "launch_ms": ms}


def run_gpu(args, rank, world, local_rank):
    import torch

    from compressed_attention_head_b200 import sq

    dev = f"cuda:{local_rank}"
    torch.cuda.set_device(local_rank)
    sq.sq_init()
    sq.sq_set_option(sq.SQ_OPT_ATTN_PATH, args.attn_path)
    peak, peak_kind = _peaks()
    headline = args.config == "headline"
    dec_name = HEADLINE_DECODE if headline else args.config
    cfg = workload_cfg(dec_name, args.layers, args.bits, not args.no_qjl)
    clocks = ClockSampler(local_rank)
    clocks.start()
    if cfg["mode"] == "decode":
        main = measure_decode(cfg, args, world, dev)
    else:
        main = measure_prefill(cfg, args, world, dev)
    comp = None
    if headline:
        ccfg = workload_cfg(HEADLINE_COMPRESS, None, None, True)
        comp = measure_prefill(ccfg, args, world, dev)
    clk = clocks.stop()
    flag_val = int(main["flags"].item()) | (int(comp["flags"].item()) if comp else 0)
    value = main["tokens"] * world / main["step_s"]
    B, T = cfg["batch"], cfg["ctx"]
    att = _roofline(main.get("kernel", "sq_attn_decode (prepare + partials + combine)"),
                    "k_decode_tc" if args.attn_path == 0 else "k_attn_partial_tc", main["attn_bytes"],
                    main["att_ms"], B * cfg["layers"] * cfg["n_kv"] * (T + 1), peak, peak_kind)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * main["step_s"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16",
        "dtype_detail": "fp16 tensor-core contractions with f32 accumulation (attention scores and PV, the "
                        "compress rotation); f64 for the key signal coordinates and exact recomputation of codes "
                        "near a threshold", "data": "synthetic",
        "config": workload_config(cfg, world),
    }
    if cfg["mode"] == "decode":
        line["roofline"] = att
        cm = main.get("cache_compress")
        if cm:
            kname = ("tcc::k_compress_tc" if cm["tensor_core"] else
                     "blk::k_compress_blk (float64, block-tiled)" if cfg["d"] in (64, 128, 256) and T >= 16 else
                     "k_compress_ref (float64, one warp per vector)")
            line["compress_decode_shape"] = {
                "workload": f"prompt compress of {cm['rows']} batch rows x {cfg['n_kv']} KV heads x {T} tokens "
                            f"(one layer), {cfg['dtype']}, head_dim {cfg['d']}",
                "kernel": kname, "l2": "flushed before each step (256 MB write, outside the timed launches)",
                "compress_k_ms": cm["k_ms"], "compress_v_ms": cm["v_ms"],
                "compress_tokens_per_s": cm["n"] * world / ((cm["k_ms"] + cm["v_ms"]) / 1e3),
                "roofline": _roofline(kname + " (mean of the K and V launches)",
                                      "k_compress_tc" if cm["tensor_core"] else "k_compress_blk",
                                      (cm["k_bytes"] + cm["v_bytes"]) / 2, (cm["k_ms"] + cm["v_ms"]) / 2, cm["n"],
                                      peak, peak_kind)}
        line["config"]["cache"] = (f"packed records of layer 0's {cfg['n_kv']} KV heads for {main['base_rows']} "
                                   f"batch rows, compressed from synthetic draws and repeated over the "
                                   f"{cfg['layers']} layers and {B} rows ({main['cache_bytes'] / 1e9:.1f} GB "
                                   f"read per step)")
    else:
        line["roofline"] = _roofline("k_compress_tc (prompt compress; mean of the K and V launches)",
                                     "k_compress_tc", main["comp_bytes"], main["comp_ms"],
                                     B * cfg["layers"] * cfg["n_kv"] * T, peak, peak_kind)
        line["roofline_attention"] = att
    if comp is not None:
        cc = comp["cfg"]
        ntok = cc["batch"] * cc["layers"] * cc["n_kv"] * cc["ctx"]
        line["roofline_compress"] = _roofline("k_compress_tc (prompt compress; mean of the K and V launches)",
                                              "k_compress_tc", comp["comp_bytes"], comp["comp_ms"], ntok, peak,
                                              peak_kind)
        line["compress"] = {
            "workload": workload_config(cc, world)["workload"],
            "compress_GBps": (comp["comp_k"] + comp["comp_v"]) / ((comp["ck_ms"] + comp["cv_ms"]) / 1e3) / 1e9,
            "compress_tokens_per_s": cc["batch"] * cc["ctx"] * world / ((comp["ck_ms"] + comp["cv_ms"]) / 1e3),
            "compress_k_ms": comp["ck_ms"], "compress_v_ms": comp["cv_ms"],
            "bytes_per_token_head": {"k": comp["comp_k"] / ntok, "v": comp["comp_v"] / ntok},
            "step_ms": 1e3 * comp["step_s"], "step_tokens_per_s": comp["tokens"] * world / comp["step_s"],
            "attention_ms": comp["att_ms"], "append_ms": comp["app_ms"],
            "e2e": comp.get("e2e"), "gpu_launches_per_step": comp["launches"],
            "prefill_attention": comp.get("prefill_attn"),
        }
    line["cpu_baseline"] = None
    if world == 1 and not args.no_cpu:
        if cfg["mode"] == "decode":
            t_o, secs, desc = oracle_decode_sample(cfg, pairs=args.cpu_pairs)
        else:
            t_o, secs, desc = oracle_prefill_sample(cfg, tokens=args.cpu_tokens, ctx=args.cpu_ctx)
        line["cpu_baseline"] = {"value": main["tokens"] / t_o, "unit": "tokens/s", "cores": cpu_threads(),
                                "kind": "oracle", "sample": desc}
    line["e2e"] = main.get("e2e")
    line["gpu_launches"] = args.steps * main["launches"]
    line["clocks"] = clk
    bd = {"step_ms_eager": 1e3 * main["eager_s"],
          "step_ms_graph": None if main["graph_s"] is None else 1e3 * main["graph_s"],
          "append_ms": main["app_ms"], "attention_ms": main["att_ms"],
          "attention_GBps": att["achieved"], "attention_frac_of_hbm": att["frac"],
          "attention_bytes_per_token_head": main["rec_k"] + main["rec_v"],
          "decode_tokens_per_s": B * world / ((main["app_ms"] + main["att_ms"]) / 1e3)}
    if cfg["mode"] == "prefill":
        bd.update({"compress_k_ms": main["ck_ms"], "compress_v_ms": main["cv_ms"],
                   "compress_GBps": (main["comp_k"] + main["comp_v"]) / ((main["ck_ms"] + main["cv_ms"]) / 1e3)
                   / 1e9})
    line["breakdown"] = bd
    if main.get("prefill_attn"):
        line["prefill_attention"] = main["prefill_attn"]
    line["calibration"] = {"ms": main["calib_ms"], "heads": main["calib_heads"],
                           "tokens_per_head": cfg["n_cal"], "status_nonzero": main["n_bad"]}
    line["device_flags"] = flag_val
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sq", choices=["sq", "reference"])
    ap.add_argument("--config", default="headline",
                    help="headline (Gemma-shaped decode + Llama-shaped prompt compress) or a workload name")
    ap.add_argument("--bits", type=float, default=None, help="bits per coordinate for K and V (Gemma sweep)")
    ap.add_argument("--no-qjl", action="store_true")
    ap.add_argument("--separate", action="store_true",
                    help="decode step as separate calls (compress one token, then attention) instead of sq_decode_step")
    ap.add_argument("--attn-path", type=int, default=0,
                    help="attention partial kernel: 0 tcgen05 (default), 1 SIMT, 2 mma.sync (comparison runs)")
    ap.add_argument("--base-rows", type=int, default=2, help="distinct batch rows of a decode cache")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=0,
                    help="batch-row chunks of the end-to-end decode step (copies overlap compute); "
                         "0: four when the step copies at least 16 MB, else one")
    ap.add_argument("--no-graph", action="store_true", help="time the eager launches only")
    ap.add_argument("--layers", type=int, default=0, help="fewer layers (profiling captures only)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-cache-compress", action="store_true",
                    help="skip the prompt-compress line of a decode workload")
    ap.add_argument("--no-prefill-attn", action="store_true",
                    help="skip the prefill-attention line of the compress workload")
    ap.add_argument("--cpu-tokens", type=int, default=32768)
    ap.add_argument("--cpu-ctx", type=int, default=8192)
    ap.add_argument("--cpu-pairs", type=int, default=96)
    ap.add_argument("--ref-tokens", type=int, default=8192)
    ap.add_argument("--ref-ctx", type=int, default=8192)
    ap.add_argument("--ref-pairs", type=int, default=4)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = "nccl" if (args.impl == "sq" and torch.cuda.is_available()) else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
