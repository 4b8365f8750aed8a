#!/usr/bin/env python
"""Benchmark of the compressed-KV hot path (one JSON line on rank 0).

A step is one pass of the per-batch hot path over one batch of synthetic
input: compress the prompt's keys and values of every layer into packed
records (rotation, Lloyd-Max codes, QJL signs, packing), append one decode
token per layer, and run decode attention of every query head over the
packed cache. Calibration is per model, not per batch (the SpectralQuant
README calls it a one-time calibration): it runs once before the timed steps
and is timed and reported on its own in the same line.

Default workload: Llama-3.1-8B-shaped (32 layers, 32 query / 8 KV heads,
head_dim 128, fp16, a 2048-token prompt, batch 1 per GPU, 3 bits per
coordinate for keys and values). Layers are folded into the head index so
each kernel covers all layers in one launch.

End to end (the ``e2e`` key): the same step with every input in pinned host
memory, through the C ABI: the prompt through sq_compress_kv_host (its
host-to-device copies overlap the compression of the previous piece), the
decode token and query copied in, the output copied back, all inside the
timed region.

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


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return HBM_FALLBACK_GBS, "fallback"


# --------------------------------------------------------------------------- workload
def build_workload(name: str, device: str, layers: int | None = None):
    """All layers of one replica, layers folded into the head index. Tensors are
    preallocated and filled layer by layer (the largest shape holds ~90 GB of fp16 KV)."""
    import torch

    from synthetic.workloads import CONFIGS, TORCH_DTYPE, make_workload

    cfg = dict(CONFIGS[name])
    cfg["name"] = name
    if layers:
        cfg["layers"] = layers
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


def record_bytes_per_token(cfg, words_k, words_v, qjl):
    """Algorithmic bytes moved per (token, head) by compress: input + record + side scalars."""
    esz = 4 if cfg["dtype"] == "f32" else 2
    kin = cfg["d"] * esz
    k_out = 4 * words_k + 4 + (4 if qjl else 0)
    v_out = 4 * words_v + 4
    return kin + k_out, kin + v_out, k_out, v_out


# Source files each profiled kernel is built from (its DRAM traffic in
# profiles/traffic.json is used only while these files are unchanged).
KERNEL_SOURCES = {
    "k_compress_tc": ["tc_compress.cuh", "sm100.cuh", "sq_common.cuh"],
    "k_attn_partial_tc": ["fast_attn.cuh", "attention.cuh", "sq_common.cuh"],
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


def profiled_traffic(kernel: str, tokens_per_launch: int):
    """DRAM bytes per launch of `kernel` from profiles/traffic.json (written from an ncu
    capture of the same sources), scaled to this launch's tokens; None if stale or absent."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            ent = json.load(f)["kernels"][kernel]
        if ent["source_hash"] != kernel_source_hash(kernel):
            return None
        return ent["dram_bytes"] * tokens_per_launch / ent["tokens"]
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
def oracle_sample(name: str, tokens: int, q_heads: int, ctx: int):
    """Times the oracle on one layer's KV heads: compress `tokens` tokens (K and V) and
    decode attention of `q_heads` query heads over `ctx` packed tokens. Returns a dict of
    rates (head-tokens/s for compress, context head-tokens/s for attention)."""
    import numpy as np

    from oracle import attention as oattn
    from oracle import calibration as ocal
    from oracle import codec as ocodec
    from synthetic import CONFIGS, make_workload

    cfg = CONFIGS[name]
    n_kv = cfg["n_kv"]
    w = make_workload(name, 0, batch=1, tokens=max(tokens, ctx))
    ck = [ocal.calibrate(w.k_cal[h].double().numpy(), avg_bits=cfg["bits_k"], is_key=True, stream=h)
          for h in range(n_kv)]
    cv = [ocal.calibrate(w.v_cal[h].double().numpy(), avg_bits=cfg["bits_v"], is_key=False, stream=h)
          for h in range(n_kv)]
    t0 = time.perf_counter()
    packed = []
    for h in range(n_kv):
        ok = ocodec.compress(w.k[0, h, :tokens].double().numpy(), ck[h])
        ov = ocodec.compress(w.v[0, h, :tokens].double().numpy(), cv[h])
        packed.append((ok, ov))
    t_c = time.perf_counter() - t0
    # attention over ctx tokens (reuse compressed records, tiled to ctx)
    group = cfg["n_q"] // n_kv
    reps = max(1, math.ceil(ctx / tokens))
    kw = np.stack([np.tile(p[0]["words"], (reps, 1))[:ctx] for p in packed])[None]
    kn = np.stack([np.tile(p[0]["norm"], reps)[:ctx] for p in packed])[None]
    kr = np.stack([np.tile(p[0]["rnorm"], reps)[:ctx] for p in packed])[None]
    vw = np.stack([np.tile(p[1]["words"], (reps, 1))[:ctx] for p in packed])[None]
    vn = np.stack([np.tile(p[1]["norm"], reps)[:ctx] for p in packed])[None]
    nq = min(q_heads, n_kv * group)
    nkv_used = max(1, nq // group)
    q = w.q[:, :nkv_used * group].double().numpy()
    t0 = time.perf_counter()
    oattn.attn_decode(q, kw[:, :nkv_used], kn[:, :nkv_used], kr[:, :nkv_used], vw[:, :nkv_used],
                      vn[:, :nkv_used], ck[:nkv_used], cv[:nkv_used], [ctx], None)
    t_a = time.perf_counter() - t0
    return {"compress_rate": n_kv * tokens / t_c, "attn_rate": nkv_used * group * ctx / t_a,
            "seconds": t_c + t_a, "tokens": tokens, "ctx": ctx, "q_heads": nkv_used * group}


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_step_seconds(name: str, s: dict) -> float:
    """Oracle seconds of one full step, extrapolated linearly from the sample rates."""
    from synthetic import CONFIGS

    cfg = CONFIGS[name]
    H = cfg["layers"] * cfg["n_kv"]
    HQ = cfg["layers"] * cfg["n_q"]
    B = cfg["batch"]
    if cfg["mode"] == "prefill":
        compress = B * H * (cfg["ctx"] + 1) / s["compress_rate"]
        attn = B * HQ * (cfg["ctx"] + 1) / s["attn_rate"]
    else:
        compress = B * H * 1 / s["compress_rate"]
        attn = B * HQ * (cfg["ctx"] + 1) / s["attn_rate"]
    return compress + attn


def step_tokens(cfg) -> int:
    return cfg["batch"] * ((cfg["ctx"] + 1) if cfg["mode"] == "prefill" else 1)


# --------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return
    from synthetic import CONFIGS

    cfg = CONFIGS[args.config]
    times = []
    sample = None
    for i in range(args.warmup + args.steps):
        s = oracle_sample(args.config, tokens=64, q_heads=cfg["n_q"] // cfg["n_kv"], ctx=256)
        if i >= args.warmup:
            times.append(oracle_step_seconds(args.config, s))
            sample = s
    t = statistics.mean(times)
    value = step_tokens(cfg) / t
    desc = (f"oracle (NumPy float64) per step on one layer's {cfg['n_kv']} KV heads: compress of "
            f"{sample['tokens']} tokens (K and V) and decode attention of {sample['q_heads']} query heads over "
            f"{sample['ctx']} tokens; extrapolated linearly to the full step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(cfg, world):
    return {"workload": f"{cfg_name(cfg)}: {cfg['layers']} layers x {cfg['n_kv']} KV / {cfg['n_q']} query heads, "
                        f"head_dim {cfg['d']}, {cfg['dtype']} KV, "
                        + (f"prompt {cfg['ctx']} tokens + 1 decode token" if cfg["mode"] == "prefill"
                           else f"1 decode token over a {cfg['ctx']}-token packed cache")
                        + f", batch {cfg['batch']} per GPU, K {cfg['bits_k']} / V {cfg['bits_v']} bits per coordinate",
            "global_batch": cfg["batch"] * world, "layers": cfg["layers"], "head_dim": cfg["d"],
            "context": cfg["ctx"], "l2": "inputs larger than L2 every step (no flush needed)"}


def cfg_name(cfg):
    from synthetic import CONFIGS
    if "name" in cfg:
        return cfg["name"]
    for k, v in CONFIGS.items():
        if v is cfg:
            return k
    return "custom"


# --------------------------------------------------------------------------- GPU arm
def run_gpu(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from compressed_attention_head_b200 import sq

    dev = f"cuda:{local_rank}"
    torch.cuda.set_device(local_rank)
    sq.sq_init()
    wl = build_workload(args.config, dev, args.layers)
    cfg, H, HQ, d, T, B = wl["cfg"], wl["H"], wl["HQ"], wl["d"], wl["T"], wl["batch"]
    prefill = cfg["mode"] == "prefill"
    stream = torch.cuda.current_stream()

    # ---- calibration (once per model; timed on its own)
    pk = sq.calib_params(d, H, cfg["bits_k"], True)
    pv = sq.calib_params(d, H, cfg["bits_v"], False)
    rk, rv = sq.alloc_records(H, d, dev), sq.alloc_records(H, d, dev)
    ncal = wl["k_cal"].shape[1]
    cws = torch.empty(sq.sq_calibrate_workspace(pk, ncal), dtype=torch.uint8, device=dev)
    st = torch.zeros(2 * H, dtype=torch.int32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    sq.sq_calibrate(pk, wl["k_cal"], ncal, ncal * d, d, rk, cws, st[:H])
    sq.sq_calibrate(pv, wl["v_cal"], ncal, ncal * d, d, rv, cws, st[H:])
    e1.record()
    torch.cuda.synchronize()
    calib_ms = e0.elapsed_time(e1)
    n_bad = int((st != 0).sum().item())
    words_k, words_v = sq.sq_record_words(pk), sq.sq_record_words(pv)
    del cws

    cap = ((T + 1 + 15) // 16) * 16
    kc = sq.alloc_cache(B, H, cap, words_k, True, dev)
    vc = sq.alloc_cache(B, H, cap, words_v, False, dev)
    pos0 = torch.zeros(B, dtype=torch.int32, device=dev)
    posT = torch.full((B,), T, dtype=torch.int32, device=dev)
    lens = torch.full((B,), T + 1, dtype=torch.int32, device=dev)
    max_ctx = T + 1
    aws = torch.empty(sq.sq_attn_workspace(B, HQ, H, d, max_ctx), dtype=torch.uint8, device=dev)
    out = torch.empty(B, HQ, d, dtype=torch.float32, device=dev)
    flags = torch.zeros(1, dtype=torch.int32, device=dev)
    if not prefill:
        # decode configs: the cache of ctx tokens is filled once, outside the timed steps,
        # and the fp16 prompt is released
        sq.sq_compress_kv(rk, rv, wl["k"], wl["v"], B, H, d, T, pos0, kc, vc, flags)
        torch.cuda.synchronize()
        del wl["k"], wl["v"]
        torch.cuda.empty_cache()

    n_ev = 6
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]

    def step(ev=None):
        if ev: ev[0].record()
        if prefill:
            sq.sq_compress_kv(rk, None, wl["k"], None, B, H, d, T, pos0, kc, None, flags)
            if ev: ev[1].record()
            sq.sq_compress_kv(None, rv, None, wl["v"], B, H, d, T, pos0, None, vc, flags)
        if ev: ev[2].record()
        sq.sq_compress_kv(rk, rv, wl["k_new"], wl["v_new"], B, H, d, 1, posT, kc, vc, flags)
        if ev: ev[3].record()
        sq.sq_attn_decode(rk, rv, kc, vc, lens, B, HQ, H, d, max_ctx, wl["q"], 0.0, out, None, aws, flags)
        if ev: ev[4].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(local_rank)
    clocks.start()
    torch.cuda.synchronize()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(args.steps):
        step(evs[i])
    t_end.record()
    torch.cuda.synchronize()
    clk = clocks.stop()
    elapsed = max_over_ranks(t_start.elapsed_time(t_end) / 1e3, dev)
    per_step = elapsed / args.steps
    # The same step captured once as a CUDA graph and replayed: the launch gaps of the
    # eager loop go away (every call is asynchronous, allocates nothing, and the
    # per-device tables were uploaded by sq_init before capture).
    graph_step = None
    if not args.no_graph:
        try:
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                step()
            torch.cuda.current_stream().wait_stream(side)
            torch.cuda.synchronize()
            with torch.cuda.graph(g):
                step()
            for _ in range(args.warmup):
                g.replay()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(args.steps):
                g.replay()
            b_.record()
            torch.cuda.synchronize()
            graph_step = max_over_ranks(a.elapsed_time(b_) / 1e3, dev) / args.steps
            del g
        except Exception as exc:       # report, keep the eager number
            print(f"graph capture failed: {exc}", file=sys.stderr)
            graph_step = None
    eager_step = per_step
    if graph_step is not None:
        per_step = graph_step
    if prefill:
        ck_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
        cv_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    else:
        ck_ms = cv_ms = 0.0
    app_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    att_ms = statistics.mean(e[3].elapsed_time(e[4]) for e in evs)
    flag_val = int(flags.item())

    # ---- algorithmic bytes
    kb, vb, k_out, v_out = record_bytes_per_token(cfg, words_k, words_v, True)
    comp_bytes_k = B * H * T * kb
    comp_bytes_v = B * H * T * vb
    attn_bytes = B * H * (T + 1) * (k_out + v_out)
    peak, peak_kind = _peaks()
    tokens = step_tokens(cfg) * world
    value = tokens / per_step
    if prefill:
        dom = {"kernel": "k_compress_tc (prompt compress; mean of the K and V launches)",
               "bytes": (comp_bytes_k + comp_bytes_v) / 2, "ms": (ck_ms + cv_ms) / 2,
               "ncu_name": "k_compress_tc", "tokens": B * H * T}
    else:
        dom = {"kernel": "sq_attn_decode (prepare + partial + combine)", "bytes": attn_bytes, "ms": att_ms,
               "ncu_name": "k_attn_partial_tc", "tokens": B * H * (T + 1)}
    achieved = dom["bytes"] / (dom["ms"] / 1e3) / 1e9
    breakdown = {
        "step_ms_eager": 1e3 * eager_step, "step_ms_graph": None if graph_step is None else 1e3 * graph_step,
        "compress_k_ms": ck_ms, "compress_v_ms": cv_ms, "append_ms": app_ms, "attention_ms": att_ms,
        "compress_GBps": ((comp_bytes_k + comp_bytes_v) / ((ck_ms + cv_ms) / 1e3) / 1e9) if prefill else None,
        "attention_GBps": attn_bytes / (att_ms / 1e3) / 1e9,
        "attention_frac_of_hbm": attn_bytes / (att_ms / 1e3) / 1e9 / peak,
        "decode_tokens_per_s": B * world / ((app_ms + att_ms) / 1e3),
        "compress_tokens_per_s": (B * T * world / ((ck_ms + cv_ms) / 1e3)) if prefill else None,
        "compress_bytes_per_token_head": {"k": kb, "v": vb}, "attention_bytes_per_token_head": k_out + v_out,
    }

    # ---- end to end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        hk = wl["k"].cpu().pin_memory() if prefill else None
        hv = wl["v"].cpu().pin_memory() if prefill else None
        hkn, hvn, hq = wl["k_new"].cpu().pin_memory(), wl["v_new"].cpu().pin_memory(), wl["q"].cpu().pin_memory()
        hout = torch.empty_like(out, device="cpu").pin_memory()

        # the prompt goes through the library's host-input compress (its copies
        # overlap the compression of the previous piece); the decode inputs are
        # small and copied directly
        staging = torch.empty(sq.sq_compress_host_staging(B, H, d, wl["k"].dtype, T), dtype=torch.uint8,
                              device=dev) if prefill else None

        def e2e_step():
            wl["k_new"].copy_(hkn, non_blocking=True)
            wl["v_new"].copy_(hvn, non_blocking=True)
            wl["q"].copy_(hq, non_blocking=True)
            if prefill:
                sq.sq_compress_kv_host(rk, rv, hk, hv, B, H, d, T, pos0, kc, vc, staging, flags)
            sq.sq_compress_kv(rk, rv, wl["k_new"], wl["v_new"], B, H, d, 1, posT, kc, vc, flags)
            sq.sq_attn_decode(rk, rv, kc, vc, lens, B, HQ, H, d, max_ctx, wl["q"], 0.0, out, None, aws, flags)
            hout.copy_(out, non_blocking=True)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(args.steps):
            e2e_step()
        b.record()
        torch.cuda.synchronize()
        t_e2e = max_over_ranks(a.elapsed_time(b) / 1e3, dev)
        h2d = (hk.numel() * hk.element_size() + hv.numel() * hv.element_size() if prefill else 0) + \
            hkn.numel() * hkn.element_size() + hvn.numel() * hvn.element_size() + hq.numel() * hq.element_size()
        e2e = {"value": tokens / (t_e2e / args.steps), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": hout.numel() * hout.element_size()}

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu:
        s = oracle_sample(args.config, tokens=args.cpu_tokens, q_heads=cfg["n_q"], ctx=args.cpu_ctx)
        t_oracle = oracle_step_seconds(args.config, s)
        cpu = {"value": step_tokens(cfg) / t_oracle, "unit": "tokens/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"one layer ({cfg['n_kv']} KV heads): compress of {s['tokens']} tokens K+V and decode "
                         f"attention of {s['q_heads']} query heads over {s['ctx']} tokens, {s['seconds']:.1f} s of "
                         f"CPU work, extrapolated linearly to the full step"}
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16",
        "dtype_detail": "fp16 tensor-core rotation and attention with f32 accumulation; f64 for the key signal "
                        "coordinates and for exact recomputation of codes near a threshold", "data": "synthetic",
        "config": workload_config(cfg, world),
        "roofline": {"bound": "hbm", "kernel": dom["kernel"], "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": profiled_traffic(dom["ncu_name"], dom["tokens"]),
                     "bytes_per_launch": dom["bytes"], "launch_ms": dom["ms"]},
        "cpu_baseline": cpu, "e2e": e2e,
        # per step: prompt compress K and V (tensor-core kernel + the pass for heads with
        # more than 16 QJL dimensions, each), two appends, prepare + partial + combine
        "gpu_launches": args.steps * ((4 if prefill else 0) + 2 + 3),
        "clocks": clk, "breakdown": breakdown,
        "calibration": {"ms": calib_ms, "heads": 2 * H, "tokens_per_head": ncal, "status_nonzero": n_bad},
        "device_flags": flag_val,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="sq", choices=["sq", "reference"])
    ap.add_argument("--config", default="llama8b")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time the eager launches only")
    ap.add_argument("--layers", type=int, default=0, help="fewer layers (profiling captures only)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--cpu-tokens", type=int, default=32768)
    ap.add_argument("--cpu-ctx", type=int, default=8192)
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
