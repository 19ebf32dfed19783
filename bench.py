"""Benchmark of the AXELRAM decode hot path on B200 (one JSON line on stdout, rank 0).

Step = one decode step over a resident quantized KV cache: the new token's key and value of every (batch row, KV
head) go through the write path (rotate + quantize + pack, appended at position T-1), then decode attention runs
over all T cached tokens (LUT scores, split-T online softmax, value product, split merge, one inverse transform for
quantized values).  The codebook is design-time (computed once at setup); sign selection is offline
(``--workload select`` times it separately).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl axr|reference]

Multi-GPU: every rank runs an independent replica of the workload (decode units are independent; no collective on
the data path), value = units of all ranks / max over ranks of the device time ("scaling": "weak").
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from kv_cache_quantized_b200 import workloads as W  # noqa: E402

METRIC = "quantized-KV decode attention: keys·heads/s and HBM GB/s vs B200 peak"
UNIT = "keys·heads/s"
L2_BYTES = 126 * 1024 * 1024

# DRAM traffic (read + write bytes) per launch of the timed decode kernel, from an ncu capture of dram__bytes_read.sum
# and dram__bytes_write.sum on the same workload at B=4 (half the units), scaled by the units processed.  Valid for
# the kernel version that capture was taken on; a workload without an entry reports null.
TRAFFIC = {
    "long_context_b8_t32768_hq32_hkv8_d128_b4_kvquant": 2 * (138.560768e6 + 3.692800e6),
}

WORKLOADS = {
    "long_context": W.LONG_CONTEXT,
    "llama8b": W.LLAMA8B_DECODE,
}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _bytes_per_key_head(w):
    """Algorithmic HBM bytes per (cached token, KV head) of one attend launch: key codes + key norm + values."""
    R = w.d * w.bits // 8
    kb = R + 2
    vb = (R + 2) if w.v_quant else 2 * w.d
    return kb + vb


class ClockSampler:
    """SM clock, power and throttle reasons sampled every 200 ms (nvidia-smi single-shot queries from a thread)
    while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, period_s=0.2):
        self.index = index
        self.period = period_s
        self.lines = []
        self._stop = None
        self._thread = None

    def _poll(self):
        while True:  # one sample at entry, then every period, and one more when stopped
            try:
                out = subprocess.run(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5)
                self.lines += [ln for ln in out.stdout.splitlines() if ln.strip()]
            except (OSError, subprocess.SubprocessError):
                return
            if self._stop.is_set():
                return
            self._stop.wait(self.period)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._poll, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._thread.join(timeout=10)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def cpu_baseline(w, seconds=10.0):
    """The fp64 oracle, as it stands, on one core: decode steps of single (batch row, KV head) units of the same
    workload (G query heads over T cached tokens, plus the new token's write), repeated for about `seconds`."""
    import oracle
    try:
        from threadpoolctl import threadpool_limits
    except ImportError:  # pragma: no cover
        threadpool_limits = None
    inp = W.decode_inputs(w, B=1)
    k, v, q, s = inp["k"][0], inp["v"][0], inp["q"][0], inp["signs"]
    scale = 1.0 / math.sqrt(w.d)
    ctx = threadpool_limits(1) if threadpool_limits else None
    if ctx:
        ctx.__enter__()
    try:
        units = 0
        t_total = 0.0
        hk = 0
        while t_total < seconds and hk < w.Hkv:
            kc, kn = oracle.write(k[hk], s, w.bits)  # cache state (setup, not timed)
            vc, vn = oracle.write(v[hk], s, w.bits) if w.v_quant else (None, None)
            t0 = time.perf_counter()
            nk = oracle.write(k[hk, -1:], s, w.bits)  # the step's append of the new token
            if w.v_quant:
                oracle.write(v[hk, -1:], s, w.bits)
            qq = q[hk * w.G:(hk + 1) * w.G][None]
            kc[-1:], kn[-1:] = nk
            if w.v_quant:
                oracle.decode_attention(qq, kc[None, None], kn[None, None], s, w.bits, scale, vcodes=vc[None, None],
                                        vn16=vn[None, None])
            else:
                oracle.decode_attention(qq, kc[None, None], kn[None, None], s, w.bits, scale, v=v[None, hk:hk + 1])
            t_total += time.perf_counter() - t0
            units += 1
            hk += 1
    finally:
        if ctx:
            ctx.__exit__(None, None, None)
    key_heads = units * w.T * w.G
    return {"value": key_heads / t_total, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{units} of {w.B * w.Hkv} (batch row, KV head) units of {w.name}: {w.G} query heads x "
                      f"{w.T} tokens each, plus the new token's write; fp64 numpy, 1 thread, {t_total:.1f} s"}


def _packed_inputs(tensors, device=None, pinned=False):
    """One byte buffer holding `tensors` back to back, each at a 16-byte aligned offset, and a view of each (its
    dtype and shape) into it; filled with the tensors' values.  On the host, pinned if asked."""
    import torch

    offs, n = [], 0
    for t in tensors:
        n = (n + 15) // 16 * 16
        offs.append(n)
        n += t.numel() * t.element_size()
    buf = torch.empty(n, dtype=torch.uint8, device=device if device is not None else "cpu")
    if pinned:
        buf = buf.pin_memory()
    views = []
    for t, o in zip(tensors, offs):
        v = buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
        v.copy_(t)
        views.append(v)
    return buf, views


def _gen_rows(gen, shape, seed, dev):
    """A synthetic fp16 tensor [B, ...] drawn one batch row at a time (bounded temporary memory)."""
    import torch
    out = torch.empty(shape, dtype=torch.float16, device=dev)
    for b in range(shape[0]):
        out[b] = gen(tuple(shape[1:]), seed + 7919 * b, dev)
    return out


def _sweep(args, dev, time_calls):
    """Decode sweep: B in {1, 8, 64} x T in {4096, 32768, 131072} x b in 1..4 x d in {64, 128}, Hq=32, Hkv=8,
    fp16 V; the LUT attend and the dense fp16 kernel on caches of the same shape, L2 flushed before every call."""
    import torch
    from kv_cache_quantized_b200 import ops
    rows = []
    peak = _peaks()[0]
    for w in W.SWEEP:
        B, Hq, Hkv, T, d, bits = w.B, w.Hq, w.Hkv, w.T, w.d, w.bits
        signs = torch.as_tensor(W.sign_vector(d, w.seed + 4), device=dev)
        k = _gen_rows(W.lognormal_rows_device, (B, Hkv, T, d), w.seed, dev)
        kc, kn = ops.write_keys(k, signs, bits)
        v = _gen_rows(W.lognormal_rows_device, (B, Hkv, T, d), w.seed + 2, dev)
        q = W.normal_device((B, Hq, d), w.seed + 3, dev, dtype=torch.float32)
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
        ws = torch.empty(max(ops.attend_workspace_bytes(B, Hq, Hkv, T, d), 16), dtype=torch.uint8, device=dev)
        ms_lut = time_calls(lambda: ops.attend_decode(q, kc, kn, signs, bits, v=v, out=out, workspace=ws))
        ms_dense = time_calls(lambda: ops.dense_decode(q, k, v, out=out, workspace=ws))
        lut_b = (d * bits // 8 + 2 + 2 * d) * B * Hkv * T
        dense_b = 4 * d * B * Hkv * T
        rows.append({"B": B, "T": T, "bits": bits, "d": d,
                     "lut_ms": ms_lut, "lut_gbs": lut_b / (ms_lut / 1e3) / 1e9,
                     "lut_frac": lut_b / (ms_lut / 1e3) / 1e9 / peak,
                     "dense_ms": ms_dense, "dense_gbs": dense_b / (ms_dense / 1e3) / 1e9,
                     "dense_frac": dense_b / (ms_dense / 1e3) / 1e9 / peak,
                     "lut_speedup_over_dense": ms_dense / ms_lut})
        del k, kc, kn, v, q, out, ws
        torch.cuda.empty_cache()
    return rows


def run_axr(args, w):
    import torch
    import torch.distributed as dist
    from kv_cache_quantized_b200 import ops

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    B, Hq, Hkv, T, d, bits = w.B, w.Hq, w.Hkv, w.T, w.d, w.bits
    R = d * bits // 8
    seed = w.seed + 1000 * rank
    signs = torch.as_tensor(W.sign_vector(d, w.seed + 4), device=dev)
    # --- setup: cache written once through the write path (not timed) ---
    if w.keys == "outlier":
        k = W.outlier_keys_device((B, Hkv, T, d), seed, dev)
    else:
        k = W.lognormal_rows_device((B, Hkv, T, d), seed, dev)
    v = (W.lognormal_rows_device if w.v_quant else W.normal_device)((B, Hkv, T, d), seed + 2, dev)
    kc, kn = ops.write_keys(k, signs, bits)
    vt = vtn = None
    if w.v_quant:
        vc, vn = ops.write_keys(v, signs, bits)
        if not args.no_variants and d == 128:  # the tiled value layout, for the variants below
            vt, vtn = ops.write_values_tiled(v, signs, bits)
        del v
        v = None
    del k
    q = W.normal_device((B, Hq, d), seed + 3, dev, dtype=torch.float32)
    knew = W.normal_device((B, Hkv, d), seed + 5, dev)
    vnew = W.normal_device((B, Hkv, d), seed + 6, dev)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    wsb = ops.attend_workspace_bytes(B, Hq, Hkv, T, d)
    wsp = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def step(q_in, k_in, v_in):  # one axr_decode_step: write the new K, V at T - 1 and attend over [0, T)
        if w.v_quant:
            ops.decode_step(q_in, k_in, v_in, kc, kn, signs, bits, vcodes=vc, vnorms=vn, out=out, workspace=wsp)
        else:
            ops.decode_step(q_in, k_in, v_in, kc, kn, signs, bits, v=v, out=out, workspace=wsp)

    launches_per_step = 2  # the decode kernel (with the new token's write) + the split merge

    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        step(q, knew, vnew)
    torch.cuda.synchronize()

    # --- timed region: K steps, L2 flushed between steps (outside the per-step events) ---
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush.zero_()
            e0, e1, e2 = ev[i]
            e0.record(stream)
            step(q, knew, vnew)
            e2.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    step_ms = sum(e0.elapsed_time(e2) for e0, _, e2 in ev)
    attend_ms = [e0.elapsed_time(e2) for e0, _, e2 in ev]  # the whole step is one decode call
    clocks = clk.summary()

    # --- end to end through the public API: pinned host inputs in, result out, every step ---
    # The step's three inputs (q, K_new, V_new) sit back to back in one pinned staging buffer and cross in one copy
    # into one device buffer whose views the call takes.
    in_h, views_h = _packed_inputs([q.cpu(), knew.cpu(), vnew.cpu()], pinned=True)
    in_d, (q_d, k_d, v_d) = _packed_inputs([q, knew, vnew], device=dev)
    o_h = torch.empty_like(out, device="cpu").pin_memory()
    e2e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        a, b_ = e2e[i]
        a.record(stream)
        in_d.copy_(in_h, non_blocking=True)
        step(q_d, k_d, v_d)
        o_h.copy_(out, non_blocking=True)
        b_.record(stream)
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b_) for a, b_ in e2e)
    h2d = in_h.numel()
    d2h = o_h.numel() * 4

    def time_calls(fn):  # mean ms per call, L2 flushed before each call, outside the events
        for _ in range(3):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for a_, b2 in evs:
            flush.zero_()
            a_.record(stream)
            fn()
            b2.record(stream)
        torch.cuda.synchronize()
        return float(np.mean([a_.elapsed_time(b2) for a_, b2 in evs]))

    # attend_decode over the tiled value layout (same cache contents): value product as warp-level MMAs, and the
    # tcgen05 kernel (key scores and value product from tensor memory)
    variants = {}
    if vt is not None:
        ab = _bytes_per_key_head(w) * B * Hkv * T
        for name, mode in (("tiled_values_mma", "mma"), ("tiled_values_tcgen05", "tensor")):
            ops.set_gather(mode)
            ms = time_calls(lambda: ops.attend_decode(q, kc, kn, signs, bits, vcodes=vt, vnorms=vtn, out=out,
                                                      workspace=wsp))
            variants[name] = {"ms": ms, "achieved_gbs": ab / (ms / 1e3) / 1e9, "algorithmic_bytes": ab}
        ops.set_gather("mma")
        variants["rows_decode_step"] = {"ms": float(np.mean(attend_ms)),
                            "achieved_gbs": ab / (float(np.mean(attend_ms)) / 1e3) / 1e9, "algorithmic_bytes": ab}

    # the scorer alone (axr_score) on the same cache, every table read mode, L2 flushed before each call
    scorer = {}
    if not args.no_scorer:
        sc_out = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
        for mode in ("mma", "tensor", "factored", "table"):
            ops.set_gather(mode)
            for _ in range(3):
                ops.score(q, kc, kn, signs, bits, scale=1.0 / math.sqrt(d), out=sc_out)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for a_, b2 in evs:
                flush.zero_()
                a_.record(stream)
                ops.score(q, kc, kn, signs, bits, scale=1.0 / math.sqrt(d), out=sc_out)
                b2.record(stream)
            torch.cuda.synchronize()
            ms = float(np.mean([a_.elapsed_time(b2) for a_, b2 in evs]))
            sbytes = (R + 2 + 4 * w.G) * B * Hkv * T
            scorer[mode] = {"ms": ms, "achieved_gbs": sbytes / (ms / 1e3) / 1e9, "algorithmic_bytes": sbytes}
        ops.set_gather("mma")
        del sc_out

    # the build's own dense fp16 decode kernel on the same shape (fp16 K and V), the bandwidth reference
    dense = None
    if not args.no_dense:
        kd = _gen_rows(W.lognormal_rows_device, (B, Hkv, T, d), seed + 7, dev)
        vd = _gen_rows(W.normal_device, (B, Hkv, T, d), seed + 8, dev)
        ms = time_calls(lambda: ops.dense_decode(q, kd, vd, out=out, workspace=wsp))
        dbytes = 4 * d * B * Hkv * T
        dense = {"kernel": "attend_partial_kernel<DENSE> + attend_reduce_kernel (axr_dense_decode)", "ms": ms,
                 "value": B * T * Hq / (ms / 1e3), "unit": UNIT, "achieved_gbs": dbytes / (ms / 1e3) / 1e9,
                 "frac": dbytes / (ms / 1e3) / 1e9 / _peaks()[0], "algorithmic_bytes": dbytes}
        del kd, vd

    # the decode sweep (--sweep): the LUT attend with fp16 values next to the dense fp16 kernel, per shape
    sweep = _sweep(args, dev, time_calls) if args.sweep else None

    # max over ranks
    from kv_cache_quantized_b200 import dist as D
    step_ms, e2e_ms, attend_avg_ms = D.max_over_ranks([step_ms, e2e_ms, float(np.mean(attend_ms))], device=dev)
    if ws > 1:
        dist.destroy_process_group()
    if rank != 0:
        return None

    key_heads = B * T * Hq * ws * args.steps
    value = key_heads / (step_ms / 1e3)
    alg_bytes = _bytes_per_key_head(w) * B * Hkv * T
    achieved = alg_bytes / (attend_avg_ms / 1e3) / 1e9
    peak, peak_src = _peaks()
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms / args.steps, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u8 codes / f32 math", "data": "synthetic",
        "config": {"workload": w.name, "B": B, "T": T, "Hq": Hq, "Hkv": Hkv, "d": d, "bits": bits,
                   "values": "quantized b=%d" % bits if w.v_quant else "fp16", "parallelism": f"replicas x{ws}",
                   "l2": "flushed between steps (256 MiB write outside the per-step events)"},
        "hbm_gbs": alg_bytes * ws * args.steps / (step_ms / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "kernel": "attend_rows_kernel (with the new token's write) + "
                     "attend_reduce_kernel (one axr_decode_step call)", "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": TRAFFIC.get(w.name) if args.batch is None else None,
                     "algorithmic_bytes": alg_bytes, "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_src == "measured" else "fallback 6.65 TB/s"},
        "e2e": {"value": key_heads / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "scorer": {m: dict(v_, frac=v_["achieved_gbs"] / _peaks()[0]) for m, v_ in scorer.items()},
        "attend_variants": {m: dict(v_, frac=v_["achieved_gbs"] / _peaks()[0]) for m, v_ in variants.items()},
        "dense_reference": dense,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if sweep is not None:
        line["sweep"] = sweep
    return line


def run_reference(args, w):
    """The oracle as it stands on this host's cores, in place of the reference implementation (the pages ship no
    code); one bounded sample per step."""
    ws, rank, _ = _dist()
    if rank != 0:
        return None
    for _ in range(args.warmup):
        pass
    vals = []
    cb = None
    for _ in range(args.steps):
        cb = cpu_baseline(w, seconds=args.cpu_seconds / max(args.steps, 1))
        vals.append(cb["value"])
    value = float(np.mean(vals))
    cb["value"] = value
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 0,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "bits": w.bits},
            "cpu_baseline": cb, "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["axr", "reference"], default="axr")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="long_context")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU time budget of the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch size (small ncu cases)")
    ap.add_argument("--no-scorer", action="store_true", help="skip the separate axr_score measurement")
    ap.add_argument("--no-variants", action="store_true", help="skip the tiled-value attend variants")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense fp16 bandwidth reference")
    ap.add_argument("--sweep", action="store_true",
                    help="also run the decode sweep (B x T x bits x d, fp16 V) against the dense fp16 kernel")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    if args.batch is not None:
        import dataclasses
        w = dataclasses.replace(w, B=args.batch, name=w.name.replace(f"_b{w.B}_", f"_b{args.batch}_"))
    if args.impl == "reference":
        line = run_reference(args, w)
    else:
        line = run_axr(args, w)
        if line is not None:
            line["cpu_baseline"] = None if args.no_cpu_baseline else cpu_baseline(w, args.cpu_seconds)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
