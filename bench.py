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
# What the timed kernel computes: u8 packed codes; key scores as fp16 x fp16 -> fp32 MMAs on hi/lo planes of the
# centroids and the query (about 22 bits each); the value product as fp16 x fp16 -> fp32 MMAs of the weights and the
# hi plane of the value centroids; softmax and the merge in fp32.
DTYPE = "u8 codes; fp16 hi/lo x fp16 hi/lo -> fp32 MMA (keys), fp16 x fp16 -> fp32 MMA (values), fp32 softmax"
NOMINAL_HBM_GBS = 8000.0  # the HBM bandwidth the target is stated against (about 8 TB/s), beside the measured copy
UNIT = "keys·heads/s"
L2_BYTES = 126 * 1024 * 1024

# DRAM traffic (read + write bytes) per launch of the timed decode kernel: an ncu counters-only capture
# (dram__bytes_read.sum, dram__bytes_write.sum, three launches) of the same workload at B=4 (half the units) read
# 138.582 MB and wrote 1.457 MB per launch on average; scaled by the units processed.  Valid for the kernel version
# that capture was taken on; a workload without an entry reports null.
class _L2Flush:
    """Between timed calls: write a buffer of twice the L2 size (every line of the L2 now holds it, dirty), then read
    another one of the same size, so that those dirty lines are written back here and the timed call starts on an L2
    of clean lines that hold none of its inputs (otherwise up to the L2's size of write-backs would land inside the
    timed call)."""

    def __init__(self, dev):
        import torch

        self.w = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
        self.r = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


LEAD_CYCLES = 200_000  # about 100 us of SM clock


def _lead_in():
    """A spin of about 100 us on the stream, queued after the L2 flush and before a timed call's start event: the
    call's launches are queued behind it while it runs, so the event pair brackets the call's device work and not the
    host's time to issue it (the host side of a call is in the end-to-end figure)."""
    import torch

    torch.cuda._sleep(LEAD_CYCLES)


def _step_kernel(w) -> str:
    """The decode kernel the library runs for a contiguous decode step of this workload: the streaming kernel for
    fp16 values, and for quantized values from 2^18 (token, KV head) units or at eight query heads per KV head; the
    row kernel otherwise."""
    stream = (not w.v_quant) or w.Hq // w.Hkv == 8 or w.B * w.Hkv * w.T >= 1 << 18
    return "attend_stream_kernel" if stream else "attend_rows_kernel"


TRAFFIC = {
    # attend_stream_kernel<128, 4, 4, quantized V> (16 warps per SM), DRAM read + write per launch at B = 4 (mean of
    # three launches of the counters-only ncu capture kept under profiles/), scaled by the units to B = 8
    "long_context_b8_t32768_hq32_hkv8_d128_b4_kvquant": 2 * (138.575189e6 + 1.367979e6),
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
    """SM clock, power and throttle reasons sampled every 200 ms while the timed region runs: read-only NVML queries
    from a thread (no process is forked while calls are timed: a fork of a large process stalls its threads, and a
    stalled launch would leave the GPU idle inside a step's events).  Without NVML bindings, one nvidia-smi process
    in its looping mode, started before the region and stopped after it.  Samples are kept in nvidia-smi's CSV form
    (the fields of FIELDS)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, period_s=0.2):
        self.index = index
        self.period = period_s
        self.lines = []
        self._stop = None
        self._thread = None
        self._proc = None

    def _nvml_line(self, nv, h):
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
        r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        act = lambda bit: "Active" if r & bit else "Not Active"
        return (f"{self.index}, {sm}, {mx}, {pw:.2f}, {r:#x}, {act(nv.nvmlClocksThrottleReasonHwSlowdown)}, "
                f"{act(nv.nvmlClocksThrottleReasonHwThermalSlowdown)}, "
                f"{act(nv.nvmlClocksThrottleReasonSwThermalSlowdown)}, {act(nv.nvmlClocksThrottleReasonSwPowerCap)}")

    def _poll(self, nv, h):
        while True:  # one sample at entry, then every period, and one more when stopped
            try:
                self.lines.append(self._nvml_line(nv, h))
            except Exception:  # noqa: BLE001 -- a failed query ends the sampling, not the benchmark
                return
            if self._stop.is_set():
                return
            self._stop.wait(self.period)

    def __enter__(self):
        import threading
        try:
            import pynvml as nv
            import torch
            nv.nvmlInit()
            try:
                nidx = torch.cuda._get_nvml_device_index(self.index)
            except Exception:  # noqa: BLE001
                nidx = self.index
            h = nv.nvmlDeviceGetHandleByIndex(nidx)
            self._nvml_line(nv, h)
        except Exception:  # noqa: BLE001 -- no NVML bindings: nvidia-smi's looping mode
            try:
                self._proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                                               "--format=csv,noheader,nounits", "-lms",
                                               str(int(self.period * 1000))],
                                              stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                time.sleep(0.3)
            except OSError:
                self._proc = None
            return self
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._poll, args=(nv, h), daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=10)
        if self._proc is not None:
            time.sleep(0.25)
            self._proc.terminate()
            try:
                out, _ = self._proc.communicate(timeout=10)
            except subprocess.TimeoutExpired:
                self._proc.kill()
                out, _ = self._proc.communicate()
            self.lines += [ln for ln in (out or "").splitlines() if ln.strip()]

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


def _oracle_unit(w, kc, kn, vc, vn, k, v, q, s, hk):
    """One (batch row, KV head) unit of the decode step through the oracle: the new token's write, then G query
    heads over the T cached tokens."""
    import oracle
    scale = 1.0 / math.sqrt(w.d)
    nk = oracle.write(k[-1:], s, w.bits)
    if w.v_quant:
        oracle.write(v[-1:], s, w.bits)
    kc[-1:], kn[-1:] = nk
    qq = q[hk * w.G:(hk + 1) * w.G][None]
    if w.v_quant:
        oracle.decode_attention(qq, kc[None, None], kn[None, None], s, w.bits, scale, vcodes=vc[None, None],
                                vn16=vn[None, None])
    else:
        oracle.decode_attention(qq, kc[None, None], kn[None, None], s, w.bits, scale, v=v[None, None])


def _oracle_proc(w, seed, cmd_q, res_q, ready):
    """Spawned oracle process: draws one (batch row, KV head) unit of the workload's shape from its own seed, then
    for every command `seconds` runs decode steps of that unit through the oracle on one thread for that long and
    reports (unit-steps, seconds).  None ends it."""
    from threadpoolctl import threadpool_limits
    import oracle
    with threadpool_limits(1):
        if w.keys == "outlier":
            k = W.outlier_keys((w.T, w.d), seed)
        else:
            k = W.lognormal_rows((w.T, w.d), seed, dtype=np.float16)
        v = (W.lognormal_rows((w.T, w.d), seed + 1, dtype=np.float16) if w.v_quant
             else W.normal((w.T, w.d), seed + 1, np.float16))
        q = W.normal((w.Hq, w.d), seed + 2, np.float32)
        s = W.sign_vector(w.d, w.seed + 4)
        kc, kn = oracle.write(k, s, w.bits)
        vc, vn = oracle.write(v, s, w.bits) if w.v_quant else (None, None)
        ready.wait()
        while True:
            seconds = cmd_q.get()
            if seconds is None:
                return
            t0 = time.perf_counter()
            units = 0
            while units == 0 or time.perf_counter() - t0 < seconds:
                _oracle_unit(w, kc, kn, vc, vn, k, v, q, s, 0)
                units += 1
            res_q.put((units, time.perf_counter() - t0))


class OracleCores:
    """One spawned oracle process per available core (os.sched_getaffinity), each on one thread with its own unit;
    step(seconds) runs them concurrently and returns key-heads per second of all of them together."""

    def __init__(self, w):
        import multiprocessing as mp
        self.w = w
        self.n = len(os.sched_getaffinity(0))
        ctx = mp.get_context("spawn")
        self.res_q = ctx.Queue()
        self.cmd_q = [ctx.Queue() for _ in range(self.n)]
        ready = ctx.Barrier(self.n + 1)
        self.procs = [ctx.Process(target=_oracle_proc, args=(w, 900_000 + 10 * i, self.cmd_q[i], self.res_q, ready),
                                  daemon=True) for i in range(self.n)]
        for p_ in self.procs:
            p_.start()
        ready.wait(timeout=600)
        self.units = 0
        self.seconds = 0.0

    def step(self, seconds):
        for q_ in self.cmd_q:
            q_.put(seconds)
        res = [self.res_q.get(timeout=600 + 10 * seconds) for _ in range(self.n)]
        units = sum(u for u, _ in res)
        t = max(t_ for _, t_ in res)
        self.units += units
        self.seconds += t
        return units * self.w.T * self.w.G / t

    def close(self):
        for q_ in self.cmd_q:
            q_.put(None)
        for p_ in self.procs:
            p_.join(timeout=30)


def cpu_baseline(w, seconds=10.0, all_cores=True):
    """The fp64 oracle, as it stands, on the host cores: decode steps of single (batch row, KV head) units of the
    workload (G query heads over T cached tokens, plus the new token's write) for about `seconds`.  First on one
    thread; then, with all_cores, on every available core at once (OracleCores, one process and one unit per
    core, the same time): the reported value is the all-core one, the one-thread figure rides along."""
    import oracle
    from threadpoolctl import threadpool_limits
    inp = W.decode_inputs(w, B=1)
    k, v, q, s = inp["k"][0], inp["v"][0], inp["q"][0], inp["signs"]
    with threadpool_limits(1):
        units, t_total, hk = 0, 0.0, 0
        while t_total < seconds and hk < w.Hkv:
            kc, kn = oracle.write(k[hk], s, w.bits)  # cache state (setup, not timed)
            vc, vn = oracle.write(v[hk], s, w.bits) if w.v_quant else (None, None)
            t0 = time.perf_counter()
            _oracle_unit(w, kc, kn, vc, vn, k[hk], v[hk], q, s, hk)
            t_total += time.perf_counter() - t0
            units += 1
            hk += 1
    one = units * w.T * w.G / t_total
    one_sample = (f"{units} of {w.B * w.Hkv} (batch row, KV head) units of {w.name}: {w.G} query heads x {w.T} "
                  f"tokens each, plus the new token's write; fp64 numpy, 1 thread, {t_total:.1f} s")
    out = {"value": one, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": one_sample}
    if not all_cores:
        return out
    pool = OracleCores(w)
    try:
        many = pool.step(seconds)
    finally:
        pool.close()
    out.update({"value": many, "cores": pool.n, "single_core_value": one,
                "sample": f"{pool.n} processes, one thread and one (batch row, KV head) unit of {w.name}'s shape "
                          f"each ({w.G} query heads x {w.T} tokens, plus the new token's write), fp64 numpy: "
                          f"{pool.units} unit-steps in {pool.seconds:.1f} s; single_core_value: {one_sample}"})
    return out


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


def _codecs(w, dev, time_calls, signs, kc, kn, q, wsp):
    """LOOKAT and PoT decode paths (and the AXELRAM literal table) at the workload's shape over fp16 values: mean ms
    per call (L2 flushed before each), algorithmic HBM bytes (codes + per-token scale + fp16 values, or codes +
    scale + fp32 scores for the scorers) and the fraction of the measured copy peak."""
    import torch
    from kv_cache_quantized_b200 import ops
    B, Hq, Hkv, T, d, G = w.B, w.Hq, w.Hkv, w.T, w.d, w.G
    peak = _peaks()[0]
    units = B * Hkv * T
    v = _gen_rows(W.normal_device, (B, Hkv, T, d), w.seed + 11, dev)
    k = _gen_rows(W.lognormal_rows_device, (B, Hkv, T, d), w.seed + 12, dev)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
    res = {}

    def rec(name, ms, per_unit):
        gb = per_unit * units / (ms / 1e3) / 1e9
        res[name] = {"ms": ms, "bytes_per_token_head": per_unit, "achieved_gbs": gb, "frac": gb / peak,
                     "keys_heads_per_s": B * T * Hq / (ms / 1e3)}

    # LOOKAT: codebooks by k-means on a slice of the keys (setup, not timed), codes written on the GPU
    m, K = 8, 256
    cbs = torch.empty((Hkv, m, K, d // m), dtype=torch.float32, device=dev)
    for h in range(Hkv):
        x = k[0, h, :65536].contiguous()
        init = x[torch.arange(K, device=dev) * (x.shape[0] // K)].view(K, m, d // m).transpose(0, 1).contiguous()
        cbs[h] = ops.pq_train(x, init.float(), 4)
    pcodes = ops.pq_encode(k, cbs)
    rec("lookat_attend", time_calls(lambda: ops.pq_attend_decode(q, pcodes, cbs, v, out=out, workspace=wsp)),
        m + 2 * d)
    rec("lookat_score", time_calls(lambda: ops.pq_score(q, pcodes, cbs, scale=1.0 / math.sqrt(d))), m + 4 * G)
    del pcodes
    # PoT, 4-bit codes (E = 3, M = 0)
    pc, pa = ops.pot_write(k, 3, 0)
    R = ops.pot_row_bytes(d, 3, 0)
    rec("pot_attend", time_calls(lambda: ops.pot_attend_decode(q, pc, pa, v, 3, 0, out=out, workspace=wsp)),
        R + 2 + 2 * d)
    rec("pot_score", time_calls(lambda: ops.pot_score(q, pc, pa, 3, 0, scale=1.0 / math.sqrt(d))), R + 2 + 4 * G)
    del pc, pa
    # the AXELRAM literal table read over fp16 values, and the default read path on the same cache
    ops.set_gather("table")
    rec("axelram_table_attend_f16v", time_calls(lambda: ops.attend_decode(q, kc, kn, signs, w.bits, v=v, out=out,
                                                                          workspace=wsp)), w.d * w.bits // 8 + 2 + 2 * d)
    ops.set_gather("mma")
    rec("axelram_mma_attend_f16v", time_calls(lambda: ops.attend_decode(q, kc, kn, signs, w.bits, v=v, out=out,
                                                                        workspace=wsp)), w.d * w.bits // 8 + 2 + 2 * d)
    del v, k
    torch.cuda.empty_cache()
    return res


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
        if args.variants and d == 128:  # the tiled value layout, for the variants below
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
    flush = _L2Flush(dev)

    def step(q_in, k_in, v_in):  # one axr_decode_step: write the new K, V at T - 1 and attend over [0, T)
        if w.v_quant:
            ops.decode_step(q_in, k_in, v_in, kc, kn, signs, bits, vcodes=vc, vnorms=vn, out=out, workspace=wsp)
        else:
            ops.decode_step(q_in, k_in, v_in, kc, kn, signs, bits, v=v, out=out, workspace=wsp)

    launches_per_step = 2  # the decode kernel (with the new token's write) + the split merge

    stream = torch.cuda.current_stream()
    # --- timed region: K steps, L2 flushed between steps (outside the per-step events) ---
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    # The clock sampler starts first and the W warm-up steps (flushed like the timed ones) run right before the timed
    # steps, so that no idle gap (the sampler's start-up) separates the two.
    with ClockSampler(local) as clk:
        for _ in range(args.warmup):
            flush()
            _lead_in()
            step(q, knew, vnew)
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(args.steps):
            flush()
            _lead_in()
            e0, e1, e2 = ev[i]
            e0.record(stream)
            step(q, knew, vnew)
            e2.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    step_ms = sum(e0.elapsed_time(e2) for e0, _, e2 in ev)
    attend_ms = [e0.elapsed_time(e2) for e0, _, e2 in ev]  # the whole step is one decode call
    step_stats = {"min": min(attend_ms), "median": float(np.median(attend_ms)), "max": max(attend_ms)}
    clocks = clk.summary()

    # --- end to end through the public API: pinned host inputs in, result out, every step ---
    # The step's three inputs (q, K_new, V_new) sit back to back in one pinned staging buffer and cross in one copy
    # into one device buffer whose views the call takes.
    in_h, views_h = _packed_inputs([q.cpu(), knew.cpu(), vnew.cpu()], pinned=True)
    in_d, (q_d, k_d, v_d) = _packed_inputs([q, knew, vnew], device=dev)
    o_h = torch.empty_like(out, device="cpu").pin_memory()
    e2e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush()
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
            flush()
            _lead_in()
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

    # the scorer alone (axr_score) on the same cache, L2 flushed before each call: the default read (the factored
    # table on mma.sync) and the literal table as its ablation; with --variants also the other read modes (codes
    # loaded straight into registers, the tcgen05 tensor cores, the CUDA cores)
    scorer = {}
    roles = {"mma": "default read: factored table on mma.sync", "table": "ablation: the literal table in shared memory",
             "direct": "variant: codes straight into registers", "tensor": "variant: tcgen05 with TMEM operands",
             "factored": "variant: factored table on the CUDA cores"}
    if not args.no_scorer:
        sc_out = torch.empty((B, Hq, T), dtype=torch.float32, device=dev)
        modes = ("mma", "table") + (("direct", "tensor", "factored") if args.variants else ())
        for mode in modes:
            ops.set_gather(mode)
            for _ in range(3):
                ops.score(q, kc, kn, signs, bits, scale=1.0 / math.sqrt(d), out=sc_out)
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for a_, b2 in evs:
                flush()
                _lead_in()
                a_.record(stream)
                ops.score(q, kc, kn, signs, bits, scale=1.0 / math.sqrt(d), out=sc_out)
                b2.record(stream)
            torch.cuda.synchronize()
            ms = float(np.mean([a_.elapsed_time(b2) for a_, b2 in evs]))
            sbytes = (R + 2 + 4 * w.G) * B * Hkv * T   # codes + norms read, fp32 scores written
            cbytes = (R + 2) * B * Hkv * T             # codes + norms only
            scorer[mode] = {"ms": ms, "achieved_gbs": sbytes / (ms / 1e3) / 1e9, "algorithmic_bytes": sbytes,
                            "achieved_gbs_codes_norms": cbytes / (ms / 1e3) / 1e9,
                            "algorithmic_bytes_codes_norms": cbytes, "role": roles[mode]}
        ops.set_gather("mma")
        # the literal table where byte-indexed multi-coordinate tables apply (b <= 2: 8 or 4 coordinates per
        # 8-bit field), against the factored MMA read of the same codes, at this shape
        klow = _gen_rows(W.lognormal_rows_device, (B, Hkv, T, d), seed + 21, dev)
        for lb in (1, 2):
            lc, ln = ops.write_keys(klow, signs, lb)
            for mode in ("mma", "table"):
                ops.set_gather(mode)
                for _ in range(3):
                    ops.score(q, lc, ln, signs, lb, scale=1.0 / math.sqrt(d), out=sc_out)
                evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(args.steps)]
                for a_, b2 in evs:
                    flush()
                    _lead_in()
                    a_.record(stream)
                    ops.score(q, lc, ln, signs, lb, scale=1.0 / math.sqrt(d), out=sc_out)
                    b2.record(stream)
                torch.cuda.synchronize()
                ms = float(np.mean([a_.elapsed_time(b2) for a_, b2 in evs]))
                sbytes = (d * lb // 8 + 2 + 4 * w.G) * B * Hkv * T
                scorer[f"{mode}_b{lb}"] = {"ms": ms, "achieved_gbs": sbytes / (ms / 1e3) / 1e9, "algorithmic_bytes": sbytes,
                                           "achieved_gbs_codes_norms": (d * lb // 8 + 2) * B * Hkv * T / (ms / 1e3) / 1e9,
                                           "algorithmic_bytes_codes_norms": (d * lb // 8 + 2) * B * Hkv * T}
            del lc, ln
        ops.set_gather("mma")
        del sc_out, klow

    # the build's own dense fp16 decode kernel on the same shape (fp16 K and V), the bandwidth reference
    dense = None
    if not args.no_dense:
        kd = _gen_rows(W.lognormal_rows_device, (B, Hkv, T, d), seed + 7, dev)
        vd = _gen_rows(W.normal_device, (B, Hkv, T, d), seed + 8, dev)
        ms = time_calls(lambda: ops.dense_decode(q, kd, vd, out=out, workspace=wsp))
        dbytes = 4 * d * B * Hkv * T
        dense = {"kernel": "dense_stream_kernel + attend_reduce_kernel (axr_dense_decode)", "ms": ms,
                 "value": B * T * Hq / (ms / 1e3), "unit": UNIT, "achieved_gbs": dbytes / (ms / 1e3) / 1e9,
                 "frac": dbytes / (ms / 1e3) / 1e9 / _peaks()[0], "algorithmic_bytes": dbytes}
        del kd, vd

    # the same decode step through paged pools (shuffled block tables) at three block sizes: blocks of 32 tokens and
    # more go through the streaming kernel (a tile never spans two blocks), 16-token blocks through the row kernel
    paged = None
    if not args.no_codecs and w.v_quant:
        paged = {}
        for bt in (16, 32, 256):
            nb = T // bt
            perm = torch.randperm(B * nb, generator=torch.Generator().manual_seed(bt)).to(dev)
            table = perm.view(B, nb).to(torch.int32).contiguous()

            def pool(x):  # [B, Hkv, T, ...] -> [B * nb, Hkv, bt, ...] with block (b, j) at table[b, j]
                y = x.view(B, Hkv, nb, bt, *x.shape[3:]).transpose(1, 2).reshape(B * nb, Hkv, bt, *x.shape[3:])
                out_ = torch.empty_like(y)
                out_[perm] = y
                return out_
            pk, pn, pvc, pvn = pool(kc), pool(kn), pool(vc), pool(vn)
            ms = time_calls(lambda: ops.decode_step_paged(q, knew, vnew, pk, pn, signs, bits, table, vcodes=pvc,
                                                          vnorms=pvn, out=out, workspace=wsp))
            ab = _bytes_per_key_head(w) * B * Hkv * T
            paged[f"bt{bt}"] = {"ms": ms, "achieved_gbs": ab / (ms / 1e3) / 1e9,
                                "frac": ab / (ms / 1e3) / 1e9 / _peaks()[0], "algorithmic_bytes": ab,
                                "kernel": "attend_stream_kernel" if bt >= 32 else "attend_rows_kernel"}
            del pk, pn, pvc, pvn
        paged["contiguous"] = {"ms": float(np.mean(attend_ms))}

    # the other codecs through the same reducer, at this shape with fp16 values: LOOKAT product-quantized keys
    # (m = 8 one-byte indices, K = 256) and power-of-two shift-accumulate keys (E = 3, M = 0: 4 bits), scores alone
    # and decode attention; the AXELRAM literal-table read (AXR_GATHER_TABLE) over the same fp16 values beside them
    codecs = _codecs(w, dev, time_calls, signs, kc, kn, q, wsp) if not args.no_codecs else None

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
        "dtype": DTYPE, "data": "synthetic", "step_ms_rank0": step_stats,
        "config": {"workload": w.name, "B": B, "T": T, "Hq": Hq, "Hkv": Hkv, "d": d, "bits": bits,
                   "values": "quantized b=%d" % bits if w.v_quant else "fp16", "parallelism": f"replicas x{ws}",
                   "l2": "flushed between steps outside the per-step events: a 256 MiB write, then a 256 MiB read of "
                         "another buffer (the timed step starts on clean L2 lines holding none of its inputs)"},
        "hbm_gbs": alg_bytes * ws * args.steps / (step_ms / 1e3) / 1e9,
        "roofline": {"bound": "hbm", "kernel": f"{_step_kernel(w)} (with the new token's write) + "
                     "attend_reduce_kernel (one axr_decode_step call)", "achieved": achieved,
                     "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
                     "traffic": TRAFFIC.get(w.name) if args.batch is None else None,
                     "algorithmic_bytes": alg_bytes, "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                     if peak_src == "measured" else "fallback 6.65 TB/s"},
        "e2e": {"value": key_heads / (e2e_ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "scorer": {m: dict(v_, frac=v_["achieved_gbs"] / peak, frac_codes_norms=v_["achieved_gbs_codes_norms"] / peak,
                           frac_of_nominal_8tbs=v_["achieved_gbs"] / NOMINAL_HBM_GBS,
                           frac_codes_norms_of_nominal_8tbs=v_["achieved_gbs_codes_norms"] / NOMINAL_HBM_GBS)
                   for m, v_ in scorer.items()},
        "attend_variants": {m: dict(v_, frac=v_["achieved_gbs"] / _peaks()[0]) for m, v_ in variants.items()},
        "dense_reference": dense,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if sweep is not None:
        line["sweep"] = sweep
    if codecs is not None:
        line["codecs"] = codecs
    if paged is not None:
        line["paged_decode_step"] = paged
    return line


def _fp32_alu_peak():
    """FP32 FMA-pipe peak of one B200, from unit counts and the maximum SM clock: 148 SMs x 128 FP32 lanes x 2 flop
    per FMA x clocks.max.sm (MEASURED_PEAKS.json sm_max_mhz, else 1965 MHz)."""
    mhz = 1965.0
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            mhz = float(json.load(f).get("sm_max_mhz", mhz))
    return 148 * 128 * 2 * mhz * 1e6 / 1e12


def _tensor_peak():
    """Dense bf16 tensor throughput measured on this machine (sustained, for kernels inside a long loop)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops_sustained"]), "measured (MEASURED_PEAKS.json bf16_tflops_sustained)"
    return 1400.0, "fallback 1.4 PFLOP/s sustained"


def select_flops(c, n_cand):
    """Algorithmic flops of one selection: per candidate, layer, sequence and query head, causal attention over N
    positions is N(N+1)/2 (query, key) pairs, each a d-long dot product for the score and a d-long update of the
    output: 2 x 2d flops per pair."""
    return n_cand * c.layers * c.seqs * c.Hq * (c.tokens * (c.tokens + 1) // 2) * 4 * c.d


def run_select(args):
    """Sign selection at the calibration set's full size (36 layers x 8 sequences x 512 tokens, Hq=16, Hkv=2, d=128,
    200 candidates): one step = one axr_select_signs call per bit width b in {2, 3, 4} (the whole-model pick),
    timed with CUDA events on the stream; inputs resident on the device."""
    import torch
    from kv_cache_quantized_b200 import ops
    c = W.QWEN3B_SELECT
    if args.batch is not None:  # fewer layers (small ncu cases)
        import dataclasses
        c = dataclasses.replace(c, layers=args.batch, name=c.name.replace("_l36_", f"_l{args.batch}_"))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    shape_q = (c.layers, c.seqs, c.Hq, c.tokens, c.d)
    shape_k = (c.layers, c.seqs, c.Hkv, c.tokens, c.d)
    q = W.normal_device(shape_q, c.seed, dev, dtype=torch.float32)
    k = W.layer_scaled_keys_device(shape_k, c.seed + 1, dev)
    v = W.normal_device(shape_k, c.seed + 2, dev)
    cands = torch.as_tensor(W.candidate_signs(c.n_cand, c.d, c.seed + 3), device=dev)
    ws = torch.empty(ops.select_workspace_bytes(c.layers, c.seqs, c.tokens, c.Hq, c.Hkv, c.d, c.n_cand),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    per_bits = {}
    for bits in c.bits:
        for _ in range(args.warmup):
            ops.select_signs(q, k, v, cands, bits, workspace=ws)
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        with ClockSampler(0) as clk:
            for a_, b_ in evs:
                a_.record(stream)
                mse, best = ops.select_signs(q, k, v, cands, bits, workspace=ws)
                b_.record(stream)
            torch.cuda.synchronize()
        ms = [a_.elapsed_time(b_) for a_, b_ in evs]
        per_bits[bits] = {"ms": float(np.mean(ms)), "best": int(best.item()), "clocks": clk.summary()}
    flops = select_flops(c, c.n_cand)
    step_ms = sum(v_["ms"] for v_ in per_bits.values())
    # the candidate attention runs on the tensor cores (mma.sync, fp16 operands): the scores as three products of
    # hi/lo planes, the value product as two, so the MMAs execute 2.5x the algorithmic flops; the peak is the
    # measured sustained dense bf16 rate (a seconds-long loop), the fp16 rate being the same
    peak, peak_src = _tensor_peak()
    achieved = flops * len(c.bits) / (step_ms / 1e3) / 1e12
    qpos = c.n_cand * c.layers * c.seqs * c.Hq * c.tokens * len(c.bits)
    # the oracle on a bounded sample: 1 layer x 1 sequence x 4 candidates at the full head count and length
    import oracle
    from threadpoolctl import threadpool_limits
    inp = W.calibration_inputs(c, layers=1, seqs=1, n_cand=4)
    with threadpool_limits(1):
        t0 = time.perf_counter()
        oracle.select_signs(inp["q"], inp["k"], inp["v"], inp["candidates"], 4)
        t_cpu = time.perf_counter() - t0
    cpu_qpos = 4 * c.Hq * c.tokens
    return {
        "metric": "sign selection at full calibration size: candidate-query evaluations/s (and FP32 TFLOP/s)",
        "value": qpos / (step_ms / 1e3), "unit": "candidate·query/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp16 hi/lo x fp16 hi/lo -> fp32 MMA attention, f64 reference and error sums",
        "data": "synthetic",
        "config": {"workload": c.name, "layers": c.layers, "seqs": c.seqs, "tokens": c.tokens, "Hq": c.Hq,
                   "Hkv": c.Hkv, "d": c.d, "bits": list(c.bits), "n_cand": c.n_cand, "causal": True,
                   "l2": "inputs (1.4 GB) and workspace (1.8 GB) larger than L2"},
        "per_bits": {str(b): v_ for b, v_ in per_bits.items()},
        "roofline": {"bound": "tensor", "kernel": "select_attn_tc_kernel<128> (candidate attention, mma.sync)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "executed_mma_tflops": 2.5 * achieved, "executed_frac": 2.5 * achieved / peak,
                     "traffic": None, "algorithmic_flops_per_selection": flops, "peak_source": peak_src,
                     "fp32_alu_peak": _fp32_alu_peak()},
        "gpu_launches": len(c.bits) * args.steps * (3 + 2 * -(-c.n_cand // 8)),
        "cpu_baseline": {"value": cpu_qpos / t_cpu, "unit": "candidate·query/s", "cores": 1, "kind": "oracle",
                         "sample": f"1 layer x 1 sequence x 4 candidates of {c.name} at b=4 "
                                   f"({c.Hq} heads x {c.tokens} positions), fp64 numpy, 1 thread, {t_cpu:.1f} s"},
    }


def run_reference(args, w):
    """The oracle as it stands on this host's cores, in place of the reference implementation (the pages ship no
    code): one OracleCores step (all cores at once, a bounded sample of the workload) per benchmark step."""
    ws, rank, _ = _dist()
    if rank != 0:
        return None
    per_step = max(args.cpu_seconds / max(args.steps, 1), 0.5)
    pool = OracleCores(w)
    try:
        for _ in range(args.warmup):
            pool.step(0.2)
        pool.units, pool.seconds = 0, 0.0
        vals = [pool.step(per_step) for _ in range(args.steps)]
    finally:
        pool.close()
    value = float(np.mean(vals))
    cb = {"value": value, "unit": UNIT, "cores": pool.n, "kind": "oracle",
          "sample": f"{pool.n} processes, one thread and one (batch row, KV head) unit of {w.name}'s shape each "
                    f"({w.G} query heads x {w.T} tokens, plus the new token's write), fp64 numpy; {args.steps} "
                    f"steps of {per_step:.1f} s: {pool.units} unit-steps"}
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
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["select"], default="long_context")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU time budget of the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size, or the selector's layer count (small ncu cases)")
    ap.add_argument("--no-scorer", action="store_true", help="skip the separate axr_score measurement")
    ap.add_argument("--variants", action="store_true",
                    help="also time the attend over the tiled value layout (MMA and tcgen05 value products) and the "
                         "scorer's other read modes (direct register loads, tcgen05, CUDA cores)")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense fp16 bandwidth reference")
    ap.add_argument("--no-codecs", action="store_true", help="skip the LOOKAT / PoT / literal-table measurements")
    ap.add_argument("--sweep", action="store_true",
                    help="also run the decode sweep (B x T x bits x d, fp16 V) against the dense fp16 kernel")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload == "select":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the select workload's oracle timing rides in its "
                              "own line's cpu_baseline"}), flush=True)
            return
        if _dist()[1] == 0:
            print(json.dumps(run_select(args)), flush=True)
        return
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
