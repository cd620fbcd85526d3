#!/usr/bin/env python
"""GQE causal-prefill benchmark.

One step = the whole routed hot path on one batch of synthetic input that is
already resident in HBM: gqe_route (router, softmax, exact top-k, weights)
then gqe_attention_prefill (V conversion, bucketing, scheduling, routed +
shared-head attention, combine).  The dense-GQA baseline from the same
library is timed the same way for the routed/dense speedup.

Prints ONE JSON line on rank 0.  Under torchrun every rank runs its own
replica on its own GPU (weak scaling; batches are independent, so there is no
collective on the data path); ranks only meet for barriers and the max-over-
ranks of the device time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--no-configs] [--impl ours|reference] [--no-cpu-baseline]
                  [--no-decode] [--decode]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import WORKLOADS, make_inputs  # noqa: E402

METRIC = "GQE prefill tokens/s & useful TFLOP/s (% bf16 TC peak), S=2k–1M, vs dense GQA"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def kernel_traffic(key):
    """DRAM bytes per launch recorded by an ncu capture (profiles/traffic.json),
    or None when the attention kernel's source changed since that capture."""
    import hashlib
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))[key]
    except (OSError, ValueError, KeyError):
        return None
    h = hashlib.sha256()
    for f in ("gqe_attn.cu", "gqe_device.cuh", "gqe_internal.h"):
        with open(os.path.join(ROOT, "moe_routed_grouped_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return rec["dram_bytes"] if h.hexdigest()[:16] == rec["kernel_sha"] else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every ~0.5 ms."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, torch_dev):
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            h = None
            try:
                import torch
                pr = torch.cuda.get_device_properties(torch_dev)
                bus = "%08x:%02x:%02x.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
                h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(int(torch_dev))
            self.nv, self.h = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report that, do not guess
            self.err = str(e)

    def _reasons(self):
        nv = self.nv
        try:
            return nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append((time.perf_counter(),
                                     self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM),
                                     int(self._reasons())))
            except Exception:
                pass
            time.sleep(0.0005)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "nvml unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        window = "timed region"
        if len(inside) < 3:
            inside = self.samples
            window = "warm-up + timed region (timed region shorter than the sampling period)"
        mhz = [s[1] for s in inside]
        bits = 0
        for s in inside:
            bits |= s[2]
        reasons = sorted(v for k, v in self.REASONS.items() if bits & k and k != 0x1)
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside), "window": window}


# ----------------------------------------------------------------- helpers
def dev_bf16(torch, bits, device):
    a = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def gpu_inputs(torch, w, device, rank, host_gen):
    """bf16 inputs on the device.  host_gen: the seeded synth generator (same
    bits the oracle sees); otherwise torch's generator with the same
    distributions (used for the very large sweep workloads)."""
    if host_gen:
        inp = make_inputs(w, seed_base=1000 * w.cid + 100 * rank)
        out = {k: dev_bf16(torch, v, device) for k, v in inp.items() if k != "bias"}
        out["bias"] = torch.from_numpy(inp["bias"]).to(device) if "bias" in inp else None
        return out, inp
    g = torch.Generator(device=device)
    g.manual_seed(1000 * w.cid + 100 * rank)
    def rn(*shape, std=1.0):
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        t.normal_(0.0, std, generator=g)
        return t
    out = dict(x=rn(w.B, w.S, w.d_model), W_r=rn(w.G, w.d_model, w.M, std=w.wr_std),
               Q=rn(w.B, w.S, w.N, w.d), Qs=rn(w.B, w.S, w.d), K=rn(w.B, w.S, w.G, w.d),
               V=rn(w.B, w.S, w.G, w.d))
    out["bias"] = None
    if w.bias0:
        b = torch.zeros(w.G, w.M, dtype=torch.float32, device=device)
        b[:, 0] = w.bias0
        out["bias"] = b
    return out, None


def timed_loop(torch, fn, steps, warmup, flush, attn_events=False):
    """Per-step device times (ms) with CUDA events on the launching stream.
    The L2 flush before each step is outside the events."""
    import moe_routed_grouped_b200 as gqe
    for _ in range(warmup):
        flush()
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    aev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)] if attn_events else []
    for a, b in aev:  # create the event handles before handing them to the library
        a.record(); b.record()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(steps):
        flush()
        if attn_events:
            gqe.gqe_set_profile_events(*aev[i])
        ev[i][0].record()
        fn()
        ev[i][1].record()
    torch.cuda.synchronize()
    t1 = time.perf_counter()
    if attn_events:
        gqe.gqe_set_profile_events(None, None)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    attn_ms = [a.elapsed_time(b) for a, b in aev]
    return step_ms, attn_ms, t0, t1


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(w, inp, budget_s=12.0, rows_per_seq=None):
    """Time the CPU oracle (router + routed attention of all G*k + 1 heads)
    on whole sequences of the workload until ~budget_s of CPU work."""
    import oracle
    done_tokens, t_total, seqs = 0, 0.0, 0
    for b in range(w.B):
        rows = np.arange(w.S) if rows_per_seq is None else \
            np.unique(np.linspace(0, w.S - 1, rows_per_seq).astype(np.int64))
        t0 = time.perf_counter()
        xb = inp["x"][b:b + 1, rows]
        idx, p, wts, _ = oracle.route(xb, inp["W_r"], inp.get("bias"), w.k)
        full_idx = np.zeros((1, w.S, w.G, w.k), np.int32)
        full_w = np.zeros((1, w.S, w.G, w.k))
        full_idx[0, rows] = idx[0]
        full_w[0, rows] = wts[0]
        oracle.gqe_prefill_rows(inp["Q"][b:b + 1], inp["Qs"][b:b + 1], inp["K"][b:b + 1],
                                inp["V"][b:b + 1], full_idx, full_w, [rows])
        t_total += time.perf_counter() - t0
        done_tokens += len(rows)
        seqs += 1
        if t_total >= budget_s:
            break
    return done_tokens, t_total, seqs


# ----------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    inp = make_inputs(w)
    # each step: the oracle on an evenly spaced sample of one sequence's rows
    rows_per_step = max(64, min(w.S, 512))
    for _ in range(args.warmup):
        oracle_sample(w, inp, budget_s=0.0, rows_per_seq=min(rows_per_step, 64))
    toks, secs = 0, 0.0
    for _ in range(args.steps):
        n, t, _ = oracle_sample(w, inp, budget_s=0.0, rows_per_seq=rows_per_step)
        toks += n
        secs += t
    val = toks / secs
    sample = (f"{args.steps} steps; each step routes and attends (all {w.G * w.k + 1} active "
              f"heads) {rows_per_step} evenly spaced token positions of sequence 0")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * secs / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, world),
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def reduce_max(values, dist, device=None):
    """Element-wise max of per-rank values over all ranks (identity without a
    process group).  Ranks are independent replicas; this is the only
    cross-rank step of the benchmark."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(tokens_per_rank, steps, world, max_total_ms):
    """Whole-job tokens/s: every rank processed `tokens_per_rank * steps`
    tokens; the job took the slowest rank's device time."""
    return world * tokens_per_rank * steps / (max_total_ms / 1e3)


def config_of(w, world):
    return {"workload": w.name, "B": w.B, "S": w.S, "N": w.N, "G": w.G, "M": w.M, "k": w.k,
            "d": w.d, "d_model": w.d_model, "router_bias_expert0": w.bias0,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "output": "float32 concat buffer (W_O input)",
            "l2": "256 MiB buffer written between steps; the write is outside the step time"}


# ----------------------------------------------------------------- decode mode
DECODE_METRIC = "GQE decode tokens/s (one new token per sequence over a full T-token KV cache)"


def measure_decode(torch, w, device, rank, steps, warmup, flush):
    """One decode step per sequence of the workload, its KV cache full (T = S,
    position T-1): gqe_route on the B new tokens, then gqe_attention_decode
    (split-KV partials + merge).  Returns this rank's step times and the mean
    time of the decode attention (the two decode kernels) alone."""
    from moe_routed_grouped_b200.layer import GqeDecode
    g = torch.Generator(device=device)
    g.manual_seed(7000 + 100 * rank)

    def rn(*shape, std=1.0):
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        t.normal_(0.0, std, generator=g)
        return t
    B, T = w.B, w.S
    dev = dict(x=rn(B, w.d_model), W_r=rn(w.G, w.d_model, w.M, std=w.wr_std), Q=rn(B, w.N, w.d),
               Qs=rn(B, w.d), Kc=rn(B, T, w.G, w.d), Vc=rn(B, T, w.G, w.d))
    pos = torch.full((B,), T - 1, dtype=torch.int32, device=device)
    L = GqeDecode(B, T, w.N, w.G, w.k, w.d, w.d_model, out_fp32=True, device=device)
    aev = []

    def step():
        L.route(dev["x"], dev["W_r"])
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        L.attention(dev["Q"], dev["Qs"], dev["Kc"], dev["Vc"], pos)
        b.record()
        aev.append((a, b))

    step_ms, _, t0, t1 = timed_loop(torch, step, steps, warmup, flush)
    torch.cuda.synchronize()
    attn = [a.elapsed_time(b) for a, b in aev[-steps:]]
    st = L.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} in the decode loop")
    return dict(step_ms=step_ms, attn_ms=statistics.mean(attn), t0=t0, t1=t1,
                kv_bytes=2 * B * T * w.G * w.d * 2)  # K and V rows 0..T-1 of every KV head


def decode_summary(w, world, steps, tot_ms, attn_ms, kv_bytes, peaks, peak_src):
    gbs = kv_bytes / (attn_ms / 1e3) / 1e9
    return {
        "metric": DECODE_METRIC, "value": world * w.B * steps / (tot_ms / 1e3),
        "unit": "tokens/s", "ms_per_step": tot_ms / steps,
        "config": dict(config_of(w, world), mode="decode", T=w.S, position=w.S - 1),
        "roofline": {"kernel": "decode_partial_kernel + decode_merge_kernel", "bound": "hbm",
                     "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": f"{peak_src} HBM copy bandwidth",
                     "attention_ms": attn_ms, "per_launch_bytes": kv_bytes,
                     "bytes_definition": "K and V cache rows 0..T-1 of all G KV heads, bf16"},
        # per step: route_prep, route, decode partial, decode merge
        "gpu_launches": steps * 4,
    }


def decode_entries(torch, device, rank, local, flush, peaks, peak_src,
                   names=("layer250m", "million"), steps=20, warmup=3):
    """The decode step at the bench's own shape and over a 1M-token cache, for
    the prefill line (one GPU).  A failure becomes an entry with its error,
    so the prefill numbers of the line stand."""
    dec = []
    for name in names:
        wd = WORKLOADS[name]
        cs = ClockSampler(local)
        cs.start()
        try:
            r = measure_decode(torch, wd, device, rank, steps, warmup, flush)
            cs.stop()
            e = decode_summary(wd, 1, steps, sum(r["step_ms"]), r["attn_ms"], r["kv_bytes"],
                               peaks, peak_src)
            e.update(workload=name, steps=steps, warmup=warmup,
                     clocks=cs.summary(r["t0"], r["t1"]))
            dec.append(e)
            del r
        except Exception as ex:  # noqa: BLE001
            dec.append({"workload": name, "error": f"{type(ex).__name__}: {ex}"[:300]})
        finally:
            cs.stop()
        torch.cuda.empty_cache()
    return dec


def run_decode(args, torch, w, device, rank, world, dist, peaks, peak_src, flush):
    """`--decode`: the decode step alone, as its own contract line."""
    clocks = ClockSampler(device.index)
    clocks.start()
    r = measure_decode(torch, w, device, rank, args.steps, args.warmup, flush)
    clocks.stop()
    tot_ms, attn_ms = reduce_max([sum(r["step_ms"]), r["attn_ms"]], dist, device)
    line = decode_summary(w, world, args.steps, tot_ms, attn_ms, r["kv_bytes"], peaks, peak_src)
    line.update({"n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                 "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                 "dtype": "bf16 in, float32 arithmetic", "data": "synthetic",
                 "clocks": clocks.summary(r["t0"], r["t1"])})
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- our arm
def measure_workload(torch, w, device, rank, steps, warmup, flush, host_gen, with_attn_events):
    from moe_routed_grouped_b200.layer import GqePrefill
    dev, host = gpu_inputs(torch, w, device, rank, host_gen)
    L = GqePrefill(w.B, w.S, w.N, w.G, w.k, w.d, w.d_model, out_fp32=True, device=device)

    def routed():
        L.route(dev["x"], dev["W_r"], dev["bias"])
        L.attention(dev["Q"], dev["Qs"], dev["K"], dev["V"])

    def dense():
        L.dense(dev["Q"], dev["K"], dev["V"])

    r_ms, r_attn, t0, t1 = timed_loop(torch, routed, steps, warmup, flush, with_attn_events)
    d_ms, d_attn, d0, d1 = timed_loop(torch, dense, steps, warmup, flush, with_attn_events)
    status = L.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after {w.name}")
    return dict(L=L, dev=dev, host=host, routed_ms=r_ms, routed_attn_ms=r_attn, dense_ms=d_ms,
                dense_attn_ms=d_attn, t0=t0, t1=t1, dense_t0=d0, dense_t1=d1)


def layer_entry(torch, device, local, flush, peaks, peak_src, steps=20, warmup=3):
    """The whole attention layer at the bench shape (gqe_layer_prefill: router,
    K/V/Qs projections, the selected heads' Q projection, attention, W_O)
    against the all-active GQA layer (gqe_dense_layer_prefill), plus the W_O
    projection alone against the tensor-core peak.  Random bf16 weights with
    std d_model^-1/2; inputs from torch's generator."""
    from moe_routed_grouped_b200.layer import GqeLayer
    import moe_routed_grouped_b200 as gqe
    w = WORKLOADS["layer250m"]
    B, S, N, G, k, d, dm, M = w.B, w.S, w.N, w.G, w.k, w.d, w.d_model, w.M
    g = torch.Generator(device=device)
    g.manual_seed(9100)

    def rn(*shape, std=1.0):
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        t.normal_(0.0, std, generator=g)
        return t
    row = (G * k + G + 1) * d
    sd = dm ** -0.5
    W = dict(Q=rn(N, dm, d, std=sd), K=rn(G, dm, d, std=sd), V=rn(G, dm, d, std=sd),
             s=rn(dm, d, std=sd), r=rn(G, dm, M, std=sd), O=rn(row, dm, std=row ** -0.5),
             Od=rn(N * d, dm, std=(N * d) ** -0.5))
    x = rn(B, S, dm)
    L = GqeLayer(B, S, N, G, k, d, dm, device=device)
    cs = ClockSampler(local)
    cs.start()
    try:
        r_ms, _, t0, t1 = timed_loop(
            torch, lambda: L.forward(x, W["Q"], W["K"], W["V"], W["s"], W["r"], None, W["O"]),
            steps, warmup, flush)
        d_ms, _, d0, d1 = timed_loop(
            torch, lambda: L.dense(x, W["Q"], W["K"], W["V"], W["Od"]), steps, warmup, flush)
        T = B * S
        Y = torch.empty(T, dm, dtype=torch.float32, device=device)
        o_ms, _, _, _ = timed_loop(
            torch, lambda: gqe.gqe_linear(T, row, 1, dm, L.concat, row, W["O"], Y, dm, 1),
            steps, warmup, flush)
    finally:
        cs.stop()
    if L.device_status() != 0:
        raise RuntimeError("device status after the layer loop")
    T = B * S
    attn_r, attn_d = w.useful_flop_routed(), w.useful_flop_dense()
    proj_r = 2.0 * T * dm * (2 * G * d + d + G * k * d) + 2.0 * T * row * dm + 2.0 * T * dm * G * M
    proj_d = 2.0 * T * dm * (2 * G * d + N * d) + 2.0 * T * N * d * dm
    rm, dmm, om = statistics.mean(r_ms), statistics.mean(d_ms), statistics.mean(o_ms)
    o_tf = 2.0 * T * row * dm / (om / 1e3) / 1e12
    return {"workload": "layer250m", "steps": steps, "warmup": warmup,
            "routed_ms": rm, "dense_ms": dmm, "routed_over_dense": dmm / rm,
            "routed_tokens_per_s": T / (rm / 1e3), "dense_tokens_per_s": T / (dmm / 1e3),
            "routed_flop": attn_r + proj_r, "dense_flop": attn_d + proj_d,
            "routed_tflops": (attn_r + proj_r) / (rm / 1e3) / 1e12,
            "dense_tflops": (attn_d + proj_d) / (dmm / 1e3) / 1e12,
            "w_o_gemm": {"kernel": "gemm_dense_kernel (T x %d x %d, bf16 in, fp32 out)" % (row, dm),
                         "ms": om, "tflops": o_tf, "peak": peaks["bf16_tflops"],
                         "frac": o_tf / peaks["bf16_tflops"],
                         "peak_source": f"{peak_src} bf16 dense (burst)"},
            "clocks": cs.summary(t0, d1),
            # routed layer 10 kernels (2 router, 3 projections, 2 routed Q, 2 attention,
            # W_O), dense layer 6, W_O alone 1
            "gpu_launches": steps * (10 + 6 + 1)}


def backward_entry(torch, device, local, flush, peaks, peak_src, steps=10, warmup=3):
    """The training step of the path at the bench shape: the forward that keeps
    each row's log-sum-exp (gqe_attention_prefill_train) and the backward pass
    (gqe_prefill_backward), timed separately.  Useful backward work: 5 products
    of 2d flop per visible (query, key) pair and active head (S, dP, dV, dK,
    dQ)."""
    from moe_routed_grouped_b200.layer import GqePrefill
    w = WORKLOADS["layer250m"]
    dev, _ = gpu_inputs(torch, w, device, 0, False)
    L = GqePrefill(w.B, w.S, w.N, w.G, w.k, w.d, w.d_model, out_fp32=True, device=device)
    g = torch.Generator(device=device)
    g.manual_seed(9300)
    dcat = torch.randn(w.B * w.S, L.row, generator=g, device=device)
    fwd = lambda: L.forward_train(dev["x"], dev["W_r"], dev["bias"], dev["Q"], dev["Qs"],  # noqa: E731
                                  dev["K"], dev["V"])
    cs = ClockSampler(local)
    cs.start()
    try:
        f_ms, _, t0, _ = timed_loop(torch, fwd, steps, warmup, flush)
        fwd()
        b_ms, _, _, t1 = timed_loop(torch, lambda: L.backward(dcat), steps, warmup, flush)
    finally:
        cs.stop()
    if L.device_status() != 0:
        raise RuntimeError("device status after the backward loop")
    pairs = (w.G * w.k + 1) * w.B * w.S * (w.S + 1) / 2.0
    bwd_flop = pairs * 5 * 2 * w.d
    fm, bm = statistics.mean(f_ms), statistics.mean(b_ms)
    tf = bwd_flop / (bm / 1e3) / 1e12
    return {"workload": "layer250m", "steps": steps, "warmup": warmup,
            "forward_train_ms": fm, "backward_ms": bm,
            "backward_tokens_per_s": w.B * w.S / (bm / 1e3),
            "backward_useful_tflops": tf, "backward_frac_of_peak": tf / peaks["bf16_tflops"],
            "backward_flop": bwd_flop,
            "flop_definition": "5 products x 2d flop per visible (query, key) pair, G*k+1 heads",
            "peak_source": f"{peak_src} bf16 dense (burst)",
            "clocks": cs.summary(t0, t1),
            # forward: route_prep, route, prep, attention; backward: bucket prep,
            # 2 memsets (not kernels of this library), bwd prep, bwd
            "gpu_launches": steps * 4 + steps * 3}


def chunk_entry(torch, device, local, flush, peaks, peak_src, steps=5, warmup=3, chunk=4096):
    """Chunked prefill (gqe_attention_prefill_chunk): the 32k biased workload
    processed as S / chunk chunks over a full KV cache, each chunk's queries at
    their absolute positions, against the one-shot prefill of the same
    sequence.  Same useful work; the difference is the chunks' extra work
    (each chunk re-reads the cache prefix) and launch overhead."""
    from moe_routed_grouped_b200.layer import GqeChunk, GqePrefill
    w = WORKLOADS["imbalanced32k"]
    dev, _ = gpu_inputs(torch, w, device, 0, False)
    n = w.S // chunk
    C = GqeChunk(w.B, chunk, w.S, w.N, w.G, w.k, w.d, w.d_model, device=device)
    P = GqePrefill(w.B, w.S, w.N, w.G, w.k, w.d, w.d_model, device=device)
    P.route(dev["x"], dev["W_r"], dev["bias"])
    offs = [torch.tensor([i * chunk], dtype=torch.int32, device=device) for i in range(n)]
    parts = [{k: dev[k][:, i * chunk:(i + 1) * chunk].contiguous() for k in ("x", "Q", "Qs")}
             for i in range(n)]

    def chunked():
        for i in range(n):
            C.forward(parts[i]["x"], dev["W_r"], dev["bias"], parts[i]["Q"], parts[i]["Qs"],
                      dev["K"], dev["V"], offs[i])
    cs = ClockSampler(local)
    cs.start()
    try:
        c_ms, _, t0, _ = timed_loop(torch, chunked, steps, warmup, flush)
        o_ms, _, _, t1 = timed_loop(torch, lambda: P.attention(dev["Q"], dev["Qs"], dev["K"],
                                                               dev["V"]), steps, warmup, flush)
    finally:
        cs.stop()
    if C.device_status() != 0 or P.device_status() != 0:
        raise RuntimeError("device status after the chunk loop")
    cm, om = statistics.mean(c_ms), statistics.mean(o_ms)
    fl = w.useful_flop_routed()
    return {"workload": "imbalanced32k", "chunk": chunk, "chunks": n, "steps": steps,
            "warmup": warmup, "chunked_ms": cm, "one_shot_attention_ms": om,
            "chunked_tokens_per_s": w.B * w.S / (cm / 1e3),
            "chunked_useful_tflops": fl / (cm / 1e3) / 1e12,
            "chunked_over_one_shot": om / cm,
            "note": "chunked includes the router per chunk; one-shot is the attention call alone",
            "clocks": cs.summary(t0, t1), "gpu_launches": steps * n * 5 + steps * 2}


# the long-context workloads every default line also measures: (name, timed steps)
CONFIG_ENTRIES = (("imbalanced32k", 10), ("wide131k", 5), ("million", 3))


def config_entry(torch, name, steps, warmup, device, rank, local, flush, peaks, peak_src):
    """Routed GQE and dense GQA on one long-context workload, each timed over
    its own steps with its own clock record (NVML samples every ~0.5 ms, so the
    1M-token steps of about 2 s are sampled inside every step).  Inputs come
    from torch's generator on the device with the synth recipe's
    distributions (parity runs on the synth bits in the tests)."""
    ws = WORKLOADS[name]
    cs = ClockSampler(local)
    cs.start()
    try:
        r = measure_workload(torch, ws, device, rank, steps, warmup, flush, False, True)
    finally:
        cs.stop()
    rm, dm = statistics.mean(r["routed_ms"]), statistics.mean(r["dense_ms"])
    ra, da = statistics.mean(r["routed_attn_ms"]), statistics.mean(r["dense_attn_ms"])
    fr, fd = ws.useful_flop_routed(), ws.useful_flop_dense()
    attn_tf, dense_attn_tf = fr / (ra / 1e3) / 1e12, fd / (da / 1e3) / 1e12
    e = {
        "workload": name, "B": ws.B, "S": ws.S, "N": ws.N, "G": ws.G, "k": ws.k, "d": ws.d,
        "d_model": ws.d_model, "router_bias_expert0": ws.bias0, "steps": steps,
        "warmup": warmup,
        "routed_ms": rm, "routed_ms_median": statistics.median(r["routed_ms"]),
        "routed_ms_best": min(r["routed_ms"]),
        "dense_ms": dm, "dense_ms_median": statistics.median(r["dense_ms"]),
        "dense_ms_best": min(r["dense_ms"]),
        "routed_tokens_per_s": ws.B * ws.S / (rm / 1e3),
        "dense_tokens_per_s": ws.B * ws.S / (dm / 1e3),
        "routed_useful_tflops": fr / (rm / 1e3) / 1e12,
        "dense_useful_tflops": fd / (dm / 1e3) / 1e12,
        "routed_over_dense": dm / rm,
        "roofline": {"kernel": ("attn_pair_kernel" if ws.d == 64 and
                                2 * ws.B * ws.S * ws.G * ws.d * 2 >= 96 << 20
                                else "attn_kernel<%d>" % ws.d) + " (routed + shared head)",
                     "bound": "tensor", "achieved": attn_tf, "unit": "TFLOP/s",
                     "peak": peaks["bf16_tflops"], "frac": attn_tf / peaks["bf16_tflops"],
                     "peak_sustained": peaks.get("bf16_tflops_sustained"),
                     "frac_sustained": (attn_tf / peaks["bf16_tflops_sustained"]
                                        if peaks.get("bf16_tflops_sustained") else None),
                     "peak_source": f"{peak_src} bf16 dense (burst; sustained beside it)",
                     "attention_kernel_ms": ra, "per_launch_flop": fr},
        "dense_attention_kernel_ms": da, "dense_attention_kernel_tflops": dense_attn_tf,
        "dense_attention_frac": dense_attn_tf / peaks["bf16_tflops"],
        "clocks_routed": cs.summary(r["t0"], r["t1"]),
        "clocks_dense": cs.summary(r["dense_t0"], r["dense_t1"]),
        "inputs": "torch generator on the device, the synth recipe's distributions",
        "gpu_launches": steps * (4 + (1 if ws.k > 1 else 0)) + steps * 2,
    }
    del r
    torch.cuda.empty_cache()
    return e


def e2e_measure(torch, w, L, dev, steps, warmup):
    """Through the public API with host buffers, as a serving loop runs it:
    every step uploads its inputs from pinned host memory, runs route +
    attention and downloads the concat output and the top-k indices.  Two
    sets of device buffers let step i+1's upload and step i-1's download run
    on their own streams while step i computes; every copy of every step is
    inside the timed region."""
    from moe_routed_grouped_b200.layer import GqePrefill
    host_in = {k: v.to("cpu").pin_memory() for k, v in dev.items() if v is not None}
    Ls = [L, GqePrefill(w.B, w.S, w.N, w.G, w.k, w.d, w.d_model, out_fp32=True,
                        device=dev["x"].device)]
    devs = [dev, {k: (None if v is None else torch.empty_like(v)) for k, v in dev.items()}]
    outs = [(torch.empty_like(Li.concat, device="cpu").pin_memory(),
             torch.empty_like(Li.topk_idx, device="cpu").pin_memory()) for Li in Ls]
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = outs[0][0].numel() * outs[0][0].element_size() + \
        outs[0][1].numel() * outs[0][1].element_size()
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    in_done = [torch.cuda.Event() for _ in range(2)]
    cmp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def step(i):
        b = i & 1
        Li, di, (oh, ih) = Ls[b], devs[b], outs[b]
        if used[b]:  # buffer b's inputs are free once its last compute is done
            s_in.wait_event(cmp_done[b])
        with torch.cuda.stream(s_in):
            for k, v in host_in.items():
                di[k].copy_(v, non_blocking=True)
        in_done[b].record(s_in)
        s_cmp.wait_event(in_done[b])
        if used[b]:  # and its outputs once their download is done
            s_cmp.wait_event(out_done[b])
        Li.route(di["x"], di["W_r"], di["bias"], stream=s_cmp)
        Li.attention(di["Q"], di["Qs"], di["K"], di["V"], stream=s_cmp)
        cmp_done[b].record(s_cmp)
        s_out.wait_event(cmp_done[b])
        with torch.cuda.stream(s_out):
            oh.copy_(Li.concat, non_blocking=True)
            ih.copy_(Li.topk_idx, non_blocking=True)
        out_done[b].record(s_out)
        used[b] = True

    # The PCIe link and the host side of the copies take some tens of
    # milliseconds of traffic to reach full speed (an idle GPU's first 100 MB
    # uploads run at about 40 GB/s, later ones at about 55), so the warm-up
    # runs long enough for that; the buffer parity stays as in the timed loop.
    for i in range(2 * max(1, (warmup + 1) // 2)):
        step(i)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(s_in)
    for i in range(steps):
        step(i)
    s_out.wait_event(out_done[(steps - 1) & 1])
    e.record(s_out)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    for Li in Ls:
        st = Li.device_status()
        if st != 0:
            raise RuntimeError(f"device status {st} in the end-to-end loop")
    return ms, h2d, d2h


# Small cases that run a kernel a few times without timing, for a profiler to
# capture one launch (inputs from torch's generator; a few hundred MB on the
# device at most, more than the 126 MB L2).
NCU_CASES = ("attn_d64_32k", "attn_d128_32k", "pair_d64_32k", "layer250m", "bwd_d64_8k",
             "decode_32k", "decode_b8_2k", "route_32k")


def run_ncu_case(torch, name, device, reps=2):
    import moe_routed_grouped_b200 as gqe
    from moe_routed_grouped_b200.layer import GqeDecode, GqeLayer, GqePrefill
    g = torch.Generator(device=device)
    g.manual_seed(5)

    def rn(*shape, std=1.0):
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        t.normal_(0.0, std, generator=g)
        return t
    if name == "layer250m":
        w = WORKLOADS["layer250m"]
        B, S, N, G, k, d, dm, M = w.B, w.S, w.N, w.G, w.k, w.d, w.d_model, w.M
        row, sd = (G * k + G + 1) * d, dm ** -0.5
        W = [rn(N, dm, d, std=sd), rn(G, dm, d, std=sd), rn(G, dm, d, std=sd), rn(dm, d, std=sd),
             rn(G, dm, M, std=sd)]
        Wo, x = rn(row, dm, std=row ** -0.5), rn(B, S, dm)
        L = GqeLayer(B, S, N, G, k, d, dm, device=device)
        for _ in range(reps):
            L.forward(x, *W, None, Wo)
    elif name == "route_32k":  # the router alone on the 32k biased shape (W_r-resident kernel)
        B, S, N, G, k, d, dm = 1, 32768, 16, 8, 1, 64, 1024
        M = N // G
        bias = torch.zeros(G, M, dtype=torch.float32, device=device)
        bias[:, 0] = 1.5
        x, Wr = rn(B, S, dm), rn(G, dm, M, std=dm ** -0.5)
        L = GqePrefill(B, S, N, G, k, d, dm, device=device)
        for _ in range(reps):
            L.route(x, Wr, bias)
    elif name.startswith("decode"):  # one sequence over 32k cached tokens, or the bench's B = 8, T = 2k
        B, T = (1, 32768) if name == "decode_32k" else (8, 2048)
        N, G, k, d, dm = 16, 8, 1, 64, 1024
        L = GqeDecode(B, T, N, G, k, d, dm, device=device)
        args = (rn(B, dm), rn(G, dm, N // G, std=dm ** -0.5), None, rn(B, N, d), rn(B, d),
                rn(B, T, G, d), rn(B, T, G, d),
                torch.full((B,), T - 1, dtype=torch.int32, device=device))
        for _ in range(reps):
            L.forward(*args)
    else:
        shapes = {"attn_d64_32k": (1, 32768, 16, 8, 1, 64, 1024, 1.5),
                  "attn_d128_32k": (1, 32768, 32, 8, 2, 128, 1024, 0.0),
                  "pair_d64_32k": (1, 32768, 16, 8, 1, 64, 1024, 1.5),
                  "bwd_d64_8k": (1, 8192, 16, 8, 1, 64, 1024, 0.0)}
        B, S, N, G, k, d, dm, b0 = shapes[name]
        M = N // G
        bias = None
        if b0:
            bias = torch.zeros(G, M, dtype=torch.float32, device=device)
            bias[:, 0] = b0
        x, Wr = rn(B, S, dm), rn(G, dm, M, std=dm ** -0.5)
        Q, Qs, K, V = rn(B, S, N, d), rn(B, S, d), rn(B, S, G, d), rn(B, S, G, d)
        L = GqePrefill(B, S, N, G, k, d, dm, device=device)
        prev = gqe.gqe_set_pair_threshold(0 if name.startswith("pair") else -1)
        try:
            if name.startswith("bwd"):
                L.forward_train(x, Wr, bias, Q, Qs, K, V)
                dcat = torch.randn(B * S, L.row, generator=g, device=device)
                for _ in range(reps):
                    L.backward(dcat)
            else:
                L.route(x, Wr, bias)
                for _ in range(reps):
                    L.attention(Q, Qs, K, V)
        finally:
            gqe.gqe_set_pair_threshold(prev)
    torch.cuda.synchronize()
    st = L.device_status()
    print(json.dumps({"ncu_case": name, "device_status": st}), flush=True)
    return 0 if st == 0 else 1


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="layer250m", choices=sorted(WORKLOADS))
    ap.add_argument("--no-configs", action="store_true",
                    help="leave the S=32k, 131k and 1M entries out of the line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="leave the decode-step measurements out of the prefill line")
    ap.add_argument("--ncu-case", choices=NCU_CASES, default=None,
                    help="run one small case's kernels a few times, untimed, for a profiler")
    ap.add_argument("--decode", action="store_true",
                    help="time one decode step per sequence over a full cache of S tokens "
                         "instead of the prefill (prints its own line)")
    args = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    import torch
    import moe_routed_grouped_b200  # noqa: F401  (fails loudly if libgqe.so is missing)

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    def barrier():
        if dist is not None:
            dist.barrier()

    peaks, peak_src = load_peaks()
    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    flush = lambda: flush_buf.zero_()  # noqa: E731

    if args.ncu_case:
        return run_ncu_case(torch, args.ncu_case, device)

    w = WORKLOADS[args.workload]
    if args.decode:
        rc = run_decode(args, torch, w, device, rank, world, dist, peaks, peak_src, flush)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return rc
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    res = measure_workload(torch, w, device, rank, args.steps, args.warmup, flush, True, True)
    barrier()
    clocks.stop()

    tot_ms = sum(res["routed_ms"])
    dense_tot_ms = sum(res["dense_ms"])
    attn_ms = statistics.mean(res["routed_attn_ms"])
    dense_attn_ms = statistics.mean(res["dense_attn_ms"])
    tot_ms, dense_tot_ms, attn_ms, dense_attn_ms = reduce_max(
        [tot_ms, dense_tot_ms, attn_ms, dense_attn_ms], dist, device)

    tokens = w.B * w.S
    value = job_throughput(tokens, args.steps, world, tot_ms)
    dense_value = job_throughput(tokens, args.steps, world, dense_tot_ms)
    ms_step = tot_ms / args.steps
    fl_r, fl_d = w.useful_flop_routed(), w.useful_flop_dense()
    useful_tf = fl_r / (ms_step / 1e3) / 1e12
    dense_tf = fl_d / (dense_tot_ms / args.steps / 1e3) / 1e12
    peak_tf = peaks["bf16_tflops"]
    attn_tf = fl_r / (attn_ms / 1e3) / 1e12
    dense_attn_tf = fl_d / (dense_attn_ms / 1e3) / 1e12

    e2e_ms, h2d, d2h = e2e_measure(torch, w, res["L"], res["dev"], max(10, args.steps),
                                   max(10, args.warmup))
    e2e_val = world * tokens / (e2e_ms / 1e3)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        # this rank's per-step spread (the mean above is the max over ranks)
        "ms_per_step_median": statistics.median(res["routed_ms"]),
        "ms_per_step_best": min(res["routed_ms"]),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 inputs; random-init router)",
        "config": config_of(w, world),
        "useful_tflops_per_gpu": useful_tf,
        "useful_frac_of_peak": useful_tf / peak_tf,
        "dense_gqa": {"value": dense_value, "unit": "tokens/s",
                      "ms_per_step": dense_tot_ms / args.steps,
                      "useful_tflops_per_gpu": dense_tf, "attention_kernel_ms": dense_attn_ms,
                      "attention_kernel_tflops": dense_attn_tf},
        "routed_over_dense": dense_tot_ms / tot_ms,
        "roofline": {"kernel": "attn_kernel<%d> (routed + shared head)" % w.d, "bound": "tensor",
                     "achieved": attn_tf, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": attn_tf / peak_tf,
                     "traffic": kernel_traffic(f"attn_kernel<{w.d}>:routed:{w.name}"),
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "peak_source": f"{peak_src} bf16 dense (burst)",
                     "attention_kernel_ms": attn_ms,
                     "per_launch_flop": fl_r,
                     "flop_definition": "4*d per visible (query, key) pair, (G*k+1)*B*S*(S+1)/2 pairs"},
        "e2e": {"value": e2e_val, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "pipeline": "two buffer sets; upload, compute and download on their own streams",
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        # per routed step: route_prep, route, prep (bucket + V fp16 + sort), attention
        # (+ combine when k > 1)
        "gpu_launches": args.steps * (4 + (1 if w.k > 1 else 0)),
        "clocks": clocks.summary(res["t0"], res["t1"]),
    }

    if world == 1 and not args.no_configs:
        for key, fn, wl in (("layer", layer_entry, "layer250m"),
                            ("backward", backward_entry, "layer250m"),
                            ("chunked", chunk_entry, "imbalanced32k")):
            try:
                line[key] = fn(torch, device, local, flush, peaks, peak_src)
                line["gpu_launches"] += line[key]["gpu_launches"]
            except Exception as ex:  # noqa: BLE001  (reported in the entry, not hidden)
                line[key] = {"workload": wl, "error": f"{type(ex).__name__}: {ex}"[:300]}
            torch.cuda.empty_cache()
        # the S >= 32k workloads, each with its own timing and clock record
        del res
        torch.cuda.empty_cache()
        entries = []
        for name, k_steps in CONFIG_ENTRIES:
            try:
                entries.append(config_entry(torch, name, k_steps, 3, device, rank, local, flush,
                                            peaks, peak_src))
            except Exception as ex:  # noqa: BLE001  (reported in the entry, not hidden)
                entries.append({"workload": name, "error": f"{type(ex).__name__}: {ex}"[:300]})
                torch.cuda.empty_cache()
        line["configs"] = entries
        line["gpu_launches"] += sum(e.get("gpu_launches", 0) for e in entries)

    if world == 1 and not args.no_decode:
        if "res" in locals():
            del res
        torch.cuda.empty_cache()
        line["decode"] = decode_entries(torch, device, rank, local, flush, peaks, peak_src)

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = make_inputs(w)
        n, secs, seqs = oracle_sample(w, host)
        line["cpu_baseline"] = {"value": n / secs, "unit": "tokens/s", "cores": blas_threads(),
                                "kind": "oracle",
                                "sample": f"{seqs} whole sequence(s) of {w.S} tokens: router + "
                                          f"all {w.G * w.k + 1} active heads, float64 numpy"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
