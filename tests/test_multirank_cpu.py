"""The benchmark's multi-rank path on CPU: two gloo ranks on 127.0.0.1.

Ranks are independent replicas (batches do not interact); the only
cross-rank step is the max of the per-rank device times, from which the
whole-job throughput is computed."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 5.0 - rank, 1.5 * (rank + 1)]
        got = bench.reduce_max(mine, dist)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r] == [11.0, 5.0, 3.0]


def test_job_throughput_is_weak_scaling():
    # 2 ranks x 16384 tokens x 10 steps in the slowest rank's 2 ms
    assert bench.job_throughput(16384, 10, 2, 2.0) == pytest.approx(2 * 16384 * 10 / 2e-3)
    assert bench.reduce_max([1.0, 2.0], None) == [1.0, 2.0]


def _bench(env_extra, *args):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], cwd=root, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_reference_arm_line_on_cpu():
    """The reference arm times the oracle on the host and prints the same
    contract line, marked as the reference, with its sample described."""
    (line,) = _bench({"RANK": "0", "WORLD_SIZE": "1"}, "--impl", "reference", "--workload",
                     "tiny", "--steps", "2", "--warmup", "3")
    assert line["impl"] == "reference"
    assert line["unit"] == "tokens/s" and line["value"] > 0 and line["higher_is_better"]
    assert line["config"]["workload"] == "tiny" and line["config"]["S"] == 128
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    assert _bench({"RANK": "1", "WORLD_SIZE": "2"}, "--impl", "reference", "--workload", "tiny",
                  "--steps", "2", "--warmup", "3") == []


def test_decode_summary_counts_cache_bytes():
    """The decode roofline divides the cache bytes a step must read (K and V
    rows of every KV head, bf16) by the decode kernels' time."""
    from synth import WORKLOADS
    w = WORKLOADS["million"]
    kv = 2 * w.B * w.S * w.G * w.d * 2
    assert kv == 2 * 2 ** 30                       # 1M tokens x 8 heads x 64 x (K, V) x 2 B
    s = bench.decode_summary(w, 1, 20, 20 * 0.5, 0.4, kv, {"hbm_gbs": 6650.0}, "measured")
    assert s["value"] == pytest.approx(1 * 20 / (10.0 / 1e3))   # B = 1 token per step
    assert s["roofline"]["achieved"] == pytest.approx(kv / 0.4e-3 / 1e9)
    assert s["roofline"]["frac"] == pytest.approx(kv / 0.4e-3 / 1e9 / 6650.0)
    assert s["roofline"]["bound"] == "hbm" and s["gpu_launches"] == 80
    assert s["config"]["mode"] == "decode" and s["config"]["position"] == w.S - 1


def test_decode_measurement_code_path_on_host(monkeypatch):
    """bench.measure_decode end to end on the host with the device parts
    stubbed (CUDA events, synchronisation and the two library calls), so its
    Python plumbing - input shapes, step loop, event bookkeeping, summary -
    is exercised without a GPU."""
    from synth import WORKLOADS
    from moe_routed_grouped_b200.layer import GqeDecode

    class FakeEvent:
        def __init__(self, enable_timing=False):
            pass

        def record(self, stream=None):
            pass

        def elapsed_time(self, other):
            return 0.25

    calls = []
    monkeypatch.setattr(torch.cuda, "Event", FakeEvent)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(GqeDecode, "route", lambda self, x, W, bias=None, stream=None:
                        calls.append(("route", tuple(x.shape), tuple(W.shape))))
    monkeypatch.setattr(GqeDecode, "attention", lambda self, Q, Qs, Kc, Vc, pos, kv_start=None,
                        stream=None: calls.append(("attn", tuple(Q.shape), tuple(Kc.shape),
                                                   int(pos[0]))))
    monkeypatch.setattr(GqeDecode, "device_status", lambda self, clear=True, stream=None: 0)
    w = WORKLOADS["tiny"]
    r = bench.measure_decode(torch, w, torch.device("cpu"), 0, 4, 3, lambda: None)
    assert len(r["step_ms"]) == 4 and r["attn_ms"] == 0.25
    assert r["kv_bytes"] == 2 * w.B * w.S * w.G * w.d * 2
    assert calls[0] == ("route", (w.B, w.d_model), (w.G, w.d_model, w.M))
    assert calls[1] == ("attn", (w.B, w.N, w.d), (w.B, w.S, w.G, w.d), w.S - 1)
    assert len(calls) == 2 * (4 + 3)
    s = bench.decode_summary(w, 1, 4, sum(r["step_ms"]), r["attn_ms"], r["kv_bytes"],
                             {"hbm_gbs": 6650.0}, "measured")
    assert s["value"] == pytest.approx(w.B * 4 / (sum(r["step_ms"]) / 1e3))


def test_decode_entries_report_failures_in_place(monkeypatch):
    """The prefill line's decode list: one entry per workload, and a failing
    measurement becomes an entry with its error instead of ending the run."""
    def fake(torch_, w, device, rank, steps, warmup, flush):
        if w.name == "layer250m":
            raise RuntimeError("device status 8 in the decode loop")
        return dict(step_ms=[0.5] * steps, attn_ms=0.4, t0=0.0, t1=1.0,
                    kv_bytes=2 * w.B * w.S * w.G * w.d * 2)
    monkeypatch.setattr(bench, "measure_decode", fake)
    dec = bench.decode_entries(torch, torch.device("cpu"), 0, 0, lambda: None,
                               {"hbm_gbs": 6650.0}, "measured", names=("tiny", "layer250m"),
                               steps=5, warmup=3)
    assert [e["workload"] for e in dec] == ["tiny", "layer250m"]
    assert dec[0]["unit"] == "tokens/s" and dec[0]["steps"] == 5 and "clocks" in dec[0]
    assert dec[1] == {"workload": "layer250m",
                      "error": "RuntimeError: device status 8 in the decode loop"}


def test_config_entry_numbers_from_fake_timings(monkeypatch):
    """A long-context entry of the default line: tokens/s, useful TFLOP/s,
    the routed/dense ratio and the attention roofline against both peaks come
    from the measured times by the stated formulas; each arm carries its own
    clock record."""
    def fake(torch_, w, device, rank, steps, warmup, flush, host_gen, ev):
        assert not host_gen and ev and warmup == 3
        return dict(routed_ms=[2.0] * steps, dense_ms=[3.0] * steps,
                    routed_attn_ms=[1.5] * steps, dense_attn_ms=[2.5] * steps,
                    t0=0.0, t1=1.0, dense_t0=1.0, dense_t1=2.0)
    monkeypatch.setattr(bench, "measure_workload", fake)
    peaks = {"bf16_tflops": 1652.2, "bf16_tflops_sustained": 1379.2, "hbm_gbs": 6548.2}
    e = bench.config_entry(torch, "imbalanced32k", 4, 3, torch.device("cpu"), 0, 0,
                           lambda: None, peaks, "measured")
    w = bench.WORKLOADS["imbalanced32k"]
    assert e["routed_tokens_per_s"] == pytest.approx(w.S / 2e-3)
    assert e["routed_over_dense"] == pytest.approx(1.5)
    tf = w.useful_flop_routed() / 1.5e-3 / 1e12
    assert e["roofline"]["achieved"] == pytest.approx(tf)
    assert e["roofline"]["frac"] == pytest.approx(tf / 1652.2)
    assert e["roofline"]["frac_sustained"] == pytest.approx(tf / 1379.2)
    assert "clocks_routed" in e and "clocks_dense" in e
