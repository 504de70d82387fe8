#!/usr/bin/env python
"""Benchmark of the fast-weight chunk scan on B200 (one JSON line on rank 0).

Default workload: the TTT-Linear mini-batch scan, B=8 sequences x H=12 heads of width 64,
T=2048, inner mini-batch 16 (TTT layers page). A step is one ttt_chunk_scan over the whole
batch with inputs resident in HBM. The K timed steps run back to back between two CUDA
events (the state is reset once before the warm-up; consecutive steps continue one scan, as
successive calls do) and take their inputs from copies whose total is over three times the
126 MB L2, so every step reads from HBM rather than from L2. The other four workloads
(In-Place fp32, In-Place 4B-class, In-Place 128k with fused target, SR-TTT gate), the two
richer inner models at the TTT-Linear workload's shapes (LayerNorm TTT-Linear, TTT-MLP) and
the further forms of the path (context-parallel In-Place, the cache read path, packed
sequences) are measured the same way and reported under "workloads".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]
                  [--only-main]

With N > 1 (launched by torch.distributed.run) every rank runs an independent replica of
the workload (the (sequence, head) problems are independent; no collective on the data
path): scaling is weak and value = all ranks' tokens / the slowest rank's time.
"""

from __future__ import annotations

import argparse
import functools
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from gen import workloads as wl  # noqa: E402

METRIC = "fast-weight scan tokens/s and TFLOP/s per layer on 1 B200; % of BF16/HBM roofline"
MAIN = wl.LINEAR_GD.name


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "sm_max_mhz": d.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


# --------------------------------------------------------------------------------------------
# algorithmic work per workload (flops, compulsory bytes)
# --------------------------------------------------------------------------------------------

def work(spec) -> dict:
    if isinstance(spec, wl.InnerSpec):
        # K, V, Q read and O written (bf16), the weights read and written once (fp32); the MLP's
        # algorithmic flops outweigh its bytes at the measured peaks, the LayerNorm model's do not.
        n = spec.B * spec.H * spec.T * spec.D
        per_head = spec.D * spec.D if spec.model == "linear_ln" else 2 * spec.D * spec.hidden
        byts = (2 + 2 * spec.with_queries) * n * 2 + 2 * spec.B * spec.H * per_head * 4
        return {"tokens": spec.B * spec.T, "flops": spec.flops, "bytes": byts,
                "bound": "hbm" if spec.model == "linear_ln" else "tensor"}
    if isinstance(spec, wl.LinearSpec):
        n = spec.B * spec.H * spec.T * spec.D
        io_b = 2
        byts = (2 + spec.with_queries) * n * io_b  # K, V (, Q) read
        byts += spec.with_queries * n * io_b       # O written
        byts += 2 * spec.B * spec.H * spec.D * spec.D * 4  # W0 read, W written
        if spec.gate:
            byts += spec.B * spec.H * spec.T * 4     # losses written
            byts += spec.B * spec.H * (256 * 3 + 2) * 4  # cache
        return {"tokens": spec.B * spec.T, "flops": spec.flops, "bytes": byts, "bound": "hbm"}
    io_b = 4 if spec.dtype == "f32" else 2
    byts = spec.T * spec.f * io_b + spec.T * spec.d * io_b * 2 + 2 * spec.d * spec.f * 4
    if spec.target:
        byts += spec.d * spec.d * 2 + spec.d * 3 * 4
    bound = "alu" if spec.dtype == "f32" else "tensor"
    return {"tokens": spec.T, "flops": spec.flops, "bytes": byts, "bound": bound}


def fp32_alu_peak_tflops(peaks) -> float:
    """148 SMs x 128 fp32 lanes x 2 flops (FFMA) x max SM clock."""
    return 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12


# --------------------------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------------------------

L2_BYTES = 126 * 2**20


class Runner:
    """Builds the state and inputs of one workload and runs its steps.

    A step is one ttt_chunk_scan over the whole batch. Consecutive steps continue one scan
    (the state is not reset between them) and take their inputs and outputs from ``n_sets``
    copies in turn, enough copies that together they are over three times the 126 MB L2:
    by the time a copy comes round again, the steps in between have moved more than the L2
    holds, so every step reads its inputs from HBM."""

    def __init__(self, spec, device, prefix=False):
        import chunked_weight_layers_b200 as cwl
        self.spec = spec
        self.cwl = cwl
        self.device = device
        if isinstance(spec, wl.InnerSpec):
            x = wl.inner_inputs(spec, device=device)
            cfg = cwl.config(spec.model, batch=spec.B, heads=spec.H, eta=spec.eta, ln_eps=spec.eps,
                             token_weights=int(spec.token_weights))
            self.state = cwl.FastWeightState(cfg, x["W0"])
            self.state.set_layernorm(x["gamma"], x["beta"])
            args = dict(keys=x["K"], targets=x["V"], queries=x.get("Q"))
            out = torch.empty_like(x["K"]) if spec.with_queries else None
            loss = None
        elif isinstance(spec, wl.LinearSpec):
            x = wl.linear_inputs(spec, device=device)
            cfg = cwl.config("linear", batch=spec.B, heads=spec.H, chunk=spec.b, eta=spec.eta,
                             gate_enable=int(spec.gate))
            self.state = cwl.FastWeightState(cfg, x["W0"])
            args = dict(keys=x["K"], targets=x["V"], queries=x.get("Q"))
            out = torch.empty_like(x["K"]) if spec.with_queries else None
            loss = (torch.empty((spec.B, spec.H, spec.T), device=device, dtype=torch.float32)
                    if spec.gate else None)
        else:
            x = wl.inplace_inputs(spec, device=device)
            io = 0 if spec.dtype == "f32" else 1
            cfg = cwl.config("inplace", io_dtype=io, d_key=spec.f, d_val=spec.d, chunk=spec.C, eta=spec.eta,
                             target_mode=int(spec.target), conv_pad_mode=spec.conv_pad_mode)
            self.state = cwl.FastWeightState(cfg, x["W0"], x.get("Wtarget"), x.get("convw"))
            if prefix:
                self.state.set_option(cwl.abi.TTT_OPT_INPLACE_PREFIX, 1)
            args = dict(keys=x["Z"], targets=x["X0"] if spec.target else x["Vhat"], queries=None)
            out = torch.empty((spec.T, spec.d), device=device, dtype=x["Z"].dtype)
            loss = None
        self.inputs = x
        step_bytes = work(spec)["bytes"]
        self.n_sets = max(1, -(-3 * L2_BYTES // step_bytes))
        clone = lambda t: None if t is None else t.clone()  # noqa: E731
        self.sets = [(args, out, loss)] + [
            ({k: clone(v) for k, v in args.items()}, clone(out), clone(loss)) for _ in range(self.n_sets - 1)]
        self.args, self.out, self.loss = self.sets[0]
        self.set_bytes = self.n_sets * step_bytes

    def step(self, i=0):
        a, out, loss = self.sets[i % self.n_sets]
        self.state.chunk_scan(a["keys"], a["targets"], a["queries"], out=out, loss_out=loss, T=self.spec.T)

    def host_buffers(self):
        pin = lambda t: None if t is None else t.cpu().pin_memory()  # noqa: E731
        h = {k: pin(v) for k, v in self.args.items()}
        h["out"] = None if self.out is None else torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        h["loss"] = None if self.loss is None else torch.empty(self.loss.shape, dtype=torch.float32).pin_memory()
        return h

    def l2_note(self):
        return (f"inputs larger than L2: {self.n_sets} copies of the step's inputs and outputs "
                f"({self.set_bytes / 2**20:.0f} MiB in all) taken in turn, so each step reads from HBM")


def timed_pass(runner, steps, stream):
    """EXACTLY ``steps`` back-to-back steps between two CUDA events on the launching stream
    (synchronised on both sides): total ms and library launches. A second pass with an event
    between every two steps gives the per-step times (for the median); it is not the value."""
    torch.cuda.synchronize()
    n0 = runner.state.launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h0 = time.perf_counter()
    for k in range(steps):
        runner.step(k)
    runner.host_ms = (time.perf_counter() - h0) * 1e3 / max(1, steps)  # host time to enqueue one step
    e1.record(stream)
    e1.synchronize()
    total = e0.elapsed_time(e1)
    launches = runner.state.launch_count() - n0
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for k in range(steps):
        runner.step(k)
        ev[k + 1].record(stream)
    ev[-1].synchronize()
    per_step = [ev[k].elapsed_time(ev[k + 1]) for k in range(steps)]
    torch.cuda.synchronize()
    return total, launches, per_step


def time_steps(runner, steps, warmup):
    stream = torch.cuda.current_stream()
    runner.state.reset()
    for k in range(warmup):
        runner.step(k)
    torch.cuda.synchronize()
    runner.state.poll()
    total, launches, per_step = timed_pass(runner, steps, stream)
    runner.state.poll()
    return total, launches, per_step


def time_e2e(runner, steps, warmup):
    h = runner.host_buffers()
    st = runner.state

    def once():
        st.reset()
        st.chunk_scan_host(h["keys"], h["targets"], h["queries"], out=h["out"], loss_out=h["loss"], T=runner.spec.T)

    for _ in range(max(1, warmup)):
        once()
    torch.cuda.synchronize()
    t = []
    for _ in range(steps):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        once()
        e1.record()
        e1.synchronize()
        t.append(e0.elapsed_time(e1))
    h2d = sum(v.numel() * v.element_size() for k, v in h.items() if k in ("keys", "targets", "queries") and v is not None)
    d2h = sum(v.numel() * v.element_size() for k, v in h.items() if k in ("out", "loss") and v is not None)
    return statistics.mean(t), h2d, d2h


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 50 ms from before the main workload's
    warm-up steps (so through its timed region) until every workload has been measured."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, max_mhz):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": max_mhz, "reasons": ["unsampled"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": max_mhz, "reasons": ["unsampled"]}
        mhz = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(mhz) if mhz else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else max_mhz,
                "reasons": reasons, "samples": len(rows)}


def dominant_kernel(spec) -> str:
    if isinstance(spec, wl.InnerSpec):
        return "k_inner_ln" if spec.model == "linear_ln" else "k_inner_mlp"
    if isinstance(spec, wl.LinearSpec):
        return "k_linear_b16" if spec.b == 16 else "k_linear_scan"
    return "k_f32_chunk" if spec.dtype == "f32" else "k_inplace_tc"


def traffic_per_launch(spec):
    """DRAM bytes per step of the workload's dominant kernel (its bytes per launch times its
    launches per step) from the committed ncu record, or None when there is none or the
    kernel's source changed since the capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(f"{dominant_kernel(spec)}@{spec.name.split('@')[0]}")
    if rec is None:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src):
        return None
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    if not digest.startswith(rec["sha256_prefix"]):
        return None
    return rec["bytes_per_launch"] * rec.get("launches_per_step", 1)


def recorded_traffic(key, chunks=None):
    """DRAM bytes per step of a further form's dominant kernel from the committed ncu record
    ``key`` (kernel@line): per padded chunk times ``chunks`` when the record was captured on a
    smaller case, else its bytes per launch times launches per step; None when there is no
    record or the kernel's source changed since the capture."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(key)
    if rec is None:
        return None
    src = os.path.join(ROOT, rec["source"])
    if not os.path.exists(src) or not hashlib.sha256(open(src, "rb").read()).hexdigest().startswith(rec["sha256_prefix"]):
        return None
    if "bytes_per_chunk" in rec:
        return None if chunks is None else rec["bytes_per_chunk"] * chunks
    return rec["bytes_per_launch"] * rec.get("launches_per_step", 1)


def padded_chunks(T, C, starts):
    """Chunks of a packed layout with every document padded to whole chunks."""
    ends = starts[1:] + [T]
    return sum(-(-(e - a) // C) for a, e in zip(starts, ends))


SUSTAINED_MS = 50.0  # a timed region at least this long runs in the power-capped regime


def roofline(spec, w, ms, peaks, traffic=None, timed_ms=0.0):
    """Roofline object of the dominant kernel. A tensor-bound kernel is compared with the burst
    bf16 peak when its timed region is short and with the sustained one (the same GEMM held for
    seconds under the power cap) when the K back-to-back steps run for SUSTAINED_MS or longer;
    both fractions are reported."""
    if w["bound"] == "hbm":
        achieved = w["bytes"] / (ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peaks["source"]}
    if w["bound"] == "tensor":
        achieved = w["flops"] / (ms * 1e-3) / 1e12
        sustained = timed_ms >= SUSTAINED_MS
        peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic, "peak_source": peaks["source"],
                "peak_kind": (f"sustained (the {timed_ms:.0f} ms timed region runs back to back under the power cap)"
                              if sustained else f"burst (a {timed_ms:.1f} ms timed region)"),
                "frac_of_burst": achieved / peaks["bf16_tflops"],
                "frac_of_sustained": achieved / peaks["bf16_tflops_sustained"]}
    achieved = w["flops"] / (ms * 1e-3) / 1e12
    peak = fp32_alu_peak_tflops(peaks)
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
            "traffic": traffic, "peak_source": "148 SMs x 128 FP32 lanes x 2 x max SM clock"}


def oracle_threads() -> int:
    """Threads of the BLAS pool behind numpy's matmul, the oracle's only multi-threaded step."""
    try:
        import threadpoolctl
        n = [i["num_threads"] for i in threadpoolctl.threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


@functools.lru_cache(maxsize=2)
def _host_inputs(spec):
    """The inputs a CPU baseline sample reads, made once per workload (the reference arm takes
    many samples of the same workload): the generator's tensors on the host, and for the
    In-Place workloads their first two chunks with the targets the oracle makes from X0."""
    from oracle import inplace as oinp
    if isinstance(spec, wl.InnerSpec):
        return wl.inner_inputs(spec)
    if isinstance(spec, wl.LinearSpec):
        return wl.linear_inputs(spec)
    x = wl.inplace_inputs(wl.scaled(spec, T=min(spec.T, spec.C * 2)) if spec.dtype == "bf16" else spec)
    if x.get("Vhat") is None:
        x["Vhat"] = torch.from_numpy(oinp.target_values(x["X0"], x["convw"], x["Wtarget"], spec.C))
    return x


def cpu_baseline(spec, limit_s=12.0, prefix=False) -> dict:
    """The oracle as it stands on this host's cores, on a bounded sample of the workload.

    ``cores`` is the BLAS pool the oracle's matmuls run on; ``busy_threads`` is the process's
    CPU time over the sample's wall time, i.e. how many of them were busy on average."""
    import numpy as np  # noqa: F401
    from oracle import gate as ogate
    from oracle import inner as oinn
    from oracle import inplace as oinp
    from oracle import linear as olin
    cores = oracle_threads()
    t0, c0 = time.perf_counter(), time.process_time()
    if isinstance(spec, wl.InnerSpec):
        x = _host_inputs(spec)
        BH = spec.B * spec.H
        K, V, Q = (x[k].reshape(BH, 1, spec.T, spec.D) for k in "KVQ")
        g, be = x["gamma"], x["beta"]
        done_heads = 0
        t0, c0 = time.perf_counter(), time.process_time()
        while done_heads < BH and time.perf_counter() - t0 < limit_s:
            h = done_heads
            hs = slice(h, h + 1)
            gh, bh_ = g[h % spec.H:h % spec.H + 1], be[h % spec.H:h % spec.H + 1]
            if spec.model == "linear_ln":
                oinn.ttt_linear_ln_scan(K[hs], V[hs], Q[hs], x["W0"].reshape(BH, 1, spec.D, spec.D)[hs], gh, bh_,
                                        spec.eta, spec.b, spec.eps, token_weights=spec.token_weights)
            else:
                oinn.ttt_mlp_scan(K[hs], V[hs], Q[hs], x["W1"].reshape(BH, 1, spec.D, spec.hidden)[hs],
                                  x["W2"].reshape(BH, 1, spec.hidden, spec.D)[hs], gh, bh_, spec.eta, spec.b, spec.eps,
                                  token_weights=spec.token_weights)
            done_heads += 1
        dt = time.perf_counter() - t0
        tokens = spec.T * done_heads / spec.H
        sample = f"{done_heads} of {BH} (sequence, head) scans, one at a time"
    elif isinstance(spec, wl.LinearSpec):
        x = _host_inputs(spec)
        done_heads = 0
        BH = spec.B * spec.H
        K = x["K"].reshape(BH, 1, spec.T, spec.D)
        V = x["V"].reshape(BH, 1, spec.T, spec.D)
        Q = x["Q"].reshape(BH, 1, spec.T, spec.D) if "Q" in x else None
        W0 = x["W0"].reshape(BH, 1, spec.D, spec.D)
        t0, c0 = time.perf_counter(), time.process_time()
        while done_heads < BH and time.perf_counter() - t0 < limit_s:
            h = done_heads
            _, _, L = olin.ttt_linear_scan(K[h:h + 1], V[h:h + 1], None if Q is None else Q[h:h + 1],
                                          W0[h:h + 1], spec.eta, spec.b)
            if spec.gate:
                ogate.surprisal_route(L.astype("float32"), ogate.GateState(1, 1))
            done_heads += 1
        dt = time.perf_counter() - t0
        tokens = spec.T * done_heads / spec.H
        sample = f"{done_heads} of {BH} (sequence, head) scans, one at a time"
    else:
        Cs = spec.C
        x = _host_inputs(spec)
        t0, c0 = time.perf_counter(), time.process_time()
        chunks = 0
        W = x["W0"]
        Vh = x["Vhat"]
        T = x["Z"].shape[0]
        scan_fn = oinp.inplace_scan_prefix if prefix else oinp.inplace_scan
        while time.perf_counter() - t0 < limit_s and chunks * Cs < T:
            sl = slice(chunks * Cs, (chunks + 1) * Cs)
            _, W = scan_fn(x["Z"][sl], Vh[sl], W, spec.eta, Cs)
            chunks += 1
        dt = time.perf_counter() - t0
        tokens = chunks * Cs
        sample = f"{chunks} chunk(s) of {Cs} tokens"
    busy = (time.process_time() - c0) / dt if dt > 0 else 0.0
    return {"value": tokens / dt, "unit": "tokens/s", "cores": cores, "busy_threads": round(busy, 2),
            "kind": "oracle", "sample": sample, "seconds": dt}


def measure(spec, steps, warmup, peaks, device, with_e2e, cpu_limit_s=None, prefix=False):
    """One workload measured like the main line: device time per scan (mean over the timed
    steps, median beside it), its roofline, end-to-end time through the host-buffer call, and
    (with ``cpu_limit_s``) the oracle on a bounded sample of it."""
    r = Runner(spec, device, prefix=prefix)
    total, launches, times = time_steps(r, steps, warmup)
    ms = total / steps
    w = work(spec)
    rl = roofline(spec, w, ms, peaks, traffic_per_launch(spec), timed_ms=total)
    rl["kernel"] = "k_gemm_tc" if prefix else dominant_kernel(spec)
    if prefix:
        # The two GEMM launches of a step, from a capture on fewer chunks (every chunk moves the
        # same data).
        rl["traffic"] = recorded_traffic(f"k_gemm_tc@{spec.name} (context-parallel form)", spec.T // spec.C)
    out = {"workload": spec.name + (" (context-parallel form)" if prefix else ""), "ms_per_step": ms, "ms_median": statistics.median(times),
           "tokens_per_s": w["tokens"] / (ms * 1e-3), "tflops": w["flops"] / (ms * 1e-3) / 1e12,
           "roofline": rl, "gpu_launches_per_step": launches / max(1, steps), "times_ms": times,
           "host_ms_per_step": r.host_ms, "l2": r.l2_note()}
    if with_e2e:
        try:
            e2e_ms, h2d, d2h = time_e2e(r, max(3, min(steps, 10) // 2), 1)
            out["e2e"] = {"value": w["tokens"] / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                          "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
        except Exception as ex:  # report, do not hide
            out["e2e"] = {"error": str(ex)}
    r.state.close()
    del r
    torch.cuda.empty_cache()
    if cpu_limit_s is not None:
        out["cpu_baseline"] = cpu_baseline(spec, cpu_limit_s)
    return out


CACHE_READ = "srttt_cache_read_B4_H16_T8192"


def _cache_read_setup(device):
    """A gated scan of the SR-TTT workload with queries drawn as well (its cache is what the read
    path reads), and a gate vector α."""
    import chunked_weight_layers_b200 as cwl
    spec = wl.scaled(wl.SR_TTT_GATE, with_queries=True)
    x = wl.linear_inputs(spec, device=device)
    cfg = cwl.config("linear", batch=spec.B, heads=spec.H, chunk=spec.b, eta=spec.eta, gate_enable=1)
    st = cwl.FastWeightState(cfg, x["W0"])
    O = torch.empty_like(x["K"])
    st.chunk_scan(x["K"], x["V"], x["Q"], out=O, loss_out=torch.empty((spec.B, spec.H, spec.T), device=device))
    alpha = torch.full((spec.H, 64), 0.25, device=device)
    return spec, x, st, O, alpha


def cache_read_work(spec, counts, entries) -> dict:
    """Bytes (Q and o_ttt read, out written, cached K and V rows gathered per query block) and
    flops (4·64 per query and visible entry, for Q·Kᵀ and P·V) of one read-path call."""
    n = spec.B * spec.H * spec.T * 64
    flops, gathered = 0, 0
    E = entries.cpu().numpy()
    C = counts.cpu().numpy()
    for b in range(spec.B):
        for h in range(spec.H):
            m = min(int(C[b, h, 0]), E.shape[2])
            toks = E[b, h, :m, 2]
            for g in range(spec.T // 64):
                vis = int((toks < 64 * g).sum())
                flops += 4 * 64 * 64 * vis
                gathered += 2 * vis * 128
    return {"tokens": spec.B * spec.T, "flops": flops, "bytes": 3 * n * 2 + gathered, "bound": "hbm"}


def measure_cache_read(steps, warmup, peaks, device):
    spec, x, st, O, alpha = _cache_read_setup(device)
    E = torch.empty((spec.B, spec.H, 256, 3), device=device, dtype=torch.int32)
    C = torch.empty((spec.B, spec.H, 2), device=device, dtype=torch.int32)
    st.cache_read(E, C)
    w = cache_read_work(spec, C, E)
    n_sets = max(1, -(-3 * L2_BYTES // w["bytes"]))
    sets = [(x["Q"], O, torch.empty_like(O))] + [(x["Q"].clone(), O.clone(), torch.empty_like(O))
                                                 for _ in range(n_sets - 1)]
    stream = torch.cuda.current_stream()
    for k in range(warmup):
        q, o, out = sets[k % n_sets]
        st.cache_attention(q, x["K"], x["V"], o, alpha, out=out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    h0 = time.perf_counter()
    for k in range(steps):
        q, o, out = sets[k % n_sets]
        st.cache_attention(q, x["K"], x["V"], o, alpha, out=out)
    host_ms = (time.perf_counter() - h0) * 1e3 / steps
    e1.record(stream)
    e1.synchronize()
    st.poll()
    ms = e0.elapsed_time(e1) / steps
    achieved = w["bytes"] / (ms * 1e-3) / 1e9
    # End to end: the call's inputs (queries, keys, values, the scan's outputs, α) from pinned host
    # memory, the call, its outputs back.
    hin = [t.cpu().pin_memory() for t in (x["Q"], x["K"], x["V"], O, alpha)]
    din = [torch.empty_like(t) for t in (x["Q"], x["K"], x["V"], O, alpha)]
    hout = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    dout = torch.empty_like(O)
    e2e = []
    for _ in range(3):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for d, h in zip(din, hin):
            d.copy_(h, non_blocking=True)
        st.cache_attention(din[0], din[1], din[2], din[3], din[4], out=dout)
        hout.copy_(dout, non_blocking=True)
        torch.cuda.synchronize()
        e2e.append((time.perf_counter() - t0) * 1e3)
    e2e_ms = statistics.median(e2e)
    out = {"workload": CACHE_READ, "ms_per_step": ms, "tokens_per_s": w["tokens"] / (ms * 1e-3),
           "tflops": w["flops"] / (ms * 1e-3) / 1e12,
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": achieved / peaks["hbm_gbs"], "traffic": recorded_traffic("k_cache_attn@" + CACHE_READ),
                        "peak_source": peaks["source"], "kernel": "k_cache_attn",
                        "tensor_frac": w["flops"] / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"]},
           "gpu_launches_per_step": 1.0, "host_ms_per_step": host_ms,
           "l2": f"inputs larger than L2: {n_sets} copies of the call's queries and outputs taken in turn",
           "e2e": {"value": w["tokens"] / (e2e_ms * 1e-3), "unit": "tokens/s",
                   "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hin),
                   "d2h_bytes_per_step": hout.numel() * hout.element_size(), "ms_per_step": e2e_ms,
                   "note": "through ttt_cache_attention with its inputs copied from pinned host memory"}}
    st.close()
    torch.cuda.empty_cache()
    return out


DOCS = wl.INPLACE_4B.name + " packed (7 documents, clipped)"
DOCS_SEED, DOCS_N, DOCS_CLIP = 1006, 7, 1.0


def measure_docs(steps, warmup, peaks, device):
    """ttt_chunk_scan_docs on the 4B-class widths: T=32768 tokens as seven documents of seeded
    ragged lengths, every chunk delta clipped to Frobenius norm 1.0. Work counts the real tokens
    only (the padding that fills each document's last chunk is overhead)."""
    import chunked_weight_layers_b200 as cwl
    spec = wl.INPLACE_4B
    starts = wl.document_starts(spec.T, DOCS_N, DOCS_SEED)
    x = wl.inplace_inputs(spec, device=device)
    cfg = cwl.config("inplace", io_dtype=1, d_key=spec.f, d_val=spec.d, chunk=spec.C, eta=spec.eta)
    st = cwl.FastWeightState(cfg, x["W0"])
    O = torch.empty((spec.T, spec.d), device=device, dtype=torch.bfloat16)
    w = work(spec)
    for _ in range(warmup):
        st.chunk_scan_docs(x["Z"], x["Vhat"], starts, clip=DOCS_CLIP, out=O)
    torch.cuda.synchronize()
    n0 = st.launch_count()
    stream = torch.cuda.current_stream()
    times = []
    for _ in range(steps):  # the call synchronises (its layout goes up from host memory): time each
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        st.chunk_scan_docs(x["Z"], x["Vhat"], starts, clip=DOCS_CLIP, out=O)
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    st.poll()
    launches = (st.launch_count() - n0) / steps
    ms = sum(times) / steps
    tf = w["flops"] / (ms * 1e-3) / 1e12
    # End to end: the inputs from pinned host memory, the call, the outputs back.
    hz, hv = x["Z"].cpu().pin_memory(), x["Vhat"].cpu().pin_memory()
    ho = torch.empty((spec.T, spec.d), dtype=torch.bfloat16).pin_memory()
    dz, dv = torch.empty_like(x["Z"]), torch.empty_like(x["Vhat"])
    e2e = []
    for k in range(3):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        dz.copy_(hz, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        st.chunk_scan_docs(dz, dv, starts, clip=DOCS_CLIP, out=O)
        ho.copy_(O, non_blocking=True)
        torch.cuda.synchronize()
        e2e.append((time.perf_counter() - t0) * 1e3)
    e2e_ms = statistics.median(e2e)
    out = {"workload": DOCS, "doc_starts": starts, "clip_norm": DOCS_CLIP, "ms_per_step": ms,
           "ms_median": statistics.median(times), "tokens_per_s": w["tokens"] / (ms * 1e-3), "tflops": tf,
           "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": tf / peaks["bf16_tflops"],
                        "traffic": recorded_traffic("k_gemm_tc@" + DOCS, padded_chunks(spec.T, spec.C, starts)),
                        "peak_source": peaks["source"], "kernel": "k_gemm_tc",
                        "peak_kind": "burst (each call timed alone: it synchronises to upload its layout)"},
           "gpu_launches_per_step": launches, "times_ms": times,
           "l2": "inputs larger than L2 (the 4B-class Z alone is 637 MB)",
           "e2e": {"value": w["tokens"] / (e2e_ms * 1e-3), "unit": "tokens/s",
                   "h2d_bytes_per_step": hz.numel() * 2 + hv.numel() * 2, "d2h_bytes_per_step": ho.numel() * 2,
                   "ms_per_step": e2e_ms}}
    st.close()
    del x, O, dz, dv
    torch.cuda.empty_cache()
    return out


def cpu_baseline_docs(limit_s) -> dict:
    """The oracle's packed scan (resets and clipping) on the first chunks of the measured
    layout's first document, within the time limit."""
    from oracle import packed as opk
    spec = wl.INPLACE_4B
    x = wl.inplace_inputs(wl.scaled(spec, T=spec.C * 2))
    cores = oracle_threads()
    t0, c0 = time.perf_counter(), time.process_time()
    chunks = 0
    while time.perf_counter() - t0 < limit_s and chunks < 2:
        sl = slice(chunks * spec.C, (chunks + 1) * spec.C)
        opk.inplace_scan_docs(x["Z"][sl], x["Vhat"][sl], x["W0"], spec.eta, spec.C, [0], DOCS_CLIP)
        chunks += 1
    dt = time.perf_counter() - t0
    busy = (time.process_time() - c0) / dt if dt > 0 else 0.0
    return {"value": chunks * spec.C / dt, "unit": "tokens/s", "cores": cores, "busy_threads": round(busy, 2),
            "kind": "oracle", "sample": f"{chunks} chunk(s) of {spec.C} tokens (one document, clipped)", "seconds": dt}


PACKED = wl.LINEAR_GD.name + " packed (4 documents per sequence)"
PACKED_SEED, PACKED_N = 1009, 4


def packed_starts(spec):
    """Seeded ragged document starts of every sequence (at least 16 tokens a document)."""
    return [wl.document_starts(spec.T, PACKED_N, PACKED_SEED + b, min_len=16) for b in range(spec.B)]


def measure_packed(steps, warmup, peaks, device):
    """ttt_chunk_scan_packed on the TTT-Linear workload: every sequence as four documents of seeded
    ragged lengths, each scanned from W0 with its own mini-batches (a shorter last one). The
    scan runs in the LayerNorm kernel's plain mode over a padded copy, with gather and scatter
    launches around it; work counts the real tokens."""
    import chunked_weight_layers_b200 as cwl
    spec = wl.LINEAR_GD
    starts = packed_starts(spec)
    x = wl.linear_inputs(spec, device=device)
    cfg = cwl.config("linear", batch=spec.B, heads=spec.H, chunk=spec.b, eta=spec.eta)
    st = cwl.FastWeightState(cfg, x["W0"])
    O = torch.empty_like(x["K"])
    w = work(spec)
    for _ in range(warmup):
        st.chunk_scan_packed(x["K"], x["V"], starts, queries=x["Q"], out=O)
    torch.cuda.synchronize()
    n0 = st.launch_count()
    stream = torch.cuda.current_stream()
    times = []
    for _ in range(steps):  # the call synchronises (its layout goes up from host memory): time each
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        st.chunk_scan_packed(x["K"], x["V"], starts, queries=x["Q"], out=O)
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    st.poll()
    launches = (st.launch_count() - n0) / steps
    ms = sum(times) / steps
    achieved = w["bytes"] / (ms * 1e-3) / 1e9
    hk, hv, hq = (x[k].cpu().pin_memory() for k in "KVQ")
    ho = torch.empty(O.shape, dtype=O.dtype).pin_memory()
    dk, dv, dq = torch.empty_like(x["K"]), torch.empty_like(x["V"]), torch.empty_like(x["Q"])
    e2e = []
    for _ in range(3):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        dq.copy_(hq, non_blocking=True)
        st.chunk_scan_packed(dk, dv, starts, queries=dq, out=O)
        ho.copy_(O, non_blocking=True)
        torch.cuda.synchronize()
        e2e.append((time.perf_counter() - t0) * 1e3)
    e2e_ms = statistics.median(e2e)
    out = {"workload": PACKED, "doc_starts": starts, "ms_per_step": ms, "ms_median": statistics.median(times),
           "tokens_per_s": w["tokens"] / (ms * 1e-3), "tflops": w["flops"] / (ms * 1e-3) / 1e12,
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": achieved / peaks["hbm_gbs"], "traffic": recorded_traffic("k_inner_ln@" + PACKED),
                        "peak_source": peaks["source"], "kernel": "k_inner_ln (plain mode)"},
           "gpu_launches_per_step": launches, "times_ms": times,
           "l2": "each call timed alone (it synchronises to upload its layout); its 100 MB of inputs are gathered into a padded copy",
           "e2e": {"value": w["tokens"] / (e2e_ms * 1e-3), "unit": "tokens/s",
                   "h2d_bytes_per_step": 3 * hk.numel() * 2, "d2h_bytes_per_step": ho.numel() * 2,
                   "ms_per_step": e2e_ms}}
    st.close()
    del x, O, dk, dv, dq
    torch.cuda.empty_cache()
    return out


def cpu_baseline_packed(limit_s) -> dict:
    """The oracle's packed TTT-Linear scan, one (sequence, head) at a time, within the limit."""
    from oracle import packed as opk
    spec = wl.LINEAR_GD
    starts = packed_starts(spec)
    x = wl.linear_inputs(spec)
    cores = oracle_threads()
    t0, c0 = time.perf_counter(), time.process_time()
    done = 0
    while done < spec.B * spec.H and time.perf_counter() - t0 < limit_s:
        b, h = divmod(done, spec.H)
        sl = (slice(b, b + 1), slice(h, h + 1))
        opk.ttt_linear_scan_docs(x["K"][sl], x["V"][sl], x["Q"][sl], x["W0"][sl], spec.eta, spec.b, [starts[b]])
        done += 1
    dt = time.perf_counter() - t0
    busy = (time.process_time() - c0) / dt if dt > 0 else 0.0
    return {"value": spec.T * done / spec.H / dt, "unit": "tokens/s", "cores": cores, "busy_threads": round(busy, 2),
            "kind": "oracle", "sample": f"{done} of {spec.B * spec.H} (sequence, head) scans, one at a time",
            "seconds": dt}


def cpu_baseline_cache_read(limit_s) -> dict:
    """The oracle's read path (attention over the visible entries, α fusion) on (sequence, head)
    pairs of the gate workload's cache, one at a time, within the time limit."""
    from oracle import cache_attention as oca
    from oracle import gate as ogate
    from oracle import linear as olin
    spec = wl.scaled(wl.SR_TTT_GATE, with_queries=True)
    x = wl.linear_inputs(spec)
    cores = oracle_threads()
    t0, c0 = time.perf_counter(), time.process_time()
    done = 0
    for h in range(spec.H):
        if time.perf_counter() - t0 >= limit_s:
            break
        sl = (slice(0, 1), slice(h, h + 1))
        K, V, Q = x["K"][sl], x["V"][sl], x["Q"][sl]
        O, _, L = olin.ttt_linear_scan(K, V, Q, x["W0"][sl], spec.eta, spec.b)
        gs = ogate.GateState(1, 1)
        ogate.surprisal_route(L.astype("float32"), gs)
        A = oca.cache_attention(Q, K, V, gs.entries, gs.counts())
        oca.alpha_fusion(O, A, torch.full((1, 64), 0.25).numpy())
        done += 1
    dt = time.perf_counter() - t0
    busy = (time.process_time() - c0) / dt if dt > 0 else 0.0
    return {"value": spec.T * done / spec.H / dt, "unit": "tokens/s", "cores": cores, "busy_threads": round(busy, 2),
            "kind": "oracle", "sample": f"{done} of {spec.B * spec.H} (sequence, head) pairs: scan, gate and read path",
            "seconds": dt}


def run_row_sharded(spec, a, world, rank, local, peaks):
    """One In-Place layer split over the ranks, strong scaling: value = T / the slowest rank's
    time per step. ``--shard rows`` (RowShardedInplace): every rank holds the whole Z and V̂
    (same seed) and its rows of W; a step is one scan of the T tokens plus the all-gather of the
    output columns. ``--shard sequence`` (SequenceShardedInplace, the context-parallel form
    across devices): every rank holds its own run of whole chunks of Z and V̂ and the whole W; a
    step is its two scans of those chunks plus the all-gather of the ranks' delta sums, and its
    outputs stay on the rank."""
    import datetime

    import torch.distributed as dist
    from chunked_weight_layers_b200 import build
    from chunked_weight_layers_b200.dist import RowShardedInplace, SequenceShardedInplace, max_over_ranks, shard_range
    if not isinstance(spec, wl.InplaceSpec) or spec.target or spec.dtype != "bf16":
        raise SystemExit(f"--shard {a.shard} takes an In-Place bf16 workload with given targets")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    import chunked_weight_layers_b200 as cwl
    x = wl.inplace_inputs(spec, device=device)
    cfg = cwl.config("inplace", io_dtype=1, d_key=spec.f, d_val=spec.d, chunk=spec.C, eta=spec.eta)
    if a.shard == "rows":
        layer = RowShardedInplace(cfg, x["W0"])
    else:
        c0, c1 = shard_range(spec.T // spec.C, rank, world)
        x["Z"], x["Vhat"] = x["Z"][c0 * spec.C:c1 * spec.C].contiguous(), x["Vhat"][c0 * spec.C:c1 * spec.C].contiguous()
        layer = SequenceShardedInplace(cfg, x["W0"])
    for _ in range(a.warmup):
        layer.scan(x["Z"], x["Vhat"])
    torch.cuda.synchronize()
    layer.state.poll()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    clk = ClockSampler(local)
    clk.__enter__()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = layer.state.launch_count()
    e0.record(stream)
    for _ in range(a.steps):
        layer.scan(x["Z"], x["Vhat"])
    e1.record(stream)
    e1.synchronize()
    launches = layer.state.launch_count() - n0
    if world > 1:
        dist.barrier()
    clk.__exit__(None, None, None)
    layer.state.poll()
    ms = max_over_ranks(e0.elapsed_time(e1), device) / a.steps
    w = work(spec)
    # End to end: inputs copied from pinned host memory, the sharded scan, the gathered output read back.
    hZ, hV = x["Z"].cpu().pin_memory(), x["Vhat"].cpu().pin_memory()
    hO = torch.empty((x["Z"].shape[0] if a.shard == "sequence" else spec.T, spec.d), dtype=torch.bfloat16).pin_memory()
    t = []
    for k in range(3):
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record()
        layer.reset()
        O = layer.scan(hZ.to(device, non_blocking=True), hV.to(device, non_blocking=True))
        hO.copy_(O, non_blocking=True)
        f1.record()
        f1.synchronize()
        t.append(f0.elapsed_time(f1))
    e2e_ms = max_over_ranks(statistics.mean(t), device)
    if rank == 0:
        rl = roofline(spec, w, ms, peaks, None, timed_ms=ms * a.steps)
        rl["kernel"] = dominant_kernel(spec)
        print(json.dumps({
            "metric": METRIC, "value": w["tokens"] / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(bench_config(spec, world), parallelism=f"{'rows' if a.shard == 'rows' else 'sequence'}{world}",
                           l2="inputs larger than L2 (one step moves over 1 GB)"),
            "tflops": w["flops"] / (ms * 1e-3) / 1e12, "roofline": rl,
            "e2e": {"value": w["tokens"] / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": (hZ.numel() + hV.numel()) * 2, "d2h_bytes_per_step": hO.numel() * 2,
                    "ms_per_step": e2e_ms},
            "gpu_launches": launches, "clocks": clk.summary(peaks["sm_max_mhz"])}))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def profile_form(form, spec, device, calls):
    """``calls`` calls of a further form (for profilers): the packed In-Place scan on the In-Place
    workload ``spec`` (its seeded document layout for spec.T tokens), the cache read path on the
    gate workload's cache, or packed TTT-Linear on the TTT-Linear workload."""
    import chunked_weight_layers_b200 as cwl
    if form == "docs":
        starts = wl.document_starts(spec.T, DOCS_N, DOCS_SEED)
        x = wl.inplace_inputs(spec, device=device)
        st = cwl.FastWeightState(cwl.config("inplace", io_dtype=1, d_key=spec.f, d_val=spec.d, chunk=spec.C,
                                            eta=spec.eta), x["W0"])
        O = torch.empty((spec.T, spec.d), device=device, dtype=torch.bfloat16)
        for _ in range(calls):
            st.chunk_scan_docs(x["Z"], x["Vhat"], starts, clip=DOCS_CLIP, out=O)
        print(f"profiled {spec.name} packed: {calls} calls, {padded_chunks(spec.T, spec.C, starts)} padded chunks")
    elif form == "cache_read":
        spec_c, x, st, O, alpha = _cache_read_setup(device)
        out = torch.empty_like(O)
        for _ in range(calls):
            st.cache_attention(x["Q"], x["K"], x["V"], O, alpha, out=out)
        print(f"profiled {CACHE_READ}: {calls} calls")
    else:
        spec_p = wl.LINEAR_GD
        starts = packed_starts(spec_p)
        x = wl.linear_inputs(spec_p, device=device)
        st = cwl.FastWeightState(cwl.config("linear", batch=spec_p.B, heads=spec_p.H, chunk=spec_p.b, eta=spec_p.eta),
                                 x["W0"])
        O = torch.empty_like(x["K"])
        for _ in range(calls):
            st.chunk_scan_packed(x["K"], x["V"], starts, queries=x["Q"], out=O)
        print(f"profiled {PACKED}: {calls} calls")
    torch.cuda.synchronize()
    st.poll()


def bench_config(spec, world) -> dict:
    """The workload description both arms report."""
    return {"workload": spec.name, "B": getattr(spec, "B", 1), "H": getattr(spec, "H", 1), "T": spec.T,
            "chunk": getattr(spec, "b", getattr(spec, "C", None)),
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2: copies of the step's inputs taken in turn (over 3x the 126 MB L2)"}


def spec_by_name(name):
    for s in list(wl.WORKLOADS.values()) + list(wl.INNER_WORKLOADS.values()):
        if s.name == name:
            return s
    raise SystemExit(f"unknown workload {name}; choose from {list(wl.WORKLOADS) + list(wl.INNER_WORKLOADS)}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # 500 back-to-back scans of the main workload (~17 ms): long enough that the start-up of the
    # first launches is a small part of the mean and the 50 ms clock samples see the region.
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=MAIN)
    ap.add_argument("--only-main", action="store_true", help="skip the other workloads")
    ap.add_argument("--tokens", type=int, default=None,
                    help="run the named workload with this many tokens instead (same widths and chunk; a smaller "
                         "case for profilers, not a bench line)")
    ap.add_argument("--shard", choices=["replicas", "rows", "sequence"], default="replicas",
                    help="with N ranks: 'replicas' (default) runs an independent copy of the workload per rank "
                         "(weak scaling); 'rows' splits one In-Place layer's Wdown rows over the ranks and "
                         "all-gathers the output columns each step; 'sequence' gives each rank its own chunks of the "
                         "sequence and all-gathers the ranks' delta sums each step (strong scaling; In-Place "
                         "workloads)")
    ap.add_argument("--form", choices=["scan", "prefix", "docs", "cache_read", "packed"], default="scan",
                    help="with --profile: the further form to run (the context-parallel In-Place scan, the packed "
                         "In-Place scan or packed TTT-Linear on the named workload's inputs, the cache read path)")
    ap.add_argument("--profile", type=int, default=None, metavar="N",
                    help="for profilers: build the named workload, run one warm-up step and N more steps, print "
                         "nothing else (no timing, no end-to-end pass, no oracle)")
    a = ap.parse_args()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    spec = spec_by_name(a.workload)
    if a.tokens is not None:
        spec = wl.scaled(spec, T=a.tokens, name=f"{spec.name}@T{a.tokens}")
    if world > 1 and a.shard == "replicas":
        # Weak scaling: every rank scans its own batch of independent problems (its own seed).
        spec = wl.scaled(spec, seed=spec.seed + 7919 * rank)
    w = work(spec)
    peaks = load_peaks()

    if a.impl == "reference":
        # The oracle on the host cores: W untimed and K timed steps, each a bounded sample of
        # the workload sized so the whole run stays within a few minutes; the value is the
        # tokens of the timed samples over their time.
        if rank != 0:
            return
        per_step = max(0.05, min(12.0, 90.0 / max(1, a.steps + a.warmup)))
        for _ in range(a.warmup):
            cpu_baseline(spec, per_step)
        samples = [cpu_baseline(spec, per_step) for _ in range(max(1, a.steps))]
        secs = sum(x["seconds"] for x in samples)
        val = sum(x["value"] * x["seconds"] for x in samples) / secs
        cb = dict(samples[-1])
        cb.update(value=val, seconds=secs,
                  sample=f"{len(samples)} timed steps, each at most {per_step:.1f} s; last: {samples[-1]['sample']}")
        print(json.dumps({"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": a.gpus,
                          "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * secs / len(samples),
                          "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                          "data": "synthetic", "config": bench_config(spec, world), "cpu_baseline": cb,
                          "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}))
        return

    if a.profile is not None:
        torch.cuda.set_device(local)
        from chunked_weight_layers_b200 import build
        build.build()
        device = torch.device("cuda", local)
        if a.form in ("scan", "prefix"):
            runner = Runner(spec, device, prefix=a.form == "prefix")
            runner.state.reset()
            for k in range(1 + a.profile):
                runner.step(k)
            torch.cuda.synchronize()
            runner.state.poll()
            print(f"profiled {spec.name} ({a.form}): 1 + {a.profile} steps, {runner.state.launch_count()} library launches")
            return
        profile_form(a.form, spec, device, 1 + a.profile)
        return

    if a.warmup < 3:
        a.warmup = 3
    if a.shard in ("rows", "sequence"):
        run_row_sharded(spec, a, world, rank, local, peaks)
        return
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
        pg = dist
    from chunked_weight_layers_b200 import build
    if rank == 0:
        build.build()
    if pg is not None:
        pg.barrier()
    runner = Runner(spec, device)
    # The clock sampler starts (and its start-up pause ends) before the warm-up steps, so the
    # GPU comes out of that idle pause through the warm-up rather than inside the timed steps
    # (measured: a 0.3 s idle pause right before 20 timed steps of 33 us read 37 us a step).
    clk = ClockSampler(local)
    clk.__enter__()
    runner.state.reset()
    for k in range(a.warmup):
        runner.step(k)
    torch.cuda.synchronize()
    runner.state.poll()
    stream = torch.cuda.current_stream()
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    total, launches, times = timed_pass(runner, a.steps, stream)
    if pg is not None:
        pg.barrier()
    runner.state.poll()
    l2_note = runner.l2_note()
    host_ms = runner.host_ms
    from chunked_weight_layers_b200.dist import max_over_ranks
    total_ms = max_over_ranks(total, device)
    ms = total_ms / a.steps
    value = world * w["tokens"] / (ms * 1e-3)
    e2e_ms, h2d, d2h = None, 0, 0
    runner_e2e = None
    try:
        e2e_ms, h2d, d2h = time_e2e(runner, max(3, min(a.steps, 100) // 2), 1)
        e2e_ms = max_over_ranks(e2e_ms, device)
        runner_e2e = world * w["tokens"] / (e2e_ms * 1e-3)
    except Exception as ex:  # report, do not hide
        runner_e2e = None
        print(f"e2e measurement failed: {ex}", file=sys.stderr)
    runner.state.close()
    del runner
    torch.cuda.empty_cache()

    # The other workloads, each a full measurement of its own (device time, roofline,
    # end-to-end through the host-buffer call, oracle baseline on a bounded sample). The clock
    # sampler keeps running through them, so its samples cover the whole of the GPU's work.
    extra = {}
    if not a.only_main and world == 1:
        for s in list(wl.WORKLOADS.values()) + list(wl.INNER_WORKLOADS.values()):
            if s.name == spec.name:
                continue
            try:
                extra[s.name] = measure(s, max(5, min(a.steps, 20)), 3, peaks, device, with_e2e=True)
            except Exception as ex:
                extra[s.name] = {"error": str(ex)}
        # The two further forms of the path: the context-parallel In-Place scan on the 4B-class
        # workload, and the residual-cache read path on the gate workload's cache.
        cp_name = wl.INPLACE_4B.name + " (context-parallel form)"
        try:
            extra[cp_name] = measure(wl.INPLACE_4B, max(5, min(a.steps, 20)), 3, peaks, device, with_e2e=True,
                                     prefix=True)
        except Exception as ex:
            extra[cp_name] = {"error": str(ex)}
        try:
            extra[CACHE_READ] = measure_cache_read(max(5, min(a.steps, 20)), 3, peaks, device)
        except Exception as ex:
            extra[CACHE_READ] = {"error": str(ex)}
        try:
            extra[DOCS] = measure_docs(max(3, min(a.steps, 5)), 2, peaks, device)
        except Exception as ex:
            extra[DOCS] = {"error": str(ex)}
        try:
            extra[PACKED] = measure_packed(max(5, min(a.steps, 20)), 3, peaks, device)
        except Exception as ex:
            extra[PACKED] = {"error": str(ex)}
    clk.__exit__(None, None, None)
    # The oracle baselines run after the sampler stops (the GPU idles meanwhile).
    for s in list(wl.WORKLOADS.values()) + list(wl.INNER_WORKLOADS.values()):
        if s.name in extra and "error" not in extra[s.name]:
            extra[s.name]["cpu_baseline"] = cpu_baseline(s, 6.0)
    if "error" not in extra.get(wl.INPLACE_4B.name + " (context-parallel form)", {"error": 1}):
        extra[wl.INPLACE_4B.name + " (context-parallel form)"]["cpu_baseline"] = cpu_baseline(wl.INPLACE_4B, 6.0,
                                                                                               prefix=True)
    if "error" not in extra.get(CACHE_READ, {"error": 1}):
        extra[CACHE_READ]["cpu_baseline"] = cpu_baseline_cache_read(6.0)
    if "error" not in extra.get(DOCS, {"error": 1}):
        extra[DOCS]["cpu_baseline"] = cpu_baseline_docs(6.0)
    if "error" not in extra.get(PACKED, {"error": 1}):
        extra[PACKED]["cpu_baseline"] = cpu_baseline_packed(6.0)

    if rank == 0:
        rl = roofline(spec, w, ms, peaks, traffic_per_launch(spec), timed_ms=total_ms)
        rl["kernel"] = dominant_kernel(spec)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": ms, "ms_median": statistics.median(times),
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(bench_config(spec, world), l2=l2_note),
            "tflops": world * w["flops"] / (ms * 1e-3) / 1e12,
            "roofline": rl,
            "e2e": {"value": runner_e2e, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms},
            "gpu_launches": launches,
            "host_ms_per_step": host_ms,
            "clocks": clk.summary(peaks["sm_max_mhz"]),
        }
        if world == 1:
            line["cpu_baseline"] = cpu_baseline(spec)
        if extra:
            line["workloads"] = extra
        print(json.dumps(line))
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
