#!/usr/bin/env python
"""Benchmark of the CKDA recurrence library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload fwdbwd|kda|fwd|varlen|varlen_fwdbwd|long|long_fwdbwd|
                                decode|decode_multi|prologue]

Default workload (the headline): one step = ckda_chunk_fwd (saving its
per-chunk results for the backward) + ckda_chunk_bwd on B=8, H=16, T=4096,
dk=dv=128, bf16 I/O, fp32 gate and state -- the shape of one 1.3B-model
token-mixer layer.  Inputs are
seeded synthetic tensors (chunked_gated_delta_ckda_b200.workloads), resident
in HBM when the timed region starts; each step streams ~2 GB, more than L2.

At N=1 the default run also times every secondary workload (decode,
multi-token decode, packed documents, the long sequence, forward only, KDA,
the prologue) with fewer steps and its own clock record, in the line's
"secondary" object (--no-secondary: headline only).  Every value is timed
with the library's per-launch profiling off; per-kernel times come from a
separate pass of identical steps.

Prints ONE JSON line (rank 0).  Under torchrun each rank runs its own batch
(weak scaling, no collective on the data path); ``value`` = tokens of all
ranks / the slowest rank's device time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from chunked_gated_delta_ckda_b200 import workloads as W  # noqa: E402

METRIC = "CKDA fwd+bwd tokens/s (H=16,d=128,T=4096,bf16); % tensor/HBM roofline"
METRIC_KDA = "KDA (gate sign +1) fwd+bwd tokens/s (H=16,d=128,T=4096,bf16), same kernels"
METRIC_LONG = "CKDA long-sequence fwd+bwd tokens/s (B=1,T=65536,H=16,d=128,bf16, with S0)"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal

# Algorithmic work per token per head (chunk 64, dk = dv = 128; causal masks
# counted at half; recomputation and padding excluded):
#   forward  139 264 flop, 1666 B (q, k, v bf16; g fp32; sign int8; beta; o)
#   backward 278 528 flop, 2948 B (inputs and dO again; dq, dk, dv, dg, dbeta)
FWD_FLOP, FWD_BYTES = 139264, 1666
BWD_FLOP, BWD_BYTES = 278528, 2948
DECODE_BYTES_PER_NH = 131072 + 1666  # state read + write, per-token inputs and output
# prologue per token-head (bf16 I/O, fp32 gate): forward reads xq, xk, xv 768 +
# a 512 + b 2, writes q, k, v 768 + g 512 + sign 128 + beta 2; backward reads
# the forward's inputs 1282 and dq, dk, dv 768 + dg 512 + dbeta 2, writes
# dxq, dxk, dxv 768 + da 512 + db 2 (the taps' gradients are per channel)
PROLOGUE_FWD_BYTES, PROLOGUE_BWD_BYTES = 2692, 3846

# Which per-unit figure a kernel's roofline uses (the call it implements).
KERNEL_UNITS = {
    "tc_grad": ("bwd", BWD_BYTES, BWD_FLOP),
    "tc_state_bwd": ("bwd", BWD_BYTES, BWD_FLOP),
    "tc_intra": ("fwd", FWD_BYTES, FWD_FLOP),
    "tc_state_fwd": ("fwd", FWD_BYTES, FWD_FLOP),
    "v1_grad": ("bwd", BWD_BYTES, BWD_FLOP),
    "v1_state_bwd": ("bwd", BWD_BYTES, BWD_FLOP),
    "v1_intra": ("fwd", FWD_BYTES, FWD_FLOP),
    "v1_state_fwd": ("fwd", FWD_BYTES, FWD_FLOP),
    "v1_state_fwd_recompute": ("fwd", FWD_BYTES, FWD_FLOP),
    "decode": ("decode", DECODE_BYTES_PER_NH, 0),
}

# DRAM traffic measured by ncu (dram__bytes_read.sum + dram__bytes_write.sum)
# for the kernel as it stands, per chunk-head, keyed by kernel and workload:
# captured on a B=2 launch (inputs still larger than L2), traffic being
# proportional to the chunk-heads a launch processes (profiles/).
NCU_TRAFFIC = {
    ("tc_grad", "layer_fwdbwd_bf16"): (470960896 + 135686912) / (2 * 64 * 16),
}


# ---------------------------------------------------------------------------
# host-side helpers (unit-tested on CPU with gloo)
# ---------------------------------------------------------------------------

def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling)."""
    return base + 1000 * rank


def reduce_max(x: float, world: int) -> float:
    """Slowest rank's value (max over ranks); identity for one process."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(tokens_per_rank: int, world: int, max_ms_per_step: float) -> float:
    """Whole-job throughput: tokens of all ranks per second of the slowest rank."""
    return tokens_per_rank * world / (max_ms_per_step / 1e3)


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=d.get("hbm_gbs", FALLBACK_HBM_GBS),
                    bf16_tflops=d.get("bf16_tflops", FALLBACK_BF16_TFLOPS),
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained", FALLBACK_BF16_TFLOPS),
                    source="measured")
    return dict(hbm_gbs=FALLBACK_HBM_GBS, bf16_tflops=FALLBACK_BF16_TFLOPS,
                bf16_tflops_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        self.dev = device_index
        self.base = 0
        self.extended = False

    def start(self):
        try:
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", sel, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            t0 = time.time()  # the sampler is running before anything is timed
            while self.count() < 1 and time.time() - t0 < 3.0 and self.proc.poll() is None:
                time.sleep(0.01)
        except Exception:
            self.proc = None

    def count(self) -> int:
        try:
            with open(self.path) as f:
                return sum(1 for _ in f)
        except Exception:
            return 0

    def mark(self):
        """The timed region starts: samples before it are not reported."""
        self.base = self.count()

    def keep_loaded(self, step, min_samples=3, max_s=1.5):
        """A timed region shorter than the sampling interval yields too few
        samples: run the same (untimed) step until min_samples have been taken
        since mark(), for at most max_s seconds."""
        if self.proc is None:
            return
        t0 = time.time()
        while self.count() - self.base < min_samples and time.time() - t0 < max_s:
            step()
            torch.cuda.synchronize()
            self.extended = True

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for n, line in enumerate(f):
                parts = [p.strip() for p in line.split(",")]
                if n >= self.base and len(parts) == 7:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows),
                "window": ("the timed region and the identical untimed steps right after it"
                           if self.extended else "the timed region")}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

def _fwdbwd_setup(inp, dev, kda=False):
    from chunked_gated_delta_ckda_b200 import _abi, api
    d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    if kda:  # standard KDA: no sign tensor (every gate sign +1)
        d["sign"] = None
    B, T, H, dk = d["q"].shape
    dv = d["v"].shape[-1]
    NC = (T + 63) // 64
    e = lambda *s, dt: torch.empty(*s, dtype=dt, device=dev)
    io = d["q"].dtype
    buf = dict(o=e(B, T, H, dv, dt=io), ST=e(B, H, dk, dv, dt=torch.float32),
               cs=e(B, H, NC, dk, dv, dt=torch.float32), dq=e(B, T, H, dk, dt=io),
               dk=e(B, T, H, dk, dt=io), dv=e(B, T, H, dv, dt=io),
               dg=e(B, T, H, dk, dt=torch.float32), dbeta=e(B, T, H, dt=io),
               dS0=e(B, H, dk, dv, dt=torch.float32))
    wsf = api.workspace(_abi.CKDA_OP_CHUNK_FWD, B, T, H, dk, dv, device=dev, cache=False)
    wsb = api.workspace(_abi.CKDA_OP_CHUNK_BWD, B, T, H, dk, dv, device=dev, cache=False)
    code = api.io_code(io)
    # the forward hands its per-chunk results (intra-chunk products and the
    # chunk-start states) to the backward (training use); fp32 chunk states
    # are only materialised where there is no saved form
    sv = api.saved_buffer(B, T, H, dk, dv, io, dev)
    cs = None if sv is not None else buf["cs"]

    S0 = d.get("S0")  # (the long-sequence workload starts from a state)

    def step():
        _abi.ckda_chunk_fwd(B, T, H, dk, dv, code, d["q"], d["k"], d["v"], d["g"], d["sign"],
                            d["beta"], S0, buf["o"], buf["ST"], cs, wsf, saved=sv)
        _abi.ckda_chunk_bwd(B, T, H, dk, dv, code, d["q"], d["k"], d["v"], d["g"], d["sign"],
                            d["beta"], S0, d["dO"], None, cs, buf["dq"], buf["dk"],
                            buf["dv"], buf["dg"], buf["dbeta"], buf["dS0"], wsb, saved=sv)
    return d, buf, step


def _time_steps(step, steps, warmup, world):
    import torch.distributed as dist
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s)
    for _ in range(steps):
        step()
    b.record(s)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def _profile_pass(step, steps, world):
    """Per-kernel live times: `steps` identical steps with the library's
    per-launch CUDA events on (the launch stream's own events).  Returns the
    per-kernel (launches, total ms) and this pass's ms per step."""
    from chunked_gated_delta_ckda_b200 import _abi
    _abi.ckda_profile_reset()
    _abi.ckda_profile_enable(True)
    try:
        ms = _time_steps(step, steps, 0, world)
    finally:
        _abi.ckda_profile_enable(False)
    return _abi.ckda_profile_collect(), ms


def run_ours(args, rank, world, local_rank):
    from chunked_gated_delta_ckda_b200 import _abi
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    long_seq = args.workload == "long_fwdbwd"
    wl = W.Workload(**{**W.LONG.__dict__, "name": "long_fwdbwd_bf16", "with_dO": True}) if long_seq \
        else W.LAYER_FWDBWD
    w = W.Workload(**{**wl.__dict__, "seed": rank_seed(wl.seed, rank),
                      "B": args.batch or wl.B})
    inp = W.make(w)
    B, T, H = w.B, w.T, w.H
    tokens = B * T
    kda = args.workload == "kda"
    d, buf, step = _fwdbwd_setup(inp, dev, kda=kda)

    clocks = ClockSampler(local_rank)
    clocks.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # the headline: library profiling off, nothing but the step's own launches
    clocks.mark()
    ms = _time_steps(step, args.steps, 0, world)
    clocks.keep_loaded(step)
    clk = clocks.stop()
    ms_max = reduce_max(ms, world)
    value = aggregate(tokens, world, ms_max)
    # per-kernel breakdown: a separate pass of the same number of identical
    # steps with a CUDA event pair recorded around every launch
    prof, ms_prof = _profile_pass(step, args.steps, world)

    # dominant kernel, timed live with CUDA events on the launch stream
    peaks = measured_peaks()
    total = sum(t for _, t in prof.values())
    kernels = {k: {"launches": n, "ms_per_launch": t / n, "share": t / total if total else None}
               for k, (n, t) in sorted(prof.items(), key=lambda kv: -kv[1][1])}
    top = max(prof.items(), key=lambda kv: kv[1][1])[0] if prof else None
    roof = None
    if top is not None:
        n, t = prof[top]
        unit, bytes_per, _ = KERNEL_UNITS.get(top, ("bwd", BWD_BYTES, BWD_FLOP))
        alg_bytes = bytes_per * B * T * H
        achieved = alg_bytes / (t / n / 1e3) / 1e9
        roof = {"bound": "hbm", "kernel": top, "achieved": achieved, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                "traffic": (NCU_TRAFFIC[(top, w.name)] * B * ((T + 63) // 64) * H
                            if (top, w.name) in NCU_TRAFFIC else None),
                "algorithmic_bytes_per_launch": alg_bytes, "per_unit": "%d B per token-head (%s)" % (bytes_per, unit),
                "peak_source": peaks["source"]}
    # whole step against both roofs
    t_hbm = (FWD_BYTES + BWD_BYTES) * B * T * H / (peaks["hbm_gbs"] * 1e9) * 1e3
    t_tc = (FWD_FLOP + BWD_FLOP) * B * T * H / (peaks["bf16_tflops_sustained"] * 1e12) * 1e3
    step_roof = {"t_hbm_ms": t_hbm, "t_tensor_ms": t_tc, "hbm_frac": t_hbm / ms_max,
                 "tensor_frac": t_tc / ms_max, "binding_frac": max(t_hbm, t_tc) / ms_max}

    # end to end through the public API with host buffers
    e2e = None if (args.no_e2e or kda or long_seq) else run_e2e(inp, dev, args, world)

    metric = METRIC_KDA if kda else (METRIC_LONG if long_seq else METRIC)
    out = {"metric": metric, "value": value, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
           "dtype": "bf16", "data": "synthetic",
           "config": {"workload": w.name, "B": B, "T": T, "H": H, "dk": w.dk, "dv": w.dv,
                      "io_dtype": "bf16", "gate_dtype": "f32", "state_dtype": "f32",
                      "contraction": "bf16 tensor-core operands, f32 accumulate",
                      "step": "ckda_chunk_fwd(saved buffer for the backward) + ckda_chunk_bwd(saved)",
                      "global_batch": B * world, "seq_len": T, "parallelism": "dp%d" % world,
                      "l2": "inputs larger than L2 (about %.1f GB streamed per step)"
                            % ((FWD_BYTES + BWD_BYTES) * B * T * H / 1e9),
                      "gate_sign": "none: every sign +1 (standard KDA)" if kda else "int8 +-1 (CKDA)"},
           "roofline": roof, "step_roofline": step_roof, "kernels": kernels,
           "kernel_times": ("from a separate pass of %d identical steps with a CUDA event pair around every "
                            "launch (%.4f ms per step there); the headline value is timed without them"
                            % (args.steps, ms_prof)),
           "gpu_launches": int(sum(n for n, _ in prof.values())), "clocks": clk, "e2e": e2e}
    return out, inp


def run_secondary(args, rank, world, local_rank):
    """Secondary workloads (not the headline line): forward only, packed
    variable-length forward, recurrent decode."""
    from chunked_gated_delta_ckda_b200 import _abi, api
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks = measured_peaks()
    clocks = ClockSampler(local_rank)
    kernel_bytes = {}
    if args.workload == "decode":
        w = W.DECODE
        N, H, dk, dv = w.B, w.H, w.dk, w.dv
        # two independent sets of N sequences, stepped in turn: a state is
        # read again only after the other set's 256 MiB have gone through L2
        states = [W.make_decode_state(w).to(dev), W.make_decode_state(w).to(dev)]
        pool = [{k: v.to(dev) for k, v in W.make_decode_step(w, t).items()} for t in range(16)]
        o = torch.empty(N, H, dv, dtype=w.io_dtype, device=dev)
        code = api.io_code(w.io_dtype)
        it = [0]

        def step():
            x = pool[it[0] % len(pool)]
            state = states[it[0] % 2]
            it[0] += 1
            _abi.ckda_decode_step(N, H, dk, dv, code, x["q"], x["k"], x["v"], x["g"], x["sign"],
                                  x["beta"], state, o)
        units, per_unit, unit_name = N * H, DECODE_BYTES_PER_NH, "B per (sequence, head) step"
        tokens = N
        metric = "CKDA decode tokens/s (N=256,H=16,d=128,bf16 I/O,fp32 state)"
        cfg = {"workload": w.name, "N": N, "H": H, "dk": dk, "dv": dv, "io_dtype": "bf16",
               "state_dtype": "f32",
               "l2": "two state sets of 256 MiB stepped in turn (512 MiB of other states between a state's uses)"}
    elif args.workload == "decode_multi":
        w = W.DECODE_MULTI
        N, K, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
        pool = W.make_decode_pool(w).to(dev)
        calls = [{k: v.to(dev) for k, v in W.make_decode_multi(w, c).items()} for c in range(8)]
        # odd calls use the pool's other N slots: the two halves of the pool are
        # stepped in turn, so a state is read again only after the other
        # half's 256 MiB have gone through L2
        taken = set(calls[0]["slots"].tolist())
        other = torch.tensor([s_ for s_ in range(pool.shape[0]) if s_ not in taken][:N], dtype=torch.int32, device=dev)
        for c in range(1, len(calls), 2):
            calls[c]["slots"] = other
        o = torch.empty(N, K, H, dv, dtype=w.io_dtype, device=dev)
        code = api.io_code(w.io_dtype)
        it = [0]

        def step():
            x = calls[it[0] % len(calls)]
            it[0] += 1
            _abi.ckda_decode_multi(N, K, H, dk, dv, code, x["q"], x["k"], x["v"], x["g"], x["sign"], x["beta"],
                                   None, x["slots"], pool.shape[0], pool, True, o)
        units, per_unit, unit_name = N * H, DECODE_BYTES_PER_NH + (K - 1) * FWD_BYTES, \
            "B per (sequence, head) call of %d tokens" % K
        tokens = N * K
        metric = "CKDA multi-token decode tokens/s (N=256,K=4,H=16,d=128,bf16 I/O,fp32 state pool)"
        cfg = {"workload": w.name, "N": N, "K": K, "H": H, "dk": dk, "dv": dv, "io_dtype": "bf16",
               "state_dtype": "f32", "n_slots": pool.shape[0],
               "l2": "the pool's two halves (256 MiB each) stepped in turn"}
    elif args.workload == "prologue":
        w = W.LAYER_FWDBWD
        x = {k: v.to(dev) for k, v in W.make_prologue(w, B=args.batch or None).items()}
        B, T, H, dk, dv = x["xq"].shape[0], w.T, w.H, w.dk, w.dv
        code = api.io_code(w.io_dtype)
        e = lambda t, dt=None: torch.empty_like(t, dtype=dt) if dt else torch.empty_like(t)
        outs = dict(q=e(x["xq"]), k=e(x["xk"]), v=e(x["xv"]), g=e(x["a"]), sign=e(x["a"], torch.int8),
                    beta=e(x["b"]))
        grads = dict(dxq=e(x["xq"]), dxk=e(x["xk"]), dxv=e(x["xv"]), dwq=e(x["wq"]), dwk=e(x["wk"]),
                     dwv=e(x["wv"]), da=e(x["a"]), db=e(x["b"]))
        args_in = (x["xq"], x["xk"], x["xv"], x["wq"], x["wk"], x["wv"], x["a"], x["b"], -5.0)

        def step():
            _abi.ckda_prologue_fwd(B, T, H, dk, dv, code, *args_in, outs["q"], outs["k"], outs["v"], outs["g"],
                                   outs["sign"], outs["beta"])
            _abi.ckda_prologue_bwd(B, T, H, dk, dv, code, *args_in, x["dq"], x["dk"], x["dv"], x["dg"], x["dbeta"],
                                   grads["dxq"], grads["dxk"], grads["dxv"], grads["dwq"], grads["dwk"],
                                   grads["dwv"], grads["da"], grads["db"])
        units, per_unit, unit_name = B * T * H, PROLOGUE_FWD_BYTES + PROLOGUE_BWD_BYTES, \
            "B per token-head (prologue fwd + bwd)"
        kernel_bytes = {"prologue_fwd": PROLOGUE_FWD_BYTES, "prologue_bwd": PROLOGUE_BWD_BYTES}
        tokens = B * T
        metric = "CKDA prologue fwd+bwd tokens/s (short conv + q/k L2 norm + signed gate + beta; B=8,T=4096,H=16,d=128,bf16)"
        cfg = {"workload": "prologue_" + w.name, "B": B, "T": T, "H": H, "dk": dk, "dv": dv, "io_dtype": "bf16",
               "g_floor": -5.0, "l2": "inputs larger than L2"}
    elif args.workload in ("varlen", "varlen_fwdbwd"):
        w = W.VARLEN
        inp = W.make_varlen(w)
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        T, H, dk, dv = inp["q"].shape[1], w.H, w.dk, w.dv
        Nd = len(inp["lens"])
        o = torch.empty(1, T, H, dv, dtype=w.io_dtype, device=dev)
        ST = torch.empty(Nd, H, dk, dv, dtype=torch.float32, device=dev)
        ws = api.workspace(_abi.CKDA_OP_VARLEN_FWD, 1, T, H, dk, dv, Nd, device=dev, cache=False)
        cu = d["cu_seqlens"]
        mx = max(inp["lens"])
        code = api.io_code(w.io_dtype)

        def step():
            _abi.ckda_varlen_fwd(T, Nd, cu, mx, H, dk, dv, code, d["q"], d["k"], d["v"], d["g"],
                                 d["sign"], d["beta"], None, o, ST, ws)
        units, per_unit, unit_name = T * H, FWD_BYTES, "B per token-head (fwd)"
        tokens = T
        metric = "CKDA varlen fwd tokens/s (65536 packed tokens,H=16,d=128,bf16)"
        cfg = {"workload": w.name, "total_T": T, "docs": Nd, "H": H, "dk": dk, "dv": dv,
               "io_dtype": "bf16", "l2": "inputs larger than L2"}
        if args.workload == "varlen_fwdbwd":  # the packed training step: forward then backward
            gen = torch.Generator().manual_seed(w.seed + 100)
            dO = torch.randn(1, T, H, dv, generator=gen).to(w.io_dtype).to(dev)
            gb = dict(dq=torch.empty_like(d["q"]), dk=torch.empty_like(d["k"]), dv=torch.empty_like(d["v"]),
                      dg=torch.empty_like(d["g"]), dbeta=torch.empty_like(d["beta"]))
            wsb = api.workspace(_abi.CKDA_OP_VARLEN_BWD, 1, T, H, dk, dv, Nd, device=dev, cache=False)
            # the forward hands its per-chunk results to the backward (as in the headline step)
            n_sv = _abi.ckda_varlen_saved_size(T, Nd, H, dk, dv, code)
            sv = torch.empty(n_sv, dtype=torch.uint8, device=dev) if n_sv > 0 else None

            def step():
                _abi.ckda_varlen_fwd(T, Nd, cu, mx, H, dk, dv, code, d["q"], d["k"], d["v"], d["g"],
                                     d["sign"], d["beta"], None, o, ST, ws, saved=sv)
                _abi.ckda_varlen_bwd(T, Nd, cu, mx, H, dk, dv, code, d["q"], d["k"], d["v"], d["g"],
                                     d["sign"], d["beta"], None, dO, None, gb["dq"], gb["dk"], gb["dv"],
                                     gb["dg"], gb["dbeta"], None, wsb, saved=sv)
            per_unit, unit_name = FWD_BYTES + BWD_BYTES, "B per token-head (fwd + bwd)"
            kernel_bytes = {"tc_grad": BWD_BYTES, "tc_intra": FWD_BYTES}
            metric = "CKDA varlen fwd+bwd tokens/s (65536 packed tokens,H=16,d=128,bf16)"
            cfg["workload"] = "varlen_fwdbwd_bf16"
    elif args.workload == "long":
        w = W.LONG
        inp = W.make(w)
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
        o = torch.empty(B, T, H, dv, dtype=w.io_dtype, device=dev)
        ST = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
        ws = api.workspace(_abi.CKDA_OP_CHUNK_FWD, B, T, H, dk, dv, device=dev, cache=False)
        code = api.io_code(w.io_dtype)
        S0 = d["S0"].float().contiguous()

        def step():
            _abi.ckda_chunk_fwd(B, T, H, dk, dv, code, d["q"], d["k"], d["v"], d["g"], d["sign"],
                                d["beta"], S0, o, ST, None, ws)
        units, per_unit, unit_name = B * T * H, FWD_BYTES, "B per token-head (fwd)"
        tokens = B * T
        metric = "CKDA long-sequence fwd tokens/s (B=1,T=65536,H=16,d=128,bf16)"
        cfg = {"workload": w.name, "B": B, "T": T, "H": H, "dk": dk, "dv": dv, "io_dtype": "bf16",
               "S0": True, "l2": "inputs larger than L2"}
    else:  # fwd
        w = W.LAYER_FWD
        inp = W.make(w)
        d = {k: (v.to(dev) if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
        B, T, H, dk, dv = w.B, w.T, w.H, w.dk, w.dv
        o = torch.empty(B, T, H, dv, dtype=w.io_dtype, device=dev)
        ST = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
        ws = api.workspace(_abi.CKDA_OP_CHUNK_FWD, B, T, H, dk, dv, device=dev, cache=False)
        code = api.io_code(w.io_dtype)

        def step():
            _abi.ckda_chunk_fwd(B, T, H, dk, dv, code, d["q"], d["k"], d["v"], d["g"], d["sign"],
                                d["beta"], None, o, ST, None, ws)
        units, per_unit, unit_name = B * T * H, FWD_BYTES, "B per token-head (fwd)"
        tokens = B * T
        metric = "CKDA fwd tokens/s (H=16,d=128,T=4096,bf16)"
        cfg = {"workload": w.name, "B": B, "T": T, "H": H, "dk": dk, "dv": dv, "io_dtype": "bf16",
               "l2": "inputs larger than L2"}
    clocks.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks.mark()
    ms = _time_steps(step, args.steps, 0, world)  # library profiling off
    clocks.keep_loaded(step)
    clk = clocks.stop()
    ms = reduce_max(ms, world)
    prof, ms_prof = _profile_pass(step, args.steps, world)
    total = sum(t for _, t in prof.values())
    kernels = {k: {"launches": n, "ms_per_launch": t / n, "share": t / total if total else None}
               for k, (n, t) in sorted(prof.items(), key=lambda kv: -kv[1][1])}
    top = max(prof.items(), key=lambda kv: kv[1][1])[0]
    n, t = prof[top]
    launches_per_step = n / args.steps
    step_bytes = per_unit * units
    if top in kernel_bytes:  # a step of several different kernels: the top one's own bytes
        per_unit, unit_name = kernel_bytes[top], "B per token-head (%s)" % top
        launches_per_step = 1
    alg = per_unit * units / launches_per_step if launches_per_step >= 1 else per_unit * units
    achieved = alg / (t / n / 1e3) / 1e9
    out = {"metric": metric, "value": tokens * world / (ms / 1e3), "unit": "tokens/s",
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
           "data": "synthetic", "config": cfg,
           "roofline": {"bound": "hbm", "kernel": top, "achieved": achieved, "peak": peaks["hbm_gbs"],
                        "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                        "algorithmic_bytes_per_launch": alg, "per_unit": "%d %s" % (per_unit, unit_name),
                        "peak_source": peaks["source"]},
           "step_hbm_frac": step_bytes / (peaks["hbm_gbs"] * 1e9) / (ms / 1e3),
           "kernels": kernels,
           "kernel_times": ("from a separate pass of %d identical steps with a CUDA event pair around every "
                            "launch (%.4f ms per step there); the value is timed without them" % (args.steps, ms_prof)),
           "gpu_launches": int(sum(n for n, _ in prof.values())), "clocks": clk}
    if args.workload == "decode":  # the step against the nominal HBM figure too
        out["step_hbm_frac_nominal"] = step_bytes / (NOMINAL_HBM_GBS * 1e9) / (ms / 1e3)
        out["step_achieved_gbs"] = step_bytes / (ms / 1e3) / 1e9
    return out


# Secondary workloads measured in the default run (after the headline), each
# with its own clock record: name -> (steps, warm-up) caps
SECONDARY = (("decode", 64), ("decode_multi", 32), ("varlen", 20), ("varlen_fwdbwd", 10), ("long", 10),
             ("long_fwdbwd", 6), ("fwd", 20), ("kda", 10), ("prologue", 10))


def secondary_suite(args, rank, world, local_rank):
    """Every secondary workload, timed as its own --workload run would time it
    (fewer steps), condensed to the figures a reader compares."""
    res = {}
    for name, steps in SECONDARY:
        sub = argparse.Namespace(**{**vars(args), "workload": name, "steps": steps, "warmup": 3, "batch": 0,
                                    "no_e2e": True})
        try:
            if name in ("long_fwdbwd", "kda"):
                line, _ = run_ours(sub, rank, world, local_rank)
            else:
                line = run_secondary(sub, rank, world, local_rank)
        except Exception as e:  # reported, never fatal to the headline line
            res[name] = {"error": "%s: %s" % (type(e).__name__, e)}
            continue
        r = line.get("roofline") or {}
        keep = {"metric": line["metric"], "value": line["value"], "unit": line["unit"],
                "ms_per_step": line["ms_per_step"], "steps": steps, "warmup": 3,
                "top_kernel": r.get("kernel"), "top_kernel_hbm_frac": r.get("frac"),
                "top_kernel_achieved_gbs": r.get("achieved"), "clocks": line.get("clocks"),
                "config": line.get("config")}
        for key in ("step_hbm_frac", "step_hbm_frac_nominal", "step_achieved_gbs"):
            if key in line:
                keep[key] = line[key]
        if "step_roofline" in line:
            keep["step_hbm_frac"] = line["step_roofline"]["hbm_frac"]
        res[name] = keep
        torch.cuda.empty_cache()
    return res


def run_e2e(inp, dev, args, world):
    """Same step through the public API from pinned HOST buffers: every step
    uploads its inputs and downloads every output inside the timed region.
    Steps are pipelined the way a training input pipeline runs: the next
    step's inputs upload (one copy engine) and the previous step's outputs
    download (the other) while the current step computes; two device buffer
    sets alternate, ordered by CUDA events."""
    from chunked_gated_delta_ckda_b200 import _abi, api
    names_in = ("q", "k", "v", "g", "sign", "beta", "dO")
    host_in = {k: inp[k].pin_memory() for k in names_in}
    B, T, H, dk = inp["q"].shape
    dv = inp["v"].shape[-1]
    code = api.io_code(inp["q"].dtype)
    wsf = api.workspace(_abi.CKDA_OP_CHUNK_FWD, B, T, H, dk, dv, device=dev, cache=False)
    wsb = api.workspace(_abi.CKDA_OP_CHUNK_BWD, B, T, H, dk, dv, device=dev, cache=False)
    sv = api.saved_buffer(B, T, H, dk, dv, inp["q"].dtype, dev)
    sets = []
    for _ in range(2):
        _, buf, _ = _fwdbwd_setup({**inp}, dev)
        sets.append(dict(dev_in={k: torch.empty_like(v, device=dev) for k, v in host_in.items()}, buf=buf,
                         host_out={k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True)
                                   for k, v in buf.items() if k != "cs"},
                         in_ready=torch.cuda.Event(), comp_done=torch.cuda.Event(),
                         out_done=torch.cuda.Event()))
    h2d = sum(v.numel() * v.element_size() for v in host_in.values())
    d2h = sum(v.numel() * v.element_size() for v in sets[0]["host_out"].values())
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def issue(i):
        S = sets[i % 2]
        x, buf = S["dev_in"], S["buf"]
        cs = None if sv is not None else buf["cs"]
        s_in.wait_event(S["comp_done"])  # this set's inputs were last read two steps ago
        with torch.cuda.stream(s_in):
            for k, v in host_in.items():
                x[k].copy_(v, non_blocking=True)
        S["in_ready"].record(s_in)
        s_comp.wait_event(S["in_ready"])
        s_comp.wait_event(S["out_done"])  # this set's outputs have been downloaded
        _abi.ckda_chunk_fwd(B, T, H, dk, dv, code, x["q"], x["k"], x["v"], x["g"], x["sign"],
                            x["beta"], None, buf["o"], buf["ST"], cs, wsf, saved=sv, stream=s_comp)
        _abi.ckda_chunk_bwd(B, T, H, dk, dv, code, x["q"], x["k"], x["v"], x["g"], x["sign"],
                            x["beta"], None, x["dO"], None, cs, buf["dq"], buf["dk"],
                            buf["dv"], buf["dg"], buf["dbeta"], buf["dS0"], wsb, saved=sv,
                            stream=s_comp)
        S["comp_done"].record(s_comp)
        s_out.wait_event(S["comp_done"])
        with torch.cuda.stream(s_out):
            for k, v in S["host_out"].items():
                v.copy_(buf[k], non_blocking=True)
        S["out_done"].record(s_out)

    import torch.distributed as dist
    steps = max(1, min(args.steps, 10))
    for i in range(max(1, min(args.warmup, 3))):
        issue(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    s_comp.wait_event(t0)
    s_out.wait_event(t0)
    for i in range(steps):
        issue(i)
    s_out.wait_event(sets[(steps - 1) % 2]["out_done"])
    t1.record(s_out)
    torch.cuda.synchronize(dev)
    ms = reduce_max(t0.elapsed_time(t1) / steps, world)
    return {"value": aggregate(B * T, world, ms), "unit": "tokens/s", "ms_per_step": ms,
            "steps": steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelined": "upload of step i+1 and download of step i-1 overlap step i's kernels"}


# ---------------------------------------------------------------------------
# the fp64 CPU oracle (baseline / reference arm)
# ---------------------------------------------------------------------------

def oracle_fwdbwd_sample(inp, pairs, nthreads):
    """Oracle forward + backward over the sampled (batch, head) sequences."""
    import numpy as np
    import oracle
    T = inp["q"].shape[1]
    P = lambda x, b, h: x[b, :, h:h + 1].to(torch.float64).numpy()
    # pack the sampled sequences as independent documents of one head
    cat = lambda key: np.concatenate([P(inp[key], b, h) for b, h in pairs], axis=0)
    sg = np.concatenate([inp["sign"][b, :, h:h + 1].numpy() for b, h in pairs], axis=0)
    cu = np.arange(len(pairs) + 1, dtype=np.int64) * T
    q, k, v, g, beta, dO = (cat(x) for x in ("q", "k", "v", "g", "beta", "dO"))
    t0 = time.perf_counter()
    oracle.fwd(cu, q, k, v, g, sg, beta, nthreads=nthreads)
    oracle.bwd(cu, q, k, v, g, sg, beta, dO, nthreads=nthreads)
    return time.perf_counter() - t0


def oracle_fwd_sample(inp, pairs, nthreads):
    """Oracle forward over the sampled (batch, head) sequences."""
    import numpy as np
    import oracle
    T = inp["q"].shape[1]
    P = lambda x, b, h: x[b, :, h:h + 1].to(torch.float64).numpy()
    cat = lambda key: np.concatenate([P(inp[key], b, h) for b, h in pairs], axis=0)
    sg = np.concatenate([inp["sign"][b, :, h:h + 1].numpy() for b, h in pairs], axis=0)
    cu = np.arange(len(pairs) + 1, dtype=np.int64) * T
    q, k, v, g, beta = (cat(x) for x in ("q", "k", "v", "g", "beta"))
    t0 = time.perf_counter()
    oracle.fwd(cu, q, k, v, g, sg, beta, nthreads=nthreads)
    return time.perf_counter() - t0


def cpu_baseline_secondary(workload):
    """The oracle on the host cores for the forward and decode workloads
    (bounded samples, the same seeded inputs)."""
    import oracle
    cores = oracle.default_threads()
    if workload == "fwd":
        w = W.LAYER_FWD
        inp = W.make(w)
        n_pairs = max(8, min(128, 16 * cores))
        pairs = [(i % w.B, (i * 7) % w.H) for i in range(n_pairs)]
        threads = min(cores, n_pairs)
        dt = oracle_fwd_sample(inp, pairs, threads)
        return {"value": n_pairs * w.T / w.H / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                "sample": "%d of %d (batch, head) sequences of %d tokens, forward, fp64, %d threads, %.1f s"
                          % (n_pairs, w.B * w.H, w.T, threads, dt)}
    w = W.DECODE  # decode: consecutive steps of every (sequence, head) state
    x = W.make_decode_step(w, 0)
    st = W.make_decode_state(w).to(torch.float64).numpy()
    f = lambda t: t.to(torch.float64).numpy()
    args = (f(x["q"]), f(x["k"]), f(x["v"]), f(x["g"]), x["sign"].numpy(), f(x["beta"]))
    steps, t0 = 0, time.perf_counter()
    while steps < 2 or (time.perf_counter() - t0 < 5.0 and steps < 64):
        _, st = oracle.decode(*args, st, nthreads=cores)
        steps += 1
    dt = time.perf_counter() - t0
    return {"value": steps * w.B / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "%d steps of all %d x %d states, fp64, %d threads, %.1f s" % (steps, w.B, w.H, cores, dt)}


def cpu_baseline(inp, H, n_pairs=None):
    import oracle
    cores = oracle.default_threads()
    n_pairs = n_pairs or max(8, min(128, 12 * cores))
    B = inp["q"].shape[0]
    pairs = [(i % B, (i * 7) % H) for i in range(n_pairs)]
    threads = min(cores, n_pairs)
    dt = oracle_fwdbwd_sample(inp, pairs, threads)
    T = inp["q"].shape[1]
    tokens = n_pairs * T / H  # a token carries H heads
    return {"value": tokens / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": "%d of %d (batch, head) sequences of %d tokens, forward + backward, fp64, "
                      "%d threads, %.1f s" % (n_pairs, B * H, T, threads, dt)}


def run_reference(args, rank, world):
    """The oracle as it stands, timed on the host cores, on this workload."""
    import oracle
    if rank != 0:
        return None
    oracle.build()
    w = W.LAYER_FWDBWD
    inp = W.make(w)
    cores = oracle.default_threads()
    n_pairs = max(2, min(32, cores))  # one sequence per host thread: every core busy
    pairs = [(i % w.B, (i * 5) % w.H) for i in range(n_pairs)]
    threads = min(cores, n_pairs)
    for _ in range(args.warmup):
        oracle_fwdbwd_sample(inp, pairs[:1], 1)
    dts = [oracle_fwdbwd_sample(inp, pairs, threads) for _ in range(args.steps)]
    dt = sum(dts) / len(dts)
    value = n_pairs * w.T / w.H / dt
    sample = ("%d of %d (batch, head) sequences of %d tokens per step, forward + backward, "
              "fp64, %d threads" % (n_pairs, w.B * w.H, w.T, threads))
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "dk": w.dk, "dv": w.dv,
                       "io_dtype": "bf16", "global_batch": w.B, "seq_len": w.T,
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer pass")
    ap.add_argument("--workload", choices=["fwdbwd", "kda", "fwd", "varlen", "varlen_fwdbwd", "long", "long_fwdbwd", "decode",
                             "decode_multi", "prologue"], default="fwdbwd",
                    help="fwdbwd is the headline; the others are secondary measurements")
    ap.add_argument("--no-secondary", action="store_true",
                    help="headline only: skip the secondary workloads of the default run")
    ap.add_argument("--batch", type=int, default=0,
                    help="override B (profiling a smaller case; not a bench line)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0

    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.workload not in ("fwdbwd", "kda", "long_fwdbwd"):
            out = run_secondary(args, rank, world, local_rank)
            if rank == 0:
                if world == 1 and not args.no_cpu_baseline and args.workload in ("fwd", "decode"):
                    out["cpu_baseline"] = cpu_baseline_secondary(args.workload)
                print(json.dumps(out), flush=True)
            return 0
        out, inp = run_ours(args, rank, world, local_rank)
        if world == 1 and args.workload == "fwdbwd" and not args.no_secondary:
            out["secondary"] = secondary_suite(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline and args.workload == "fwdbwd":
                out["cpu_baseline"] = cpu_baseline(inp, W.LAYER_FWDBWD.H)
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
