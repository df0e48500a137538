#!/usr/bin/env python
"""Benchmark of the tree-ordered invariant hot path on B200.

One step = one pass of every kernel of the path over one batch of M = 4096
tokens, with the sizes of the lm_head / down_proj / reduction workloads:

  residual RMSNorm   x, res bf16 [4096, 4096]          -> y, res_out
  RoPE (fp32)        q, k bf16 [4096, 32, 128], pos     -> q', k'
  SwiGLU (fp32)      g, u bf16 [4096, 14336]            -> A bf16
  down_proj GEMM     A [4096, 14336] x B [14336, 4096], leaf 256, T = 1, tensor cores -> h bf16
  lm_head logprob    h [4096, 4096] x W_lm [151936, 4096]^T, targets -> logprob fp32 [4096]

``value`` is whole-job tokens/s (all ranks; each rank runs its own batch:
weak scaling, no collective on the data path).  ``--impl reference`` times the
CPU oracle on a bounded sample of the same step instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

M_TOK = 4096
H = 4096
F = 14336
V = 151936
HEADS, HEAD_DIM, MAX_POS = 32, 128, 32768
LEAF = 256
METRIC = "invariant GEMM TFLOP/s + logprob tokens/s, bitwise-stable over T/batch"
WORKLOAD = ("tbik hot path, M=4096 tokens/step: residual RMSNorm H=4096 -> RoPE fp32 q,k [32x128] -> "
            "SwiGLU fp32 [14336] -> down_proj tree GEMM [4096x14336]x[14336x4096] leaf 256 T=1 (tcgen05) -> "
            "lm_head logprob V=151936 H=4096 leaf 256 (fused tcgen05 + tree log-softmax)")
GEMM_FLOP = 2.0 * M_TOK * F * H
LOGPROB_FLOP = 2.0 * M_TOK * V * H
KERNELS_PER_STEP = 6  # rmsnorm, rope, swiglu, gemm, logprob gemm+stats, logprob row tree
# fp32 FMA peak of the exact-order (CUDA-core) mode: 148 SMs x 128 fp32 lanes x
# 2 flop x 1.965 GHz (the maximum SM clock)
FP32_FMA_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# Timed regions at least this long are compared with the sustained bf16 peak.
SUSTAINED_REGION_S = 3.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="tbik", choices=["tbik", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decoder", action="store_true", help="skip the end-to-end decoder component")
    ap.add_argument("--profile-case", choices=["logprob", "gemm", "gemm-t8", "gemm-exact", "attention",
                                               "attention-tc", "swiglu", "rmsnorm"],
                    default=None,
                    help="run only one call of the path, `--steps` times, for ncu captures (no JSON line)")
    ap.add_argument("--tokens", type=int, default=M_TOK, help="tokens per call in --profile-case")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sus=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), src="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # pragma: no cover
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.02)

    def start(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------- profile-backed traffic

TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "logprob_tc_m4096.md")
KERNEL_SOURCES = ["device_common.cuh", "gemm_tc.cuh", "logprob.cuh", "tbik_api.cu"]


def kernel_source_hash() -> str:
    """sha256 over the sources of the logprob kernels (changes invalidate old counters)."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "invariant_tree_ordered_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic():
    """DRAM bytes per logprob launch from the committed ncu summary, if it was
    taken on the current kernel sources; else None."""
    try:
        with open(TRAFFIC_PROFILE) as f:
            text = f.read()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith(("traffic_bytes_per_launch", "source_sha256")):
            k, v = line.strip().strip("`").split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("source_sha256") != kernel_source_hash() or "traffic_bytes_per_launch" not in fields:
        return None
    return int(fields["traffic_bytes_per_launch"])


# ------------------------------------------------- multi-rank aggregation

def max_over_ranks(value: float, world: int, device=None) -> float:
    """Largest `value` over all ranks (all-reduce MAX); the identity for one rank."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(ms_total_max: float, steps: int, world: int, tokens_per_rank: int = M_TOK) -> float:
    """Weak scaling: every rank runs its own batch; the job's time is the slowest rank's."""
    return world * tokens_per_rank * steps / (ms_total_max * 1e-3)


# ------------------------------------------------------------- CPU oracle

def host_cpu() -> dict:
    """The host the oracle ran on: logical CPUs available and the CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        avail = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        avail = os.cpu_count()
    return {"host_cores": os.cpu_count(), "host_cores_available": avail, "cpu_model": model}


_ORACLE_INPUTS = {}


def oracle_step_sample(tokens: int):
    """Time the CPU oracle on `tokens` tokens of the step (every kernel of the path)."""
    import oracle
    if "weights" not in _ORACLE_INPUTS:  # the same weights for every sample size
        _ORACLE_INPUTS["weights"] = dict(b=synth.down_proj_weight(F, H, "kn"),
                                         w=synth.normal_bf16(31, (V, H), std=0.02),
                                         table=oracle.rope_table(MAX_POS, HEAD_DIM, 1e6))
    if tokens not in _ORACLE_INPUTS:
        std = 0.02 * np.sqrt(H)
        _ORACLE_INPUTS[tokens] = dict(
            d=synth.reduction_inputs(tokens), g=synth.normal_bf16(11, (tokens, F), std=std),
            u=synth.normal_bf16(12, (tokens, F), std=std), targets=synth.uniform_int32(32, tokens, 0, V))
    c_, wt = _ORACLE_INPUTS[tokens], _ORACLE_INPUTS["weights"]
    d, g, u, targets = c_["d"], c_["g"], c_["u"], c_["targets"]
    b, w, table = wt["b"], wt["w"], wt["table"]
    t0 = time.perf_counter()
    oracle.rmsnorm_residual(d["x"], d["res"], d["gamma"], eps=1e-6)
    oracle.rope(d["q"], d["pos"], table)
    oracle.rope(d["k"], d["pos"], table)
    a = oracle.swiglu(g, u)
    c = oracle.gemm_tree(a, b, b_nk=False, T=1, leaf=LEAF)
    hid = oracle.bf16_rne_array(c)
    oracle.logprob(hid, w, targets, T=1, leaf=LEAF)
    return time.perf_counter() - t0


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    tokens = 1
    for _ in range(args.warmup):
        oracle_step_sample(tokens)
    times = [oracle_step_sample(tokens) for _ in range(args.steps)]
    total = sum(times)
    value = tokens * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32 (bf16 inputs)",
        "data": "synthetic (seeded SplitMix64/Box-Muller)",
        "config": {"workload": WORKLOAD, "tokens_per_step": M_TOK, "sample_tokens_per_step": tokens,
                   "T": 1, "leaf": LEAF},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"{tokens} token(s) of the step per step: RMSNorm, RoPE q/k, SwiGLU, one "
                                   f"down_proj row, one lm_head logprob row (single-threaded C oracle)",
                         **host_cpu()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- GPU path

def run_tbik(args):
    import torch
    import torch.distributed as dist

    import invariant_tree_ordered_b200 as tbik
    from invariant_tree_ordered_b200 import build as libbuild

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not os.path.exists(libbuild.LIB):
        libbuild.build_library()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])
        torch.cuda.synchronize()


    def bf(a):
        return synth.as_torch_bf16(a)

    # ---- inputs (seeded, synthetic), resident in HBM
    d = synth.reduction_inputs(M_TOK)
    std = 0.02 * np.sqrt(H)
    host = {
        "x": bf(d["x"]), "res": bf(d["res"]), "q": bf(d["q"]), "k": bf(d["k"]),
        "pos": torch.from_numpy(d["pos"]),
        "g": bf(synth.normal_bf16(11, (M_TOK, F), std=std)), "u": bf(synth.normal_bf16(12, (M_TOK, F), std=std)),
        "targets": torch.from_numpy(synth.uniform_int32(32, M_TOK, 0, V)),
    }
    gamma = bf(d["gamma"]).to(dev)
    B = bf(synth.down_proj_weight(F, H, "kn")).to(dev)
    W = bf(synth.normal_bf16(31, (V, H), std=0.02)).to(dev)
    table = tbik.rope_table(MAX_POS, HEAD_DIM, 1e6, device=dev)
    inp = {k: v.to(dev) for k, v in host.items()}
    y = torch.empty_like(inp["x"])
    res_out = torch.empty_like(inp["x"])
    qo = torch.empty_like(inp["q"])
    ko = torch.empty_like(inp["k"])
    A = torch.empty((M_TOK, F), dtype=torch.bfloat16, device=dev)
    hid = torch.empty((M_TOK, H), dtype=torch.bfloat16, device=dev)
    out = torch.empty(M_TOK, dtype=torch.float32, device=dev)
    gws = torch.empty(max(tbik.gemm_workspace(M_TOK, H, F, 1, LEAF, tbik.TC | tbik.OUT_BF16), 256),
                      dtype=torch.uint8, device=dev)
    lws = torch.empty(tbik.logprob_workspace(M_TOK, V, H, 1, LEAF, tbik.TC), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    ev = {k: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for k in ("rms", "rope", "swiglu", "gemm", "logprob")}
    acc = {k: 0.0 for k in ev}

    def step(src, timed=False, lp_events=None):
        def mark(k, i):
            if timed:
                ev[k][i].record(stream)
        mark("rms", 0)
        tbik.rmsnorm_residual(src["x"], src["res"], gamma, eps=1e-6, T=1, y=y, res_out=res_out, stream=stream)
        mark("rms", 1)
        mark("rope", 0)
        tbik.rope_swiglu(q=src["q"], k=src["k"], pos=src["pos"], table=table, q_out=qo, k_out=ko, stream=stream)
        mark("rope", 1)
        mark("swiglu", 0)
        tbik.rope_swiglu(g=src["g"], u=src["u"], out=A, stream=stream)
        mark("swiglu", 1)
        mark("gemm", 0)
        tbik.gemm(A, B, T=1, leaf=LEAF, tc=True, out_bf16=True, out=hid, workspace=gws, stream=stream)
        mark("gemm", 1)
        mark("logprob", 0)
        if lp_events is not None:
            lp_events[0].record(stream)
        tbik.logprob(hid, W, src["targets"], T=1, leaf=LEAF, tc=True, out=out, workspace=lws, stream=stream)
        if lp_events is not None:
            lp_events[1].record(stream)
        mark("logprob", 1)

    for _ in range(args.warmup):
        step(inp)
    if tbik.get_error(stream) != tbik.TBIK_OK:
        raise RuntimeError("device error during warm-up")

    # ---- device-timed region: inputs resident in HBM
    clocks = ClockSampler(local)
    barrier()
    clocks.start()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    lp_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    torch.cuda.nvtx.range_push("tbik_timed_steps")
    t0.record(stream)
    for i in range(args.steps):
        step(inp, lp_events=lp_ev[i])
    t1.record(stream)
    torch.cuda.nvtx.range_pop()
    barrier()
    clk = clocks.stop()
    # dominant kernel: average duration of the logprob call inside the timed region
    lp_step_ms = [a.elapsed_time(b) for a, b in lp_ev]
    lp_live_ms = float(np.mean(lp_step_ms))
    ms_total = max_over_ranks(t0.elapsed_time(t1), world, dev)
    status = tbik.get_error(stream)
    if status != tbik.TBIK_OK:
        raise RuntimeError(f"device error in timed region: {status}")

    # ---- per-kernel durations (same stream, events around each call, averaged)
    comp = {k: [] for k in ev}
    barrier()
    for _ in range(min(args.steps, 20)):
        # a ~0.5 ms device-side spin first, so the host has queued every launch
        # of the step before its first kernel starts: the events then bracket
        # kernel time only, not Python launch latency
        torch.cuda._sleep(1_000_000)
        step(inp, timed=True)
        torch.cuda.synchronize()
        for k, (a, b) in ev.items():
            comp[k].append(a.elapsed_time(b))
    comp_ms = {k: float(np.mean(v)) for k, v in comp.items()}

    # ---- end to end: host buffers in pinned memory, copies inside the timed region.
    # Every step copies its inputs host -> device and reads its logprobs back.
    # The input copies run on a copy stream into two alternating sets of device
    # buffers, so step i+1's copy overlaps step i's kernels (a pipelined
    # serving loop); the compute stream waits for its set's copy, and the copy
    # into a set waits until the step that last read it is done.
    pinned = {k: v.pin_memory() for k, v in host.items()}
    out_host = torch.empty(M_TOK, dtype=torch.float32).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = out_host.numel() * out_host.element_size()
    dst = [{k: torch.empty_like(v) for k, v in inp.items()} for _ in range(2)]
    copy_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(copy_stream):
            if used[b]:
                copy_stream.wait_event(consumed[b])
            for k, v in pinned.items():
                dst[b][k].copy_(v, non_blocking=True)
            copied[b].record(copy_stream)
        stream.wait_event(copied[b])
        step(dst[b])
        consumed[b].record(stream)
        used[b] = True
        out_host.copy_(out, non_blocking=True)

    for i in range(3):
        e2e_step(i)
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_stream.wait_event(e0)  # no copy of the timed steps starts before the region does
    for i in range(args.steps):
        e2e_step(i)
    e1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)

    # ---- overhead of the invariant path over the non-invariant baseline (T = 1)
    def avg_ms(fn, n=10):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    nws = torch.empty(max(tbik.gemm_workspace(M_TOK, H, F, 1, LEAF, tbik.TC | tbik.NONINV | tbik.OUT_BF16), 256),
                      dtype=torch.uint8, device=dev)
    nlws = torch.empty(tbik.logprob_workspace(M_TOK, V, H, 1, LEAF, tbik.TC | tbik.NONINV), dtype=torch.uint8,
                       device=dev)
    hid2 = torch.empty_like(hid)
    out2 = torch.empty_like(out)
    g_inv = avg_ms(lambda: tbik.gemm(A, B, T=1, leaf=LEAF, tc=True, out_bf16=True, out=hid2, workspace=gws))
    g_non = avg_ms(lambda: tbik.gemm(A, B, T=1, leaf=LEAF, tc=True, noninv=True, out_bf16=True, out=hid2,
                                     workspace=nws))
    l_inv = avg_ms(lambda: tbik.logprob(hid, W, inp["targets"], T=1, leaf=LEAF, tc=True, out=out2, workspace=lws), 5)
    l_non = avg_ms(lambda: tbik.logprob(hid, W, inp["targets"], T=1, leaf=LEAF, tc=True, noninv=True, out=out2,
                                        workspace=nlws), 5)
    gws8 = torch.empty(tbik.gemm_workspace(M_TOK, H, F, 8, LEAF, tbik.TC | tbik.OUT_BF16), dtype=torch.uint8,
                       device=dev)
    g_t8 = avg_ms(lambda: tbik.gemm(A, B, T=8, leaf=LEAF, tc=True, out_bf16=True, out=hid2, workspace=gws8))
    tbik.get_error(stream)
    try:  # the exact-order (CUDA-core) mode of the same down_proj call: an extra measurement
        ex_ms = avg_ms(lambda: tbik.gemm(A, B, T=1, leaf=LEAF, tc=False, out_bf16=True, out=hid2), 3)
        ex_tf = GEMM_FLOP / (ex_ms * 1e-3) / 1e12
        exact = {"down_proj_exact_ms": ex_ms, "down_proj_exact_tflops": ex_tf, "bound": "alu",
                 "peak_tflops": FP32_FMA_PEAK_TFLOPS, "frac": ex_tf / FP32_FMA_PEAK_TFLOPS,
                 "status": int(tbik.get_error(stream))}
    except Exception as e:  # noqa: BLE001
        exact = {"error": f"{type(e).__name__}: {e}"[:300]}
        torch.cuda.synchronize()
    try:  # the backward GEMMs of the down_proj (an extra measurement): dA = dY B^T with B read as [N', K']
        # (K' = 4096 in leaves of 256), dB = A^T dY reducing over the 4096 tokens in leaves of 256
        dY = hid  # any bf16 [M, 4096] gradient of the output
        dA = torch.empty((M_TOK, F), dtype=torch.float32, device=dev)
        dB = torch.empty((F, H), dtype=torch.float32, device=dev)
        At = torch.empty((F, M_TOK), dtype=torch.bfloat16, device=dev)
        wdx = torch.empty(max(tbik.gemm_workspace(M_TOK, F, H, 1, LEAF, tbik.TC | tbik.B_NK), 256),
                          dtype=torch.uint8, device=dev)
        wdw = torch.empty(max(tbik.gemm_workspace(F, H, M_TOK, 1, LEAF, tbik.TC), 256), dtype=torch.uint8,
                          device=dev)
        dx_ms = avg_ms(lambda: tbik.gemm(dY, B, T=1, leaf=LEAF, tc=True, b_nk=True, out=dA, workspace=wdx))
        tr_ms = avg_ms(lambda: tbik.transpose(A, out=At))
        dw_ms = avg_ms(lambda: tbik.gemm(At, dY, T=1, leaf=LEAF, tc=True, out=dB, workspace=wdw))
        backward = {"dA_ms": dx_ms, "dA_tflops": GEMM_FLOP / (dx_ms * 1e-3) / 1e12,
                    "dB_gemm_ms": dw_ms, "dB_gemm_tflops": GEMM_FLOP / (dw_ms * 1e-3) / 1e12,
                    "transpose_A_ms": tr_ms, "transpose_A_gbs": 2 * M_TOK * F * 2 / (tr_ms * 1e-3) / 1e9,
                    "fp32_outputs": True, "status": int(tbik.get_error(stream))}
        del dA, dB, At, wdx, wdw
    except Exception as e:  # noqa: BLE001
        backward = {"error": f"{type(e).__name__}: {e}"[:300]}
        torch.cuda.synchronize()
    pk = peaks()
    red8k = reductions_component(8192, dev, stream, gamma, table, pk["hbm"])
    dec = None
    if not args.no_decoder:
        try:  # an extra measurement: a failure here must not cost the main line
            dec = decoder_component(dev, stream)
        except Exception as e:  # noqa: BLE001
            dec = {"error": f"{type(e).__name__}: {e}"[:300]}
            torch.cuda.synchronize()

    lp_ms = lp_live_ms
    achieved = LOGPROB_FLOP / (lp_ms * 1e-3) / 1e12
    # The peak that matches the timing conditions: a short timed region runs at
    # the burst clock (the burst cuBLAS figure), a region of several seconds
    # settles under the power cap (the sustained figure).
    region_s = ms_total * 1e-3
    peak_kind = "burst" if region_s < SUSTAINED_REGION_S else "sustained"
    peak = pk["bf16"] if peak_kind == "burst" else pk["bf16_sus"]
    ms_step = ms_total / args.steps
    value = whole_job_tokens_per_s(ms_total, args.steps, world)
    gb = lambda nbytes, ms: nbytes / (ms * 1e-3) / 1e9  # noqa: E731
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 in, f32 accumulate/reduce",
        "data": "synthetic (seeded SplitMix64/Box-Muller, shapes and distributions of the lm_head/down_proj/"
                "reduction workloads)",
        "config": {"workload": WORKLOAD, "tokens_per_step_per_gpu": M_TOK, "T": 1, "leaf": LEAF,
                   "parallelism": f"{world} independent batches (weak scaling, no data-path collective)",
                   "l2": "inputs larger than L2: every step streams W_lm (1.24 GB) and B (117 MB)"},
        "components": {
            "down_proj_gemm_tflops": GEMM_FLOP / (comp_ms["gemm"] * 1e-3) / 1e12,
            "down_proj_gemm_tflops_T8": GEMM_FLOP / (g_t8 * 1e-3) / 1e12,
            "logprob_tokens_per_s": M_TOK / (lp_ms * 1e-3),
            "logprob_tflops": achieved,
            "logprob_ms_mean_median_best": [lp_live_ms, float(np.median(lp_step_ms)), float(np.min(lp_step_ms))],
            "logprob_frac_of_spec_2250_tflops": achieved / 2250.0,
            "rmsnorm_gbs": gb(4 * M_TOK * H * 2, comp_ms["rms"]),
            "rope_gbs": gb(2 * 2 * M_TOK * HEADS * HEAD_DIM * 2 + M_TOK * (4 + HEAD_DIM * 4), comp_ms["rope"]),
            "swiglu_gbs": gb(3 * M_TOK * F * 2, comp_ms["swiglu"]),
            "ms": comp_ms,
            "reductions_8192_tokens": dict(red8k, copy_peak_gbs=pk["hbm"], copy_peak_source=pk["src"]),
            "exact_mode": exact,
            "backward_down_proj_tc": backward,
            "overhead_vs_noninv": {"gemm": g_inv / g_non - 1.0, "logprob": l_inv / l_non - 1.0,
                                   "gemm_ms": [g_inv, g_non], "logprob_ms": [l_inv, l_non]},
            "decoder_e2e": dec,
        },
        "roofline": {"kernel": "tbik_logprob (fused tcgen05 GEMM + vocab stats, then row tree)",
                     "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": profiled_traffic(),
                     "peak_source": f"{pk['src']} bf16 {peak_kind} (timed region {region_s:.2f} s; burst "
                                    f"below {SUSTAINED_REGION_S:.0f} s)",
                     "frac_of_burst": achieved / pk["bf16"], "frac_of_sustained": achieved / pk["bf16_sus"],
                     "achieved_formula": "2*M*V*H / mean in-step CUDA-event time of the logprob call"},
        "e2e": {"value": whole_job_tokens_per_s(e2e_ms, args.steps, world), "unit": "tokens/s",
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "note": "every step copies its inputs from pinned host memory and reads its logprobs back inside "
                        "the timed region; input copies run on a copy stream into two alternating device "
                        "buffer sets, overlapping the previous step's kernels"},
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tok = 16  # about 10-15 s of single-threaded oracle work
        dt = oracle_step_sample(tok)
        line["cpu_baseline"] = {"value": tok / dt, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{tok} tokens of the step (RMSNorm, RoPE, SwiGLU, down_proj rows, "
                                          f"lm_head logprob rows), single-threaded C oracle, {dt:.1f} s",
                                **host_cpu()}
        try:  # the same oracle built with OpenMP: its GEMM outputs and logprob rows on every host core
            import oracle
            tok_all = 64
            with oracle.library(oracle.build_all_cores()):
                dt_all = oracle_step_sample(tok_all)
            threads = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
            line["cpu_baseline_all_cores"] = {
                "value": tok_all / dt_all, "unit": "tokens/s", "cores": threads,
                "kind": "oracle (same source built with -fopenmp; same bits)",
                "sample": f"{tok_all} tokens of the step, the down_proj outputs and logprob rows spread over "
                          f"{threads} threads, {dt_all:.1f} s"}
        except Exception as e:  # noqa: BLE001  (an extra figure: its failure must not cost the line)
            line["cpu_baseline_all_cores"] = {"error": f"{type(e).__name__}: {e}"[:200]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    return 0


def reductions_component(tokens, dev, stream, gamma, table, copy_gbs):
    """RMSNorm, RoPE and SwiGLU at `tokens` tokens (8192: the size their HBM
    bar is set at): each averaged over 20 back-to-back calls after 3 warm-up
    calls; every call moves more than the 126 MB L2 (268, 273 and 705 MB)."""
    import torch

    import invariant_tree_ordered_b200 as tbik

    d = synth.reduction_inputs(tokens, F=F)
    t = {k: (synth.as_torch_bf16(v) if v.dtype == np.uint16 else torch.from_numpy(v)).to(dev)
         for k, v in d.items() if k != "gamma"}
    y, ro = torch.empty_like(t["x"]), torch.empty_like(t["x"])
    qo, ko = torch.empty_like(t["q"]), torch.empty_like(t["k"])
    act = torch.empty_like(t["g"])
    calls = {
        "rmsnorm": lambda: tbik.rmsnorm_residual(t["x"], t["res"], gamma, eps=1e-6, T=1, y=y, res_out=ro,
                                                 stream=stream),
        "rope": lambda: tbik.rope_swiglu(q=t["q"], k=t["k"], pos=t["pos"], table=table, q_out=qo, k_out=ko,
                                         stream=stream),
        "swiglu": lambda: tbik.rope_swiglu(g=t["g"], u=t["u"], out=act, stream=stream),
    }
    nbytes = {"rmsnorm": 4 * tokens * H * 2,
              "rope": 2 * 2 * tokens * HEADS * HEAD_DIM * 2 + tokens * (4 + HEAD_DIM * 4),
              "swiglu": 3 * tokens * F * 2}
    out = {"tokens": tokens}
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for k, fn in calls.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(20):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / 20
        gbs = nbytes[k] / (ms * 1e-3) / 1e9
        out[k] = {"us": ms * 1e3, "gbs": gbs, "frac_of_copy_peak": gbs / copy_gbs}
    return out


def decoder_component(dev, stream):
    """The end-to-end decoder (4 layers, d 2048, 16 heads of 128, ffn 5632,
    vocab 32000, batch 8 x seq 2048): forward + target logprobs in tensor-core
    mode at T = 1 (tokens/s, CUDA events), the same with the residual add fused
    into the o and down projections, the same with the attention on the tensor
    cores, the attention kernels alone (exact order and tensor cores), the
    bitwise checks against T = 8, and the non-invariant baseline's divergence."""
    import torch

    import invariant_tree_ordered_b200 as tbik
    from invariant_tree_ordered_b200.decoder import Decoder, DecoderConfig, interleave_gate_up, positions

    cfg = synth.DECODER_FULL
    w = synth.decoder_weights(cfg)
    up = lambda a: synth.as_torch_bf16(a).to(dev)  # noqa: E731
    layers = []
    tr = lambda a: np.ascontiguousarray(a.T)  # noqa: E731  weights stored [out, in], as in nn.Linear
    for L in w["layers"]:
        dl = {k: up(tr(L[k])) for k in ("wq", "wk", "wv", "wo", "wd")}
        dl["wgu"] = up(tr(interleave_gate_up(L["wg"], L["wu"])))
        layers.append(dl)
    dc = DecoderConfig(d=cfg["d"], heads=cfg["heads"], head_dim=cfg["head_dim"], ffn=cfg["ffn"],
                       vocab=cfg["vocab"], layers=cfg["layers"], leaf=cfg["leaf"], leaf_ffn=cfg["leaf_ffn"],
                       w_out_in=True)
    dec = Decoder(dc, up(w["emb"]), up(w["lm_head"]), up(w["gamma"]), layers)
    ids_h, tg_h = synth.decoder_tokens(cfg)
    B, S = ids_h.shape
    ids = torch.from_numpy(ids_h).to(dev)
    tg = torch.from_numpy(tg_h).to(dev)
    pos = torch.from_numpy(positions(B, S)).to(dev)
    fwd = lambda **kw: dec.forward(ids, tg, pos, stream=stream, **kw)  # noqa: E731
    base = fwd(T=1, tc=True)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = 3
    a.record(stream)
    for _ in range(n):
        fwd(T=1, tc=True)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / n
    fused = fwd(T=1, tc=True, fuse_residual=True)  # residual add in the o and down projections
    a.record(stream)
    for _ in range(n):
        fwd(T=1, tc=True, fuse_residual=True)
    b.record(stream)
    torch.cuda.synchronize()
    ms_fused = a.elapsed_time(b) / n
    tca = fwd(T=1, tc=True, attention_tc=True)  # attention on the tensor cores
    a.record(stream)
    for _ in range(n):
        fwd(T=1, tc=True, attention_tc=True)
    b.record(stream)
    torch.cuda.synchronize()
    ms_tca = a.elapsed_time(b) / n
    tca8 = fwd(T=8, tc=True, attention_tc=True)
    fused8 = fwd(T=8, tc=True, fuse_residual=True)
    t8 = fwd(T=8, tc=True)
    non1, non8 = fwd(T=1, tc=True, noninv=True), fwd(T=8, tc=True, noninv=True)
    q = torch.randn(B, S, cfg["heads"], cfg["head_dim"], device=dev).to(torch.bfloat16)
    tbik.attention(q, q, q, stream=stream)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n):
        tbik.attention(q, q, q, stream=stream)
    b.record(stream)
    torch.cuda.synchronize()
    att_ms = a.elapsed_time(b) / n
    aws = torch.empty(tbik.attention_tc_workspace(B, S, cfg["heads"], cfg["head_dim"]), dtype=torch.uint8,
                      device=dev)
    tbik.attention(q, q, q, tc=True, workspace=aws, stream=stream)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n):
        tbik.attention(q, q, q, tc=True, workspace=aws, stream=stream)
    b.record(stream)
    torch.cuda.synchronize()
    att_tc_ms = a.elapsed_time(b) / n
    att_flop = 4.0 * B * cfg["heads"] * cfg["head_dim"] * (S * (S + 1) / 2)
    status = tbik.get_error(stream)
    return {"workload": "4 layers, d 2048, 16x128 heads, ffn 5632, vocab 32000, batch 8 x seq 2048, TC, T=1, "
                        "projection weights stored [out, in]",
            "tokens_per_s": B * S / (ms * 1e-3), "ms_per_forward": ms,
            "bitwise_T1_vs_T8": bool(torch.equal(base.view(torch.int32), t8.view(torch.int32))),
            "ms_per_forward_fused_residual": ms_fused,
            "fused_residual_bitwise_T1_vs_T8": bool(torch.equal(fused.view(torch.int32), fused8.view(torch.int32))),
            "noninv_max_abs_dlogprob_T8_vs_T1": float((non8 - non1).abs().max()),
            "attention_ms_per_layer": att_ms, "attention_tflops": att_flop / (att_ms * 1e-3) / 1e12,
            "tc_attention": {"tokens_per_s": B * S / (ms_tca * 1e-3), "ms_per_forward": ms_tca,
                             "bitwise_T1_vs_T8": bool(torch.equal(tca.view(torch.int32), tca8.view(torch.int32))),
                             "mean_abs_dlogprob_vs_exact_attention": float((tca - base).abs().mean()),
                             "attention_ms_per_layer": att_tc_ms,
                             "attention_tflops": att_flop / (att_tc_ms * 1e-3) / 1e12},
            "status": int(status)}


def run_profile_case(args):
    """One call of the path, repeated: the launches an ncu capture selects from."""
    import torch

    import invariant_tree_ordered_b200 as tbik

    dev = torch.device("cuda", 0)
    M = args.tokens
    if args.profile_case in ("attention", "attention-tc"):
        # decoder attention: sequences of 2048 positions, 16 heads of 128; --tokens = batch * 2048
        S, NH, D = 2048, 16, 128
        Bq = max(1, M // S)
        qkv = [synth.as_torch_bf16(synth.normal_bf16(450 + i, (Bq, S, NH, D))).to(dev) for i in range(3)]
        out = torch.empty_like(qkv[0])
        if args.profile_case == "attention":
            call = lambda: tbik.attention(*qkv, out=out)  # noqa: E731
        else:
            aws = torch.empty(tbik.attention_tc_workspace(Bq, S, NH, D), dtype=torch.uint8, device=dev)
            call = lambda: tbik.attention(*qkv, out=out, tc=True, workspace=aws)  # noqa: E731
    elif args.profile_case in ("swiglu", "rmsnorm"):
        d = synth.reduction_inputs(M, F=F)
        t = {k: synth.as_torch_bf16(d[k]).to(dev) for k in ("x", "res", "gamma", "g", "u")}
        if args.profile_case == "swiglu":
            out = torch.empty_like(t["g"])
            call = lambda: tbik.rope_swiglu(g=t["g"], u=t["u"], out=out)  # noqa: E731
        else:
            y, ro = torch.empty_like(t["x"]), torch.empty_like(t["x"])
            call = lambda: tbik.rmsnorm_residual(t["x"], t["res"], t["gamma"], eps=1e-6, y=y, res_out=ro)  # noqa: E731
    elif args.profile_case == "logprob":
        h = synth.as_torch_bf16(synth.normal_bf16(30, (M, H))).to(dev)
        w = synth.as_torch_bf16(synth.normal_bf16(31, (V, H), std=0.02)).to(dev)
        t = torch.from_numpy(synth.uniform_int32(32, M, 0, V)).to(dev)
        ws = torch.empty(tbik.logprob_workspace(M, V, H, 1, LEAF, tbik.TC), dtype=torch.uint8, device=dev)
        out = torch.empty(M, dtype=torch.float32, device=dev)
        call = lambda: tbik.logprob(h, w, t, T=1, leaf=LEAF, tc=True, out=out, workspace=ws)  # noqa: E731
    else:
        T = 8 if args.profile_case == "gemm-t8" else 1
        tc = args.profile_case != "gemm-exact"
        std = 0.02 * np.sqrt(H)
        g = synth.as_torch_bf16(synth.normal_bf16(11, (M, F), std=std)).to(dev)
        u = synth.as_torch_bf16(synth.normal_bf16(12, (M, F), std=std)).to(dev)
        a = tbik.rope_swiglu(g=g, u=u)[2]
        b = synth.as_torch_bf16(synth.down_proj_weight(F, H, "kn")).to(dev)
        mode = (tbik.TC if tc else tbik.EXACT) | tbik.OUT_BF16
        ws = torch.empty(max(tbik.gemm_workspace(M, H, F, T, LEAF, mode), 256), dtype=torch.uint8, device=dev)
        out = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
        call = lambda: tbik.gemm(a, b, T=T, leaf=LEAF, tc=tc, out_bf16=True, out=out, workspace=ws)  # noqa: E731
    call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps - 1):
        call()
    e1.record()
    torch.cuda.synchronize()
    status = tbik.get_error()
    ms = e0.elapsed_time(e1) / max(args.steps - 1, 1)
    print(f"profile case {args.profile_case}: {args.steps} calls, {ms:.3f} ms per call after the first, "
          f"status {status}", flush=True)
    return 0 if status == tbik.TBIK_OK else 1


def main():
    args = parse()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_case:
        return run_profile_case(args)
    return run_tbik(args)


if __name__ == "__main__":
    sys.exit(main())
