"""Benchmark of the fused attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one attention forward (one C-ABI `attn_fwd` launch) over the whole
workload: causal GQA attention at the LLaMA3-8B head shape, B=64, Hq=32,
Hkv=8, S=8192, D=128, fp16 in / fp32 accumulate, inputs already in HBM.
Metric: TFLOP/s = 4*B*Hq*S^2*D (halved when causal) / device time per step.
With N > 1 (torchrun, one process per GPU) every rank runs its own batch of
the same shape (weak scaling, no collective on the data path); time is the
max over ranks.  Rank 0 prints one JSON line.

Other keys: `e2e` (the same metric through the host-buffer C entry point,
H2D and D2H copies inside the timed region), `roofline` (tensor-core bound
against the measured burst bf16 GEMM peak: the kernel is timed on its own;
`traffic` is the DRAM bytes per launch of the committed ncu capture, given
only for the workload and inputs it was taken on and while the kernel
sources match it; `hbm` is the algorithmic bytes per second against the
measured copy bandwidth; `launch_ms` the mean, median, min and max launch
time), `cpu_baseline` (the fp64 oracle on a bounded sample, timed on this
host's cores), `clocks` (nvidia-smi sampled during the timed region),
`gpu_launches`, `exact_pass` (work items recomputed with hi + lo weights).

`--impl reference` times the reference arm, which for this operator is the
fp64 CPU oracle, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

NOMINAL_DENSE_FP16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "attn_fwd_llama3-8b-s8192-b64.md")
# the workload and input mix that summary's DRAM figure holds for
PROFILED_CASE = ("llama3-8b-s8192-b64", "normal")
KERNEL_SOURCES = [os.path.join(ROOT, "dnn_compiler_pipelining_b200", "csrc", f)
                  for f in ("attn_fwd_sm100.cuh", "ptx_sm100.cuh", "attn_api.cu",
                            "variant_table.inc")]
LAYER_PROFILE = os.path.join(ROOT, "profiles", "decoder_layer_llama3-8b-s8192-b1.md")
GEMM_SOURCES = [os.path.join(ROOT, "dnn_compiler_pipelining_b200", "csrc", f)
                for f in ("gemm_sm100.cuh", "ptx_sm100.cuh", "decoder_api.cu")]


def attn_flops(B, Hq, S, D, causal):
    f = 4.0 * B * Hq * S * S * D
    return f / 2 if causal else f


def n_items(w, sms=148):
    """Work items of one attn_fwd call of this workload, for the variant the
    library's table picks: 256-row items (two 128-row tiles of one head, or
    the same rows of two heads), or 128-row items for the double-buffered
    kernel and for calls whose 256-row items would leave SMs idle."""
    from dnn_compiler_pipelining_b200 import attn
    B, Hq, Hkv, S, D = w["B"], w["Hq"], w["Hkv"], w["S"], w["D"]
    var = attn.variant_select(B, Hq, Hkv, S, S, D, 1 if w["causal"] else 0)
    structure = var // 5
    n_qb = -(-S // 128)
    heads = B * Hq
    if D == 256 or structure >= 2 or heads * (-(-n_qb // 2)) < sms:
        return heads * n_qb
    if structure == 1 and (Hq // Hkv) % 2 == 0:
        return heads // 2 * n_qb
    return heads * (-(-n_qb // 2))


def launches_per_call(w, sms=148, per_cta=2048):
    """Kernel launches of one attn_fwd call: one per batch range of at most
    sms * per_cta work items (the library's split of large calls)."""
    per_b = n_items(w, sms) // w["B"]
    chunk_b = max(1, (sms * per_cta) // per_b)
    return -(-w["B"] // chunk_b)


def row_flops(n_keys, D):
    """Algorithmic FLOPs of one query row: QK^T and PV over its visible keys."""
    return 4.0 * D * n_keys


def code_tokens(text):
    """C/C++/CUDA source with comments removed and whitespace runs collapsed:
    what the compiler sees, so edits to comments or layout keep the hash."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":  # string or character literal, copied verbatim
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
            out.append(" ")
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash(sources=None):
    """Hash of the code (comments and layout ignored) of the sources that
    make the timed kernel; profiles/ records it next to the counters."""
    h = hashlib.sha256()
    for f in (sources or KERNEL_SOURCES):
        with open(f) as fh:
            h.update(code_tokens(fh.read()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def profiled_traffic(path=PROFILE_SUMMARY, sources=None):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source; else None."""
    try:
        text = open(path).read()
    except OSError:
        return None
    m_h = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]{16})", text)
    m_t = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not (m_h and m_t) or m_h.group(1) != kernel_source_hash(sources):
        return None
    return float(m_t.group(1))


def algorithmic_bytes(B, Hq, Hkv, S, D):
    """Bytes one attention call must move at the least: Q, K, V read once (fp16),
    O (fp16) and LSE (fp32) written once."""
    return 2 * S * D * (2 * B * Hq + 2 * B * Hkv) + 4 * B * Hq * S


def hbm_figure(nbytes, launch_ms, peak_gbs, peak_src):
    """The call's algorithmic bytes per second against the measured copy
    bandwidth: the bound that matters where the launch is too short for the
    tensor pipe to dominate (a single short sequence)."""
    gbs = nbytes / (launch_ms * 1e-3) / 1e9
    return {"algorithmic_bytes_per_launch": nbytes, "achieved_gbs": gbs, "peak_gbs": peak_gbs,
            "frac": gbs / peak_gbs, "peak_source": "%s HBM copy bandwidth" % peak_src}


def attn_traffic(workload, inputs):
    """The fused pass's DRAM bytes per launch for `workload` on `inputs`: the
    committed capture's figure for the case it was taken on, None for any
    other (another shape, or stress inputs whose exact pass reads K and V
    again)."""
    return profiled_traffic() if (workload, inputs) == PROFILED_CASE else None


# --------------------------------------------------------------------------- ranks
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own batch (weak scaling: independent problems)."""
    return base_seed + 1000 * rank


def reduce_max(value: float, device=None) -> float:
    """Max over ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), max=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], cap=parts[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r["power"] > 300.0] or rows
        reasons = set()
        for r in loaded:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("cap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in loaded),
                "sm_max_mhz": max(r["max"] for r in rows),
                "power_w_median": statistics.median(r["power"] for r in loaded),
                "samples": len(loaded), "reasons": sorted(reasons)}


# --------------------------------------------------------------------------- oracle timing
def oracle_sample(w, seconds: float, seed: int = 0):
    """Time the fp64 oracle on rows of the workload until about `seconds` of
    CPU work: whole batches of random rows of random heads, full K/V of their
    kv head.  Returns (flops done, seconds, rows, threads)."""
    import numpy as np
    import torch
    import oracle
    from dnn_compiler_pipelining_b200.inputs import make_qkv

    B, Hq, Hkv, S, D, causal = w["B"], w["Hq"], w["Hkv"], w["S"], w["D"], w["causal"]
    # one (b=0) slice of the workload's inputs, same recipe, on the CPU
    q, k, v = make_qkv(1, Hq, Hkv, S, D, seed=seed, device="cpu")
    qd, kd, vd = q[0].double().numpy(), k[0].double().numpy(), v[0].double().numpy()
    rng = np.random.default_rng(seed)
    group = Hq // Hkv
    flops = 0.0
    rows = 0
    t0 = time.perf_counter()
    while True:
        h = int(rng.integers(Hq))
        pos = np.sort(rng.integers(0, S, size=64)).astype(np.int64)
        oracle.attention_rows(qd[h, pos], pos, kd[h // group], vd[h // group], causal)
        flops += sum(row_flops(int(i) + 1 if causal else S, D) for i in pos)
        rows += len(pos)
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return flops, el, rows, oracle.num_threads()


def run_reference(args, w, name):
    world, rank, _ = dist_env()
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        if rank != 0:
            dist.destroy_process_group()
            return
    import oracle
    oracle.build()
    per_step = []
    tot_f = tot_t = 0.0
    rows = threads = 0
    for i in range(args.warmup + args.steps):
        f, t, r, threads = oracle_sample(w, args.ref_seconds, seed=i)
        if i >= args.warmup:
            per_step.append(t)
            tot_f += f
            tot_t += t
            rows += r
    value = tot_f / tot_t / 1e12
    sample = ("%d query rows (random heads and positions of one batch element) per step, "
              "%.1f s of fp64 oracle work per step" % (rows // max(1, args.steps), args.ref_seconds))
    line = {
        "impl": "reference",
        "metric": "attention fwd TFLOP/s (fp16, causal) and % of B200 dense tensor peak",
        "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, name, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


L2_BYTES = 126 * 2 ** 20          # B200 L2
FLUSH_BYTES = 256 * 2 ** 20       # written between timed launches when the inputs fit in L2


def input_bytes(w):
    B, Hq, Hkv, S, D = w["B"], w["Hq"], w["Hkv"], w["S"], w["D"]
    return 2 * B * S * D * (Hq + 2 * Hkv)


def needs_l2_flush(w):
    return input_bytes(w) <= 2 * L2_BYTES


INPUTS = {
    "normal": (1.0, "Q,K,V iid N(0,1) fp16, seeded per rank"),
    # the stress sweep's recipe: logits with std 16 make the softmax peaked, so
    # most rows' outputs follow single values of V and most work items meet
    # the exact pass's |O| threshold
    "stress": (4.0, "Q,K iid N(0,4^2), V iid N(0,1) fp16 (logit std 16), seeded per rank"),
}


def workload_config(w, name, n, inputs="normal"):
    return {"workload": name, "B_per_gpu": w["B"], "Hq": w["Hq"], "Hkv": w["Hkv"], "S": w["S"],
            "D": w["D"], "causal": w["causal"], "global_batch": w["B"] * n,
            "parallelism": "replicas%d" % n if n > 1 else "single",
            "l2": ("L2 flushed (256 MiB written) between timed launches; time = sum of "
                   "per-launch device times" if needs_l2_flush(w) else
                   "inputs larger than L2 (no flush needed)"),
            "inputs": INPUTS[inputs][1]}


# --------------------------------------------------------------------------- GPU arm
def run_gpu(args, w, name):
    import torch
    import torch.distributed as dist
    from dnn_compiler_pipelining_b200 import attn
    from dnn_compiler_pipelining_b200.inputs import make_qkv

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    attn.load()
    B, Hq, Hkv, S, D, causal = w["B"], w["Hq"], w["Hkv"], w["S"], w["D"], w["causal"]
    q, k, v = make_qkv(B, Hq, Hkv, S, D, seed=rank_seed(0, rank), qk_std=INPUTS[args.inputs][0],
                       device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = int(stream.cuda_stream)
    args_c = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
              B, Hq, Hkv, S, D, causal, sp)

    def step():
        st = attn.attn_fwd_raw(*args_c)
        if st != attn.ATTN_OK:
            raise attn.AttnError(st, "attn_fwd")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st, site = attn.device_status()
    if st != attn.ATTN_OK:
        raise RuntimeError("device status %d at site %#x after warm-up" % (st, site))

    # ---- timed region: K launches, per-launch events on the launching stream.
    # Inputs that fit in L2 get a 256 MiB write between launches (outside the
    # per-launch events) and the step time is the sum of launch times.
    flush = (torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
             if needs_l2_flush(w) else None)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        barrier(dev)
        torch.cuda.synchronize(dev)
        t_all0 = torch.cuda.Event(enable_timing=True)
        t_all1 = torch.cuda.Event(enable_timing=True)
        t_all0.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(float(i))
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        t_all1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(dev)
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(launch_ms) if flush is not None else t_all0.elapsed_time(t_all1)
    del flush
    st, site, exact_items = attn.device_status_ex()
    if st != attn.ATTN_OK:
        raise RuntimeError("device status %d at site %#x in the timed region" % (st, site))
    total_ms = reduce_max(total_ms, dev)
    ms_per_step = total_ms / args.steps
    flops = attn_flops(B, Hq, S, D, causal)
    value = flops * world / (ms_per_step * 1e-3) / 1e12
    clocks = clk.summary()

    # ---- e2e through the host-buffer entry point (pinned host memory)
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory()
        oh = torch.empty_like(qh).pin_memory()
        lh = torch.empty((B, Hq, S), dtype=torch.float32).pin_memory()
        del o
        ws = torch.empty(attn.host_workspace_bytes(B, Hq, Hkv, S, D), dtype=torch.uint8,
                         device=dev)
        attn.attn_fwd_host(qh, kh, vh, oh, lh, causal, ws, stream)  # warm
        barrier(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            attn.attn_fwd_host(qh, kh, vh, oh, lh, causal, ws, stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = reduce_max(e0.elapsed_time(e1) / args.e2e_steps, dev)
        h2d = (qh.numel() + kh.numel() + vh.numel()) * 2
        d2h = oh.numel() * 2 + lh.numel() * 4
        e2e = {"value": flops * world / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": args.e2e_steps, "host_memory": "pinned"}
        del ws, qh, kh, vh, oh, lh

    # ---- roofline of the one kernel (it is the whole step).  The kernel is
    # timed on its own for well under a second, so the denominator is the
    # burst GEMM figure; the sustained one (measured at a lower clock under
    # the power cap) is reported beside it.
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    avg_launch_ms = statistics.mean(launch_ms)
    achieved = flops / (avg_launch_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": attn_traffic(name, args.inputs),
                "peak_source": "%s bf16 dense GEMM, burst (fp16 has the same nominal rate)"
                               % src,
                "frac_of_sustained_peak": achieved / peak_sus,
                "frac_of_nominal_2250": achieved / NOMINAL_DENSE_FP16_TFLOPS,
                "algorithmic_flops_per_launch": flops,
                "launch_ms": {"mean": avg_launch_ms, "median": statistics.median(launch_ms),
                              "min": min(launch_ms), "max": max(launch_ms)},
                "hbm": hbm_figure(algorithmic_bytes(B, Hq, Hkv, S, D), avg_launch_ms,
                                  float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])),
                                  src)}

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        f, t, r, threads = oracle_sample(w, args.cpu_seconds)
        cpu = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": "%d query rows of one batch element (random heads and positions), "
                         "%.1f s of fp64 oracle work" % (r, t)}

    if rank == 0:
        line = {
            "metric": "attention fwd TFLOP/s (fp16, causal) and % of B200 dense tensor peak",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic", "config": workload_config(w, name, world, args.inputs),
            "e2e": e2e, "roofline": roofline, "cpu_baseline": cpu, "clocks": clocks,
            "exact_pass": {"items_per_step": exact_items / args.steps,
                           "items_per_step_of": n_items(w),
                           "note": "work items recomputed with hi+lo P because a row's "
                                   "max|O| reached the threshold (rank 0)"},
            "gpu_launches": launches_per_call(w) * args.steps,
            "pct_of_nominal_fp16_peak": 100.0 * value / world / NOMINAL_DENSE_FP16_TFLOPS,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier(dev)
        dist.destroy_process_group()


# --------------------------------------------------------------------------- decoder layer
def layer_flops(B, S, hidden, Hq, Hkv, D, inter):
    """GEMM FLOPs of one decoder layer plus its causal attention."""
    T = B * S
    gemm = 2.0 * T * hidden * ((Hq + 2 * Hkv) * D + Hq * D + 2 * inter + inter)
    return gemm + attn_flops(B, Hq, S, D, True)


def blas_threads():
    """Threads numpy's BLAS runs the oracle's matrix products on."""
    try:
        from threadpoolctl import threadpool_info
        n = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except ImportError:
        return os.cpu_count()


def layer_oracle_sample(m, seconds: float, S: int = 128, seed: int = 0):
    """Time the fp64 decoder-layer oracle on whole B=1 sequences of S tokens at
    the model's dimensions until about `seconds` of CPU work.  Returns (flops
    done, seconds, tokens)."""
    from oracle import decoder as oracle_decoder
    from dnn_compiler_pipelining_b200.inputs import make_decoder_inputs

    hidden, Hq, Hkv, D, inter = m["hidden"], m["Hq"], m["Hkv"], m["D"], m["inter"]
    x, w = make_decoder_inputs(1, S, hidden, Hq, Hkv, D, inter, seed=seed, device="cpu")
    xd = x.double().numpy()
    wd = {k: v.double().numpy() for k, v in w.items()}
    flops, tokens = 0.0, 0
    t0 = time.perf_counter()
    while True:
        oracle_decoder.decoder_layer(xd, Hq=Hq, Hkv=Hkv, D=D, eps=1e-5, theta=500000.0, **wd)
        flops += layer_flops(1, S, hidden, Hq, Hkv, D, inter)
        tokens += S
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return flops, el, tokens


def run_layer(args):
    """One LLaMA3 decoder layer (attn_decoder_layer_fwd) per step, 1 GPU; prints
    its own JSON line (not the attention headline)."""
    import torch
    from dnn_compiler_pipelining_b200 import attn
    from dnn_compiler_pipelining_b200.inputs import DECODER_MODELS, make_decoder_inputs, make_qkv

    m = DECODER_MODELS[args.layer]
    B, S = args.layer_batch, args.layer_seq
    hidden, Hq, Hkv, D, inter = m["hidden"], m["Hq"], m["Hkv"], m["D"], m["inter"]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    attn.load()
    x, w = make_decoder_inputs(B, S, hidden, Hq, Hkv, D, inter, seed=0, device=dev)
    y = torch.empty_like(x)
    ws = torch.empty(attn.decoder_layer_workspace_bytes(B, S, hidden, Hq, Hkv, D, inter),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        attn.decoder_layer_fwd(x, w, Hq, Hkv, D, y=y, workspace=ws, stream=stream)

    def timed(fn, n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n

    for _ in range(args.warmup):
        step()
    with ClockSampler(0) as clk:
        ms = timed(step, args.steps)
    clocks = clk.summary()
    st, site = attn.device_status()
    if st != attn.ATTN_OK:
        raise RuntimeError("device status %d at site %#x" % (st, site))
    # the attention alone on the same shape, for the split of the step
    q, k, v = make_qkv(B, Hq, Hkv, S, D, seed=1, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, S), dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        attn.attn_fwd(q, k, v, True, o=o, lse=lse, stream=stream)
    attn_ms = timed(lambda: attn.attn_fwd(q, k, v, True, o=o, lse=lse, stream=stream), args.steps)
    flops = layer_flops(B, S, hidden, Hq, Hkv, D, inter)
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    value = flops / (ms * 1e-3) / 1e12
    line = {
        "metric": "decoder layer fwd TFLOP/s (fp16, LLaMA3 single-layer proxy)",
        "value": value, "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic (random weights)",
        "config": {"workload": "%s-layer-s%d-b%d" % (args.layer, S, B), "B": B, "S": S,
                   "hidden": hidden, "Hq": Hq, "Hkv": Hkv, "D": D, "inter": inter,
                   "causal": True, "l2": "activations and weights larger than L2"},
        "roofline": {"bound": "tensor", "achieved": value, "peak": peak, "unit": "TFLOP/s",
                     "frac": value / peak,
                     "traffic": (profiled_traffic(LAYER_PROFILE, GEMM_SOURCES)
                                 if args.layer == "llama3-8b" and S == 8192 and B == 1 else None),
                     "traffic_of": "the gate/up GEMM (the layer's largest kernel), one launch, "
                                   "DRAM read + write from the committed ncu capture",
                     "peak_source": "%s bf16 dense GEMM, sustained (the layer runs for several ms "
                                    "per step, back to back)" % src,
                     "algorithmic_flops_per_step": flops},
        "split": {"attention_ms": attn_ms, "rest_ms": ms - attn_ms,
                  "attention_flops": attn_flops(B, Hq, S, D, True)},
        "clocks": clocks,
        # per step: rope table, 2 RMSNorm, the attention, 4 GEMMs with fused
        # epilogues (and a head merge when S is not a multiple of 128)
        "gpu_launches": (8 + (1 if S % 128 else 0)) * args.steps, "library_gemm_calls": 0,
    }
    if not args.no_cpu_baseline:
        f, t, n = layer_oracle_sample(m, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": f / t / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": "%d tokens in whole 128-token sequences (B=1) at the model's dimensions, "
                      "%.1f s of fp64 oracle work (numpy BLAS threads)" % (n, t)}
    print(json.dumps(line), flush=True)


def main(argv=None):
    from dnn_compiler_pipelining_b200.inputs import WORKLOADS
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3-8b-s8192-b64", choices=sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--inputs", choices=sorted(INPUTS), default="normal",
                    help="input distribution: normal (N(0,1)) or stress (logit std 16)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-seconds", type=float, default=8.0)
    ap.add_argument("--layer", choices=["llama3-8b", "llama3-70b"], default=None,
                    help="time the decoder-layer proxy instead of the attention headline")
    ap.add_argument("--layer-batch", type=int, default=1)
    ap.add_argument("--layer-seq", type=int, default=8192)
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be at least 3")
    w = WORKLOADS[args.workload]
    if args.layer is not None:
        if args.impl != "ours":
            ap.error("--layer times this library only")
        run_layer(args)
    elif args.impl == "reference":
        run_reference(args, w, args.workload)
    else:
        run_gpu(args, w, args.workload)


if __name__ == "__main__":
    main()
