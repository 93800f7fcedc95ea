"""Profile-guided choice of the fused-kernel variant, per shape class.

Times every compiled variant of the fused kernel (attn_variant_count(): four
pipeline structures -- the two-tile ping-pong over two row blocks of one
query head or over the same rows of two query heads of a group, and one tile
with S double-buffered in TMEM with one or two softmax warps per lane
quadrant -- times how many exponentials the FMA-pipe polynomial takes from
the MUFU unit) on the current GPU over a grid of shape classes, and writes the rule table that libattn_b200.so compiles in
(csrc/variant_table.inc).  This is the
pages' search-with-profile-feedback idea (PipeThreader, sections 核心方法 and
设计取舍) reduced to a handful of candidates chosen once per GPU model.

    python -m dnn_compiler_pipelining_b200.tune --table OUT.inc --report OUT.md

Then copy OUT.inc over csrc/variant_table.inc and rebuild.  Every launch goes
through the library's C ABI (attn_fwd_variant); nothing here computes
attention.
"""
from __future__ import annotations

import argparse
import math
import statistics
import time

import torch

from . import attn

HEAD_SHAPE = (32, 8)           # Hq, Hkv: the LLaMA3-8B head shape
SEQS = (512, 1024, 2048, 4096, 8192)
HEAD_DIMS = (128, 64, 256)
TOKENS = 16 * 8192             # B * S per timed launch: Q alone is 1 GiB at D = 128 (> L2)
MARGIN = 0.02                  # a variant must beat variant 0 by this fraction to be chosen
O_AGREE = 2e-3                 # every variant's O must agree with variant 0's within this


def flops(B, Hq, S, D, causal):
    f = 4.0 * B * Hq * S * S * D
    return f / 2 if causal else f


def time_class(D, causal, S, reps, warmup, seed=0):
    """Median device time (ms) of one attn_fwd_variant call, per variant."""
    Hq, Hkv = HEAD_SHAPE
    B = max(1, TOKENS // S)
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((B, Hq, S, D), generator=g, device="cuda", dtype=torch.float16)
    k = torch.randn((B, Hkv, S, D), generator=g, device="cuda", dtype=torch.float16)
    v = torch.randn((B, Hkv, S, D), generator=g, device="cuda", dtype=torch.float16)
    n = attn.variant_count()
    # head dimension 256 has one pipeline structure: variants v and v + 5k
    # run the same kernel there, so only the first five are timed
    timed = range(5) if D == 256 else range(n)
    outs = [(torch.empty_like(q), torch.empty((B, Hq, S), device="cuda", dtype=torch.float32))
            for _ in range(n)]
    for var in timed:
        for _ in range(warmup):
            attn.attn_fwd_variant(q, k, v, causal, var, o=outs[var][0], lse=outs[var][1])
    torch.cuda.synchronize()
    times = [[] for _ in range(n)]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    for _ in range(reps):
        for var in timed:  # interleaved, so clock drift hits every variant alike
            ev[0].record()
            attn.attn_fwd_variant(q, k, v, causal, var, o=outs[var][0], lse=outs[var][1])
            ev[1].record()
            ev[1].synchronize()
            times[var].append(ev[0].elapsed_time(ev[1]))
    st, site = attn.device_status()
    if st != attn.ATTN_OK:
        raise RuntimeError("device status %s (site %#x) for D=%d causal=%d S=%d"
                           % (attn.STATUS_NAMES.get(st), site, D, causal, S))
    o0, l0 = outs[0]
    agree = []
    for var in range(n):
        if var not in timed:
            agree.append(False)
            continue
        do = (outs[var][0].float() - o0.float()).abs().max().item()
        dl = (outs[var][1] - l0).abs().max().item()
        agree.append(do <= O_AGREE and dl <= 1e-3 and math.isfinite(do) and math.isfinite(dl))
    med = [statistics.median(t) if t else float("inf") for t in times]
    return B, med, agree


def choose(med, agree):
    """Variant 0 unless another (that agrees with it) is faster by MARGIN."""
    best = 0
    for var in range(1, len(med)):
        if agree[var] and med[var] < med[best] and med[var] < med[0] * (1 - MARGIN):
            best = var
    return best


def rules_for(choices):
    """[(S, variant)] over ascending S -> [(sk_lo, sk_hi, variant)]: each
    measured S owns the keys from the geometric midpoint with its lower
    neighbour up to the one with its upper neighbour; runs of one variant
    merge."""
    out = []
    for i, (s, var) in enumerate(choices):
        lo = 1 if i == 0 else int(math.floor(math.sqrt(choices[i - 1][0] * s))) + 1
        hi = (2 ** 31 - 1) if i == len(choices) - 1 else int(math.floor(math.sqrt(s * choices[i + 1][0])))
        if out and out[-1][2] == var:
            out[-1] = (out[-1][0], hi, var)
        else:
            out.append((lo, hi, var))
    return out


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--table", required=True, help="where to write the VARIANT_RULE table")
    ap.add_argument("--report", required=True, help="where to write the timing report (markdown)")
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=2)
    args = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("tune: needs a CUDA device (sm_100)")
    n = attn.variant_count()
    names = [attn.variant_name(i) for i in range(n)]
    props = torch.cuda.get_device_properties(0)

    def run_name(var, D):
        # at D = 256 every structure runs the double-buffered kernel
        # (structure 2), so variant v runs what variant 10 + v % 5 names
        return names[10 + var % 5] if D == 256 and n >= 15 else names[var]

    t0 = time.time()
    lines = ["| D | causal | S | B | " + " | ".join("%s TFLOP/s" % nm for nm in names)
             + " | chosen |", "|" + "---|" * (n + 5)]
    table_rules = []
    for D in HEAD_DIMS:
        for causal in (1, 0):
            choices = []
            for S in SEQS:
                B, med, agree = time_class(D, causal, S, args.reps, args.warmup)
                var = choose(med, agree)
                choices.append((S, var))
                tf = [flops(B, HEAD_SHAPE[0], S, D, causal) / (m * 1e-3) / 1e12 for m in med]
                tf = [t if t > 0 else float("nan") for t in tf]
                timed = range(5) if D == 256 else range(n)
                cells = ["%.1f%s" % (t, "" if ok else " (disagrees)") if v in timed
                         else "= v%d" % (v % 5) for v, (t, ok) in enumerate(zip(tf, agree))]
                lines.append("| %d | %d | %d | %d | %s | %s |" % (D, causal, S, B,
                                                                  " | ".join(cells),
                                                                  run_name(var, D)))
                print(lines[-1], flush=True)
            for lo, hi, var in rules_for(choices):
                table_rules.append((D, causal, lo, hi, var))
    head = ("// Fused-kernel variant per shape class: VARIANT_RULE(D, causal, smallest Sk,\n"
            "// largest Sk, variant index); first match wins, no match ->\n"
            "// variant 0.  Written by `python -m dnn_compiler_pipelining_b200.tune` on\n"
            "// %s (%d SMs): median of %d interleaved launches per variant, Hq=%d,\n"
            "// Hkv=%d, B*S=%d; a variant replaces 0 only when %.0f%% faster.\n"
            % (props.name, props.multi_processor_count, args.reps, HEAD_SHAPE[0], HEAD_SHAPE[1],
               TOKENS, MARGIN * 100))
    with open(args.table, "w") as f:
        f.write(head)
        for r in table_rules:
            f.write("VARIANT_RULE(%d, %d, %d, %d, %d)  // %s\n" % (r + (run_name(r[4], r[0]),)))
    with open(args.report, "w") as f:
        f.write("# Fused-pass variant timings (%s, %d SMs)\n\n" % (props.name,
                                                                props.multi_processor_count))
        f.write("Median of %d interleaved calls per variant (one launch each, exact pass "
                "included; CUDA events), Q/K/V iid N(0,1) fp16, Hq=%d, Hkv=%d, B*S=%d; %.0f s. "
                "At D = 256 every structure runs the double-buffered kernel, so only variants "
                "0-4 are timed there (\"= vN\": the same kernel as variant N).\n\n"
                % (args.reps, HEAD_SHAPE[0], HEAD_SHAPE[1], TOKENS, time.time() - t0))
        f.write("\n".join(lines) + "\n")
    print("wrote %s and %s" % (args.table, args.report))


if __name__ == "__main__":
    main()
