"""Device timeline of one denoising step (the library built with DLM_TRACE).

    python -m masked_block_diffusion_denoise_b200.trace [--workload 8b_b1] [--blocks 3]
                                                        [--json FILE] [--md FILE]

Builds libdlm_trace.so, runs whole blocks of the workload as CUDA-graph
replays and reports, for the last step of the last block, every kernel's CTA
entry, programmatic-launch wait and exit, and its phase marks, in
microseconds from the step's first CTA entry (the embedding kernel), read
from the GPU's global timer.  The trace build adds a few stores per CTA: its
times show where a step's time goes; the benchmark's numbers come from the
default library.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np

KINDS = ["embed", "qkv_gemm", "qkv_epilogue", "attention", "attn_combine", "wo_gemm",
         "wo_epilogue", "quantize", "lm_head", "commit"]
_GEMM = {3: "first stage full", 4: "last stage full", 5: "first accumulator ready",
         6: "last epilogue done"}
PHASES = {
    "qkv_gemm": _GEMM, "wo_gemm": _GEMM, "lm_head": _GEMM,
    "attention": {3: "query + first K/V tile", 4: "O complete", 5: "cluster barrier",
                  6: "peers' rows received", 7: "combined"},
    "commit": {3: "rows reduced", 4: "keys sorted", 5: "done"},
}


def _summary(table: np.ndarray) -> dict:
    """Per kind: CTA count, entry / wait / exit and phase marks (us from the
    step's first CTA entry; min, median, max over the CTAs)."""
    live = {}
    for k, name in enumerate(KINDS):
        rows = table[k]
        rows = rows[rows[:, 0] > 0]
        if len(rows):
            live[name] = rows
    if "embed" not in live:
        raise RuntimeError("no embedding kernel in the trace")
    t0 = int(live["embed"][:, 0].min())

    def stats(v):
        v = v[v > 0]
        if not len(v):
            return None
        x = (v.astype(np.int64) - t0) / 1e3
        return {"min": round(float(x.min()), 2), "med": round(float(np.median(x)), 2),
                "max": round(float(x.max()), 2)}

    out = {"kernels": {}, "order": [n for n in KINDS if n in live]}
    for name, rows in live.items():
        rec = {"ctas": int(len(rows)), "entry": stats(rows[:, 0]), "exit": stats(rows[:, 1]),
               "wait": stats(rows[:, 2]), "phases": {}}
        for slot, label in PHASES.get(name, {}).items():
            s = stats(rows[:, slot])
            if s is not None:
                rec["phases"][label] = s
        out["kernels"][name] = rec
    last = out["order"][-1]
    out["step_span_us"] = out["kernels"][last]["exit"]["max"]
    return out


def collect(workload: str, blocks: int) -> dict:
    from . import build as B
    os.environ["DLM_LIBRARY"] = B.build(trace=True)
    import torch
    from . import dlm_trace_clear, dlm_trace_layout, dlm_trace_read
    from .session import Session, sampler_params
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import workloads as W

    dlm_trace_layout()   # raises unless the trace build was loaded

    wl = W.WORKLOADS[workload]
    sh = wl.shape
    weights = W.make_weights(sh, seed=wl.seed)
    lens, toks, kp, vp = W.make_prefix(wl)
    sess = Session(sh, weights, max_batch=wl.batch, max_prefix=wl.prefix_cap,
                   max_canvas=wl.canvas)
    try:
        for b in range(wl.batch):
            if toks is not None:
                sess.kv_append_tokens(b, toks[b])
            else:
                n = int(lens[b])
                sess.kv_append_kv(b, np.ascontiguousarray(kp[b][:, :n]),
                                  np.ascontiguousarray(vp[b][:, :n]))
        p = sampler_params(canvas=wl.canvas, steps=wl.steps, threshold=wl.threshold,
                           quota=wl.quota, corruption=wl.corruption,
                           entropy_bound=wl.entropy_bound, temperature=wl.temperature,
                           t_max=wl.t_max, t_min=wl.t_min, seed=wl.seed)
        cv = sess.new_canvas(wl.batch, wl.canvas)
        table = None
        for _ in range(blocks):
            sess.init(cv, p)
            torch.cuda.synchronize()
            dlm_trace_clear()
            sess.block(cv, p)
            sess.check()
            table = dlm_trace_read()
    finally:
        sess.close()
    out = _summary(table)
    out["workload"] = workload
    out["blocks"] = blocks
    return out


def markdown(s: dict) -> str:
    lines = ["| kernel | CTAs | entry (min / med / max) | wait (med) | exit (med / max) |",
             "|---|---|---|---|---|"]
    for name in s["order"]:
        k = s["kernels"][name]
        e, w, x = k["entry"], k["wait"], k["exit"]
        lines.append("| %s | %d | %.2f / %.2f / %.2f | %s | %.2f / %.2f |" % (
            name, k["ctas"], e["min"], e["med"], e["max"],
            "%.2f" % w["med"] if w else "-", x["med"], x["max"]))
    lines.append("")
    lines.append("Phase marks (median over the CTAs, max in brackets):")
    lines.append("")
    for name in s["order"]:
        ph = s["kernels"][name]["phases"]
        if ph:
            lines.append("- %s: " % name + "; ".join(
                "%s %.2f (%.2f)" % (lab, v["med"], v["max"]) for lab, v in ph.items()))
    lines.append("")
    lines.append("Step span (first embedding CTA in to last commit CTA out): %.2f us"
                 % s["step_span_us"])
    return "\n".join(lines)


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--workload", default="8b_b1")
    ap.add_argument("--blocks", type=int, default=3)
    ap.add_argument("--json", default=None, help="write the summary as JSON")
    ap.add_argument("--md", default=None, help="write the summary as a markdown table")
    a = ap.parse_args()
    s = collect(a.workload, a.blocks)
    text = markdown(s)
    print(text)
    if a.json:
        with open(a.json, "w") as f:
            json.dump(s, f, indent=1)
    if a.md:
        with open(a.md, "w") as f:
            f.write(text + "\n")


if __name__ == "__main__":
    main()
