#!/usr/bin/env python
"""Throughput of the masked block-diffusion denoise step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload batched]
    python bench.py --impl reference ...        # the CPU oracle, same line format

One "step" is one denoising step over the whole batch: embed, QKV + RoPE,
attention, output projection, fused LM-head reduction, cross-tile reduce,
commit / re-noise.  The default workload is the batched-serving shape (16
canvases of 64 positions over prefixes of 1024-4096 keys, the 8B-class
model), the largest single-GPU configuration.  Steps run as CUDA-graph
replays: K steps are K // S whole blocks (``dlm_decode_block``, S steps each,
every block from the same initial canvas) and the first K % S steps of one
more block as one graph (``dlm_decode_steps``).  W warm-up steps (at least
3) run the same way first; the graphs of the timed region are captured
before it by one replay over finished canvases, which does no work.  K steps
are timed with CUDA events on the launch stream between a barrier and device
synchronisation on both sides; with N ranks each rank decodes its own batch
(weak scaling, no collective on the data path) and the time is the maximum
over ranks.  Rank 0 prints one JSON line.

Besides the headline, the line carries: the LM head's roofline (HBM- or
tensor-bound, by its arithmetic intensity) from CUDA events recorded around
its launches inside the replayed graph; the attention + reduce/commit stages'
achieved HBM bandwidth; ``e2e``, the same metric through the host-buffer
entry point (``dlm_decode_block_host``: canvas state copied in and out every
block, inside the timed region); and, at N = 1, ``configs``: one block of
every other workload measured the same way.

Inputs exceed L2: the LM head streams its 1.07 GB weight every step, so no
L2 flush is needed between steps.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402
from masked_block_diffusion_denoise_b200 import roofline as RL  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=320)
    ap.add_argument("--warmup", type=int, default=32)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="batched", choices=sorted(W.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload map of the other configurations")
    ap.add_argument("--profile", action="store_true",
                    help="a few eager steps only, for ncu captures")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        p["source"] = "measured"
        return p
    except Exception:
        return dict(FALLBACK_PEAKS)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_init(n_gpus, backend="nccl"):
    """One process per GPU (RANK / LOCAL_RANK / WORLD_SIZE from the launcher);
    returns (world, rank, local_rank, torch.distributed or None)."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus and world > 1:
        raise SystemExit("WORLD_SIZE %d != --gpus %d" % (world, n_gpus))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
        pg = dist
    return world, rank, local, pg


def barrier(pg, device):
    """All ranks meet, then the device drains (the same collective on every rank)."""
    import torch
    if pg is not None:
        t = torch.zeros(1, device=device)
        pg.all_reduce(t)
    if device.type == "cuda":
        torch.cuda.synchronize(device)


def max_over_ranks(pg, value, device):
    import torch
    if pg is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world, units_per_rank, ms_max):
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return world * units_per_rank / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def workload_config(workload, wl, lens, world):
    """The `config` object of the JSON line (the same for both arms)."""
    sh = wl.shape
    return {"workload": workload, "batch": wl.batch, "canvas": wl.canvas,
            "prefix": [int(min(lens)), int(max(lens))], "steps_per_block": wl.steps,
            "threshold": wl.threshold, "quota": wl.quota_eff, "corruption": wl.corruption,
            "d_model": sh.d_model, "heads": [sh.n_heads, sh.n_kv_heads, sh.head_dim],
            "vocab": sh.vocab, "parallelism": "replicas" if world > 1 else "single",
            "l2": "inputs larger than L2 (the LM head streams 1.07 GB of weights every step); "
                  "no flush"}


class Runner:
    """One workload on one GPU: a library session with the workload's
    weights and prefixes, a template canvas (initial state plus EOS plant)
    and the working canvas the steps update."""

    def __init__(self, wl, device, upload=None):
        import torch
        from masked_block_diffusion_denoise_b200.session import Session, sampler_params
        self.torch = torch
        self.wl = wl
        sh = wl.shape
        weights = W.make_weights(sh, seed=wl.seed) if upload is None else None
        lens, toks, kp, vp = W.make_prefix(wl)
        self.lens = [int(x) for x in lens]
        self.sess = Session(sh, weights, max_batch=wl.batch, max_prefix=wl.prefix_cap,
                            max_canvas=wl.canvas, device=device, upload=upload)
        del weights
        for b in range(wl.batch):
            if toks is not None:
                self.sess.kv_append_tokens(b, toks[b])
            else:
                n = int(lens[b])
                self.sess.kv_append_kv(b, np.ascontiguousarray(kp[b][:, :n]),
                                       np.ascontiguousarray(vp[b][:, :n]))
        del kp, vp
        self.p = sampler_params(canvas=wl.canvas, steps=wl.steps, threshold=wl.threshold,
                                quota=wl.quota, corruption=wl.corruption,
                                entropy_bound=wl.entropy_bound, temperature=wl.temperature,
                                t_max=wl.t_max, t_min=wl.t_min, seed=wl.seed)
        self.S = wl.steps
        self.stream = torch.cuda.Stream(device)
        self.tmpl = self.sess.new_canvas(wl.batch, wl.canvas)
        with torch.cuda.stream(self.stream):
            self.sess.init(self.tmpl, self.p, stream=self.stream)
            for (b, slot) in W.make_eos_plant(wl):
                self.tmpl.tokens[b, slot] = sh.eos_id
                self.tmpl.committed[b, slot] = 1
        self.stream.synchronize()
        self.cv = self.sess.new_canvas(wl.batch, wl.canvas)

    def reset(self, finished=False):
        """The working canvas back to the initial state (or every canvas
        marked done, so that a replay does no work)."""
        c, t = self.cv, self.tmpl
        for dst, src in ((c.tokens, t.tokens), (c.committed, t.committed), (c.step, t.step),
                         (c.done, t.done), (c.eos_pos, t.eos_pos)):
            dst.copy_(src, non_blocking=True)
        if finished:
            c.done.fill_(1)

    def run(self, k):
        """k steps: whole blocks, then the first k % S steps of one more
        block, each a graph replay from the initial canvas."""
        import masked_block_diffusion_denoise_b200 as dlm
        full, rest = divmod(k, self.S)
        st = self.stream
        with self.torch.cuda.stream(st):
            for _ in range(full):
                self.reset()
                self.sess.block(self.cv, self.p, stream=st)
            if rest:
                self.reset()
                dlm.dlm_decode_steps(self.sess.ctx, self.cv.c, self.wl.batch, self.p, rest,
                                     stats=self.cv.stats, stream=st)

    def capture(self, k):
        """Capture (and replay over finished canvases) the graphs run(k) uses."""
        import masked_block_diffusion_denoise_b200 as dlm
        full, rest = divmod(k, self.S)
        st = self.stream
        with self.torch.cuda.stream(st):
            for n in ([self.S] if full else []) + ([rest] if rest else []):
                self.reset(finished=True)
                dlm.dlm_decode_steps(self.sess.ctx, self.cv.c, self.wl.batch, self.p, n,
                                     stats=self.cv.stats, stream=st)
        st.synchronize()

    def timed(self, k):
        """Device time (ms) of run(k) on the launch stream."""
        torch = self.torch
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        self.run(k)
        e1.record(self.stream)
        self.stream.synchronize()
        return e0.elapsed_time(e1)

    def stage_us(self, stage, n_blocks):
        """Mean duration (us) of one stage over the S steps of a block, from
        events recorded around it inside the replayed graph (after n_blocks
        blocks of replays, the last one read)."""
        import masked_block_diffusion_denoise_b200 as dlm
        torch = self.torch
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * self.S)]
        for e in evs:            # torch creates the CUDA event on its first record
            e.record(self.stream)
        self.stream.synchronize()
        dlm.dlm_set_stage_events(self.sess.ctx, stage, [e.cuda_event for e in evs])
        self.run(n_blocks * self.S)
        self.stream.synchronize()
        dlm.dlm_set_stage_events(self.sess.ctx, 0, [])
        return [1e3 * evs[2 * i].elapsed_time(evs[2 * i + 1]) for i in range(self.S)]

    def plan(self):
        import masked_block_diffusion_denoise_b200 as dlm
        if self.wl.shape.dtype != "bf16":
            return None
        return dlm.dlm_attention_plan(self.sess.ctx, self.wl.batch, self.wl.canvas)

    def close(self):
        self.sess.close()


STAGES = ["embed", "qkv", "attention", "wo", "lm_head", "reduce+commit"]


def kernel_figures(r, pk, n_blocks):
    """Per-stage event times of one block and the rooflines they give: the
    LM head against HBM or the bf16 tensor peak (by its arithmetic
    intensity), attention + reduce/commit against HBM."""
    wl = r.wl
    sh = wl.shape
    # a stage of a finished canvas does no work: average over the steps in
    # which every canvas was still active (the first steps of the block)
    times = {name: r.stage_us(i, n_blocks) for i, name in enumerate(STAGES)}
    n_full = r.S
    for (b, slot) in W.make_eos_plant(wl):
        # the `slot` positions before a planted EOS take ceil(slot / quota) steps
        n_full = min(n_full, max(1, -(-slot // max(1, wl.quota_eff))))
    mean = {k: statistics.mean(v[:n_full]) for k, v in times.items()}
    lm_fp8 = bool(getattr(sh, "lm_fp8", False))
    lm_nvfp4 = bool(getattr(sh, "lm_nvfp4", False))
    es = 2 if sh.dtype == "bf16" else 4
    shape = RL.StepShape(sh.d_model, sh.n_heads, sh.n_kv_heads, sh.head_dim, sh.vocab, es,
                         wl.canvas, r.lens)
    work = RL.step_work(shape, lm_tile=128 if wl.batch * wl.canvas <= 128 or lm_nvfp4 else 256,
                        lm_elem_bytes=1 if lm_fp8 else 0, lm_nvfp4=lm_nvfp4)
    out = {"stages_us": {k: round(v, 2) for k, v in mean.items()},
           "steps_averaged": n_full, "step_algorithmic_bytes": work["step"]["bytes"]}
    if sh.dtype != "bf16":
        return out, None
    lm_s = mean["lm_head"] / 1e6
    intensity = work["lm_head"]["flop"] / work["lm_head"]["bytes"]
    if intensity < 250:
        ach, peak, unit, bound = work["lm_head"]["bytes"] / lm_s / 1e9, pk["hbm_gbs"], "GB/s", "hbm"
        src = " hbm_gbs"
    else:
        ratio = 4 if lm_nvfp4 else (2 if lm_fp8 else 1)
        peak = pk.get("bf16_tflops_sustained", pk["bf16_tflops"]) * ratio
        ach, unit, bound = work["lm_head"]["flop"] / lm_s / 1e12, "TFLOP/s", "tensor"
        src = " bf16_tflops_sustained" + (
            " x %d (%s : bf16 nominal ratio)" % (ratio, "nvfp4" if lm_nvfp4 else "e4m3")
            if ratio > 1 else "")
    roof = {"kernel": "gemm_tc_kernel<EPI_LM%s> (LM head + fused vocab reduction)"
                      % (", nvfp4" if lm_nvfp4 else (", e4m3" if lm_fp8 else "")),
            "bound": bound, "achieved": round(ach, 1), "peak": peak, "unit": unit,
            "frac": round(ach / peak, 4), "traffic": _ncu_traffic(wl.name),
            "peak_source": pk.get("source", "measured") + src,
            "launch_us": round(mean["lm_head"], 2),
            "algorithmic_bytes_per_launch": work["lm_head"]["bytes"],
            "algorithmic_flop_per_launch": work["lm_head"]["flop"],
            "launches_timed": n_full}
    ac_bytes = work["attention"]["bytes"] + work["reduce"]["bytes"] + work["commit"]["bytes"]
    ac_s = (mean["attention"] + mean["reduce+commit"]) / 1e6
    out["attention_commit"] = {
        "bound": "hbm", "bytes": ac_bytes, "us": round(ac_s * 1e6, 2),
        "achieved_gbs": round(ac_bytes / ac_s / 1e9, 1), "peak": pk["hbm_gbs"],
        "frac": round(ac_bytes / ac_s / 1e9 / pk["hbm_gbs"], 4),
        "attention_gbs": round(work["attention"]["bytes"] / (mean["attention"] / 1e6) / 1e9, 1),
        "attention_frac": round(work["attention"]["bytes"] / (mean["attention"] / 1e6) / 1e9
                                / pk["hbm_gbs"], 4)}
    return out, roof


def run_ours(a):
    import torch
    import masked_block_diffusion_denoise_b200 as dlm
    from masked_block_diffusion_denoise_b200 import build as B

    world, rank, local, pg = dist_init(a.gpus)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if rank == 0:
        B.build()
    if pg is not None:
        barrier(pg, device)
    wl = W.WORKLOADS[a.workload]
    sh = wl.shape
    r = Runner(wl, device)
    S = wl.steps

    if a.profile:
        with torch.cuda.stream(r.stream):
            r.reset()
            for _ in range(max(1, a.steps)):
                r.sess.step(r.cv, r.p, stream=r.stream)
        r.stream.synchronize()
        r.sess.check(r.stream)
        if rank == 0:
            print(json.dumps({"profile": a.workload, "steps": a.steps}))
        return

    K, Wm = a.steps, max(a.warmup, 3)
    r.run(Wm)                       # warm-up, the same graph replays as the timed steps
    r.stream.synchronize()
    r.capture(K)                    # the timed region's graphs, before it
    r.sess.check(r.stream)
    launches_per_step = dlm.dlm_launches_per_step(r.sess.ctx)

    # ---- timed region ----
    clocks = Clocks(local) if rank == 0 else None
    r.cv.stats.zero_()
    barrier(pg, device)
    if clocks:
        clocks.start()
        time.sleep(0.3)
    barrier(pg, device)
    ms = r.timed(K)
    barrier(pg, device)
    ck = clocks.stop() if clocks else None
    r.sess.check(r.stream)
    ms_max = max_over_ranks(pg, ms, device)
    committed = int(r.cv.stats[:, 1].sum().item())
    committed_all = max_over_ranks(pg, committed, device) * world

    # ---- per-stage events inside the replayed graph ----
    pk = peaks()
    figs, roof = kernel_figures(r, pk, n_blocks=max(2, min(10, K // S)))

    # ---- end to end through the host-buffer entry point ----
    e2e = None
    if not a.no_e2e:
        host = {k: getattr(r.tmpl, k).cpu().pin_memory() for k in
                ("tokens", "committed", "step", "done", "eos_pos")}
        hstats = torch.zeros((wl.batch, 6), dtype=torch.int32).pin_memory()
        work = {k: v.clone().pin_memory() for k, v in host.items()}
        n_blocks = max(3, K // S)
        h2d = sum(v.numel() * v.element_size() for v in host.values()) + hstats.numel() * 4
        d2h = h2d

        def host_block():
            for k in work:
                work[k].copy_(host[k])
            dlm.dlm_decode_block_host(r.sess.ctx, work["tokens"], work["committed"],
                                      work["step"], work["done"], work["eos_pos"], wl.batch,
                                      r.p, stats=hstats, stream=r.stream)
        host_block()                # warm: the entry point's graph is captured here
        hstats.zero_()
        barrier(pg, device)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(r.stream)
        for _ in range(n_blocks):
            host_block()
        f1.record(r.stream)
        r.stream.synchronize()
        e2e_ms = max_over_ranks(pg, f0.elapsed_time(f1), device)
        e2e = {"value": round(world * n_blocks * S / (e2e_ms / 1e3), 2), "unit": "steps/s",
               "h2d_bytes_per_step": h2d / S, "d2h_bytes_per_step": d2h / S,
               "blocks": n_blocks, "call": "dlm_decode_block_host",
               "committed_tokens_per_s": round(
                   world * float(hstats[:, 1].sum().item()) / (e2e_ms / 1e3), 1)}
    plan = r.plan()

    line = None
    if rank == 0:
        step_s = ms_max / 1e3 / K
        line = {
            "metric": "denoise steps/s", "value": round(aggregate_rate(world, K, ms_max), 2),
            "unit": "steps/s", "n_gpus": world, "steps": K, "warmup": Wm,
            "ms_per_step": round(ms_max / K, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": ("bf16, LM head nvfp4" if getattr(sh, "lm_nvfp4", False) else
                      ("bf16, LM head e4m3" if getattr(sh, "lm_fp8", False) else "bf16"))
                     if sh.dtype == "bf16" else "f32",
            "data": "synthetic: seeded random-init weights N(0,0.02), embeddings and prefix "
                    "K/V N(0,1), all-mask canvas",
            "config": workload_config(a.workload, wl, r.lens, world),
            "committed_tokens_per_s": round(committed_all / (ms_max / 1e3), 1),
            "timing": "%d whole-block graph replays + one graph of %d steps, every block from "
                      "the initial canvas" % divmod(K, S),
            "stages_us": figs["stages_us"],
            "stages_steps_averaged": figs["steps_averaged"],
            "step_algorithmic_bytes": figs["step_algorithmic_bytes"],
            "step_hbm_frac": round(figs["step_algorithmic_bytes"] / step_s / 1e9
                                   / pk["hbm_gbs"], 4),
            "attention_commit": figs.get("attention_commit"),
            "attention_plan": plan,
            "roofline": roof,
            "gpu_launches": int(launches_per_step * K),
            "e2e": e2e,
            "clocks": ck,
        }
    r.close()
    del r
    torch.cuda.empty_cache()
    if rank == 0:
        if world == 1 and not a.no_configs:
            line["configs"] = measure_configs(a.workload, device, pk)
        if world == 1 and not a.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl)
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


CONFIG_WORKLOADS = ["tiny", "8b_b1", "batched", "longctx", "encdec", "encdec_eb",
                    "8b_b1_fp8", "8b_b1_nvfp4"]


def measure_configs(skip, device, pk):
    """One block (S steps, graph replay, after one warm-up block) of every
    configuration, with its stage rooflines; weights are drawn once per
    model shape."""
    import torch
    out = {}
    uploads = {}
    for name in CONFIG_WORKLOADS:
        if name == skip:
            out[name] = "the headline line"
            continue
        wl = W.WORKLOADS[name]
        # the low-bit LM-head variants share the model's weights
        key = (dataclasses.replace(wl.shape, lm_fp8=False, lm_nvfp4=False), wl.seed)
        if key not in uploads:
            from masked_block_diffusion_denoise_b200.session import host_to_device
            uploads.clear()
            torch.cuda.empty_cache()
            w = W.make_weights(wl.shape, seed=wl.seed)
            uploads[key] = {k: host_to_device(v, wl.shape.dtype, device) for k, v in w.items()}
            del w
        r = Runner(wl, device, upload=uploads[key])
        try:
            S = wl.steps
            r.run(S)
            r.stream.synchronize()
            r.cv.stats.zero_()
            ms = r.timed(S)
            r.sess.check(r.stream)
            committed = int(r.cv.stats[:, 1].sum().item())
            figs, roof = kernel_figures(r, pk, n_blocks=2)
            entry = {"steps_per_s": round(S / (ms / 1e3), 2), "ms_per_step": round(ms / S, 5),
                     "committed_tokens_per_s": round(committed / (ms / 1e3), 1),
                     "stages_us": figs["stages_us"]}
            if roof is not None:
                entry["lm_head"] = {k: roof[k] for k in ("bound", "achieved", "peak", "unit",
                                                         "frac", "launch_us", "traffic")}
                entry["attention_commit"] = figs["attention_commit"]
                entry["attention_plan"] = r.plan()
            out[name] = entry
        finally:
            r.close()
    uploads.clear()
    torch.cuda.empty_cache()
    return out


def _ncu_traffic(workload):
    """DRAM bytes per LM-head launch from the committed ncu summary, if it
    describes this workload and the kernel sources have not changed since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "lm_head_%s.json" % workload)
    try:
        with open(path) as f:
            d = json.load(f)
        h = hashlib.sha256()
        for src in d["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        return d["dram_bytes_per_launch"] if h.hexdigest() == d["source_sha256"] else None
    except Exception:
        return None


# ---------------------------------------------------------------------------
# the CPU oracle
# ---------------------------------------------------------------------------

def _threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def _oracle_setup(wl, vocab_slice=None):
    from oracle import dlm_oracle as O
    sh = wl.shape
    w = W.make_weights(sh, seed=wl.seed)
    if vocab_slice is not None:
        w = dict(w)
        w["w_lm"] = np.ascontiguousarray(w["w_lm"][:vocab_slice])
    dims = O.ModelDims.of(sh)
    if vocab_slice is not None:
        dims.vocab = vocab_slice
    om = O.OracleModel(dims, w)
    lens, toks, kp, vp = W.make_prefix(wl)
    conv = O.bf16_bits_to_f64 if sh.dtype == "bf16" else (lambda x: np.asarray(x, np.float64))
    for b in range(wl.batch):
        if toks is not None:
            om.kv_append_tokens(b, toks[b])
        else:
            n = int(lens[b])
            om.kv_append_kv(b, conv(kp[b][:, :n]), conv(vp[b][:, :n]))
    p = O.SamplerParams(canvas=wl.canvas, steps=wl.steps, threshold=wl.threshold,
                        quota=wl.quota, corruption=wl.corruption,
                        entropy_bound=wl.entropy_bound, temperature=wl.temperature,
                        t_max=wl.t_max, t_min=wl.t_min, seed=wl.seed)
    st = O.init_canvas(wl.batch, p, sh.mask_id, sh.vocab)
    return O, om, p, st


def _oracle_step_timed(O, om, p, st, vocab_full, canvases=None):
    """One oracle step over `canvases` (all when None); returns (seconds of
    forward-to-y, of LM head + scores, of selection).  The LM head may cover
    a vocabulary slice."""
    t_fwd = t_lm = t_sel = 0.0
    for b in (range(st.tokens.shape[0]) if canvases is None else canvases):
        if st.done[b]:
            continue
        t0 = time.perf_counter()
        x = om.embed(st.tokens[b])
        L = om.kv_len(b)
        q, k, v = om.project_qkv(x, np.arange(L, L + len(x)))
        o = om.attend(b, q, k, v)
        y = om.out_proj(x, o)
        t1 = time.perf_counter()
        lg = om.logits(y)
        mask = om.dims.mask_id if p.corruption == "mask" else -1
        cand, conf, H, _ = O.scores(lg, mask if mask < lg.shape[1] else -1)
        t2 = time.perf_counter()
        O.select_canvas(st, b, cand, conf, H, p, vocab=vocab_full, mask_id=om.dims.mask_id,
                        eos_id=om.dims.eos_id)
        t3 = time.perf_counter()
        t_fwd += t1 - t0
        t_lm += t2 - t1
        t_sel += t3 - t2
    return t_fwd, t_lm, t_sel


def cpu_baseline(wl):
    """The oracle, as it stands, timed on this host over full steps for about
    10-30 s (at least two steps)."""
    O, om, p, st = _oracle_setup(wl)
    times = []
    t_start = time.perf_counter()
    while len(times) < 2 or (time.perf_counter() - t_start < 10.0 and len(times) < 32):
        if st.done.all():
            st = O.init_canvas(wl.batch, p, wl.shape.mask_id, wl.shape.vocab)
        f, l, s = _oracle_step_timed(O, om, p, st, wl.shape.vocab)
        times.append(f + l + s)
    return {"value": round(len(times) / sum(times), 4), "unit": "steps/s",
            "cores": _threads(), "host_cpus": os.cpu_count(), "kind": "oracle",
            "sample": "%d full oracle steps of the %s block (float64 NumPy)" % (len(times),
                                                                            wl.name)}


def run_reference(a):
    """--impl reference: the oracle on this host, K timed steps after W
    warm-up steps.  Each step is a bounded sample of the batch's step: the
    first n_s = ceil(B / 8) canvases (every canvas up to a batch of 8), each
    with its full forward to the LM-head input, the LM head + scores on a
    vocabulary slice of 1/f of the rows of W_lm (that part's time scaled by f)
    and its selection; the sampled canvases' time is scaled by B / n_s.  When
    the sampled canvases are all done, their block starts over."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = W.WORKLOADS[a.workload]
    V = wl.shape.vocab
    f = 32
    O, om, p, st = _oracle_setup(wl, vocab_slice=V // f)
    n_s = -(-wl.batch // 8)
    sample = list(range(n_s))
    K, Wm = a.steps, max(a.warmup, 3)
    total = 0.0
    for i in range(Wm + K):
        if st.done[sample].all():
            st = O.init_canvas(wl.batch, p, wl.shape.mask_id, V)
        fw, lm, sel = _oracle_step_timed(O, om, p, st, V, canvases=sample)
        if i >= Wm:
            total += (fw + lm * f + sel) * wl.batch / n_s
    value = K / total
    line = {"metric": "denoise steps/s", "value": round(value, 4), "unit": "steps/s",
            "n_gpus": world, "steps": K, "warmup": Wm, "ms_per_step": round(1e3 * total / K, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(a.workload, wl, W.make_prefix(wl)[0], world),
            "cpu_baseline": {"value": round(value, 4), "unit": "steps/s", "cores": _threads(),
                             "kind": "oracle",
                             "sample": "each step: %d of the %d canvases, each with its full "
                                       "forward to the LM-head input, LM head and scores on "
                                       "1/%d of the vocabulary (that time scaled by %d) and "
                                       "its selection; time scaled by %d/%d"
                                       % (n_s, wl.batch, f, f, wl.batch, n_s)},
            "e2e": {"value": round(value, 4), "unit": "steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    else:
        run_ours(a)


if __name__ == "__main__":
    main()
