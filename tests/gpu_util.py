"""Helpers shared by the GPU parity tests: build a library session and a
matching oracle from the same seeded workload, compare stage by stage."""
from __future__ import annotations

import numpy as np

import workloads as W
from oracle import dlm_oracle as O


def to64(t) -> np.ndarray:
    """device tensor (bf16 / f32 / int) -> float64 numpy"""
    import torch
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy().astype(np.float64)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.maximum(np.abs(x), 1e-30)
    return 2.0 ** (np.floor(np.log2(ax)) - 7)


# Accumulation allowance of a dot product computed by the tensor cores (or an
# fp32 FMA chain): float32 accumulation, error below a small multiple of
# 2^-23 times the sum of the absolute values of the terms (measured: about
# 1 x 2^-23); 2^-21 is used.  Near-zero results of long cancelling sums
# need it: there one bf16 rounding step of the result is far smaller.
ACCUM_U = 2.0 ** -21


def abs_terms(a: np.ndarray, w: np.ndarray) -> np.ndarray:
    """sum_k |a_k w_nk| for every output n of a @ w.T"""
    return np.abs(a) @ np.abs(w).T


def assert_storage_close(got, ref, dtype, *, max_ulp=1.0, max_frac=0.02, atol=1e-6, what="",
                         terms=None):
    """Values a kernel stored after rounding to the model's element type:
    equal up to one rounding step at a rounding boundary, and rarely so, plus
    the float32 accumulation allowance ACCUM_U * terms (terms = sum of the
    absolute values of the products behind each value)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    if terms is not None:
        atol = atol + ACCUM_U * np.asarray(terms, np.float64)
    if dtype == "bf16":
        tol = max_ulp * bf16_ulp(np.maximum(np.abs(got), np.abs(ref))) * 1.001 + atol
    else:
        tol = 1e-5 * np.maximum(np.abs(ref), 1.0) + atol
    diff = np.abs(got - ref)
    bad = diff > tol
    if bad.any():
        idx = [tuple(int(i) for i in ix) for ix in np.argwhere(bad)[:8]]
        detail = ["%s got %.9g ref %.9g" % (ix, got[ix], ref[ix]) for ix in idx]
        raise AssertionError("%s: %d values beyond tolerance, max diff %g: %s" % (
            what, int(bad.sum()), float(diff.max()), "; ".join(detail)))
    frac = float((diff > 1e-6).mean())
    assert frac <= max_frac or dtype != "bf16", "%s: %.3f of values differ" % (what, frac)


def make_pair(wl: W.Workload, *, device="cuda:0", seed=None, max_batch=None, max_canvas=None):
    """Library session and oracle model with identical weights and prefixes."""
    from masked_block_diffusion_denoise_b200.session import Session
    seed = wl.seed if seed is None else seed
    sh = wl.shape
    weights = W.make_weights(sh, seed=seed)
    lens, toks, k, v = W.make_prefix(wl, seed=seed)
    sess = Session(sh, weights, max_batch=max_batch or wl.batch, max_prefix=wl.prefix_cap,
                   max_canvas=max_canvas or wl.canvas, device=device)
    om = O.OracleModel(O.ModelDims.of(sh), weights)
    for b in range(wl.batch):
        if toks is not None:
            sess.kv_append_tokens(b, toks[b])
            om.kv_append_tokens(b, toks[b])
        else:
            n = int(lens[b])
            kb, vb = np.ascontiguousarray(k[b][:, :n]), np.ascontiguousarray(v[b][:, :n])
            sess.kv_append_kv(b, kb, vb)
            conv = O.bf16_bits_to_f64 if sh.dtype == "bf16" else (lambda a: np.asarray(a, np.float64))
            om.kv_append_kv(b, conv(kb), conv(vb))
    return sess, om, weights


def oracle_params(wl: W.Workload, **over) -> "O.SamplerParams":
    kw = dict(canvas=wl.canvas, steps=wl.steps, threshold=wl.threshold, quota=wl.quota,
              corruption=wl.corruption, entropy_bound=wl.entropy_bound,
              temperature=wl.temperature, t_max=wl.t_max, t_min=wl.t_min, seed=wl.seed)
    kw.update(over)
    return O.SamplerParams(**kw)


def lib_params(wl: W.Workload, **over):
    from masked_block_diffusion_denoise_b200.session import sampler_params
    kw = dict(canvas=wl.canvas, steps=wl.steps, threshold=wl.threshold, quota=wl.quota,
              corruption=wl.corruption, entropy_bound=wl.entropy_bound,
              temperature=wl.temperature, t_max=wl.t_max, t_min=wl.t_min, seed=wl.seed)
    kw.update(over)
    return sampler_params(**kw)


def state_from(np_state) -> "O.CanvasState":
    return O.CanvasState(np_state["tokens"].copy(), np_state["committed"].copy(),
                         np_state["step"].copy(), np_state["done"].copy(),
                         np_state["eos_pos"].copy())


def near_tie_ok(values: np.ndarray, got: int, want: int, gap: float) -> bool:
    """Equal, or both within `gap` of the row maximum (a near tie)."""
    if got == want:
        return True
    top = values[want]
    return abs(values[got] - top) < gap
