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


# Near ties seen by the GPU parity tests (positions whose candidate differs
# from the oracle's only inside the near-tie gap), by test; printed in the
# pytest summary by conftest.py.
NEAR_TIES = {}


def record_near_ties(name: str, count: int, positions: int) -> None:
    n, m = NEAR_TIES.get(name, (0, 0))
    NEAR_TIES[name] = (n + int(count), m + int(positions))


# ---------------------------------------------------------------------------
# stage-by-stage check of one step
# ---------------------------------------------------------------------------

def check_one_step(sess, om, wl, cv, p_lib, p_or, *, rows_sample=None, heads_sample=None,
                   full_logits=True, report=None, canvases_sample=None):
    """One library step from the canvas state in `cv`, checked stage by stage
    against the oracle on the GPU's own inputs to each stage.  rows_sample:
    canvas positions whose projections, y and scores are checked (all when
    None); canvases_sample: canvases checked stage by stage (all active ones
    when None); the selection is checked bit for bit on every canvas."""
    import torch
    from masked_block_diffusion_denoise_b200 import (DLM_BUF_CAND, DLM_BUF_CONF, DLM_BUF_ENTROPY,
                                                     DLM_BUF_K_CACHE, DLM_BUF_O, DLM_BUF_Q,
                                                     DLM_BUF_V_CACHE, DLM_BUF_X, DLM_BUF_Y)
    sh = wl.shape
    B, C = cv.tokens.shape
    M = B * C
    dt = torch.bfloat16 if sh.dtype == "bf16" else torch.float32
    pre = cv.numpy()
    sess.step(cv, p_lib)
    sess.check()
    post = cv.numpy()
    active = [b for b in range(B) if not pre["done"][b]]
    x = to64(sess.buffer(DLM_BUF_X, (M, sh.d_model), dt))
    q = to64(sess.buffer(DLM_BUF_Q, (M, sh.n_heads, sh.head_dim), dt))
    o = to64(sess.buffer(DLM_BUF_O, (M, sh.n_heads * sh.head_dim), dt))
    y = to64(sess.buffer(DLM_BUF_Y, (M, sh.d_model), dt))
    Lcap = sess.max_prefix + sess.max_canvas
    kc = sess.buffer(DLM_BUF_K_CACHE, (sess.max_batch, sh.n_kv_heads, Lcap, sh.head_dim), dt)
    vc = sess.buffer(DLM_BUF_V_CACHE, (sess.max_batch, sh.n_kv_heads, Lcap, sh.head_dim), dt)
    cand = sess.buffer(DLM_BUF_CAND, (M,), torch.int32).cpu().numpy()
    conf = sess.buffer(DLM_BUF_CONF, (M,), torch.float32).cpu().numpy()
    ent = sess.buffer(DLM_BUF_ENTROPY, (M,), torch.float32).cpu().numpy()
    logits = sess.logits(B, C).cpu().numpy() if full_logits else None
    near_ties = compared = 0
    for b in active:
        if canvases_sample is not None and b not in canvases_sample:
            continue
        r0 = b * C
        rows = np.arange(C) if rows_sample is None else np.asarray(rows_sample)
        L = om.kv_len(b)
        # a1 embedding: exact
        assert np.array_equal(x[r0 + rows], om.embed(pre["tokens"][b][rows])), "embed"
        # a2 projections + RoPE from the GPU's x
        qo, ko, vo = om.project_qkv(x[r0 + rows], L + rows)
        xr = x[r0 + rows]
        half = sh.head_dim // 2
        rot = lambda t: np.concatenate([t[..., :half] + t[..., half:]] * 2, axis=-1)
        tq = rot(abs_terms(xr, om.w_q).reshape(qo.shape))
        tk = rot(abs_terms(xr, om.w_k).reshape(ko.shape))
        tv = abs_terms(xr, om.w_v).reshape(vo.shape)
        assert_storage_close(q[r0 + rows], qo, sh.dtype, what="q", terms=tq)
        kg = to64(kc[b, :, L:L + C]).transpose(1, 0, 2)
        vg = to64(vc[b, :, L:L + C]).transpose(1, 0, 2)
        assert_storage_close(kg[rows], ko, sh.dtype, what="canvas k", terms=tk)
        assert_storage_close(vg[rows], vo, sh.dtype, what="canvas v", terms=tv)
        # a3 attention from the GPU's q, k, v
        qb = q[r0:r0 + C]
        oo = om.attend(b, qb, kg, vg)
        err = np.abs(o[r0:r0 + C] - oo)
        if heads_sample is not None:
            cols = np.concatenate([np.arange(h * sh.head_dim, (h + 1) * sh.head_dim)
                                   for h in heads_sample])
            err = err[:, cols]
        assert err.max() < 2e-2, "attention max abs err %g" % err.max()
        if report is not None:
            report.setdefault("attn_max_err", []).append(float(err.max()))
        # a4 output projection + residual from the GPU's x and o
        yo = om.out_proj(x[r0 + rows], o[r0 + rows])
        assert_storage_close(y[r0 + rows], yo, sh.dtype, what="y",
                             terms=np.abs(xr) + abs_terms(o[r0 + rows], om.w_o))
        # a5/a6 scores
        if p_or.entropy_bound >= 0 or p_or.temperature > 0:
            continue   # sampling modes are checked in their own test
        mask = sh.mask_id if p_or.corruption == "mask" else -1
        if logits is not None:
            lg = logits[r0:r0 + C]
            lo = om.logits(y[r0:r0 + C])
            assert np.abs(lg - lo).max() < 2e-3 * max(1.0, np.abs(lo).max()), "logits"
            c32, f32, h32, _ = O.scores(lg.astype(np.float32), mask)
            assert np.array_equal(cand[r0:r0 + C], c32), "cand from identical logits"
            assert np.abs(conf[r0:r0 + C] - f32).max() < 1e-3, "confidence"
            assert np.abs(ent[r0:r0 + C] - h32).max() < 1e-3, "entropy"
            c64, _, _, z = O.scores(lo, mask)
            compared += C
            for i in range(C):
                if cand[r0 + i] != c64[i]:
                    assert near_tie_ok(z[i], int(cand[r0 + i]), int(c64[i]), 1e-3), \
                        "argmax flip outside a near tie"
                    near_ties += 1
        else:
            # the sampled rows' float64 logits in one pass over W_lm
            lo = om.logits(y[r0 + rows])
            c64, f64, h64, z = O.scores(lo, mask)
            compared += len(rows)
            for j, i in enumerate(rows):
                if cand[r0 + i] != c64[j]:
                    assert near_tie_ok(z[j], int(cand[r0 + i]), int(c64[j]), 1e-3), \
                        "argmax flip outside a near tie"
                    near_ties += 1
                else:
                    assert abs(conf[r0 + i] - f64[j]) < 1e-3
                assert abs(ent[r0 + i] - h64[j]) < 1e-3
    # a7 selection on the GPU's own cand / conf / H: bit-exact
    st = state_from(pre)
    stats = [O.CanvasStats() for _ in range(B)]
    for b in range(B):
        O.select_canvas(st, b, cand[b * C:(b + 1) * C], conf[b * C:(b + 1) * C],
                        ent[b * C:(b + 1) * C], p_or, vocab=sh.vocab, mask_id=sh.mask_id,
                        eos_id=sh.eos_id, stats=stats[b])
    assert np.array_equal(st.tokens, post["tokens"]), "tokens after commit"
    assert np.array_equal(st.committed, post["committed"]), "commit mask"
    assert np.array_equal(st.step, post["step"]) and np.array_equal(st.done, post["done"])
    assert np.array_equal(st.eos_pos, post["eos_pos"])
    dstats = post["stats"] - pre["stats"]
    for b in range(B):
        assert list(dstats[b]) == [stats[b].steps_used, stats[b].committed_by_sampler,
                                   stats[b].forced_at_budget, stats[b].eos_autofill,
                                   stats[b].frozen, stats[b].edited]
    if report is not None:
        report["near_ties"] = report.get("near_ties", 0) + near_ties
        report["compared"] = report.get("compared", 0) + compared
    return pre, post
