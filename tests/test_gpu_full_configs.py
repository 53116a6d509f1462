"""Parity at the full shapes of the batched, long-context and entropy-bound
encoder-decoder workloads, through the C ABI, against the CPU oracle.

Each step is teacher-forced (the oracle is given the GPU's own canvas state
and its own inputs to every stage) and checked with the standards of
test_gpu_parity.py: stored bf16 activations within one rounding step plus
the float32 accumulation allowance, attention within 2e-2 absolute,
candidates equal to the oracle's float64 argmax except near ties (top-2 gap
below 1e-3, counted), confidence and entropy within 1e-3, and the selection
bit for bit on the GPU's own scores.

* batched (16 canvases of 64 over prefixes of 1024-4096, EOS planted in 4
  canvases): canvases in four different 128-row tiles, one of them EOS
  planted, at step 0, at step 8 (after the EOS-planted canvas 1 finished
  early) and at the last step of the budget (index 31), where the forced
  commit fills every open position (Nemotron guide, section 6; DiffusionGemma
  page, BlockRefinementScheduler).
* long context (4 canvases of 32 over 32768-key prefixes): every canvas,
  every head, at step 0 and step 7; the split plan that ran is reported and
  must split the keys.
* entropy-bound encoder-decoder (2 canvases of 256, vocabulary 262144,
  uniform corruption, Gumbel sampling at the annealed temperature,
  DiffusionGemma page, EntropyBoundScheduler): the sampled candidates
  replayed on the GPU's float32 logits with the oracle's Gumbel noise equal
  the GPU's except near ties (perturbed top-2 gap below 1e-4), at step 0 and
  step 20.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from gpu_util import (check_one_step, lib_params, make_pair, oracle_params, record_near_ties,
                      to64)
from oracle import dlm_oracle as O
import workloads as W

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU-only hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

from masked_block_diffusion_denoise_b200 import (DLM_BUF_CAND, DLM_BUF_CONF, DLM_BUF_ENTROPY,
                                                 DLM_BUF_Y, dlm_attention_plan)


def _canvas_with_plant(sess, wl, p_lib):
    cv = sess.new_canvas(wl.batch, wl.canvas)
    sess.init(cv, p_lib)
    for (b, slot) in W.make_eos_plant(wl):
        cv.tokens[b, slot] = wl.shape.eos_id
        cv.committed[b, slot] = 1
    return cv


def test_batched_full_shape():
    wl = W.WORKLOADS["batched"]
    planted = dict(W.make_eos_plant(wl))
    assert 1 in planted      # canvas 1 carries an EOS at slot 12 and finishes early
    sess, om, _ = make_pair(wl)
    try:
        p_lib, p_or = lib_params(wl), oracle_params(wl)
        cv = _canvas_with_plant(sess, wl, p_lib)
        # canvases in row tiles 0, 0, 3, 5 and 7 (128 rows = two canvases a tile)
        canvases = [0, 1, 7, 10, 15]
        rows = np.array([0, 17, 41, wl.canvas - 1])
        report = {}
        check_one_step(sess, om, wl, cv, p_lib, p_or, rows_sample=rows, full_logits=False,
                       canvases_sample=canvases, report=report)
        # steps 1..7 on the library alone, then step 8 teacher-forced
        for _ in range(7):
            sess.step(cv, p_lib)
        sess.check()
        pre = cv.numpy()
        assert pre["done"][1] and not pre["done"][0], "canvas 1 finishes early (EOS at 12)"
        check_one_step(sess, om, wl, cv, p_lib, p_or, rows_sample=rows, full_logits=False,
                       canvases_sample=canvases, report=report)
        # the last step of the budget from the current state: every open
        # position commits (far more than the quota of 2)
        st = cv.numpy()
        open_before = (~st["committed"]).sum(axis=1)
        step = np.where(st["done"], st["step"], wl.steps - 1)
        cv.load(st["tokens"], st["committed"], step, st["done"], st["eos_pos"])
        pre, post = check_one_step(sess, om, wl, cv, p_lib, p_or, rows_sample=rows,
                                   full_logits=False, canvases_sample=canvases, report=report)
        active = ~pre["done"]
        assert (open_before[active] > wl.quota_eff).all()
        assert post["done"].all() and post["committed"].all()
        record_near_ties("batched_full_shape", report["near_ties"], report["compared"])
    finally:
        sess.close()


def test_longctx_full_shape():
    wl = W.WORKLOADS["longctx"]
    sess, om, _ = make_pair(wl)
    try:
        p_lib, p_or = lib_params(wl), oracle_params(wl)
        cv = sess.new_canvas(wl.batch, wl.canvas)
        sess.init(cv, p_lib)
        plan = dlm_attention_plan(sess.ctx, wl.batch, wl.canvas)
        print("longctx attention plan", plan)
        assert plan["nsplit"] > 1 and plan["chunk"] % 128 == 0
        rows = np.array([0, 13, wl.canvas - 1])
        report = {}
        check_one_step(sess, om, wl, cv, p_lib, p_or, rows_sample=rows, full_logits=False,
                       report=report)
        for _ in range(6):
            sess.step(cv, p_lib)
        check_one_step(sess, om, wl, cv, p_lib, p_or, rows_sample=rows, full_logits=False,
                       report=report)
        assert len(report["attn_max_err"]) == 2 * wl.batch
        record_near_ties("longctx_full_shape", report["near_ties"], report["compared"])
    finally:
        sess.close()


def _check_sampled_candidates(sess, om, wl, pre, rows, gap=1e-4):
    """Replay Gumbel sampling at the annealed temperature on the GPU's float32
    logits of the sampled rows (oracle noise, float64): the candidate equals
    the GPU's except where the perturbed top-2 gap is below `gap`; the
    confidence and entropy at the sampling temperature within 1e-3.  The
    logits themselves are compared with the oracle's of the GPU's y.
    Returns (near ties, positions compared)."""
    sh, B, C = wl.shape, wl.batch, wl.canvas
    M = B * C
    lg = sess.logits(B, C).cpu().numpy()
    y = to64(sess.buffer(DLM_BUF_Y, (M, sh.d_model), torch.bfloat16))
    cand = sess.buffer(DLM_BUF_CAND, (M,), torch.int32).cpu().numpy()
    conf = sess.buffer(DLM_BUF_CONF, (M,), torch.float32).cpu().numpy()
    ent = sess.buffer(DLM_BUF_ENTROPY, (M,), torch.float32).cpu().numpy()
    ties = n = 0
    for b in range(B):
        if pre["done"][b]:
            continue
        r = b * C + rows
        lo = om.logits(y[r])
        assert np.abs(lg[r] - lo).max() < 2e-3 * max(1.0, np.abs(lo).max()), "logits"
        st = int(pre["step"][b])
        T = O.annealed_temperature(wl.t_max, wl.t_min, st, wl.steps)
        inv = np.float32(np.float32(1.0) / T)
        G = np.stack([O.gumbel_noise(wl.seed, b, st, int(i), sh.vocab) for i in rows])
        c64, f64, h64, z = O.scores(lg[r], -1, inv_temp=inv, gumbel=G)
        for j in range(len(rows)):
            gc = int(cand[r[j]])
            g = z[j] + G[j]
            n += 1
            if gc != c64[j]:
                assert abs(g[gc] - g[c64[j]]) < gap, "sampled id outside a near tie"
                ties += 1
            else:
                assert abs(conf[r[j]] - f64[j]) < 1e-3
            assert abs(ent[r[j]] - h64[j]) < 1e-3
    return ties, n


def test_encdec_entropy_bound_full_shape():
    wl = W.WORKLOADS["encdec_eb"]
    sess, om, _ = make_pair(wl)
    try:
        p_lib, p_or = lib_params(wl), oracle_params(wl)
        cv = sess.new_canvas(wl.batch, wl.canvas)
        sess.init(cv, p_lib)
        init = cv.numpy()
        ref = O.init_canvas(wl.batch, p_or, wl.shape.mask_id, wl.shape.vocab)
        assert np.array_equal(init["tokens"], ref.tokens)     # uniform initial noise
        rows = np.array([0, 1, 77, 128, 200, wl.canvas - 1])
        ties = n = 0
        for advance in (0, 19):          # check step 0, then step 20
            for _ in range(advance):
                sess.step(cv, p_lib)
            pre, _ = check_one_step(sess, om, wl, cv, p_lib, p_or, rows_sample=rows,
                                    full_logits=False)
            assert not pre["done"].any()
            t, m = _check_sampled_candidates(sess, om, wl, pre, rows)
            ties, n = ties + t, n + m
        assert ties <= max(2, n // 50)
        record_near_ties("encdec_entropy_bound_full_shape", ties, n)
    finally:
        sess.close()
