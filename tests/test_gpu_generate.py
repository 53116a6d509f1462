"""Multi-block generation, adaptive stopping and token editing through the
C ABI (``dlm_generate``), against the oracle's ``generate``.

The float32 configuration runs free (no teacher forcing): on it the GPU's
candidates agree with the float64 oracle's at every step, so the whole
output, the cache the clean passes wrote and the counters must match.  The
bf16 configuration checks what holds at any rounding: every block finished,
and the clean pass cached each block's own tokens."""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from gpu_util import (abs_terms, assert_storage_close, lib_params, make_pair, oracle_params,
                      to64)
from oracle import dlm_oracle as O
import workloads as W

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU-only hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

from masked_block_diffusion_denoise_b200 import (DLM_BUF_K_CACHE, DLM_BUF_V_CACHE,
                                                 dlm_kv_length)

N_BLOCKS = 3


def _stats(s):
    return [s.steps_used, s.committed_by_sampler, s.forced_at_budget, s.eos_autofill, s.frozen,
            s.edited]


@pytest.mark.parametrize("mode", ["plain", "stop", "uniform", "edit"])
def test_generate_tiny_fp32_free_running(mode):
    base = W.WORKLOADS["tiny"]
    wl = base.replace(prefix_cap=base.prefix_len[1] + N_BLOCKS * base.canvas)
    over = {}
    if mode == "stop":
        # the argmax of this random model changes between steps, so only
        # stability 0 freezes (the stable-step count is covered bit-exactly
        # by the commit tests)
        over = dict(stability_steps=0, stop_entropy=100.0)
    if mode == "uniform":
        over = dict(corruption="uniform", seed=7)
    if mode == "edit":
        over = dict(editing=1, editing_threshold=0.0)
    sess, om, _ = make_pair(wl)
    try:
        C, B = wl.canvas, wl.batch
        cv = sess.new_canvas(B, C)
        out, n = sess.generate(cv, lib_params(wl, **over), N_BLOCKS, eos_early_stop=False)
        sess.check()
        stats = [O.CanvasStats() for _ in range(B)]
        ref, n_ref = O.generate(om, oracle_params(wl, **over), B, N_BLOCKS,
                                eos_early_stop=False, stats=stats)
        assert n == n_ref == N_BLOCKS
        assert np.array_equal(out.cpu().numpy(), ref)
        got = cv.numpy()["stats"]
        for b in range(B):
            assert list(got[b]) == _stats(stats[b])
        if mode == "stop":
            assert sum(s.frozen for s in stats) > 0
        if mode == "edit":
            assert sum(s.edited for s in stats) > 0
        L = om.kv_len(0)
        assert dlm_kv_length(sess.ctx, 0) == L == wl.prefix_len[1] + N_BLOCKS * C
        sh = wl.shape
        Lcap = sess.max_prefix + sess.max_canvas
        kc = to64(sess.buffer(DLM_BUF_K_CACHE, (B, sh.n_kv_heads, Lcap, sh.head_dim),
                              torch.float32))
        vc = to64(sess.buffer(DLM_BUF_V_CACHE, (B, sh.n_kv_heads, Lcap, sh.head_dim),
                              torch.float32))
        assert np.allclose(kc[0, :, :L], om.k_cache[0], atol=1e-4)
        assert np.allclose(vc[0, :, :L], om.v_cache[0], atol=1e-4)
    finally:
        sess.close()


def test_generate_bf16_clean_pass_caches_each_block():
    base = W.small_workload("gen_bf16", batch=3, canvas=32, steps=6, quota=0,
                            prefix_len=(40, 250))
    wl = base.replace(prefix_cap=base.prefix_len[1] + N_BLOCKS * base.canvas)
    sess, om, _ = make_pair(wl)
    try:
        C, B, sh = wl.canvas, wl.batch, wl.shape
        L0 = [om.kv_len(b) for b in range(B)]
        cv = sess.new_canvas(B, C)
        out, n = sess.generate(cv, lib_params(wl), N_BLOCKS, eos_early_stop=False)
        sess.check()
        out = out.cpu().numpy()
        assert n == N_BLOCKS and not (out == sh.mask_id).any()
        assert ((out >= 0) & (out < sh.vocab)).all()
        Lcap = sess.max_prefix + sess.max_canvas
        kc = sess.buffer(DLM_BUF_K_CACHE, (B, sh.n_kv_heads, Lcap, sh.head_dim), torch.bfloat16)
        vc = sess.buffer(DLM_BUF_V_CACHE, (B, sh.n_kv_heads, Lcap, sh.head_dim), torch.bfloat16)
        half = sh.head_dim // 2
        for b in range(B):
            assert dlm_kv_length(sess.ctx, b) == L0[b] + N_BLOCKS * C
            om.kv_append_tokens(b, out[b])
            L = om.kv_len(b)
            xe = om.embed(out[b])
            tk = abs_terms(xe, om.w_k).reshape(-1, sh.n_kv_heads, sh.head_dim).transpose(1, 0, 2)
            tk = np.concatenate([tk[..., :half] + tk[..., half:]] * 2, axis=-1)
            tv = abs_terms(xe, om.w_v).reshape(-1, sh.n_kv_heads, sh.head_dim).transpose(1, 0, 2)
            assert_storage_close(to64(kc[b, :, L0[b]:L]), om.k_cache[b][:, L0[b]:], "bf16",
                                 what="K", terms=tk)
            assert_storage_close(to64(vc[b, :, L0[b]:L]), om.v_cache[b][:, L0[b]:], "bf16",
                                 what="V", terms=tv)
    finally:
        sess.close()


@pytest.mark.parametrize("early", [True, False])
def test_generate_eos_early_stop(early):
    """A zero LM head: every candidate is id 0 (the EOS here) at confidence
    1/(V-1); position 0 wins the tie, commits the EOS and the rest of the
    block is filled in the same step."""
    from masked_block_diffusion_denoise_b200.session import Session
    base = W.WORKLOADS["tiny"]
    wl = base.replace(prefix_cap=base.prefix_len[1] + N_BLOCKS * base.canvas)
    sh = dataclasses.replace(wl.shape, eos_id=0)
    w = W.make_weights(sh, seed=wl.seed)
    w["w_lm"] = np.zeros_like(w["w_lm"])
    sess = Session(sh, w, max_batch=1, max_prefix=wl.prefix_cap, max_canvas=wl.canvas)
    try:
        _, toks, _, _ = W.make_prefix(wl)
        sess.kv_append_tokens(0, toks[0])
        cv = sess.new_canvas(1, wl.canvas)
        out, n = sess.generate(cv, lib_params(wl), N_BLOCKS, eos_early_stop=early)
        sess.check()
        assert n == (1 if early else N_BLOCKS)
        assert (out.cpu().numpy()[:, :n * wl.canvas] == 0).all()
        st = cv.numpy()
        assert st["eos_pos"][0] == 0 and list(st["stats"][0]) == [n, 4 * n, 0,
                                                                 n * (wl.canvas - 4), 0, 0]
        assert dlm_kv_length(sess.ctx, 0) == wl.prefix_len[1] + n * wl.canvas
    finally:
        sess.close()


def test_generate_rejects_overflow():
    from masked_block_diffusion_denoise_b200 import DlmError
    wl = W.WORKLOADS["tiny"]
    sess, _, _ = make_pair(wl)
    try:
        cv = sess.new_canvas(1, wl.canvas)
        with pytest.raises(DlmError):
            sess.generate(cv, lib_params(wl), 1)
        assert dlm_kv_length(sess.ctx, 0) == wl.prefix_len[1]
    finally:
        sess.close()


@pytest.mark.parametrize("lm_fp8", [False, True])
def test_generate_bf16_every_option(lm_fp8):
    """Two blocks with uniform corruption, adaptive stopping and token editing
    together (bf16, and with the e4m3 LM head): every position of every block
    is committed, no id is out of range, the counters add up, and the clean
    passes cached each block's own tokens."""
    base = W.small_workload("gen_all", batch=2, canvas=32, steps=5, quota=0, corruption="uniform",
                            prefix_len=(60, 200), lm_fp8=lm_fp8, seed=8)
    wl = base.replace(prefix_cap=base.prefix_len[1] + 2 * base.canvas)
    sess, om, _ = make_pair(wl)
    try:
        C, B, sh = wl.canvas, wl.batch, wl.shape
        L0 = [om.kv_len(b) for b in range(B)]
        p = lib_params(wl, stability_steps=0, stop_entropy=0.05, editing=1,
                       editing_threshold=0.0)
        cv = sess.new_canvas(B, C)
        out, n = sess.generate(cv, p, 2, eos_early_stop=False)
        sess.check()
        out = out.cpu().numpy()
        st = cv.numpy()
        assert n == 2 and ((out >= 0) & (out < sh.vocab)).all()
        assert st["committed"].all() and st["done"].all()
        stats = st["stats"]
        # per block every position is committed once: by the sampler, a freeze or the EOS fill
        for b in range(B):
            assert stats[b][1] + stats[b][4] + stats[b][3] == 2 * C
            assert stats[b][0] <= 2 * wl.steps
        Lcap = sess.max_prefix + sess.max_canvas
        kc = sess.buffer(DLM_BUF_K_CACHE, (B, sh.n_kv_heads, Lcap, sh.head_dim), torch.bfloat16)
        half = sh.head_dim // 2
        for b in range(B):
            assert dlm_kv_length(sess.ctx, b) == L0[b] + 2 * C
            om.kv_append_tokens(b, out[b])
            xe = om.embed(out[b])
            tk = abs_terms(xe, om.w_k).reshape(-1, sh.n_kv_heads, sh.head_dim).transpose(1, 0, 2)
            tk = np.concatenate([tk[..., :half] + tk[..., half:]] * 2, axis=-1)
            assert_storage_close(to64(kc[b, :, L0[b]:L0[b] + 2 * C]), om.k_cache[b][:, L0[b]:],
                                 "bf16", what="K", terms=tk)
    finally:
        sess.close()
