"""dlm_attention_noalloc: canvas attention that allocates no device memory.

Some callers cannot call cudaMalloc: a serving engine that hands all device
memory to its own pool at start-up, or code that issues work while a stream
is being captured into a CUDA graph, where an allocation would synchronise
the device or is refused.  For them the library keeps the split-KV partials
of the attention in a fixed array compiled into the library.  These tests
check, through the C ABI, that two calls in a row give the attention output
that dlm_denoise_step's own attention wrote, within the attention tolerance
of the parity tests (2e-2 absolute), and that the device error word stays
clear (dlm_attention_noalloc_check after every call).  The file name sorts
last so that a run stopping at the first failure has run every other test
already.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU-only hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

import workloads as W
from gpu_util import lib_params, make_pair
from masked_block_diffusion_denoise_b200 import (DLM_BUF_K_CACHE, DLM_BUF_O, DLM_BUF_Q,
                                                 DLM_BUF_V_CACHE, dlm_attention_noalloc,
                                                 dlm_attention_noalloc_check, dlm_attention_plan)

NOALLOC_SLOTS = 16384   # partial row slots of the library's fixed array


def _run(wl):
    """The step's own attention, then two no-alloc calls over the same q and
    cache; returns the split plan the step used."""
    sess, om, _ = make_pair(wl)
    try:
        sh = wl.shape
        B, C = wl.batch, wl.canvas
        M = B * C
        p = lib_params(wl)
        cv = sess.new_canvas(B, C)
        sess.init(cv, p)
        sess.step(cv, p)       # the library's own attention, into its context buffers
        sess.check()
        plan = dlm_attention_plan(sess.ctx, B, C)
        Lcap = sess.max_prefix + sess.max_canvas
        q = sess.buffer(DLM_BUF_Q, (M, sh.n_heads, sh.head_dim), torch.bfloat16)
        kc = sess.buffer(DLM_BUF_K_CACHE, (B, sh.n_kv_heads, Lcap, sh.head_dim), torch.bfloat16)
        vc = sess.buffer(DLM_BUF_V_CACHE, (B, sh.n_kv_heads, Lcap, sh.head_dim), torch.bfloat16)
        ref = sess.buffer(DLM_BUF_O, (M, sh.n_heads * sh.head_dim), torch.bfloat16).clone()
        lens_h = [om.kv_len(b) for b in range(B)]
        lens = torch.tensor(lens_h, dtype=torch.int32, device="cuda")
        stream = torch.cuda.current_stream()
        for call in range(2):
            out = torch.full_like(ref, float("nan"))
            dlm_attention_noalloc(q, kc, vc, lens, max(lens_h), out, B, C, sh.n_heads,
                                  sh.n_kv_heads, sh.head_dim, B, Lcap, stream=stream)
            dlm_attention_noalloc_check(stream)      # raises on a recorded device error
            err = (out.float() - ref.float()).abs().max().item()
            assert np.isfinite(err) and err <= 2e-2, "call %d: max abs diff %g" % (call, err)
        return plan
    finally:
        sess.close()


def test_attention_noalloc_matches_the_step_attention():
    wl = W.small_workload("noalloc", n_heads=8, n_kv_heads=2, batch=3, canvas=32, steps=4,
                          prefix_len=(100, 350), prefix_cap=384)
    _run(wl)


def test_attention_noalloc_partials_path(monkeypatch):
    """With in-cluster combining turned off, a multi-split plan writes its
    partials into the fixed array and the combine kernel reads them back."""
    monkeypatch.setenv("DLM_ATTN_CLUSTER", "0")
    wl = W.small_workload("noalloc_parts", n_heads=8, n_kv_heads=2, batch=3, canvas=32,
                          steps=4, prefix_len=(900, 1500), prefix_cap=1536, seed=2)
    plan = _run(wl)
    assert plan["nsplit"] > 1 and plan["cluster"] == 1, plan


def test_attention_noalloc_caps_the_splits(monkeypatch):
    """A shape whose step attention runs a partials plan needing more row
    slots than the fixed array holds (256-key splits forced): the no-alloc
    call plans within the array instead and still matches."""
    monkeypatch.setenv("DLM_ATTN_CLUSTER", "0")
    monkeypatch.setenv("DLM_ATTN_TILES", "2")
    wl = W.small_workload("noalloc_cap", n_heads=32, n_kv_heads=8, batch=4, canvas=32,
                          steps=4, prefix_len=(1500, 2000), prefix_cap=2000, seed=3)
    plan = _run(wl)
    rows = (wl.shape.n_heads // wl.shape.n_kv_heads) * wl.canvas
    need = wl.batch * wl.shape.n_kv_heads * plan["nsplit"] * rows
    assert plan["cluster"] == 1 and need > NOALLOC_SLOTS, (plan, need)
