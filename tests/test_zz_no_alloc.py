"""dlm_attention_noalloc: canvas attention that allocates no device memory.

Some callers cannot call cudaMalloc: a serving engine that hands all device
memory to its own pool at start-up, or code that issues work while a stream
is being captured into a CUDA graph, where an allocation would synchronise
the device or is refused.  For them the library keeps the split-KV partials
of the attention in a fixed array compiled into the library.  This test
checks, through the C ABI, that two calls in a row give the attention output
that dlm_denoise_step's own attention wrote, within the attention tolerance
of the parity tests (2e-2 absolute).  The file name sorts last so that a run
stopping at the first failure has run every other test already.
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
                                                 DLM_BUF_V_CACHE, dlm_attention_noalloc)


def test_attention_noalloc_matches_the_step_attention():
    wl = W.small_workload("noalloc", n_heads=8, n_kv_heads=2, batch=3, canvas=32, steps=4,
                          prefix_len=(100, 350), prefix_cap=384)
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
            torch.cuda.synchronize()
            err = (out.float() - ref.float()).abs().max().item()
            assert np.isfinite(err) and err <= 2e-2, "call %d: max abs diff %g" % (call, err)
    finally:
        sess.close()
