"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The test hook dlm_test_withhold_loads makes the next tensor-core GEMM launch
issue no TMA loads, so its MMA warp waits for a ring stage that nothing
fills (a flag nothing sets).  After the wait's limit the CTA stops issuing
work, waits for everything it has in flight, frees its tensor memory and
records DLM_ETIMEOUT; dlm_check must report it, and the context must then
run a normal step exactly as a fresh context does.  Nothing here faults,
traps or hangs the GPU: every wait is bounded and the withheld loads are
never issued.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU-only hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

import workloads as W
from gpu_util import lib_params, make_pair
from masked_block_diffusion_denoise_b200 import (DLM_BUF_Q, DLM_ETIMEOUT, DlmError,
                                                 dlm_test_withhold_loads)


@pytest.mark.parametrize("canvas,batch", [(32, 2), (64, 4)])   # one M tile; two (fused QKV)
def test_gemm_wait_timeout_is_reported_and_the_context_recovers(canvas, batch):
    wl = W.small_workload("timeout", n_heads=8, n_kv_heads=2, batch=batch, canvas=canvas,
                          steps=4, prefix_len=(100, 300), prefix_cap=320, seed=12)
    sess, _, _ = make_pair(wl)
    fresh, _, _ = make_pair(wl)
    try:
        p = lib_params(wl)
        sh = wl.shape
        M = wl.batch * wl.canvas
        cv = sess.new_canvas(wl.batch, wl.canvas)
        sess.init(cv, p)
        dlm_test_withhold_loads(sess.ctx, 1)       # the step's first GEMM (QKV) starves
        sess.step(cv, p)
        with pytest.raises(DlmError) as err:
            sess.check()
        assert err.value.code == DLM_ETIMEOUT
        sess.check()                               # the error word was cleared
        # the same context and a fresh one run the same normal step
        a, b = sess.new_canvas(wl.batch, wl.canvas), fresh.new_canvas(wl.batch, wl.canvas)
        sess.init(a, p)
        fresh.init(b, p)
        sess.step(a, p)
        fresh.step(b, p)
        sess.check()
        fresh.check()
        na, nb = a.numpy(), b.numpy()
        for key in ("tokens", "committed", "step", "done", "stats"):
            assert np.array_equal(na[key], nb[key]), key
        qa = sess.buffer(DLM_BUF_Q, (M, sh.n_heads, sh.head_dim), torch.bfloat16)
        qb = fresh.buffer(DLM_BUF_Q, (M, sh.n_heads, sh.head_dim), torch.bfloat16)
        assert torch.equal(qa, qb)
    finally:
        sess.close()
        fresh.close()
