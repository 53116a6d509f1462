"""The index-checking build (DLM_DEBUG_BOUNDS, libdlm_bounds.so): on valid
inputs it reports no violation and computes exactly what the default build
computes (the checks only guard accesses)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "masked_block_diffusion_denoise_b200")

# Two blocks of generation on a small bf16 model: prefixes appended as K/V
# (cache copy), split-K projections with their epilogue kernels (96 rows) or
# the fused epilogues of several M tiles (160 rows), clean passes, attention.
_SCRIPT = r"""
import hashlib, json, sys
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
import workloads as W
from masked_block_diffusion_denoise_b200 import DLM_BUF_K_CACHE, DLM_BUF_V_CACHE, dlm_kv_length
from masked_block_diffusion_denoise_b200.session import Session, sampler_params
out = {}
for batch in (3, 5):
    base = W.small_workload("bounds", batch=batch, canvas=32, steps=6, quota=0,
                            prefix_len=(40, 250))
    wl = base.replace(prefix_cap=base.prefix_len[1] + 2 * base.canvas)
    sh = wl.shape
    lens, toks, k, v = W.make_prefix(wl)
    sess = Session(sh, W.make_weights(sh, seed=wl.seed), max_batch=wl.batch,
                   max_prefix=wl.prefix_cap, max_canvas=wl.canvas)
    for b in range(wl.batch):
        n = int(lens[b])
        sess.kv_append_kv(b, np.ascontiguousarray(k[b][:, :n]), np.ascontiguousarray(v[b][:, :n]))
    p = sampler_params(canvas=wl.canvas, steps=wl.steps, threshold=wl.threshold, quota=wl.quota,
                       seed=wl.seed)
    cv = sess.new_canvas(wl.batch, wl.canvas)
    toks_out, nb = sess.generate(cv, p, 2, eos_early_stop=False)
    sess.check()
    Lcap = sess.max_prefix + sess.max_canvas
    shape = (wl.batch, sh.n_kv_heads, Lcap, sh.head_dim)
    kc = sess.buffer(DLM_BUF_K_CACHE, shape, torch.bfloat16)
    vc = sess.buffer(DLM_BUF_V_CACHE, shape, torch.bfloat16)
    h = hashlib.sha256()   # the written slots of each sequence (the rest is never read)
    for b in range(wl.batch):
        L = dlm_kv_length(sess.ctx, b)
        h.update(kc[b, :, :L].contiguous().view(torch.int16).cpu().numpy().tobytes())
        h.update(vc[b, :, :L].contiguous().view(torch.int16).cpu().numpy().tobytes())
    out[str(batch)] = {"tokens": toks_out.cpu().numpy().tolist(), "blocks": nb,
                       "kv_sha256": h.hexdigest()}
    sess.close()
print(json.dumps(out))
"""


def test_variants_are_exclusive():
    from masked_block_diffusion_denoise_b200 import build as B
    with pytest.raises(ValueError):
        B.build(trace=True, bounds=True)


def _run(library):
    env = dict(os.environ)
    env["DLM_LIBRARY"] = library
    r = subprocess.run([sys.executable, "-c", _SCRIPT, ROOT], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


@pytest.mark.gpu
def test_bounds_build_matches_the_default_build():
    from masked_block_diffusion_denoise_b200 import build as B
    bounds = B.build(bounds=True)
    default = B.build()
    got, want = _run(bounds), _run(default)
    assert set(got) == {"3", "5"}
    for key in want:
        assert got[key]["blocks"] == want[key]["blocks"] == 2
        assert got[key]["tokens"] == want[key]["tokens"], key
        assert got[key]["kv_sha256"] == want[key]["kv_sha256"], key
