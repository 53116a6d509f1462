"""Device timeline (DLM_TRACE build): the summary's arithmetic on a table
built by hand, the default library's refusal, and on a GPU the order the
programmatic-launch chain imposes on the stamps."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_summary_on_a_hand_built_table():
    from masked_block_diffusion_denoise_b200 import trace as T
    kinds, ctas, slots = 16, 512, 8
    t = np.zeros((kinds, ctas, slots), dtype=np.uint64)
    base = 10_000_000
    # embed: 2 CTAs in at +0 / +1000 ns, wait +500 / +1500, out +3000 / +4000
    t[0, 0, :3] = [base, base + 3000, base + 500]
    t[0, 1, :3] = [base + 1000, base + 4000, base + 1500]
    # commit: 1 CTA, phases 3..5
    t[9, 0, :6] = [base + 2000, base + 9000, base + 5000, base + 6000, base + 7000, base + 8500]
    s = T._summary(t)
    assert s["order"] == ["embed", "commit"]
    e = s["kernels"]["embed"]
    assert e["ctas"] == 2
    assert e["entry"] == {"min": 0.0, "med": 0.5, "max": 1.0}
    assert e["exit"] == {"min": 3.0, "med": 3.5, "max": 4.0}
    assert e["wait"]["med"] == 1.0
    c = s["kernels"]["commit"]
    assert c["phases"]["rows reduced"]["med"] == 6.0
    assert c["phases"]["keys sorted"]["med"] == 7.0
    assert c["phases"]["done"]["med"] == 8.5
    assert s["step_span_us"] == 9.0
    assert "| commit | 1 |" in T.markdown(s)


def test_default_library_refuses_tracing():
    import masked_block_diffusion_denoise_b200 as dlm
    if not os.path.exists(os.path.join(ROOT, "masked_block_diffusion_denoise_b200",
                                       "libdlm.so")):
        pytest.skip("library not built")
    if os.environ.get("DLM_LIBRARY"):
        pytest.skip("another library selected")
    with pytest.raises(dlm.DlmError) as ei:
        dlm.dlm_trace_layout()
    assert ei.value.code == dlm.DLM_ESTATE


@pytest.mark.gpu
def test_trace_follows_the_launch_chain(tmp_path):
    out = tmp_path / "trace.json"
    env = dict(os.environ)
    env.pop("DLM_LIBRARY", None)
    r = subprocess.run([sys.executable, "-m", "masked_block_diffusion_denoise_b200.trace",
                        "--workload", "8b_b1", "--blocks", "1", "--json", str(out)],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    s = json.loads(out.read_text())
    order = s["order"]
    assert order[0] == "embed" and order[-1] == "commit"
    for name in ("qkv_gemm", "attention", "wo_gemm", "lm_head"):
        assert name in order
    k = s["kernels"]
    for name in order:
        rec = k[name]
        assert rec["entry"]["min"] <= rec["wait"]["min"] <= rec["exit"]["max"], name
    # a kernel's wait returns only after its predecessor's grid has finished
    # (global timer, 0.5 us of slack for the stamps' own placement)
    for prev, nxt in zip(order, order[1:]):
        assert k[nxt]["wait"]["min"] >= k[prev]["exit"]["max"] - 0.5, (prev, nxt)
    # the LM head dominates the step
    lm = k["lm_head"]
    assert lm["exit"]["max"] - lm["wait"]["min"] > 0.5 * s["step_span_us"]
