"""Pins of the CPU oracle to things other than itself: the pages' worked
examples, published known answers, closed forms, library routines and
invariants.  CPU only."""
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from conftest import golden_lines, ROOT
from oracle import dlm_oracle as O
import workloads as W


# ---------------------------------------------------------------------------
# storage rounding
# ---------------------------------------------------------------------------

def test_bf16_rounding_matches_torch():
    """torch's float32 -> bfloat16 conversion rounds to nearest even."""
    r = np.random.default_rng(1)
    x = np.concatenate([r.standard_normal(100000).astype(np.float32) * 3,
                        np.float32([0.0, -0.0, 1.0, 1.00390625, 1.005859375, 65504.0, 1e-30])])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_to_bf16(x), ref)
    assert np.array_equal(W.from_bf16_bits(W.to_bf16_bits(x)).astype(np.float64), ref)


# ---------------------------------------------------------------------------
# reveal schedule (course section 6, worked example A)
# ---------------------------------------------------------------------------

def test_linear_schedule_worked_example():
    for row in golden_lines("course_schedule.txt"):
        n, s, *m = map(int, row)
        assert O.linear_mask_schedule(n, s) == tuple(m)
        assert all(a - b == 2 for a, b in zip(m, m[1:]))


@pytest.mark.parametrize("n,s", [(8, 4), (32, 32), (256, 48), (7, 3), (5, 9)])
def test_linear_schedule_closed_form(n, s):
    m = O.linear_mask_schedule(n, s)
    assert m[0] == n and m[-1] == 0 and len(m) == s + 1
    assert all(a >= b for a, b in zip(m, m[1:]))
    for i, v in enumerate(m):   # smallest integer >= N(S-i)/S
        assert v - 1 < n * (s - i) / s <= v


def test_linear_schedule_rejects_bad_args():
    for bad in [(0, 4), (8, 0), (-1, 2), (True, 2), (2.0, 2)]:
        with pytest.raises(ValueError):
            O.linear_mask_schedule(*bad)


# ---------------------------------------------------------------------------
# Philox4x32-10
# ---------------------------------------------------------------------------

def test_philox_known_answers():
    for row in golden_lines("philox4x32_10_kat.txt"):
        v = [int(x, 16) for x in row]
        out = O.philox4x32_10(v[0:4], (v[4], v[5]))
        assert [int(o) for o in out] == v[6:10]


def test_philox_matches_triton_interpreter():
    """Independent implementation: Triton's philox, run by its CPU
    interpreter, on random counters and keys."""
    pytest.importorskip("triton")
    script = r'''
import os, sys
os.environ["TRITON_INTERPRET"] = "1"
import numpy as np, torch, triton, triton.language as tl
@triton.jit
def k(out, c0p, c1p, c2p, c3p, seed, N: tl.constexpr):
    i = tl.arange(0, N)
    a, b, c, d = tl.philox(seed, tl.load(c0p + i), tl.load(c1p + i), tl.load(c2p + i), tl.load(c3p + i))
    tl.store(out + 4 * i, a); tl.store(out + 4 * i + 1, b); tl.store(out + 4 * i + 2, c); tl.store(out + 4 * i + 3, d)
r = np.random.default_rng(7)
N = 64
ctr = r.integers(0, 2**32, size=(4, N), dtype=np.uint64)
seed = int(r.integers(0, 2**63))
out = torch.zeros(4 * N, dtype=torch.int32)
k[(1,)](out, *[torch.from_numpy(c.astype(np.uint32).view(np.int32)) for c in ctr], seed, N=N)
np.savez(sys.argv[1], ctr=ctr, seed=np.uint64(seed), out=out.numpy().view(np.uint32).astype(np.uint64))
'''
    import tempfile
    with tempfile.TemporaryDirectory() as td:
        path = os.path.join(td, "p.npz")
        env = dict(os.environ, TRITON_INTERPRET="1")
        res = subprocess.run([sys.executable, "-c", script, path], env=env,
                             capture_output=True, text=True, timeout=600)
        if res.returncode != 0:
            pytest.skip("triton interpreter unavailable: " + res.stderr[-300:])
        a = np.load(path)
        N = 64
        ctr, seed = a["ctr"], int(a["seed"])
        ref = a["out"].reshape(N, 4).T
    out = O.philox4x32_10(list(ctr), O.seed_key(seed))
    for w in range(4):
        assert np.array_equal(out[w].astype(np.uint64), ref[w])


def test_uniform_ids_range_and_uniformity():
    V = 1000
    ids = np.concatenate([O.uniform_token_ids(123, b, s, np.arange(256), V)
                          for b in range(4) for s in range(40)])
    assert ids.min() >= 0 and ids.max() < V
    counts = np.bincount(ids, minlength=V)
    expected = ids.size / V
    chi2 = ((counts - expected) ** 2 / expected).sum()
    # V-1 = 999 degrees of freedom: mean 999, sd ~44.7; 6 sd bound
    assert abs(chi2 - (V - 1)) < 6 * math.sqrt(2 * (V - 1))
    # different steps / canvases give different streams
    a = O.uniform_token_ids(1, 0, 1, np.arange(64), 1 << 20)
    b = O.uniform_token_ids(1, 0, 2, np.arange(64), 1 << 20)
    c = O.uniform_token_ids(1, 1, 1, np.arange(64), 1 << 20)
    assert (a != b).mean() > 0.9 and (a != c).mean() > 0.9


def test_gumbel_max_samples_softmax():
    """Gumbel-max trick: argmax(z + G) is distributed as softmax(z)."""
    z = np.log(np.array([0.1, 0.2, 0.3, 0.4, 1e-9]))
    V = z.size
    n = 40000
    wins = np.zeros(V)
    for i in range(n):
        g = O.gumbel_noise(99, 0, i // 512, i % 512, V)
        wins[np.argmax(z + g)] += 1
    p = np.exp(z) / np.exp(z).sum()
    expected = n * p
    sel = expected > 5
    chi2 = (((wins - expected) ** 2)[sel] / expected[sel]).sum()
    assert chi2 < 25.0, (wins, expected)


# ---------------------------------------------------------------------------
# RoPE
# ---------------------------------------------------------------------------

def test_rope_textbook_properties():
    r = np.random.default_rng(3)
    dh, theta = 64, 1.0e6
    x = r.standard_normal((5, dh))
    pos = np.array([0, 1, 17, 4096, 32800])
    y = O.rope(x, pos, theta)
    assert np.allclose(y[0], x[0])                          # position 0 is the identity
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1))
    # complex form: (x_j + i x_{j+D/2}) * exp(i pos theta^(-2j/D))
    half = dh // 2
    zc = (x[:, :half] + 1j * x[:, half:]) * np.exp(
        1j * pos[:, None] * theta ** (-2.0 * np.arange(half) / dh)[None, :])
    assert np.allclose(y[:, :half], zc.real) and np.allclose(y[:, half:], zc.imag)
    # relative position: <R(q, m), R(k, n)> depends on m - n only
    q, k = r.standard_normal((1, dh)), r.standard_normal((1, dh))
    a = (O.rope(q, np.array([10]), theta) * O.rope(k, np.array([3]), theta)).sum()
    b = (O.rope(q, np.array([1010]), theta) * O.rope(k, np.array([1003]), theta)).sum()
    assert abs(a - b) < 1e-9


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def test_attention_special_cases():
    r = np.random.default_rng(4)
    q = r.standard_normal((6, 16))
    k1, v1 = r.standard_normal((1, 16)), r.standard_normal((1, 16))
    assert np.allclose(O.attention_head(q, k1, v1), np.repeat(v1, 6, axis=0))   # one key -> V
    k, v = r.standard_normal((9, 16)), r.standard_normal((9, 16))
    assert np.allclose(O.attention_head(np.zeros((3, 16)), k, v), v.mean(axis=0))  # equal scores
    perm = r.permutation(9)
    assert np.allclose(O.attention_head(q, k, v), O.attention_head(q, k[perm], v[perm]))


def test_attention_matches_torch_sdpa_with_gqa():
    """The model's head grouping against torch's scaled_dot_product_attention
    (enable_gqa) in float64."""
    r = np.random.default_rng(5)
    dims = O.ModelDims(d_model=64, n_heads=8, n_kv_heads=2, head_dim=16, vocab=50, dtype="f32",
                       rope_theta=0.0)
    w = {n: r.standard_normal(s).astype(np.float32) * 0.3 for n, s in
         [("emb", (50, 64)), ("w_q", (128, 64)), ("w_k", (32, 64)), ("w_v", (32, 64)),
          ("w_o", (64, 128)), ("w_lm", (50, 64))]}
    m = O.OracleModel(dims, w)
    m.kv_append_kv(0, r.standard_normal((2, 11, 16)), r.standard_normal((2, 11, 16)))
    C = 7
    q = r.standard_normal((C, 8, 16))
    k = r.standard_normal((C, 2, 16))
    v = r.standard_normal((C, 2, 16))
    o = m.attend(0, q, k, v)
    K = np.concatenate([m.k_cache[0], k.transpose(1, 0, 2)], axis=1)
    V = np.concatenate([m.v_cache[0], v.transpose(1, 0, 2)], axis=1)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q.transpose(1, 0, 2))[None], torch.from_numpy(K)[None],
        torch.from_numpy(V)[None], enable_gqa=True)[0]
    ref = ref.numpy().transpose(1, 0, 2).reshape(C, -1)
    assert np.allclose(o, O.round_to_f32(ref), atol=1e-6)


# ---------------------------------------------------------------------------
# scores
# ---------------------------------------------------------------------------

def test_scores_closed_forms():
    V, mask = 1000, 100
    cand, conf, H, _ = O.scores(np.zeros((3, V)), mask)
    assert (cand == 0).all()
    assert np.allclose(conf, 1.0 / (V - 1)) and np.allclose(H, math.log(V - 1))
    lg = np.zeros((2, V)); lg[:, mask] = 50.0
    cand, _, _, _ = O.scores(lg, mask)
    assert (cand == 0).all()                                   # the mask is never a candidate
    cand, conf, H, _ = O.scores(np.zeros((1, V)), -1)
    assert np.allclose(H, math.log(V))
    lg = np.zeros((1, V)); lg[0, 777] = 200.0
    cand, conf, H, _ = O.scores(lg, mask)
    assert cand[0] == 777 and abs(conf[0] - 1) < 1e-12 and abs(H[0]) < 1e-12
    lg = np.zeros((1, V)); lg[0, [5, 3, 900]] = 4.0             # tie -> lowest index
    assert O.scores(lg, mask)[0][0] == 3


def test_scores_match_scipy():
    sp = pytest.importorskip("scipy")
    from scipy.special import softmax
    from scipy.stats import entropy
    r = np.random.default_rng(6)
    lg = r.standard_normal((20, 3000)) * 2.5
    cand, conf, H, _ = O.scores(lg, -1)
    p = softmax(lg, axis=1)
    assert np.array_equal(cand, np.argmax(p, axis=1))
    assert np.allclose(conf, p.max(axis=1), rtol=1e-12)
    assert np.allclose(H, entropy(p, axis=1), rtol=1e-10)
    # temperature: softmax(z / T)
    cand, conf, H, _ = O.scores(lg, -1, inv_temp=np.float32(1 / 0.7))
    p = softmax((lg.astype(np.float32) * np.float32(1 / 0.7)).astype(np.float64), axis=1)
    assert np.allclose(H, entropy(p, axis=1), rtol=1e-10)


def test_chunked_scoring_equals_full():
    """Non-materialised chunked greedy scoring gives the argmax of the full
    hidden @ weight^T product (Nemotron guide, section 10: the chunked scorer
    is checked one by one against the full argmax)."""
    r = np.random.default_rng(8)
    V = 1000
    lg = r.standard_normal((16, V)) * 3
    lg[0, [17, 517]] = 20.0        # tie across two chunks
    lg[1, [130, 131]] = 20.0       # tie inside a chunk
    lg[2, :] = 1.0                 # all equal
    lg[3, 128:256] = -np.inf       # a whole chunk excluded
    for chunk in (128, 100, 37, 1000):
        for row in range(16):
            cand, conf, H, _ = O.scores(lg[row:row + 1], -1)
            c2, conf2, H2 = O.combine_partials(O.chunk_partials(lg[row], chunk))
            assert c2 == cand[0]
            assert abs(conf2 - conf[0]) < 1e-12 and abs(H2 - H[0]) < 1e-9


def test_annealed_temperature_end_points():
    """DiffusionGemma page: t_max at the first step, t_min at the last."""
    assert O.annealed_temperature(0.8, 0.4, 0, 48) == np.float32(0.8)
    assert O.annealed_temperature(0.8, 0.4, 47, 48) == np.float32(0.4)
    ts = [O.annealed_temperature(0.8, 0.4, s, 48) for s in range(48)]
    assert all(a > b for a, b in zip(ts, ts[1:]))
    assert O.annealed_temperature(0.8, 0.4, 0, 1) == np.float32(0.8)


# ---------------------------------------------------------------------------
# roofline calculator (course sections 1, 10, 11)
# ---------------------------------------------------------------------------

def test_course_roofline_numbers():
    from masked_block_diffusion_denoise_b200 import roofline as R
    P, Wb, bw, fl = 8e9, 16e9, 3.35e12, 990e12
    ar = R.ar_bounds(P, Wb, bw, fl)
    p1024 = R.diffusion_pass(P, 1024, Wb, bw, fl)
    q64 = R.diffusion_tokens_per_s(1024, 64, p1024["t_pass_s"])
    p256 = R.diffusion_pass(P, 256, Wb, bw, fl)
    p256_4b = R.diffusion_pass(P, 256, Wb / 4, bw, fl)
    got = {
        "ar_t_mem_ms": ar["t_mem_s"] * 1e3,
        "ar_t_compute_us": ar["t_compute_s"] * 1e6,
        "ar_compute_share_pct": ar["compute_share"] * 100,
        "ar_tokens_per_s": ar["tokens_per_s"],
        "pass1024_tflop": p1024["flop"] / 1e12,
        "pass1024_ms": p1024["t_pass_s"] * 1e3,
        "q_s64_tokens_per_s": q64,
        "speedup_vs_ar": q64 / ar["tokens_per_s"],
        "parity_steps": R.parity_steps(1024, p1024["t_pass_s"], ar["tokens_per_s"]),
        "parity_batch": 966.8 / 209.4,
        "pass256_ms": p256["t_compute_s"] * 1e3,
        "w4bit_read_ms": p256_4b["t_mem_s"] * 1e3,
        "q256_s16_tokens_per_s": R.diffusion_tokens_per_s(256, 16, p256_4b["t_pass_s"]),
    }
    assert p1024["bound"] == "compute" and p256["bound"] == "memory"
    assert p256_4b["bound"] == "compute"
    for key, val, tol in golden_lines("course_roofline.txt"):
        assert abs(got[key] - float(val)) <= float(tol) * float(val), (key, got[key], val)


def test_step_work_counts():
    from masked_block_diffusion_denoise_b200 import roofline as R
    s = R.StepShape(4096, 32, 8, 128, 131072, 2, 32, [2048])
    w = R.step_work(s)
    assert w["lm_head"]["bytes"] > 131072 * 4096 * 2
    assert abs(w["lm_head"]["flop"] - 2 * 32 * 4096 * 131072) < 1
    # K and V of 2048 + 32 keys for 8 heads of 128
    assert w["attention"]["bytes"] >= 2 * 2080 * 1024 * 2
