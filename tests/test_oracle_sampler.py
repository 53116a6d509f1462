"""Pins of the oracle's sampler: the five invariants the method fixes, the
course worked example and the selection rules' special cases.  CPU only."""
import numpy as np
import pytest

from conftest import golden_lines
from oracle import dlm_oracle as O
import workloads as W


def fixed_scores(C, r, V=50):
    cand = r.integers(0, V, size=C)
    conf = r.random(C).astype(np.float32)
    H = (r.random(C) * 3).astype(np.float32)
    return cand, conf, H


def run_fixed(C, p, cand, conf, H, *, mask_id=100, V=1000, eos_id=11, state=None, limit=None):
    """Decode one canvas with scores that do not depend on the canvas."""
    st = state or O.init_canvas(1, p, mask_id, V)
    stats = O.CanvasStats()
    trace = []
    calls = 0
    while not st.done[0] and calls < (limit or p.steps):
        before = st.copy()
        O.select_canvas(st, 0, cand, conf, H, p, vocab=V, mask_id=mask_id, eos_id=eos_id,
                        stats=stats)
        newly = np.flatnonzero(st.committed[0] & ~before.committed[0])
        trace.append((before, st.copy(), newly))
        calls += 1
    return st, stats, trace


# (1) threshold 0 -> every position commits in the first step ----------------

def test_threshold_zero_commits_all_in_step_one():
    r = np.random.default_rng(0)
    for C in (1, 7, 32, 256):
        cand, conf, H = fixed_scores(C, r)
        p = O.SamplerParams(canvas=C, steps=32, threshold=0.0, quota=1)
        st, stats, trace = run_fixed(C, p, cand, conf, H, eos_id=-5)
        assert len(trace) == 1 and st.done[0]
        assert np.array_equal(st.tokens[0], cand) and stats.committed_by_sampler == C


# (2) threshold > 1, quota 1 -> commit order is descending confidence ---------

def test_threshold_above_one_quota_one_orders_by_confidence():
    r = np.random.default_rng(1)
    C = 40
    cand, conf, H = fixed_scores(C, r)
    conf[[3, 9]] = conf[5]          # ties -> lower index first
    p = O.SamplerParams(canvas=C, steps=C, threshold=1.5, quota=1)
    st, stats, trace = run_fixed(C, p, cand, conf, H, eos_id=-5)
    order = [int(t[2][0]) for t in trace]
    assert all(len(t[2]) == 1 for t in trace)
    assert order == sorted(range(C), key=lambda i: (-conf[i], i))


# (3) committed tokens never revert -------------------------------------------

@pytest.mark.parametrize("corruption", ["mask", "uniform"])
def test_committed_never_revert(corruption):
    r = np.random.default_rng(2)
    C = 64
    for trial in range(5):
        cand, conf, H = fixed_scores(C, r)
        p = O.SamplerParams(canvas=C, steps=16, threshold=0.8, quota=3, corruption=corruption,
                            seed=trial)
        st, stats, trace = run_fixed(C, p, cand, conf, H, eos_id=-5)
        for before, after, _ in trace:
            com = before.committed[0]
            assert after.committed[0][com].all()
            assert np.array_equal(after.tokens[0][com], before.tokens[0][com])


# (4) decoding terminates within the step budget ------------------------------

@pytest.mark.parametrize("C,S,q", [(32, 32, 1), (64, 8, 1), (256, 48, 0), (33, 5, 2), (10, 1, 1)])
def test_terminates_within_budget(C, S, q):
    r = np.random.default_rng(C * S)
    cand, conf, H = fixed_scores(C, r)
    p = O.SamplerParams(canvas=C, steps=S, threshold=2.0, quota=q)
    st, stats, trace = run_fixed(C, p, cand, conf, H, eos_id=-5, limit=10 * S)
    assert st.done[0] and len(trace) <= S and stats.steps_used <= S
    if q == 0:   # the default quota ceil(C/S) finishes exactly at the budget or before
        assert len(trace) == -(-C // -(-C // S))


def test_forced_completion_on_last_step():
    C, S = 64, 8
    r = np.random.default_rng(3)
    cand, conf, H = fixed_scores(C, r)
    p = O.SamplerParams(canvas=C, steps=S, threshold=2.0, quota=1)
    st, stats, trace = run_fixed(C, p, cand, conf, H, eos_id=-5)
    assert len(trace) == S and st.done[0]
    assert stats.forced_at_budget == C - S
    assert stats.committed_by_sampler == C


# course worked example A / section 12 sampler -------------------------------

def test_course_schedule_mode_matches_worked_example():
    (n, s, *m), = list(golden_lines("course_schedule.txt"))
    n, s, m = int(n), int(s), [int(x) for x in m]
    r = np.random.default_rng(4)
    V = 12
    logits = r.standard_normal((n, V)) * 2
    cand, conf, H, _ = O.scores(logits, -1)
    p = O.SamplerParams(canvas=n, steps=s, threshold=2.0, schedule="course")
    st, stats, trace = run_fixed(n, p, cand, conf, H, mask_id=-1, V=V, eos_id=-5)
    masked_counts = [n] + [int((~t[1].committed[0]).sum()) for t in trace]
    assert masked_counts == m
    # the course's own sampler with the same fixed predictor opens the same positions
    tokens, ctrace = O.course_sampler(lambda t, k: logits, n, s, -1)
    assert [tuple(sorted(o)) for o, _ in ctrace] == [tuple(sorted(t[2])) for t in trace]
    assert np.array_equal(tokens, st.tokens[0])


def test_course_ties_go_to_lower_index():
    """Course section 12: equal scores are resolved by the lower position
    index."""
    n, s = 8, 4
    tokens, trace = O.course_sampler(lambda t, k: np.zeros((n, 5)), n, s, -1)
    assert [o for o, _ in trace] == [(0, 1), (2, 3), (4, 5), (6, 7)]
    cand, conf, H = np.zeros(n, int), np.full(n, 0.2, np.float32), np.zeros(n, np.float32)
    p = O.SamplerParams(canvas=n, steps=s, threshold=2.0, quota=2)
    st, stats, tr = run_fixed(n, p, cand, conf, H, mask_id=-1, V=5, eos_id=-5)
    assert [tuple(t[2]) for t in tr] == [(0, 1), (2, 3), (4, 5), (6, 7)]


# threshold + quota readings ---------------------------------------------------

def test_union_and_additive_agree_without_threshold_hits():
    r = np.random.default_rng(5)
    C = 32
    cand, conf, H = fixed_scores(C, r)
    conf = conf * np.float32(0.5)    # nothing reaches 0.9
    a = run_fixed(C, O.SamplerParams(canvas=C, steps=8, threshold=0.9, quota=4), cand, conf, H,
                  eos_id=-5)[0]
    b = run_fixed(C, O.SamplerParams(canvas=C, steps=8, threshold=0.9, quota=4,
                                     quota_rule="additive"), cand, conf, H, eos_id=-5)[0]
    assert np.array_equal(a.tokens, b.tokens)


def test_threshold_commits_every_confident_position():
    C = 16
    cand = np.arange(C)
    conf = np.full(C, 0.1, np.float32)
    conf[[2, 5, 11]] = [0.95, 0.9, 0.99]      # 0.9 counts ("at least")
    p = O.SamplerParams(canvas=C, steps=16, threshold=0.9, quota=1)
    st, stats, trace = run_fixed(C, p, cand, conf, np.zeros(C, np.float32), eos_id=-5, limit=1)
    assert sorted(trace[0][2]) == [2, 5, 11]


# entropy bound ---------------------------------------------------------------

def test_entropy_bound_worked_cases():
    C = 4
    H = np.array([0.05, 0.02, 0.04, 0.5], np.float32)
    cand = np.array([7, 8, 9, 10])
    conf = np.zeros(C, np.float32)
    p = O.SamplerParams(canvas=C, steps=10, entropy_bound=0.1)
    st, stats, trace = run_fixed(C, p, cand, conf, H, eos_id=-5)
    # order by H: 1 (0.02), 2 (0.06 cumulative), 0 (0.11 > 0.1) -> {1, 2}; then 0 alone
    # (0.05), then 3 alone (0.5 > bound, but at least one)
    assert [tuple(sorted(t[2])) for t in trace] == [(1, 2), (0,), (3,)]
    p = O.SamplerParams(canvas=C, steps=10, entropy_bound=100.0)
    assert len(run_fixed(C, p, cand, conf, H, eos_id=-5)[2]) == 1
    p = O.SamplerParams(canvas=C, steps=10, entropy_bound=0.0)
    tr = run_fixed(C, p, cand, conf, H, eos_id=-5)[2]
    assert [int(t[2][0]) for t in tr] == [1, 2, 0, 3]


# EOS ---------------------------------------------------------------------------

def test_eos_plant_finishes_the_canvas():
    C, eos = 32, 11
    p = O.SamplerParams(canvas=C, steps=32, threshold=2.0, quota=2)
    st = O.init_canvas(1, p, 100, 1000)
    st.tokens[0, 9] = eos
    st.committed[0, 9] = True
    cand = np.full(C, 5)
    conf = np.linspace(0.1, 0.5, C).astype(np.float32)   # later positions more confident
    st, stats, trace = run_fixed(C, p, cand, conf, np.zeros(C, np.float32), eos_id=eos, state=st)
    assert st.done[0] and st.eos_pos[0] == 9
    assert (st.tokens[0, 10:] == eos).all() and (st.tokens[0, :9] == 5).all()
    assert len(trace) == 5 and stats.committed_by_sampler == 9 and stats.eos_autofill == C - 10
    # the sampler chose at most the quota per step, all before the EOS
    assert all((t[2] < 9).sum() <= 2 for t in trace)


def test_eos_committed_by_the_sampler_truncates():
    C, eos = 16, 11
    cand = np.full(C, 3)
    cand[4] = eos
    conf = np.zeros(C, np.float32)
    conf[4] = 0.99
    p = O.SamplerParams(canvas=C, steps=16, threshold=0.9, quota=1)
    st, stats, trace = run_fixed(C, p, cand, conf, np.zeros(C, np.float32), eos_id=eos)
    assert st.eos_pos[0] == 4 and (st.tokens[0, 5:] == eos).all()
    assert stats.eos_autofill == C - 5


# re-noise -----------------------------------------------------------------------

def test_uniform_renoise_uses_the_step_stream():
    C, V = 24, 5000
    p = O.SamplerParams(canvas=C, steps=8, threshold=2.0, quota=3, corruption="uniform", seed=77)
    st = O.init_canvas(1, p, 100, V)
    assert np.array_equal(st.tokens[0], O.uniform_token_ids(77, 0, 0, np.arange(C), V))
    cand = np.arange(C) + 1000
    conf = np.linspace(0, 1, C).astype(np.float32)
    O.select_canvas(st, 0, cand, conf, np.zeros(C, np.float32), p, vocab=V, mask_id=100,
                    eos_id=-5)
    rest = np.flatnonzero(~st.committed[0])
    assert np.array_equal(st.tokens[0, rest], O.uniform_token_ids(77, 0, 1, rest, V))
    assert sorted(np.flatnonzero(st.committed[0])) == [21, 22, 23]


# resume (counter-based RNG makes the state all there is) ------------------------

def test_resume_is_bit_identical():
    r = np.random.default_rng(9)
    C = 48
    cand, conf, H = fixed_scores(C, r)
    p = O.SamplerParams(canvas=C, steps=12, threshold=0.7, quota=2, corruption="uniform", seed=5)
    full = run_fixed(C, p, cand, conf, H, eos_id=-5)[0]
    part = run_fixed(C, p, cand, conf, H, eos_id=-5, limit=5)[0]
    resumed = run_fixed(C, p, cand, conf, H, eos_id=-5, state=part.copy())[0]
    assert np.array_equal(full.tokens, resumed.tokens) and (full.step == resumed.step).all()


# model-level ------------------------------------------------------------------------

def _tiny_model(dtype="f32", V=300):
    wl = W.small_workload(d_model=64, n_heads=4, n_kv_heads=2, head_dim=16, vocab=V,
                          dtype=dtype, prefix_kind="tokens", prefix_len=(20, 29), batch=2,
                          canvas=16, steps=8)
    dims = O.ModelDims.of(wl.shape)
    w = W.make_weights(wl.shape, seed=3)
    m = O.OracleModel(dims, w)
    lens, toks, _, _ = W.make_prefix(wl, seed=3)
    for b, t in enumerate(toks):
        m.kv_append_tokens(b, t)
    return wl, m


def test_clean_pass_equals_canvas_keys():
    """The K/V a finished block gets from the clean pass equal the canvas K/V
    computed at the same absolute positions (one layer: no dependence on the
    attention pattern)."""
    wl, m = _tiny_model()
    tokens = np.arange(10, 26)
    L = m.kv_len(0)
    out = m.forward(0, tokens)
    m.kv_append_tokens(0, tokens)
    assert np.allclose(m.k_cache[0][:, L:], out["k"].transpose(1, 0, 2))
    assert np.allclose(m.v_cache[0][:, L:], out["v"].transpose(1, 0, 2))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_model_block_invariants(dtype):
    wl, m = _tiny_model(dtype)
    p = O.SamplerParams(canvas=16, steps=8, threshold=0.9, quota=2)
    st = O.init_canvas(2, p, m.dims.mask_id, m.dims.vocab)
    stats = [O.CanvasStats(), O.CanvasStats()]
    prev = st.copy()
    calls = 0
    while not st.done.all():
        O.denoise_step(m, st, p, stats)
        com = prev.committed
        assert (st.committed[com]).all() and np.array_equal(st.tokens[com], prev.tokens[com])
        assert not (st.tokens[st.committed] == m.dims.mask_id).any()
        prev = st.copy()
        calls += 1
    assert calls <= 8 and all(s.steps_used <= 8 for s in stats)
    p0 = O.SamplerParams(canvas=16, steps=8, threshold=0.0, quota=1)
    st0 = O.init_canvas(2, p0, m.dims.mask_id, m.dims.vocab)
    O.denoise_step(m, st0, p0)
    assert st0.done.all()


def test_entropy_bound_block_runs_to_completion():
    wl, m = _tiny_model("bf16")
    p = O.SamplerParams(canvas=16, steps=8, entropy_bound=0.1, corruption="uniform", seed=4)
    st = O.init_canvas(2, p, m.dims.mask_id, m.dims.vocab)
    calls = O.decode_block(m, st, p)
    assert st.done.all() and calls <= 8
