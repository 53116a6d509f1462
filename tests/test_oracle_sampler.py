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


# adaptive stopping (DiffusionGemma page: argmax stable for stability_steps
# steps and mean entropy below stop_entropy -> the canvas freezes) -------------

@pytest.mark.parametrize("k", [0, 1, 3])
def test_adaptive_stop_freezes_after_k_stable_steps(k):
    C = 32
    cand, conf, _ = fixed_scores(C, np.random.default_rng(11))
    H = np.full(C, 0.01, np.float32)
    p = O.SamplerParams(canvas=C, steps=32, threshold=2.0, quota=1, stability_steps=k,
                        stop_entropy=0.1)
    st, stats, trace = run_fixed(C, p, cand, conf, H, eos_id=-5)
    # prev_cand starts at -1, so after call j (1-based) the count is j - 1:
    # the freeze comes at call k + 1 and commits every position still open
    assert len(trace) == k + 1 and st.done[0] and st.step[0] == k + 1
    assert stats.committed_by_sampler == k and stats.frozen == C - k
    assert np.array_equal(st.tokens[0], cand)


def test_adaptive_stop_bound_is_strict():
    C = 4
    cand = np.arange(C) + 20
    conf = np.full(C, 0.5, np.float32)
    H = np.full(C, 0.25, np.float32)            # mean exactly 0.25
    at = O.SamplerParams(canvas=C, steps=4, threshold=2.0, quota=1, stability_steps=0,
                         stop_entropy=0.25)
    st, stats, _ = run_fixed(C, at, cand, conf, H, eos_id=-5, limit=1)
    assert stats.frozen == 0 and st.committed[0].sum() == 1
    above = O.SamplerParams(**{**at.__dict__,
                               "stop_entropy": float(np.nextafter(np.float32(0.25), 1))})
    st, stats, _ = run_fixed(C, above, cand, conf, H, eos_id=-5, limit=1)
    assert stats.frozen == C and st.done[0]


def test_adaptive_stop_mean_counts_every_position():
    """READING: the mean entropy runs over all C positions, committed ones
    included, so confident open positions do not freeze a canvas whose
    committed positions were uncertain."""
    C = 8
    cand = np.arange(C) + 20
    conf = np.full(C, 0.5, np.float32)
    H = np.zeros(C, np.float32)
    H[:4] = 1.0                                 # mean 0.5
    p = O.SamplerParams(canvas=C, steps=8, threshold=2.0, quota=1, stability_steps=0,
                        stop_entropy=0.4)
    st = O.init_canvas(1, p, 100, 1000)
    st.committed[0, :4] = True
    st.tokens[0, :4] = cand[:4]
    st, stats, _ = run_fixed(C, p, cand, conf, H, eos_id=-5, state=st, limit=1)
    assert stats.frozen == 0 and st.committed[0].sum() == 5


def test_adaptive_stop_without_a_freeze_matches_the_plain_sampler():
    """An argmax that changes every step never counts as stable: the run is
    the one without adaptive stopping, bit for bit."""
    r = np.random.default_rng(12)
    C = 40
    cand, conf, H = fixed_scores(C, r)
    on = O.SamplerParams(canvas=C, steps=10, threshold=0.8, quota=2, corruption="uniform",
                         seed=3, stability_steps=1, stop_entropy=100.0)
    off = O.SamplerParams(**{**on.__dict__, "stop_entropy": -1.0})
    a, b = O.init_canvas(1, on, 100, 1000), O.init_canvas(1, off, 100, 1000)
    sa, sb = O.CanvasStats(), O.CanvasStats()
    for s in range(10):
        c = cand + (s % 2)
        O.select_canvas(a, 0, c, conf, H, on, vocab=1000, mask_id=100, eos_id=-5, stats=sa)
        O.select_canvas(b, 0, c, conf, H, off, vocab=1000, mask_id=100, eos_id=-5, stats=sb)
        assert np.array_equal(a.tokens, b.tokens) and np.array_equal(a.committed, b.committed)
        assert a.stable[0] == 0
    assert sa.frozen == 0 and sa.__dict__ == sb.__dict__


def test_adaptive_stop_with_no_stable_steps_equals_threshold_zero():
    """stability_steps 0 and a bound above every mean entropy freeze at the
    first call: each canvas takes its first candidates, as threshold 0 does."""
    p = O.SamplerParams(canvas=16, steps=8, threshold=2.0, quota=1, stability_steps=0,
                        stop_entropy=100.0)
    p0 = O.SamplerParams(canvas=16, steps=8, threshold=0.0, quota=1)
    _, m = _tiny_model("bf16")
    st = O.init_canvas(2, p, m.dims.mask_id, m.dims.vocab)
    stats = [O.CanvasStats(), O.CanvasStats()]
    assert O.decode_block(m, st, p, stats) == 1
    _, m0 = _tiny_model("bf16")
    st0 = O.init_canvas(2, p0, m0.dims.mask_id, m0.dims.vocab)
    assert O.decode_block(m0, st0, p0) == 1
    assert np.array_equal(st.tokens, st0.tokens) and st.done.all()
    assert all(s.frozen == 16 and s.committed_by_sampler == 0 for s in stats)


# multi-block generation -----------------------------------------------------------

def _zero_head_model():
    """A tiny model whose LM head is zero: every logit is 0, so the candidate
    is the lowest id that is not the mask (the EOS id 0 here), confidence
    1/(V-1) and entropy log(V-1) at every position."""
    import dataclasses
    wl, m = _tiny_model("f32", V=300)
    w = W.make_weights(wl.shape, seed=3)
    w["w_lm"] = np.zeros_like(w["w_lm"])
    dims = dataclasses.replace(m.dims, eos_id=0)
    z = O.OracleModel(dims, w)
    lens, toks, _, _ = W.make_prefix(wl, seed=3)
    for b, t in enumerate(toks):
        z.kv_append_tokens(b, t)
    return wl, z


def test_zero_head_scores_closed_form():
    wl, z = _zero_head_model()
    V = z.dims.vocab
    y = np.random.default_rng(0).standard_normal((5, z.dims.d_model))
    cand, conf, H, _ = O.scores(z.logits(y), z.dims.mask_id)
    assert (cand == 0).all()
    assert np.allclose(conf, 1.0 / (V - 1), rtol=1e-6) and np.allclose(H, np.log(V - 1))


@pytest.mark.parametrize("early", [True, False])
def test_generate_stops_at_eos(early):
    wl, z = _zero_head_model()
    C = 16
    L0 = [z.kv_len(b) for b in range(2)]
    p = O.SamplerParams(canvas=C, steps=4, threshold=2.0, quota=1)
    stats = [O.CanvasStats(), O.CanvasStats()]
    out, blocks = O.generate(z, p, 2, 3, eos_early_stop=early, stats=stats)
    # position 0 wins the confidence tie and commits the EOS; the rest of the
    # block is filled with EOS in the same step
    assert blocks == (1 if early else 3) and out.shape == (2, blocks * C)
    assert (out == 0).all()
    assert all(s.steps_used == blocks and s.eos_autofill == blocks * (C - 1) for s in stats)
    assert [z.kv_len(b) - L0[b] for b in range(2)] == [blocks * C] * 2


def test_generate_blocks_condition_only_on_what_precedes():
    """Block k equals one block decoded with seed + k over the prefix plus
    blocks 0..k-1 (cached through the clean pass), and the first block does
    not depend on how many blocks follow."""
    p = O.SamplerParams(canvas=16, steps=6, threshold=0.5, quota=2, corruption="uniform",
                        seed=21)
    _, m3 = _tiny_model("bf16")
    out3, n3 = O.generate(m3, p, 2, 3, eos_early_stop=False)
    _, m1 = _tiny_model("bf16")
    out1, n1 = O.generate(m1, p, 2, 1, eos_early_stop=False)
    assert (n3, n1) == (3, 1) and np.array_equal(out3[:, :16], out1)
    _, mk = _tiny_model("bf16")
    for b in range(2):
        mk.kv_append_tokens(b, out3[b, :32])
    p2 = O.SamplerParams(**{**p.__dict__, "seed": 23})
    st = O.init_canvas(2, p2, mk.dims.mask_id, mk.dims.vocab)
    O.decode_block(mk, st, p2)
    assert np.array_equal(st.tokens, out3[:, 32:])


# token editing (DiffusionGemma page editing_threshold; course section 14,
# LLaDA2.1 token-to-token editing) ----------------------------------------------

def _edit_params(C, **kw):
    base = dict(canvas=C, steps=8, threshold=2.0, quota=1, editing=1, editing_threshold=0.9)
    base.update(kw)
    return O.SamplerParams(**base)


def test_editing_worked_case():
    C = 6
    p = _edit_params(C)
    st = O.init_canvas(1, p, 100, 1000)
    st.tokens[0, :3] = [5, 6, 7]
    st.committed[0, :3] = True
    cand = np.array([5, 9, 8, 30, 31, 32])
    conf = np.array([0.99, 0.95, 0.5, 0.3, 0.6, 0.1], np.float32)
    stats = O.CanvasStats()
    O.select_canvas(st, 0, cand, conf, np.zeros(C, np.float32), p, vocab=1000, mask_id=100,
                    eos_id=-5, stats=stats)
    # 0: same id, no edit; 1: differs at 0.95 >= 0.9 -> 9; 2: differs at 0.5 < 0.9;
    # the quota then opens position 4 (highest confidence of the open ones)
    assert list(st.tokens[0]) == [5, 9, 7, 100, 31, 100]
    assert list(st.committed[0]) == [True, True, True, False, True, False]
    assert stats.edited == 1 and stats.committed_by_sampler == 1


def test_editing_above_one_is_the_plain_sampler():
    r = np.random.default_rng(13)
    C = 40
    cand, conf, H = fixed_scores(C, r)
    on = _edit_params(C, threshold=0.7, quota=2, corruption="uniform", seed=4,
                      editing_threshold=1.5)
    off = O.SamplerParams(**{**on.__dict__, "editing": 0})
    a, b = O.init_canvas(1, on, 100, 1000), O.init_canvas(1, off, 100, 1000)
    sa, sb = O.CanvasStats(), O.CanvasStats()
    for s in range(8):
        c = (cand + s) % 50
        O.select_canvas(a, 0, c, conf, H, on, vocab=1000, mask_id=100, eos_id=-5, stats=sa)
        O.select_canvas(b, 0, c, conf, H, off, vocab=1000, mask_id=100, eos_id=-5, stats=sb)
        assert np.array_equal(a.tokens, b.tokens) and np.array_equal(a.committed, b.committed)
    assert sa.edited == 0 and sa.__dict__ == sb.__dict__


def test_editing_at_zero_tracks_the_candidates():
    """editing_threshold 0: after every step each committed position holds
    that step's candidate, and committed positions never reopen."""
    r = np.random.default_rng(14)
    C = 24
    _, conf, H = fixed_scores(C, r)
    p = _edit_params(C, threshold=0.8, quota=3, editing_threshold=0.0)
    st = O.init_canvas(1, p, 100, 1000)
    stats = O.CanvasStats()
    for s in range(8):
        if st.done[0]:
            break
        prev = st.committed[0].copy()
        c = r.integers(0, 50, size=C)
        O.select_canvas(st, 0, c, conf, H, p, vocab=1000, mask_id=100, eos_id=-5, stats=stats)
        com = st.committed[0]
        assert (com[prev]).all()
        assert np.array_equal(st.tokens[0][com], c[com])
    assert st.done[0] and stats.edited > 0


def test_editing_leaves_the_eos_and_what_follows():
    C, eos = 10, 11
    p = _edit_params(C, editing_threshold=0.0)
    st = O.init_canvas(1, p, 100, 1000)
    st.tokens[0, [1, 4, 6]] = [3, eos, 8]
    st.committed[0, [1, 4, 6]] = True
    cand = np.full(C, 20)
    O.select_canvas(st, 0, cand, np.full(C, 0.5, np.float32), np.zeros(C, np.float32), p,
                    vocab=1000, mask_id=100, eos_id=eos)
    # before the EOS: edited; the EOS and the committed token after it: kept
    assert st.tokens[0, 1] == 20 and st.tokens[0, 4] == eos and st.tokens[0, 6] == 8
    assert st.eos_pos[0] == 4 and st.committed[0, 5:].all()


def test_an_edit_to_eos_truncates():
    C, eos = 8, 11
    p = _edit_params(C, editing_threshold=0.5)
    st = O.init_canvas(1, p, 100, 1000)
    st.tokens[0, [2, 5]] = [3, 4]
    st.committed[0, [2, 5]] = True
    cand = np.full(C, 20)
    cand[2] = eos
    conf = np.full(C, 0.1, np.float32)
    conf[2] = 0.6
    stats = O.CanvasStats()
    O.select_canvas(st, 0, cand, conf, np.zeros(C, np.float32), p, vocab=1000, mask_id=100,
                    eos_id=eos, stats=stats)
    assert st.eos_pos[0] == 2 and st.tokens[0, 2] == eos and stats.edited == 1
    # uncommitted positions after the new EOS are filled; the committed one at 5 stays
    assert st.tokens[0, 5] == 4 and (st.tokens[0, [3, 4, 6, 7]] == eos).all()
