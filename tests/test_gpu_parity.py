"""Parity of the CUDA path (through the C ABI) with the CPU oracle on seeded
inputs.  Every stage is teacher-forced: the oracle is given the GPU's own
inputs to that stage, so one rounding difference cannot cascade.

Standards (the method's parity bar):
  * selection on identical float32 inputs: token ids, commit masks, step,
    done, EOS position and counters bit-exact;
  * candidates from identical float32 logits bit-exact, confidence within
    1e-3, entropy within 1e-3;
  * attention output within 2e-2 absolute of the float64 oracle;
  * stored bf16 activations equal up to one rounding step;
  * candidates from the oracle's float64 logits: equal except near ties
    (top-2 gap < 1e-3), which are counted.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from gpu_util import (abs_terms, assert_storage_close, check_one_step, lib_params, make_pair,
                      oracle_params, record_near_ties, to64)
from oracle import dlm_oracle as O
import workloads as W

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU-only hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

from masked_block_diffusion_denoise_b200 import (DLM_BUF_CAND, DLM_BUF_CONF, DLM_BUF_ENTROPY,
                                                 DLM_BUF_K_CACHE, DLM_BUF_V_CACHE, DLM_BUF_Y)


SMALL = {
    # GQA 2, vocab with a ragged 96-column tail, ragged prefixes, one M tile
    "small_gqa2": W.small_workload("small_gqa2", steps=8, quota=4),
    # GQA 4, two batches of 64 positions: 256 rows -> two M tiles, 256-wide LM tiles
    "small_mtiles": W.small_workload("small_mtiles", n_heads=8, n_kv_heads=2, batch=4,
                                     canvas=64, steps=6, quota=0, prefix_len=(64, 300),
                                     prefix_cap=320, vocab=3000),
    # canvas not a multiple of 8, single KV head, threshold 0 (all commit in one step)
    "small_c37": W.small_workload("small_c37", n_heads=2, n_kv_heads=1, canvas=37, batch=3,
                                  steps=5, threshold=0.0, quota=1, prefix_len=(1, 130),
                                  prefix_cap=160),
    # uniform corruption, quota from ceil(C/S)
    "small_uniform": W.small_workload("small_uniform", corruption="uniform", steps=7, quota=0,
                                      seed=3),
    # e4m3 LM head, one M tile (128-wide vocabulary tiles, ragged vocabulary)
    "small_fp8": W.small_workload("small_fp8", steps=6, quota=0, lm_fp8=True, seed=4),
    # e4m3 LM head over two M tiles (256-wide vocabulary tiles), uniform corruption
    "small_fp8_mtiles": W.small_workload("small_fp8_mtiles", n_heads=8, n_kv_heads=2, batch=4,
                                         canvas=64, steps=4, quota=0, prefix_len=(64, 300),
                                         prefix_cap=320, vocab=3000, lm_fp8=True,
                                         corruption="uniform"),
    # two M tiles, 256-wide LM tiles, vocabulary 20440 = 80 tiles (the last
    # ragged): on 148 SMs 74 CTAs share each M tile and 6 of them take a
    # second tile
    "small_lm_tail": W.small_workload("small_lm_tail", n_heads=8, n_kv_heads=2, batch=4,
                                      canvas=64, steps=3, quota=0, prefix_len=(64, 300),
                                      prefix_cap=320, vocab=20440, seed=7),
    # NVFP4 LM head, one M tile, ragged vocabulary
    "small_nvfp4": W.small_workload("small_nvfp4", steps=6, quota=0, lm_nvfp4=True, seed=4),
    # NVFP4 LM head over two M tiles, d 512 (two k-blocks), uniform corruption
    "small_nvfp4_mtiles": W.small_workload("small_nvfp4_mtiles", d_model=512, n_heads=8,
                                           n_kv_heads=2, batch=4, canvas=64, steps=4, quota=0,
                                           prefix_len=(64, 300), prefix_cap=320, vocab=3000,
                                           lm_nvfp4=True, corruption="uniform"),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_block_stagewise(name):
    wl = SMALL[name]
    sess, om, _ = make_pair(wl)
    try:
        cv = sess.new_canvas(wl.batch, wl.canvas)
        p_lib, p_or = lib_params(wl), oracle_params(wl)
        sess.init(cv, p_lib)
        init = cv.numpy()
        ref = O.init_canvas(wl.batch, p_or, wl.shape.mask_id, wl.shape.vocab)
        assert np.array_equal(init["tokens"], ref.tokens)
        report = {}
        for s in range(wl.steps):
            pre, post = check_one_step(sess, om, wl, cv, p_lib, p_or, report=report)
            if post["done"].all():
                break
        assert cv.numpy()["done"].all()
        record_near_ties("small_block_stagewise[%s]" % name, report.get("near_ties", 0),
                         report.get("compared", 0))
    finally:
        sess.close()


@pytest.mark.parametrize("cluster,tiles", [("1", None), ("0", None), ("0", 1)])
def test_attention_split_paths(cluster, tiles, monkeypatch):
    """The split-KV attention both ways: splits combined inside a thread-block
    cluster, and splits written as partials for the combine kernel
    (DLM_ATTN_CLUSTER=0; also with 128-key splits, one per key tile); ragged
    prefixes leave some splits without keys.  Two steps each."""
    monkeypatch.setenv("DLM_ATTN_CLUSTER", cluster)
    if tiles is not None:
        monkeypatch.setenv("DLM_ATTN_TILES", str(tiles))
    from masked_block_diffusion_denoise_b200 import dlm_attention_plan
    wl = W.small_workload("split_paths", n_heads=8, n_kv_heads=2, batch=3, canvas=16, steps=2,
                          quota=0, prefix_len=(20, 1500), prefix_cap=1600, seed=6)
    sess, om, _ = make_pair(wl)
    try:
        cv = sess.new_canvas(wl.batch, wl.canvas)
        p_lib, p_or = lib_params(wl), oracle_params(wl)
        sess.init(cv, p_lib)
        plan = dlm_attention_plan(sess.ctx, wl.batch, wl.canvas)
        if cluster == "0":
            assert plan["cluster"] == 1, plan
        if tiles is not None:
            assert plan["chunk"] == 128 and plan["nsplit"] >= 4, plan
        for _ in range(2):
            check_one_step(sess, om, wl, cv, p_lib, p_or)
    finally:
        sess.close()


@pytest.mark.parametrize("heads,canvas,tiles", [
    ((8, 2), 64, None),    # G 4, 256 rows: one CTA per KV head, planner's splits
    ((8, 2), 64, 2),       # the same with 256-key splits: partials + combine kernel
    ((8, 2), 96, 3),       # 384 rows: the second CTA holds one live row tile
    ((4, 4), 256, None),   # G 1 (encoder-decoder grouping), 256 canvas positions
    ((6, 2), 96, None),    # G 3 does not divide 128: query tiles by plain loads
])
def test_attention_two_row_tiles(heads, canvas, tiles, monkeypatch):
    """The 256-row attention CTA (two 128-row query tiles of one KV head
    share every K/V tile), forced with DLM_ATTN_ROWS=256, on ragged prefixes,
    within 2e-2 of the float64 attention over the GPU's own q, k, v."""
    from masked_block_diffusion_denoise_b200 import dlm_attention_plan
    monkeypatch.setenv("DLM_ATTN_ROWS", "256")
    if tiles is not None:
        monkeypatch.setenv("DLM_ATTN_TILES", str(tiles))
    H, Hkv = heads
    wl = W.small_workload("two_tiles", n_heads=H, n_kv_heads=Hkv, batch=3, canvas=canvas,
                          steps=2, quota=0, prefix_len=(20, 1500), prefix_cap=1600, seed=8)
    sess, om, _ = make_pair(wl)
    try:
        cv = sess.new_canvas(wl.batch, wl.canvas)
        p_lib, p_or = lib_params(wl), oracle_params(wl)
        sess.init(cv, p_lib)
        plan = dlm_attention_plan(sess.ctx, wl.batch, wl.canvas)
        assert plan["rows_per_cta"] == 256, plan
        if tiles is not None:
            assert plan["nsplit"] > 1 and plan["chunk"] == 128 * tiles, plan
        report = {}
        check_one_step(sess, om, wl, cv, p_lib, p_or, report=report)
        assert max(report["attn_max_err"]) < 2e-2
    finally:
        sess.close()


def test_tiny_fp32_reference_config():
    """The tiny fp32 configuration: batch 1, d 256, 4 heads of 64, vocab 4096,
    prefix of 128 random ids appended through the clean pass, canvas 32,
    8 steps, threshold 0.9, quota 4, seed 0."""
    wl = W.WORKLOADS["tiny"]
    sess, om, _ = make_pair(wl)
    try:
        # the clean pass wrote the same K/V as the oracle's
        Lcap = sess.max_prefix + sess.max_canvas
        kc = to64(sess.buffer(DLM_BUF_K_CACHE, (1, 4, Lcap, 64), torch.float32))
        assert np.allclose(kc[0, :, :128], om.k_cache[0], atol=1e-4)
        cv = sess.new_canvas(1, 32)
        p_lib, p_or = lib_params(wl), oracle_params(wl)
        sess.init(cv, p_lib)
        steps = 0
        while not cv.numpy()["done"].all():
            check_one_step(sess, om, wl, cv, p_lib, p_or)
            steps += 1
        assert steps == 8    # quota 4 over 32 positions
        # free-running oracle from the same start reaches the same canvas
        st = O.init_canvas(1, p_or, 100, 4096)
        O.decode_block(om, st, p_or)
        assert np.array_equal(st.tokens, cv.numpy()["tokens"])
    finally:
        sess.close()


def test_block_graph_equals_steps_and_resume():
    wl = SMALL["small_gqa2"].replace(eos_frac=0.5, seed=5)
    sess, om, _ = make_pair(wl)
    try:
        p = lib_params(wl)
        a, b, c = (sess.new_canvas(wl.batch, wl.canvas) for _ in range(3))
        for cv in (a, b, c):
            sess.init(cv, p)
        for (bb, slot) in W.make_eos_plant(wl) or [(0, 7)]:
            for cv in (a, b, c):
                cv.tokens[bb, slot] = wl.shape.eos_id
                cv.committed[bb, slot] = 1
        sess.block(a, p)
        for _ in range(wl.steps):
            sess.step(b, p)
        for _ in range(3):
            sess.step(c, p)
        sess.block(c, p)       # resume: steps of finished canvases do nothing
        sess.check()
        na, nb, nc = a.numpy(), b.numpy(), c.numpy()
        for key in ("tokens", "committed", "step", "done", "eos_pos", "stats"):
            assert np.array_equal(na[key], nb[key]), key
            assert np.array_equal(na[key], nc[key]), key
        assert na["done"].all()
        assert sess.ctx is not None
    finally:
        sess.close()


def test_entropy_bound_sampling_stage():
    """Gumbel sampling at annealed temperature and the entropy-bound rule."""
    wl = W.small_workload("small_eb", corruption="uniform", entropy_bound=0.5, steps=6,
                          vocab=2000, seed=11)
    sess, om, _ = make_pair(wl)
    try:
        p_lib, p_or = lib_params(wl), oracle_params(wl)
        cv = sess.new_canvas(wl.batch, wl.canvas)
        sess.init(cv, p_lib)
        C = wl.canvas
        flips = 0
        for s in range(wl.steps):
            pre = cv.numpy()
            if pre["done"].all():
                break
            check_one_step(sess, om, wl, cv, p_lib, p_or)
            # scores: replay the sampling on the GPU's float32 logits
            lg = sess.logits(wl.batch, C).cpu().numpy()
            cand = sess.buffer(DLM_BUF_CAND, (wl.batch * C,), torch.int32).cpu().numpy()
            conf = sess.buffer(DLM_BUF_CONF, (wl.batch * C,), torch.float32).cpu().numpy()
            ent = sess.buffer(DLM_BUF_ENTROPY, (wl.batch * C,), torch.float32).cpu().numpy()
            for b in range(wl.batch):
                if pre["done"][b]:
                    continue
                st = int(pre["step"][b])
                T = O.annealed_temperature(wl.t_max, wl.t_min, st, wl.steps)
                inv = np.float32(np.float32(1.0) / T)
                G = np.stack([O.gumbel_noise(wl.seed, b, st, i, wl.shape.vocab)
                              for i in range(C)])
                c64, f64, h64, z = O.scores(lg[b * C:(b + 1) * C], -1, inv_temp=inv, gumbel=G)
                for i in range(C):
                    gc = int(cand[b * C + i])
                    g = z[i] + G[i]
                    if gc != c64[i]:
                        assert abs(g[gc] - g[c64[i]]) < 1e-4, "sampled id outside a near tie"
                        flips += 1
                    else:
                        assert abs(conf[b * C + i] - f64[i]) < 1e-3
                    assert abs(ent[b * C + i] - h64[i]) < 1e-3
        assert flips <= 2
    finally:
        sess.close()


# ---------------------------------------------------------------------------
# kernel (c) alone: bit-exact selection on identical inputs
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("C", [1, 7, 32, 100, 256, 1024])
@pytest.mark.parametrize("mode", ["greedy", "thr0", "thr_big_q1", "eb", "uniform", "forced",
                                  "stop", "stop_high_h", "edit", "edit_all"])
def test_commit_bit_exact(C, mode):
    from masked_block_diffusion_denoise_b200.session import Session, sampler_params
    sh = W.ModelShape(d_model=64, n_heads=2, n_kv_heads=1, head_dim=32, vocab=5000, dtype="f32")
    w = W.make_weights(sh, seed=1)
    B = 5
    sess = Session(sh, w, max_batch=B, max_prefix=8, max_canvas=1024)
    try:
        r = np.random.default_rng(C * 31 + len(mode))
        S = 10
        kw = dict(canvas=C, steps=S, threshold=0.6, quota=3, seed=99)
        if mode == "thr0":
            kw.update(threshold=0.0)
        if mode == "thr_big_q1":
            kw.update(threshold=1.5, quota=1)
        if mode == "eb":
            kw.update(entropy_bound=2.0, corruption="uniform")
        if mode == "uniform":
            kw.update(corruption="uniform")
        if mode == "stop":
            kw.update(stability_steps=2, stop_entropy=0.5)
        if mode == "stop_high_h":
            kw.update(stability_steps=1, stop_entropy=0.05)
        if mode == "edit":
            kw.update(editing=1, editing_threshold=0.6)
        if mode == "edit_all":
            kw.update(editing=1, editing_threshold=0.0, corruption="uniform")
        p_lib = sampler_params(**kw)
        p_or = O.SamplerParams(**kw)
        tokens = r.integers(0, sh.vocab, size=(B, C)).astype(np.int64)
        committed = r.random((B, C)) < 0.3
        step = r.integers(0, S - 1, size=B)
        if mode == "forced":
            step[:] = S - 1
        done = np.zeros(B, bool)
        done[4] = True
        tokens[1, C // 2] = sh.eos_id          # a committed EOS mid-canvas
        committed[1, C // 2] = True
        cand = r.integers(0, sh.vocab, size=(B, C)).astype(np.int32)
        cand[2, : max(1, C // 5)] = sh.eos_id  # sampler may commit an EOS
        conf = r.random((B, C)).astype(np.float32)
        conf[:, ::3] = conf[:, :1]             # ties -> lower index first
        conf[3, :] = np.float32(0.6)           # exactly the threshold
        ent = (r.random((B, C)) * 0.5).astype(np.float32)
        ent[:, ::4] = np.float32(0.0)
        # adaptive stopping state: canvases 0-2 repeat their argmax, canvas 3
        # changes one position; canvas 0 and 1 reach two stable steps
        prev_cand = cand.astype(np.int64).copy()
        prev_cand[3, C - 1] += 1
        stable = np.array([1, 2, 0, 5, 0], dtype=np.int64)
        cv = sess.new_canvas(B, C)
        cv.load(tokens, committed, step, done, np.full(B, -1), prev_cand, stable)
        dev = lambda a: torch.as_tensor(a).cuda()
        sess.commit(cv, p_lib, dev(cand), dev(conf), dev(ent))
        sess.check()
        got = cv.numpy()
        st = O.CanvasState(tokens.copy(), committed.copy(), step.copy(), done.copy(),
                           np.full(B, -1), prev_cand.copy(), stable.copy())
        stats = [O.CanvasStats() for _ in range(B)]
        for b in range(B):
            O.select_canvas(st, b, cand[b], conf[b], ent[b], p_or, vocab=sh.vocab,
                            mask_id=sh.mask_id, eos_id=sh.eos_id, stats=stats[b])
        assert np.array_equal(got["tokens"], st.tokens)
        assert np.array_equal(got["committed"], st.committed)
        assert np.array_equal(got["step"], st.step)
        assert np.array_equal(got["done"], st.done)
        assert np.array_equal(got["eos_pos"][:4], st.eos_pos[:4])
        if mode.startswith("stop"):
            assert np.array_equal(got["prev_cand"][:4], st.prev_cand[:4])
            assert np.array_equal(got["stable"][:4], st.stable[:4])
        if mode == "stop":
            assert sum(x.frozen for x in stats) > 0
        if mode.startswith("edit") and C > 1:
            assert sum(x.edited for x in stats) > 0
        for b in range(B):
            assert list(got["stats"][b]) == [stats[b].steps_used, stats[b].committed_by_sampler,
                                             stats[b].forced_at_budget, stats[b].eos_autofill,
                                             stats[b].frozen, stats[b].edited]
    finally:
        sess.close()


def test_canvas_init_uniform_bit_exact():
    from masked_block_diffusion_denoise_b200.session import Session, sampler_params
    sh = W.ModelShape(d_model=64, n_heads=2, n_kv_heads=1, head_dim=32, vocab=262144, dtype="f32")
    sess = Session(sh, W.make_weights(sh, seed=2), max_batch=3, max_prefix=8, max_canvas=256)
    try:
        p = sampler_params(canvas=256, steps=48, corruption="uniform", seed=0xDEADBEEF12345)
        cv = sess.new_canvas(3, 256)
        sess.init(cv, p)
        ref = O.init_canvas(3, O.SamplerParams(canvas=256, steps=48, corruption="uniform",
                                               seed=0xDEADBEEF12345), 100, 262144)
        assert np.array_equal(cv.numpy()["tokens"], ref.tokens)
    finally:
        sess.close()


def test_kv_append_tokens_bf16():
    wl = W.small_workload("kv_tokens", prefix_kind="tokens", prefix_len=(150, 333), batch=2)
    sess, om, _ = make_pair(wl)
    try:
        Lcap = sess.max_prefix + sess.max_canvas
        sh = wl.shape
        kc = sess.buffer(DLM_BUF_K_CACHE, (2, sh.n_kv_heads, Lcap, sh.head_dim), torch.bfloat16)
        vc = sess.buffer(DLM_BUF_V_CACHE, (2, sh.n_kv_heads, Lcap, sh.head_dim), torch.bfloat16)
        lens, toks, _, _ = W.make_prefix(wl)
        for b in range(2):
            L = om.kv_len(b)
            xe = om.embed(toks[b])
            half = sh.head_dim // 2
            tk = abs_terms(xe, om.w_k).reshape(L, sh.n_kv_heads, sh.head_dim).transpose(1, 0, 2)
            tk = np.concatenate([tk[..., :half] + tk[..., half:]] * 2, axis=-1)
            tv = abs_terms(xe, om.w_v).reshape(L, sh.n_kv_heads, sh.head_dim).transpose(1, 0, 2)
            assert_storage_close(to64(kc[b, :, :L]), om.k_cache[b], "bf16", what="K", terms=tk)
            assert_storage_close(to64(vc[b, :, :L]), om.v_cache[b], "bf16", what="V", terms=tv)
    finally:
        sess.close()


# ---------------------------------------------------------------------------
# full-size shapes: one step, sampled outputs
# ---------------------------------------------------------------------------

def test_fp8_quantisation_bit_exact():
    """The e4m3 copies of the LM head's weights and of a step's input rows,
    and their scales, equal the oracle's quantisation bit for bit."""
    wl = SMALL["small_fp8"]
    sess, om, _ = make_pair(wl)
    try:
        from masked_block_diffusion_denoise_b200 import (DLM_BUF_LM_Q, DLM_BUF_LM_SCALE,
                                                         DLM_BUF_Y_Q, DLM_BUF_Y_SCALE)
        sh = wl.shape
        V, d = sh.vocab, sh.d_model
        as_e4m3 = lambda t: t.cpu().view(torch.float8_e4m3fn).to(torch.float64).numpy()
        q = as_e4m3(sess.buffer(DLM_BUF_LM_Q, (V, d), torch.uint8))
        sc = sess.buffer(DLM_BUF_LM_SCALE, (V,), torch.float32).cpu().numpy()
        assert np.array_equal(q, om.lm_q) and np.array_equal(sc, om.lm_scale)
        cv = sess.new_canvas(wl.batch, wl.canvas)
        p_lib = lib_params(wl)
        sess.init(cv, p_lib)
        sess.step(cv, p_lib)
        sess.check()
        M = wl.batch * wl.canvas
        y = to64(sess.buffer(DLM_BUF_Y, (M, d), torch.bfloat16))
        qy = as_e4m3(sess.buffer(DLM_BUF_Y_Q, (M, d), torch.uint8))
        sy = sess.buffer(DLM_BUF_Y_SCALE, (M,), torch.float32).cpu().numpy()
        ref_q, ref_s = O.quantize_rows_e4m3(y)
        assert np.array_equal(qy, ref_q) and np.array_equal(sy, ref_s)
    finally:
        sess.close()


E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _decode_e2m1_pairs(packed: np.ndarray, cols: int) -> np.ndarray:
    """[rows][cols/2] bytes, element 2i in the low nibble -> values"""
    b = packed.astype(np.int64)
    nib = np.stack([b & 0xF, b >> 4], axis=-1).reshape(b.shape[0], cols)
    return np.where(nib & 8, -1.0, 1.0) * E2M1[nib & 7]


def _block_scales_from_mma_layout(sf: np.ndarray, rows: int, cols: int) -> np.ndarray:
    """e4m3 block scales stored per 128-row block and 64-element k group in
    512-byte chunks, byte (m % 32) * 16 + (m / 32) * 4 + s -> [rows][cols/16]"""
    kg = cols // 64
    r = np.arange(rows)[:, None]
    j = np.arange(cols // 16)[None, :]
    m = r % 128
    idx = ((r // 128) * kg + j // 4) * 512 + (m % 32) * 16 + (m // 32) * 4 + j % 4
    return torch.from_numpy(sf[idx].astype(np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def test_nvfp4_quantisation_bit_exact():
    """The NVFP4 copies of the LM head's weights and of a step's input rows --
    e2m1 elements, e4m3 block scales in the block-scaled MMA's layout and
    float32 row scales -- equal the oracle's quantisation exactly."""
    wl = SMALL["small_nvfp4_mtiles"]
    sess, om, _ = make_pair(wl)
    try:
        from masked_block_diffusion_denoise_b200 import (DLM_BUF_LM_Q, DLM_BUF_LM_SCALE,
                                                         DLM_BUF_LM_SF, DLM_BUF_Y_Q,
                                                         DLM_BUF_Y_SCALE, DLM_BUF_Y_SF)
        sh = wl.shape
        V, d = sh.vocab, sh.d_model
        lm_q = sess.buffer(DLM_BUF_LM_Q, (V, d // 2), torch.uint8).cpu().numpy()
        assert np.array_equal(_decode_e2m1_pairs(lm_q, d), om.lm_q4)
        kgb = -(-V // 128) * (d // 64) * 512
        lm_sf = sess.buffer(DLM_BUF_LM_SF, (kgb,), torch.uint8).cpu().numpy()
        assert np.array_equal(_block_scales_from_mma_layout(lm_sf, V, d), om.lm_sb)
        sr = sess.buffer(DLM_BUF_LM_SCALE, (V,), torch.float32).cpu().numpy()
        assert np.array_equal(sr, om.lm_sr)
        cv = sess.new_canvas(wl.batch, wl.canvas)
        p_lib = lib_params(wl)
        sess.init(cv, p_lib)
        sess.step(cv, p_lib)
        sess.check()
        M = wl.batch * wl.canvas
        y = to64(sess.buffer(DLM_BUF_Y, (M, d), torch.bfloat16))
        ref_q, ref_sb, ref_sr = O.quantize_rows_nvfp4(y)
        yq = sess.buffer(DLM_BUF_Y_Q, (M, d // 2), torch.uint8).cpu().numpy()
        assert np.array_equal(_decode_e2m1_pairs(yq, d), ref_q)
        ysf = sess.buffer(DLM_BUF_Y_SF, (-(-M // 128) * (d // 64) * 512,), torch.uint8)
        assert np.array_equal(_block_scales_from_mma_layout(ysf.cpu().numpy(), M, d), ref_sb)
        ys = sess.buffer(DLM_BUF_Y_SCALE, (M,), torch.float32).cpu().numpy()
        assert np.array_equal(ys, ref_sr)
    finally:
        sess.close()


@pytest.mark.parametrize("name", ["8b_b1", "encdec", "8b_b1_fp8", "8b_b1_nvfp4"])
def test_full_size_step_sampled(name):
    wl = W.WORKLOADS[name]
    sess, om, _ = make_pair(wl)
    try:
        cv = sess.new_canvas(wl.batch, wl.canvas)
        p_lib, p_or = lib_params(wl), oracle_params(wl)
        sess.init(cv, p_lib)
        rows = np.array([0, 5, wl.canvas - 1])
        report = {}
        check_one_step(sess, om, wl, cv, p_lib, p_or, rows_sample=rows, full_logits=False,
                       report=report)
        record_near_ties("full_size_step_sampled[%s]" % name, report.get("near_ties", 0),
                         report.get("compared", 0))
    finally:
        sess.close()
