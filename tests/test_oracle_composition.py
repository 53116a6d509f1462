"""Pins of the oracle's composition that do not restate its own code.

* Uniform re-noise ids (DiffusionGemma page: uncommitted positions get
  uniform random ids) from one Philox4x32-10 known-answer word of the
  Random123 distribution, worked by hand with the multiply-shift reading
  id = floor(w * V / 2^32).  A modulo reading (w mod V) or a different
  counter word would fail here.
* The forward pass of the single-layer denoiser (x = E[t]; q, k, v = x W^T;
  one joint softmax over the keys; y = x + o W_o^T; logits = y W_lm^T) with
  permutation weight matrices and one key, so that every intermediate value
  is a small integer worked out by hand; a transposed weight (x W instead of
  x W^T) permutes the other way and fails.  One rotary rotation (Nemotron
  guide, section 7: RoPE) is checked against cos / sin of its angle.
"""
import math

import numpy as np

from oracle import dlm_oracle as O


# ---------------------------------------------------------------------------
# uniform ids from a known-answer Philox word
# ---------------------------------------------------------------------------

def test_uniform_id_from_known_answer_word():
    # Random123 known answer: counter (ffffffff, ffffffff, ffffffff,
    # ffffffff), key (ffffffff, ffffffff) -> first word 0x408f276d =
    # 1083123565.  The re-noise stream uses counter (canvas, step, position,
    # 0xffffffff) and the 64-bit seed as the key, so canvas = step =
    # position = 0xffffffff and seed = 2^64 - 1 select exactly that word.
    seed, c, s, pos = 0xFFFFFFFFFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF, 0xFFFFFFFF
    w = 1083123565
    # V = 2^17: floor(w / 2^15); 32768 * 33054 = 1083113472 <= w < +32768
    assert O.uniform_token_ids(seed, c, s, [pos], 131072)[0] == 33054
    # V = 2^18: floor(w / 2^14) = 66108 (16384 * 66108 = 1083113472)
    assert O.uniform_token_ids(seed, c, s, [pos], 262144)[0] == 66108
    # V = 1000: w * 1000 = 1083123565000 = 252 * 2^32 + 791806408 -> 252;
    # the modulo reading would give 565
    assert O.uniform_token_ids(seed, c, s, [pos], 1000)[0] == 252
    assert w % 1000 == 565


# ---------------------------------------------------------------------------
# the forward composition, worked by hand
# ---------------------------------------------------------------------------

def _perm(sigma):
    """Matrix P with P[i, sigma[i]] = 1, so that (x P^T)[i] = x[sigma[i]]."""
    n = len(sigma)
    p = np.zeros((n, n), np.float32)
    p[np.arange(n), sigma] = 1.0
    return p


def _model(rope_theta):
    dims = O.ModelDims(d_model=4, n_heads=1, n_kv_heads=1, head_dim=4, vocab=5, dtype="f32",
                       rope_theta=rope_theta, mask_id=4, eos_id=3)
    emb = np.zeros((5, 4), np.float32)
    emb[2] = [1, 2, 3, 4]
    emb[0] = [1, 1, 1, 1]
    w_lm = np.array([[1, 0, 0, 0], [0, 0, 0, 1], [0, 0, 1, 0], [0, 1, 0, 0], [1, -1, 0, 0]],
                    np.float32)
    w = {"emb": emb, "w_q": _perm([1, 2, 3, 0]), "w_k": np.eye(4, dtype=np.float32),
         "w_v": _perm([3, 0, 1, 2]), "w_o": _perm([1, 3, 0, 2]), "w_lm": w_lm}
    return O.OracleModel(dims, w)


def test_forward_composition_by_hand():
    m = _model(rope_theta=0.0)          # no rotary embedding
    out = m.forward(0, [2])             # one canvas position, empty prefix
    x = [1, 2, 3, 4]                    # E[2]
    assert out["x"].tolist() == [x]
    # q[i] = x[sigma_q[i]], sigma_q = (1, 2, 3, 0)
    assert out["q"].reshape(-1).tolist() == [2, 3, 4, 1]
    assert out["k"].reshape(-1).tolist() == [1, 2, 3, 4]
    # v[i] = x[sigma_v[i]], sigma_v = (3, 0, 1, 2)
    assert out["v"].reshape(-1).tolist() == [4, 1, 2, 3]
    # one key: the softmax weight is 1, so o = v
    assert out["o"].reshape(-1).tolist() == [4, 1, 2, 3]
    # y = x + z, z[i] = o[sigma_o[i]], sigma_o = (1, 3, 0, 2): z = (1, 3, 4, 2)
    assert out["y"].reshape(-1).tolist() == [2, 5, 7, 6]
    # logits: rows of W_lm pick y0, y3, y2, y1 and y0 - y1
    assert out["logits"].reshape(-1).tolist() == [2, 6, 7, 5, -3]


def test_forward_two_keys_softmax_weights_by_hand():
    """Canvas of two positions: every position attends to both keys with the
    softmax weights of its two scores, worked out by hand."""
    m = _model(rope_theta=0.0)
    out = m.forward(0, [0, 2])          # x0 = (1, 1, 1, 1), x1 = (1, 2, 3, 4)
    q = out["q"].reshape(2, 4)
    k = out["k"].reshape(2, 4)
    assert q.tolist() == [[1, 1, 1, 1], [2, 3, 4, 1]]
    assert k.tolist() == [[1, 1, 1, 1], [1, 2, 3, 4]]
    # softmax weights of query 0: scores (4, 10) / sqrt(4) = (2, 5)
    w1 = math.exp(5) / (math.exp(2) + math.exp(5))
    v = out["v"].reshape(2, 4)
    assert v.tolist() == [[1, 1, 1, 1], [4, 1, 2, 3]]
    want0 = (1 - w1) * np.array([1, 1, 1, 1]) + w1 * np.array([4, 1, 2, 3])
    assert np.allclose(out["o"][0], want0, rtol=1e-6)
    # query 1 = (2,3,4,1): scores (10, 2+6+12+4 = 24) / 2 = (5, 12)
    w1b = math.exp(12) / (math.exp(5) + math.exp(12))
    want1 = (1 - w1b) * np.array([1, 1, 1, 1]) + w1b * np.array([4, 1, 2, 3])
    assert np.allclose(out["o"][1], want1, rtol=1e-6)


def test_rotary_rotation_by_hand():
    """Position 1, theta 1e4, head dim 4: pair (0, 2) turns by 1 radian,
    pair (1, 3) by 1e4^(-1/2) = 0.01 radian (rotate-half pairs j, j + 2)."""
    m = _model(rope_theta=1.0e4)
    x = np.array([[1.0, 2.0, 3.0, 4.0]])
    q, k, _ = m.project_qkv(x, np.array([1]))
    a, b = 1.0, 0.01
    q0 = [2.0, 3.0, 4.0, 1.0]
    want_q = [q0[0] * math.cos(a) - q0[2] * math.sin(a),
              q0[1] * math.cos(b) - q0[3] * math.sin(b),
              q0[2] * math.cos(a) + q0[0] * math.sin(a),
              q0[3] * math.cos(b) + q0[1] * math.sin(b)]
    assert np.allclose(q.reshape(-1), want_q, rtol=1e-6, atol=1e-6)
    k0 = [1.0, 2.0, 3.0, 4.0]
    want_k = [k0[0] * math.cos(a) - k0[2] * math.sin(a),
              k0[1] * math.cos(b) - k0[3] * math.sin(b),
              k0[2] * math.cos(a) + k0[0] * math.sin(a),
              k0[3] * math.cos(b) + k0[1] * math.sin(b)]
    assert np.allclose(k.reshape(-1), want_k, rtol=1e-6, atol=1e-6)
