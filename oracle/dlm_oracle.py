"""CPU oracle for one denoising step of masked block-diffusion decoding.

TEST INFRASTRUCTURE.  This module is the plain, slow reference that the CUDA
path is checked against.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
It shares no code with the CUDA library and imports nothing from it; the only
thing both sides have in common is the seeded input generator in
``workloads/``.

What it computes (one step over a canvas of C positions per sequence), with
the passage each part restates:

* the denoiser: a random-init single attention layer plus LM head over the
  canvas.  Embedding lookup of the canvas tokens (the block is filled with the
  mask id 100 -- Nemotron guide, section 6 "masked block denoising");
  projections with RoPE, theta 1e6, rotate-half convention (Nemotron guide,
  section 7 "architecture"); one joint softmax attention of every canvas
  position over the cached prefix plus all canvas positions, no mask inside
  the block (Nemotron guide section 6, the bidirectional block mask; course
  "Diffusion LLMs" section 14: the current block reads the finished prefix and
  all of its own positions; diffusers DiffusionGemma page: the decoder attends
  to the encoder's KV cache); residual output projection; untied LM head to
  vocabulary logits [batch, canvas, vocab] (DiffusionGemma page, pipeline
  class description).
* scores: per position softmax, argmax candidate and its probability as the
  confidence (course section 12, the greedy sampler), entropy in nats
  (course section 9 and section 7 for the natural log).
* selection: threshold plus uniform per-step quota (DiffusionGemma page,
  BlockRefinementScheduler; Nemotron guide section 3.2 for the 0.9 threshold
  and 32-step budget, section 6 for forcing every remaining mask on the last
  step); confidence order with ties to the lower position index (course
  section 12); re-noising of uncommitted positions with uniform random ids
  (DiffusionGemma page: uniform corruption, mask_token_id=None) or keeping
  the mask id; entropy-bound selection with annealed temperature
  (DiffusionGemma page, EntropyBoundScheduler); EOS handling (Nemotron guide
  section 6: generation stops at EOS; text-diffusion explainer: tokens after
  EOS are discarded).

Precision: arithmetic is float64.  The denoiser is a bf16 model (Nemotron
guide, section 10: bf16 is kept through logits), so every activation the
model stores between layers (q, k, v, attention output, residual output) is
rounded to bfloat16 (float32 for the fp32 model) exactly where a bf16 model
stores it.  Decisions that turn floats into integers take them in float32,
the precision in which the kernel holds the values: confidence / entropy
comparisons in the selection, the entropy prefix sum, temperature scaling.

Readings of points the pages leave open are marked READING where they are
taken.  Pins (tests/test_oracle_*.py) tie every function to something other
than itself; no function here is parity-unpinned.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, Dict, List, Optional, Sequence, Tuple

import numpy as np

F64 = np.float64
F32 = np.float32

# ---------------------------------------------------------------------------
# storage precision
# ---------------------------------------------------------------------------


def round_to_bf16(x) -> np.ndarray:
    """Round to the nearest bfloat16 value (ties to even), via float32 -- the
    value a kernel holding a float32 accumulator stores.  Returns float64."""
    f = np.asarray(x, dtype=F64).astype(F32)
    bits = f.view(np.uint32).astype(np.uint64)
    keep_lsb = (bits >> np.uint64(16)) & np.uint64(1)
    bits = ((bits + np.uint64(0x7FFF) + keep_lsb) >> np.uint64(16)) << np.uint64(16)
    return bits.astype(np.uint32).view(F32).astype(F64)


def round_to_f32(x) -> np.ndarray:
    return np.asarray(x, dtype=F64).astype(F32).astype(F64)


def bf16_bits_to_f64(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(F32).astype(F64)


# ---------------------------------------------------------------------------
# course reveal schedule (course "Diffusion LLMs", section 6 worked example A
# and the section 12 code: m_s = ceil(N (S - s) / S), s = 0..S)
# ---------------------------------------------------------------------------


def linear_mask_schedule(length: int, steps: int) -> Tuple[int, ...]:
    """Target number of masked positions after each of S model calls, starting
    from the fully masked canvas: m_s = ceil(N (S - s) / S) for s = 0..S."""
    for v in (length, steps):
        if isinstance(v, bool) or not isinstance(v, (int, np.integer)) or v <= 0:
            raise ValueError("length and steps must be positive integers")
    out = []
    for s in range(steps + 1):
        out.append(-(-(int(length) * (int(steps) - s)) // int(steps)))
    return tuple(out)


# ---------------------------------------------------------------------------
# Philox4x32-10 counter-based generator (Salmon, Moraes, Dror, Shaw,
# "Parallel random numbers: as easy as 1, 2, 3", SC'11), written from the
# published round function: two 32x32->64 multiplications by the round
# constants, an xor with the key and a word permutation per round, and a
# Weyl-sequence key schedule between rounds.
# ---------------------------------------------------------------------------

_PHILOX_M0 = 0xD2511F53
_PHILOX_M1 = 0xCD9E8D57
_PHILOX_W0 = 0x9E3779B9
_PHILOX_W1 = 0xBB67AE85
_U32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(ctr: Sequence, key: Tuple[int, int]) -> Tuple[np.ndarray, ...]:
    """Ten Philox4x32 rounds.  ``ctr`` holds four (broadcastable) arrays of
    32-bit counter words, ``key`` two 32-bit key words.  Returns four uint32
    arrays."""
    c = [np.asarray(w, dtype=np.uint64) & _U32 for w in ctr]
    c = np.broadcast_arrays(*c)
    c0, c1, c2, c3 = [np.array(w, dtype=np.uint64) for w in c]
    k0 = int(key[0]) & 0xFFFFFFFF
    k1 = int(key[1]) & 0xFFFFFFFF
    m0 = np.uint64(_PHILOX_M0)
    m1 = np.uint64(_PHILOX_M1)
    for _ in range(10):
        prod0 = m0 * c0          # < 2**64, exact in uint64
        prod1 = m1 * c2
        hi0, lo0 = prod0 >> np.uint64(32), prod0 & _U32
        hi1, lo1 = prod1 >> np.uint64(32), prod1 & _U32
        c0, c1, c2, c3 = (hi1 ^ c1 ^ np.uint64(k0), lo1,
                          hi0 ^ c3 ^ np.uint64(k1), lo0)
        k0 = (k0 + _PHILOX_W0) & 0xFFFFFFFF
        k1 = (k1 + _PHILOX_W1) & 0xFFFFFFFF
    return tuple(w.astype(np.uint32) for w in (c0, c1, c2, c3))


def seed_key(seed: int) -> Tuple[int, int]:
    seed = int(seed) & 0xFFFFFFFFFFFFFFFF
    return seed & 0xFFFFFFFF, seed >> 32


RENOISE_WORD3 = 0xFFFFFFFF    # READING: counter word 3 of the re-noise stream


def uniform_token_ids(seed: int, canvas_index: int, step: int, positions, vocab: int) -> np.ndarray:
    """Uniform corruption ids (DiffusionGemma page: uncommitted positions are
    re-noised with uniform random ids; D3PM uniform replacement, course
    section 5).  READING: id = floor(u32 * V / 2**32) with u32 the first
    Philox word of counter (canvas, step, position, 0xFFFFFFFF); step 0 is
    the initial canvas, step s+1 the re-noise after step s."""
    pos = np.asarray(positions, dtype=np.uint64)
    w0, _, _, _ = philox4x32_10((canvas_index, step, pos, RENOISE_WORD3), seed_key(seed))
    return ((w0.astype(np.uint64) * np.uint64(vocab)) >> np.uint64(32)).astype(np.int64)


def gumbel_noise(seed: int, canvas_index: int, step: int, position: int, vocab: int) -> np.ndarray:
    """Standard Gumbel noise for every vocabulary entry of one position.
    READING: u = ((w >> 8) + 1/2) / 2**24 with w word (v mod 4) of Philox
    counter (canvas, step, position, floor(v / 4)); G = -log(-log u)."""
    v = np.arange(vocab, dtype=np.int64)
    words = philox4x32_10((canvas_index, step, position, (v >> 2).astype(np.uint64)),
                          seed_key(seed))
    w = np.choose((v & 3), words).astype(np.uint64)
    u = ((w >> np.uint64(8)).astype(F64) + 0.5) / float(1 << 24)
    return -np.log(-np.log(u))


# ---------------------------------------------------------------------------
# model pieces
# ---------------------------------------------------------------------------


def rope(x: np.ndarray, positions: np.ndarray, theta: float) -> np.ndarray:
    """Rotary position embedding, rotate-half convention.  ``x`` [..., n, Dh]
    with token positions ``positions`` [n]; pair (j, j + Dh/2) is rotated by
    angle pos * theta**(-2j/Dh).  theta = 1e6 (Nemotron guide, section 7)."""
    dh = x.shape[-1]
    half = dh // 2
    j = np.arange(half, dtype=F64)
    inv_freq = float(theta) ** (-2.0 * j / dh)
    ang = np.asarray(positions, dtype=F64)[:, None] * inv_freq[None, :]
    cos, sin = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def attention_head(q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
    """softmax(q k^T / sqrt(Dh)) v for one head, no mask: q [R][Dh],
    k, v [L][Dh]."""
    s = (q @ k.T) / math.sqrt(q.shape[-1])
    s = s - s.max(axis=1, keepdims=True)
    w = np.exp(s)
    return (w @ v) / w.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# FP8 LM head (NLD tutorial section 8.6: online BF16 -> FP8 quantisation of
# the weights, KV cache kept in BF16; course section 15: low-bit weight paths
# on Blackwell).  READING: one float32 scale per row, s = max|x| / 448 (1 for
# an all-zero row), q = e4m3(x / s) with the division in float32.  The
# tensor cores take both operands in 8 bits, so the LM head's input rows are
# quantised the same way (per row).
# ---------------------------------------------------------------------------

E4M3_MAX = 448.0


def round_to_e4m3(x) -> np.ndarray:
    """Nearest value of the e4m3 format -- sign, 4 exponent bits (bias 7), 3
    mantissa bits, no infinities, largest finite 448 -- ties to even;
    magnitudes beyond 448 saturate to 448.  Values are float64."""
    x = np.asarray(x, dtype=F64)
    a = np.abs(x)
    _, e = np.frexp(a)                 # a = m * 2^e with m in [0.5, 1)
    e = np.maximum(e - 1, -6)          # binade; below 2^-6 the subnormal spacing
    step = np.ldexp(1.0, e - 3)        # grid spacing: 3 mantissa bits
    r = np.minimum(np.rint(a / step) * step, E4M3_MAX)   # rint: ties to even
    return np.copysign(r, x)


def quantize_rows_e4m3(x) -> Tuple[np.ndarray, np.ndarray]:
    """(q, s): q [rows][cols] the e4m3 values (float64), s [rows] float32.
    Rows are independent; they are processed in blocks to bound memory."""
    x = np.asarray(x)
    q = np.empty(x.shape, dtype=F64)
    s = np.empty(x.shape[0], dtype=np.float32)
    for r0 in range(0, x.shape[0], 4096):
        x32 = np.asarray(x[r0:r0 + 4096], dtype=np.float32)
        amax = np.abs(x32).max(axis=1)
        sb = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
        q[r0:r0 + 4096] = round_to_e4m3((x32 / sb[:, None]).astype(np.float32))
        s[r0:r0 + 4096] = sb
    return q, s


# ---------------------------------------------------------------------------
# NVFP4 (the 4-bit option of the LM head; course "Diffusion LLMs" section 15
# names NVFP4 as the Blackwell low-bit path; the pages give no recipe, so the
# block layout below is a reading): e2m1 elements in blocks of 16 along the
# reduction axis, one e4m3 scale per block, one float32 scale per row.
# ---------------------------------------------------------------------------

E2M1_MAX = 6.0
NVFP4_BLOCK = 16


def round_to_e2m1(x) -> np.ndarray:
    """Nearest value of the e2m1 format -- sign, 2 exponent bits (bias 1), 1
    mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 -- ties to the even
    mantissa bit; magnitudes beyond 6 saturate to 6.  Values are float64."""
    x = np.asarray(x, dtype=F64)
    a = np.abs(x)
    _, e = np.frexp(a)                 # a = m * 2^e with m in [0.5, 1)
    e = np.maximum(e - 1, 0)           # binade; below 1 the subnormal spacing
    step = np.ldexp(1.0, e - 1)        # grid spacing: 1 mantissa bit
    r = np.minimum(np.rint(a / step) * step, E2M1_MAX)   # rint: ties to even
    return np.copysign(r, x)


def quantize_rows_nvfp4(x) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """(q, sb, sr) for rows x [rows][cols] (cols a multiple of 16):
    sr [rows] float32 = amax(row) / (448 * 6) (1 for a zero row), so that every
    block scale is within the e4m3 range; sb [rows][cols/16] the e4m3 block
    scales, e4m3(amax(block) / (6 * sr)) with the division in float32; q the
    e2m1 elements, e2m1(x / (sb * sr)) with the product and the quotient in
    float32 (0 in a block whose scale is 0).  x ~ q * sb * sr."""
    x = np.asarray(x)
    rows, cols = x.shape
    if cols % NVFP4_BLOCK:
        raise ValueError("cols must be a multiple of 16")
    x32 = np.asarray(x, dtype=np.float32)
    amax_r = np.abs(x32).max(axis=1)
    sr = np.where(amax_r > 0, amax_r / np.float32(E4M3_MAX * E2M1_MAX),
                  np.float32(1.0)).astype(np.float32)
    xb = x32.reshape(rows, cols // NVFP4_BLOCK, NVFP4_BLOCK)
    amax_b = np.abs(xb).max(axis=2)
    sb = round_to_e4m3((amax_b / (np.float32(E2M1_MAX) * sr[:, None])).astype(np.float32))
    scale = (sb.astype(np.float32) * sr[:, None]).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(scale[:, :, None] > 0, xb / scale[:, :, None], np.float32(0.0))
    q = round_to_e2m1(ratio.astype(np.float32)).reshape(rows, cols)
    return q, sb, sr


def dequantize_rows_nvfp4(q, sb, sr) -> np.ndarray:
    """q * sb * sr, float64."""
    q = np.asarray(q, dtype=F64)
    rows, cols = q.shape
    s = np.repeat(np.asarray(sb, dtype=F64), NVFP4_BLOCK, axis=1) * np.asarray(sr, F64)[:, None]
    return q * s


def quantize_rows_nvfp4_blocked(x, rows_per_block: int = 4096):
    """quantize_rows_nvfp4 over row blocks (rows are independent), keeping
    the elements as float32 (every e2m1 value is exact there) to bound
    memory for large matrices."""
    x = np.asarray(x)
    rows, cols = x.shape
    q = np.empty((rows, cols), dtype=np.float32)
    sb = np.empty((rows, cols // NVFP4_BLOCK), dtype=F64)
    sr = np.empty(rows, dtype=np.float32)
    for r0 in range(0, rows, rows_per_block):
        qb_, sbb_, srb_ = quantize_rows_nvfp4(x[r0:r0 + rows_per_block])
        q[r0:r0 + rows_per_block] = qb_
        sb[r0:r0 + rows_per_block] = sbb_
        sr[r0:r0 + rows_per_block] = srb_
    return q, sb, sr


def nvfp4_dot(qa, sba, sra, qb, sbb, srb) -> np.ndarray:
    """Rows of A times rows of B, both NVFP4 along the reduction axis, the way
    a block-scaled product runs: per block the exact sum of element products
    times the two block scales, summed over blocks, times the two row scales.
    Returns [rows_a][rows_b] float64."""
    qa = np.asarray(qa, F64)
    qb = np.asarray(qb, F64)
    ra, cols = qa.shape
    nb = cols // NVFP4_BLOCK
    pa = qa.reshape(ra, nb, NVFP4_BLOCK)
    pb = qb.reshape(qb.shape[0], nb, NVFP4_BLOCK)
    blk = np.einsum("ikj,lkj->ilk", pa, pb)            # exact: products of e2m1 values
    w = np.asarray(sba, F64)[:, None, :] * np.asarray(sbb, F64)[None, :, :]
    return (blk * w).sum(axis=2) * (np.asarray(sra, F64)[:, None] * np.asarray(srb, F64)[None, :])


def nvfp4_head_logits(qa, sba, sra, qb, sbb, srb, rows_per_block: int = 4096) -> np.ndarray:
    """The NVFP4 LM head: per pair of rows the block-scaled sum of nvfp4_dot
    without the row scales, times the two row scales' product rounded to
    float32 (READING, as for the e4m3 head: one float32 factor per logit).
    B is processed in row blocks to bound memory."""
    ra = np.asarray(qa).shape[0]
    out = np.empty((ra, np.asarray(qb).shape[0]), dtype=F64)
    ones_a = np.ones(ra)
    for r0 in range(0, out.shape[1], rows_per_block):
        sl = slice(r0, r0 + rows_per_block)
        blk = nvfp4_dot(qa, sba, ones_a, qb[sl], sbb[sl], np.ones(len(srb[sl])))
        f = (np.asarray(sra, np.float32)[:, None] * np.asarray(srb[sl], np.float32)[None, :])
        out[:, sl] = blk * f.astype(np.float32).astype(F64)
    return out


@dataclass
class ModelDims:
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    vocab: int
    dtype: str = "bf16"
    rope_theta: float = 1.0e6
    mask_id: int = 100
    eos_id: int = 11
    lm_fp8: bool = False      # LM head with e4m3 weights and activations
    lm_nvfp4: bool = False    # LM head with NVFP4 weights and activations

    @classmethod
    def of(cls, shape) -> "ModelDims":
        return cls(shape.d_model, shape.n_heads, shape.n_kv_heads, shape.head_dim,
                   shape.vocab, shape.dtype, shape.rope_theta, shape.mask_id, shape.eos_id,
                   bool(getattr(shape, "lm_fp8", False)), bool(getattr(shape, "lm_nvfp4", False)))


class OracleModel:
    """The synthetic denoiser: one attention layer and an LM head.

        x = E[tok];  q, k, v = RoPE(x Wq^T), RoPE(x Wk^T), x Wv^T
        o = attention(q; [K_prefix ; k], [V_prefix ; v]);  y = x + o Wo^T
        logits = y Wlm^T

    Weights are given as bf16 bit patterns (uint16) or float32 and held as
    float64.  Query head h reads KV head floor(h * Hkv / Hq).
    """

    def __init__(self, dims: ModelDims, weights: Dict[str, np.ndarray]):
        self.dims = dims
        conv = bf16_bits_to_f64 if dims.dtype == "bf16" else (lambda a: np.asarray(a, F64))
        self._emb_raw = weights["emb"]
        self._conv = conv
        self.w_q = conv(weights["w_q"])
        self.w_k = conv(weights["w_k"])
        self.w_v = conv(weights["w_v"])
        self.w_o = conv(weights["w_o"])
        self.w_lm = conv(weights["w_lm"])
        if dims.lm_fp8:
            self.lm_q, self.lm_scale = quantize_rows_e4m3(self.w_lm)
        if dims.lm_nvfp4:
            self.lm_q4, self.lm_sb, self.lm_sr = quantize_rows_nvfp4_blocked(self.w_lm)
        self.store = round_to_bf16 if dims.dtype == "bf16" else round_to_f32
        self.k_cache: Dict[int, np.ndarray] = {}
        self.v_cache: Dict[int, np.ndarray] = {}

    # -- KV cache ---------------------------------------------------------
    def kv_len(self, seq: int) -> int:
        return 0 if seq not in self.k_cache else self.k_cache[seq].shape[1]

    def kv_append_kv(self, seq: int, k: np.ndarray, v: np.ndarray) -> None:
        """Append given (already rotated) K/V, [Hkv][n][Dh]."""
        dh = self.dims.head_dim
        k = np.asarray(k, F64).reshape(self.dims.n_kv_heads, -1, dh)
        v = np.asarray(v, F64).reshape(self.dims.n_kv_heads, -1, dh)
        if seq in self.k_cache:
            self.k_cache[seq] = np.concatenate([self.k_cache[seq], k], axis=1)
            self.v_cache[seq] = np.concatenate([self.v_cache[seq], v], axis=1)
        else:
            self.k_cache[seq], self.v_cache[seq] = k.copy(), v.copy()

    def kv_append_tokens(self, seq: int, tokens: np.ndarray) -> None:
        """Clean pass over finished tokens (course section 14: the finished
        block is run once more and its states join the cache): K = RoPE(E[t]
        Wk^T), V = E[t] Wv^T at absolute positions L .. L+n-1."""
        x = self.embed(tokens)
        pos = np.arange(self.kv_len(seq), self.kv_len(seq) + len(tokens))
        _, k, v = self.project_qkv(x, pos)
        self.kv_append_kv(seq, k.transpose(1, 0, 2), v.transpose(1, 0, 2))

    # -- stages -------------------------------------------------------------
    def embed(self, tokens) -> np.ndarray:
        t = np.asarray(tokens, dtype=np.int64)
        return self._conv(self._emb_raw[t])

    def project_qkv(self, x: np.ndarray, positions) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
        """q [n][Hq][Dh], k, v [n][Hkv][Dh], rounded to storage precision."""
        d = self.dims
        n = x.shape[0]
        q = (x @ self.w_q.T).reshape(n, d.n_heads, d.head_dim)
        k = (x @ self.w_k.T).reshape(n, d.n_kv_heads, d.head_dim)
        v = (x @ self.w_v.T).reshape(n, d.n_kv_heads, d.head_dim)
        pos = np.asarray(positions)
        if d.rope_theta > 0:
            q = rope(q.transpose(1, 0, 2), pos, d.rope_theta).transpose(1, 0, 2)
            k = rope(k.transpose(1, 0, 2), pos, d.rope_theta).transpose(1, 0, 2)
        return self.store(q), self.store(k), self.store(v)

    def attend(self, seq: int, q: np.ndarray, k: np.ndarray, v: np.ndarray) -> np.ndarray:
        """Canvas attention for one sequence.  q [C][Hq][Dh], canvas k, v
        [C][Hkv][Dh]; keys = cached prefix of ``seq`` followed by the canvas.
        Returns o [C][Hq*Dh] rounded to storage precision."""
        d = self.dims
        C = q.shape[0]
        L = self.kv_len(seq)
        out = np.empty((C, d.n_heads, d.head_dim), dtype=F64)
        for h in range(d.n_heads):
            g = (h * d.n_kv_heads) // d.n_heads
            if L:
                keys = np.concatenate([self.k_cache[seq][g], k[:, g]], axis=0)
                vals = np.concatenate([self.v_cache[seq][g], v[:, g]], axis=0)
            else:
                keys, vals = k[:, g], v[:, g]
            out[:, h] = attention_head(q[:, h], keys, vals)
        return self.store(out.reshape(C, -1))

    def out_proj(self, x: np.ndarray, o: np.ndarray) -> np.ndarray:
        return self.store(x + o @ self.w_o.T)

    def logits(self, y: np.ndarray) -> np.ndarray:
        if self.dims.lm_nvfp4:
            # the NVFP4 head: both operands quantised per row (e2m1 elements,
            # e4m3 block scales of 16, a float32 row scale)
            qy, sby, sry = quantize_rows_nvfp4(y)
            return nvfp4_head_logits(qy, sby, sry, self.lm_q4, self.lm_sb, self.lm_sr)
        if self.dims.lm_fp8:
            # the e4m3 head: both operands quantised per row, the products
            # summed exactly, then one float32 factor a_r * s_v per logit
            qy, a = quantize_rows_e4m3(y)
            w = (a[:, None] * self.lm_scale[None, :]).astype(np.float32)
            return (qy @ self.lm_q.T) * w.astype(F64)
        return y @ self.w_lm.T

    def forward(self, seq: int, tokens) -> Dict[str, np.ndarray]:
        """All stages for one canvas; positions start after the prefix."""
        x = self.embed(tokens)
        pos = np.arange(self.kv_len(seq), self.kv_len(seq) + len(tokens))
        q, k, v = self.project_qkv(x, pos)
        o = self.attend(seq, q, k, v)
        y = self.out_proj(x, o)
        return {"x": x, "q": q, "k": k, "v": v, "o": o, "y": y, "logits": self.logits(y)}


# ---------------------------------------------------------------------------
# scores: softmax confidence, argmax / sampled candidate, entropy
# ---------------------------------------------------------------------------


def annealed_temperature(t_max: float, t_min: float, step: int, steps: int) -> np.float32:
    """READING: linear in the step index from t_max at the first step to
    t_min at the last (DiffusionGemma page gives only the end points), in
    float32: T = t_max + (t_min - t_max) * (s / (S - 1)); S = 1 gives t_max."""
    if steps <= 1:
        return F32(t_max)
    frac = F32(step) / F32(steps - 1)
    return F32(F32(t_max) + F32(F32(F32(t_min) - F32(t_max)) * frac))


def scores(logits: np.ndarray, mask_id: int = -1, *, inv_temp: Optional[float] = None,
           gumbel: Optional[np.ndarray] = None):
    """Per-row candidate, confidence and entropy.

    Greedy (``gumbel is None``, ``inv_temp is None``): candidate = argmax of
    the logits (lowest index on ties), confidence = softmax(logits)[cand]
    (course section 12), entropy H = -sum p log p in nats (course section 9).
    With ``inv_temp``, the distribution is softmax(logits * inv_temp), scaled
    in float32; with ``gumbel`` [n][V], candidate = argmax(z + G) (the
    Gumbel-max sample of softmax(z)).  The mask id, when >= 0, is excluded
    (its logit is -inf), so a commit can never write the mask.
    Returns (cand int64[n], conf float64[n], H float64[n], z float64[n][V]).
    """
    lg = np.asarray(logits)
    if inv_temp is not None:
        z = (lg.astype(F32) * F32(inv_temp)).astype(F64)
    else:
        z = lg.astype(F64)
    z = z.copy()
    if mask_id >= 0:
        z[:, mask_id] = -np.inf
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    p = e / e.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        plogp = np.where(p > 0, p * np.log(np.where(p > 0, p, 1.0)), 0.0)
    H = -plogp.sum(axis=1)
    if gumbel is None:
        cand = np.argmax(z, axis=1)
    else:
        cand = np.argmax(z + gumbel, axis=1)
    conf = p[np.arange(p.shape[0]), cand]
    return cand.astype(np.int64), conf, H, z


def chunk_partials(z_row: np.ndarray, chunk: int):
    """Per vocabulary chunk of one row of scaled logits: (m, s, t, argmax)
    with m = max z, s = sum e^(z-m), t = sum e^(z-m)(z-m) -- the quantities
    of non-materialised chunked greedy scoring (Nemotron guide, section 5.3,
    head_scoring=chunked)."""
    parts = []
    for c0 in range(0, z_row.shape[0], chunk):
        zc = z_row[c0:c0 + chunk]
        m = zc.max()
        if not np.isfinite(m):
            parts.append((-np.inf, 0.0, 0.0, -1))
            continue
        fin = np.isfinite(zc)
        dz = np.where(fin, zc - m, 0.0)
        e = np.where(fin, np.exp(dz), 0.0)
        parts.append((m, e.sum(), float(np.sum(e * dz)), c0 + int(np.argmax(zc))))
    return parts


def combine_partials(parts):
    """READING: combination of chunk partials.  m = max_j m_j, a_j =
    e^(m_j - m), s = sum a_j s_j, t = sum a_j (t_j + s_j (m_j - m)); argmax
    keeps the smaller index on equal values.  Then confidence = 1/s and
    H = log s - t/s."""
    m = max(p[0] for p in parts)
    s = t = 0.0
    best, best_m = -1, -np.inf
    for (mj, sj, tj, ij) in parts:
        if not np.isfinite(mj):
            continue
        a = math.exp(mj - m)
        s += a * sj
        t += a * (tj + sj * (mj - m))
        if mj > best_m or (mj == best_m and ij < best):
            best, best_m = ij, mj
    return best, 1.0 / s, math.log(s) - t / s


# ---------------------------------------------------------------------------
# sampler state and selection
# ---------------------------------------------------------------------------


@dataclass
class SamplerParams:
    canvas: int
    steps: int = 32
    threshold: float = 0.9
    quota: int = 0                 # 0 -> ceil(canvas / steps)
    corruption: str = "mask"       # "mask" | "uniform"
    entropy_bound: float = -1.0    # >= 0 selects the entropy-bound rule
    temperature: float = 0.0
    t_max: float = 0.8
    t_min: float = 0.4
    seed: int = 0
    # adaptive stopping (DiffusionGemma page): off when stop_entropy <= 0
    stability_steps: int = 1
    stop_entropy: float = -1.0
    # token editing (DiffusionGemma page editing_threshold): off when editing == 0
    editing: int = 0
    editing_threshold: float = 0.9
    # oracle-only readings, for pins and for the readings table
    quota_rule: str = "union"      # "union": max(n_thr, q); "additive": n_thr + q
    schedule: str = "quota"        # "quota" | "course" (m_s = ceil(N(S-s)/S))

    @property
    def quota_eff(self) -> int:
        return self.quota if self.quota > 0 else -(-self.canvas // self.steps)


@dataclass
class CanvasState:
    tokens: np.ndarray      # int64 [B][C]
    committed: np.ndarray   # bool  [B][C]
    step: np.ndarray        # int64 [B]
    done: np.ndarray        # bool  [B]
    eos_pos: np.ndarray     # int64 [B]
    prev_cand: Optional[np.ndarray] = None   # int64 [B][C], -1 before the first step
    stable: Optional[np.ndarray] = None      # int64 [B]

    def __post_init__(self):
        if self.prev_cand is None:
            self.prev_cand = np.full(self.tokens.shape, -1, dtype=np.int64)
        if self.stable is None:
            self.stable = np.zeros(self.tokens.shape[0], dtype=np.int64)

    def copy(self) -> "CanvasState":
        return CanvasState(self.tokens.copy(), self.committed.copy(), self.step.copy(),
                           self.done.copy(), self.eos_pos.copy(), self.prev_cand.copy(),
                           self.stable.copy())


@dataclass
class CanvasStats:
    steps_used: int = 0
    committed_by_sampler: int = 0
    forced_at_budget: int = 0
    eos_autofill: int = 0
    frozen: int = 0
    edited: int = 0


def init_canvas(batch: int, p: SamplerParams, mask_id: int, vocab: int,
                seed: Optional[int] = None) -> CanvasState:
    """All-mask canvas (Nemotron guide, section 6) or, in uniform mode, uniform
    random ids from the step-0 re-noise stream."""
    C = p.canvas
    seed = p.seed if seed is None else seed
    if p.corruption == "uniform":
        tok = np.stack([uniform_token_ids(seed, b, 0, np.arange(C), vocab) for b in range(batch)])
    else:
        tok = np.full((batch, C), mask_id, dtype=np.int64)
    return CanvasState(tok.astype(np.int64), np.zeros((batch, C), bool),
                       np.zeros(batch, np.int64), np.zeros(batch, bool),
                       np.full(batch, -1, np.int64))


def _eos_fill(tokens: np.ndarray, committed: np.ndarray, eos_id: int):
    """READING: positions after the first committed EOS are finished -- every
    uncommitted one there becomes EOS and committed (tokens after EOS are
    discarded; committed tokens are never rewritten).  Returns (e, filled)."""
    e = -1
    for i in range(tokens.shape[0]):
        if committed[i] and tokens[i] == eos_id:
            e = i
            break
    if e < 0:
        return -1, 0
    n = 0
    for i in range(e + 1, tokens.shape[0]):
        if not committed[i]:
            tokens[i] = eos_id
            committed[i] = True
            n += 1
    return e, n


def _canon(x) -> np.float32:
    return F32(F32(x) + F32(0.0))    # -0.0 -> +0.0


def select_canvas(state: CanvasState, b: int, cand, conf, H, p: SamplerParams, *,
                  vocab: int, mask_id: int, eos_id: int,
                  stats: Optional[CanvasStats] = None) -> None:
    """One sampler update of canvas ``b`` in place (course section 9: rank the
    hidden positions, reveal, keep the scores; DiffusionGemma page:
    BlockRefinementScheduler / EntropyBoundScheduler).

    Threshold rule: U = uncommitted positions, ordered by (confidence desc,
    index asc); n_thr = #{i in U: conf_i >= threshold}; k = min(|U|,
    max(n_thr, q)) (READING: the quota is a floor, the 'union' reading).
    Entropy-bound rule: U ordered by (H asc, index asc); k = the longest
    prefix whose float32 running sum of H stays <= bound, at least 1.
    On the last step of the budget (step >= S-1) k = |U|.  Confidence and
    entropy enter as float32.
    """
    if state.done[b]:
        return
    C = state.tokens.shape[1]
    tok, com = state.tokens[b], state.committed[b]
    s = int(state.step[b])
    e, fill0 = _eos_fill(tok, com, eos_id)
    if p.editing:
        # token editing (DiffusionGemma page: editing_threshold re-edits
        # committed tokens; course section 14: LLaDA2.1 replaces an opened
        # token that a later iteration finds weak).  READING: a position
        # committed before this step and before the first committed EOS
        # takes the model's current candidate when it differs from its token
        # and its float32 confidence is >= editing_threshold; it stays
        # committed.
        tau_e = F32(p.editing_threshold)
        for i in range(e if e >= 0 else C):
            if com[i] and int(cand[i]) != int(tok[i]) and _canon(conf[i]) >= tau_e:
                tok[i] = int(cand[i])
                if stats is not None:
                    stats.edited += 1
    U = [i for i in range(C) if not com[i]]
    conf32 = [_canon(conf[i]) for i in range(C)]
    H32 = [_canon(H[i]) for i in range(C)]
    if p.stop_entropy > 0:
        # adaptive stopping (DiffusionGemma page): READING -- the argmax of all
        # C positions unchanged since the previous step counts one stable
        # step; the mean entropy is the float32 sum over the positions in
        # order, divided by C
        same = all(int(cand[i]) == int(state.prev_cand[b][i]) for i in range(C))
        state.stable[b] = state.stable[b] + 1 if same else 0
        state.prev_cand[b][:] = [int(c) for c in cand[:C]]
        total = F32(0.0)
        for i in range(C):
            total = F32(total + H32[i])
        mean_h = F32(total / F32(C))
        if state.stable[b] >= p.stability_steps and mean_h < F32(p.stop_entropy):
            for i in U:
                tok[i] = int(cand[i])
                com[i] = True
            e2, fill1 = _eos_fill(tok, com, eos_id)
            state.done[b] = bool(com.all())
            state.step[b] = s + 1
            state.eos_pos[b] = e2
            if stats is not None:
                stats.steps_used += 1
                stats.frozen += len(U)
                stats.eos_autofill += fill0 + fill1
            return
    if p.entropy_bound >= 0:
        order = sorted(U, key=lambda i: (H32[i], i))
        k, run = 0, F32(0.0)
        for i in order:
            run = F32(run + H32[i])
            if run <= F32(p.entropy_bound):
                k += 1
            else:
                break
        k = max(k, 1) if U else 0
    else:
        order = sorted(U, key=lambda i: (-conf32[i], i))
        tau = F32(p.threshold)
        n_thr = sum(1 for i in U if conf32[i] >= tau)
        if p.schedule == "course":
            sched = linear_mask_schedule(C, p.steps)
            k = len(U) - sched[min(s + 1, p.steps)]
        elif p.quota_rule == "additive":
            k = n_thr + p.quota_eff
        else:
            k = max(n_thr, p.quota_eff)
        k = max(0, min(len(U), k))
    k_rule = k
    if s >= p.steps - 1:
        k = len(U)
    for i in order[:k]:
        tok[i] = int(cand[i])
        com[i] = True
    e2, fill1 = _eos_fill(tok, com, eos_id)
    if p.corruption == "uniform":
        rest = np.array([i for i in range(C) if not com[i]], dtype=np.int64)
        if rest.size:
            tok[rest] = uniform_token_ids(p.seed, b, s + 1, rest, vocab)
    state.done[b] = bool(com.all())
    state.step[b] = s + 1
    state.eos_pos[b] = e2
    if stats is not None:
        stats.steps_used += 1
        stats.committed_by_sampler += k
        stats.forced_at_budget += k - k_rule
        stats.eos_autofill += fill0 + fill1


# ---------------------------------------------------------------------------
# one denoising step and a block
# ---------------------------------------------------------------------------


def step_scores(model: OracleModel, state: CanvasState, b: int, p: SamplerParams,
                logits: Optional[np.ndarray] = None):
    """Model call + scores for canvas b (course section 9: one model call on
    the current canvas, then candidates and ranking)."""
    d = model.dims
    out = None
    if logits is None:
        out = model.forward(b, state.tokens[b])
        logits = out["logits"]
    mask = d.mask_id if p.corruption == "mask" else -1
    s = int(state.step[b])
    if p.entropy_bound >= 0:
        T = annealed_temperature(p.t_max, p.t_min, s, p.steps)
        inv = F32(F32(1.0) / T)
        G = np.stack([gumbel_noise(p.seed, b, s, i, d.vocab) for i in range(logits.shape[0])])
        cand, conf, H, _ = scores(logits, mask, inv_temp=inv, gumbel=G)
    elif p.temperature > 0:
        inv = F32(F32(1.0) / F32(p.temperature))
        G = np.stack([gumbel_noise(p.seed, b, s, i, d.vocab) for i in range(logits.shape[0])])
        cand, conf, H, _ = scores(logits, mask, inv_temp=inv, gumbel=G)
    else:
        cand, conf, H, _ = scores(logits, mask)
    return cand, conf, H, out


def denoise_step(model: OracleModel, state: CanvasState, p: SamplerParams,
                 stats: Optional[List[CanvasStats]] = None) -> Dict[int, dict]:
    """One step over every canvas that is not done; returns per-canvas
    intermediates."""
    d = model.dims
    inter = {}
    for b in range(state.tokens.shape[0]):
        if state.done[b]:
            continue
        cand, conf, H, out = step_scores(model, state, b, p)
        select_canvas(state, b, cand, conf, H, p, vocab=d.vocab, mask_id=d.mask_id,
                      eos_id=d.eos_id, stats=None if stats is None else stats[b])
        inter[b] = {"cand": cand, "conf": conf, "H": H, **(out or {})}
    return inter


def decode_block(model: OracleModel, state: CanvasState, p: SamplerParams,
                 stats: Optional[List[CanvasStats]] = None, max_calls: Optional[int] = None):
    """Steps until every canvas is done; the last step of the budget forces
    completion, so at most ``p.steps`` calls."""
    calls = 0
    limit = p.steps if max_calls is None else max_calls
    while not state.done.all() and calls < limit:
        denoise_step(model, state, p, stats)
        calls += 1
    return calls


def generate(model: OracleModel, p: SamplerParams, batch: int, n_blocks: int,
             eos_early_stop: bool = True, stats: Optional[List[CanvasStats]] = None):
    """Blocks one after another (Nemotron guide, section 6: until gen_length
    or EOS; DiffusionGemma page: outer loop over canvases with eos_early_stop;
    course section 14: the finished block joins the cache through a clean
    pass).  READING: block k uses seed + k for its random streams.  Returns
    (tokens int64 [batch][blocks*C], blocks run)."""
    d = model.dims
    C = p.canvas
    out = []
    blocks = 0
    for k in range(n_blocks):
        pk = SamplerParams(**{**p.__dict__, "seed": p.seed + k})
        st = init_canvas(batch, pk, d.mask_id, d.vocab)
        decode_block(model, st, pk, stats)
        out.append(st.tokens.copy())
        for b in range(batch):
            model.kv_append_tokens(b, st.tokens[b])
        blocks += 1
        if eos_early_stop and (st.eos_pos >= 0).all():
            break
    return np.concatenate(out, axis=1), blocks


# ---------------------------------------------------------------------------
# the course's own greedy sampler, for the worked-example pin
# ---------------------------------------------------------------------------


def course_sampler(predict: Callable[[np.ndarray, int], np.ndarray], length: int, steps: int,
                   mask_id: int):
    """Course section 12, greedy confidence reveal: S model calls; at call s
    the number of masks drops to m_s; the positions opened are the masked
    ones of highest confidence, ties to the lower index.  Returns final
    tokens and the per-call (opened positions, tokens) trace."""
    sched = linear_mask_schedule(length, steps)
    tokens = np.full(length, mask_id, dtype=np.int64)
    trace = []
    for s in range(1, steps + 1):
        lg = np.asarray(predict(tokens.copy(), s), dtype=F64)
        z = lg - lg.max(axis=1, keepdims=True)
        pr = np.exp(z)
        pr /= pr.sum(axis=1, keepdims=True)
        cand = pr.argmax(axis=1)
        conf = pr[np.arange(length), cand]
        masked = [i for i in range(length) if tokens[i] == mask_id]
        n_open = len(masked) - sched[s]
        ranked = sorted(masked, key=lambda i: (-conf[i], i))
        opened = ranked[:n_open]
        for i in opened:
            tokens[i] = cand[i]
        trace.append((tuple(opened), tokens.copy()))
    return tokens, trace
