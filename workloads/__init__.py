"""Seeded synthetic inputs for the masked block-diffusion denoise step.

This module draws random numbers and lays them out in the shapes of the
workloads; it computes none of the method's arithmetic (no projection,
attention, softmax, selection or random-number stream of the sampler).  Both
the CPU oracle and the CUDA path consume the arrays it returns, so that the
two sides see bit-identical inputs.

Workload shapes follow the pages' problem statement:
  * Nemotron-Labs-Diffusion-8B shape (d_model 4096, 32 query / 8 KV heads,
    head dim 128, vocab 131072, mask id 100, EOS id 11, RoPE theta 1e6) --
    "MLX-VLM runs NVIDIA Nemotron Labs Diffusion" guide, section 7
    (architecture details);
  * block length 32, 32 denoising steps, 0.9 threshold -- same guide,
    sections 3.2 and 6;
  * DiffusionGemma canvas 256, 48 steps, uniform corruption, entropy bound
    0.1 with temperature annealed 0.8 -> 0.4 -- diffusers DiffusionGemma
    pipeline page, "Usage" and "Schedulers".
The public benchmarks those pages evaluate on are not available; seeded
random-init weights and random prefixes stand in for them.

Recipe (all draws from numpy.random.default_rng([seed, stream])):
  * embedding table E[V][d] ~ N(0, 1); W_q, W_k, W_v, W_o, W_lm ~ N(0, 0.02);
    drawn in float32, then rounded to bfloat16 (round-to-nearest-even) for
    bf16 workloads, kept float32 for the fp32 workload;
  * prefix: either uniform random token ids (tiny workload; their K/V are
    computed by the library from the weights) or post-RoPE K/V ~ N(0, 1)
    (all other workloads), lengths fixed or uniform in [lo, hi];
  * EOS plant: each canvas independently with probability ``eos_frac`` gets
    the EOS id pre-committed at a uniform slot of the canvas.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Dict, List, Optional, Tuple

import numpy as np

__all__ = [
    "ModelShape", "Workload", "WORKLOADS", "to_bf16_bits", "from_bf16_bits",
    "make_weights", "make_prefix", "make_eos_plant", "small_workload",
]

# stream ids: each array has its own RNG stream, so changing one size never
# shifts the values of another array.
_STREAM = {"emb": 1, "w_q": 2, "w_k": 3, "w_v": 4, "w_o": 5, "w_lm": 6,
           "prefix_len": 10, "prefix_tok": 11, "prefix_k": 12, "prefix_v": 13,
           "eos": 20}


@dataclass(frozen=True)
class ModelShape:
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    vocab: int
    dtype: str = "bf16"            # "bf16" or "f32"
    rope_theta: float = 1.0e6
    mask_id: int = 100
    eos_id: int = 11
    lm_fp8: bool = False           # LM head in e4m3 (weights and its input rows)
    lm_nvfp4: bool = False         # LM head in NVFP4 (e2m1, e4m3 block scales of 16)

    @property
    def q_dim(self) -> int:
        return self.n_heads * self.head_dim

    @property
    def kv_dim(self) -> int:
        return self.n_kv_heads * self.head_dim


@dataclass(frozen=True)
class Workload:
    name: str
    shape: ModelShape
    batch: int
    canvas: int
    steps: int
    threshold: float = 0.9
    quota: int = 0                 # 0 -> ceil(canvas / steps)
    corruption: str = "mask"       # "mask" or "uniform"
    prefix_kind: str = "kv"        # "kv" (random post-RoPE K/V) or "tokens"
    prefix_len: Tuple[int, int] = (2048, 2048)   # inclusive range
    prefix_cap: int = 2048         # KV capacity reserved for the prefix
    eos_frac: float = 0.0
    entropy_bound: float = -1.0    # < 0: threshold + quota selection
    temperature: float = 0.0
    t_max: float = 0.8
    t_min: float = 0.4
    seed: int = 0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def quota_eff(self) -> int:
        return self.quota if self.quota > 0 else -(-self.canvas // self.steps)


_SHAPE_8B = ModelShape(d_model=4096, n_heads=32, n_kv_heads=8, head_dim=128,
                       vocab=131072, dtype="bf16")
_SHAPE_ENCDEC = ModelShape(d_model=2048, n_heads=16, n_kv_heads=16, head_dim=128,
                           vocab=262144, dtype="bf16")
_SHAPE_TINY = ModelShape(d_model=256, n_heads=4, n_kv_heads=4, head_dim=64,
                         vocab=4096, dtype="f32")

WORKLOADS: Dict[str, Workload] = {
    # tiny fp32 reference: prefix of 128 random ids, canvas 32, 8 steps, quota 4
    "tiny": Workload("tiny", _SHAPE_TINY, batch=1, canvas=32, steps=8, threshold=0.9,
                     quota=4, prefix_kind="tokens", prefix_len=(128, 128), prefix_cap=128),
    # 8B-class dense shape, batch 1, prefix KV 2048, canvas 32, 32 steps, quota 1
    "8b_b1": Workload("8b_b1", _SHAPE_8B, batch=1, canvas=32, steps=32, threshold=0.9,
                      quota=1, prefix_len=(2048, 2048), prefix_cap=2048),
    # batched serving: 16 canvases of 64, prefix lengths uniform in [1024, 4096], EOS plant
    "batched": Workload("batched", _SHAPE_8B, batch=16, canvas=64, steps=32, threshold=0.9,
                        quota=2, prefix_len=(1024, 4096), prefix_cap=4096, eos_frac=0.2),
    # long context: 4 canvases of 32 over 32768-token prefixes, 16 steps, quota 2
    "longctx": Workload("longctx", _SHAPE_8B, batch=4, canvas=32, steps=16, threshold=0.9,
                        quota=2, prefix_len=(32768, 32768), prefix_cap=32768),
    # encoder-decoder block refinement: canvas 256, 48 steps, uniform corruption
    "encdec": Workload("encdec", _SHAPE_ENCDEC, batch=2, canvas=256, steps=48, threshold=0.9,
                       quota=0, corruption="uniform", prefix_len=(1024, 1024),
                       prefix_cap=1024),
    # same shape, entropy-bound selection (bound 0.1, temperature 0.8 -> 0.4)
    "encdec_eb": Workload("encdec_eb", _SHAPE_ENCDEC, batch=2, canvas=256, steps=48,
                          threshold=0.9, quota=0, corruption="uniform",
                          prefix_len=(1024, 1024), prefix_cap=1024, entropy_bound=0.1,
                          t_max=0.8, t_min=0.4),
}
# the same workloads with the e4m3 LM head (online FP8 weight quantisation)
# and with the NVFP4 LM head (4-bit weights, the Blackwell low-bit path)
for _name in ("8b_b1", "batched", "encdec"):
    _w = WORKLOADS[_name]
    WORKLOADS[_name + "_fp8"] = _w.replace(name=_name + "_fp8",
                                           shape=dataclasses.replace(_w.shape, lm_fp8=True))
for _name in ("8b_b1", "longctx"):
    _w = WORKLOADS[_name]
    WORKLOADS[_name + "_nvfp4"] = _w.replace(name=_name + "_nvfp4",
                                             shape=dataclasses.replace(_w.shape, lm_nvfp4=True))


def small_workload(name: str = "small", *, d_model=256, n_heads=4, n_kv_heads=2,
                   head_dim=128, vocab=4096 + 96, batch=2, canvas=32, steps=8,
                   prefix_len=(200, 333), prefix_cap=384, dtype="bf16", lm_fp8=False,
                   lm_nvfp4=False, **kw) -> Workload:
    """A reduced workload that the oracle finishes in seconds; by default the
    vocabulary, prefix lengths and canvas are not multiples of the kernels'
    tile sizes, so every tiling has a ragged tail."""
    shape = ModelShape(d_model=d_model, n_heads=n_heads, n_kv_heads=n_kv_heads,
                       head_dim=head_dim, vocab=vocab, dtype=dtype, lm_fp8=lm_fp8,
                       lm_nvfp4=lm_nvfp4)
    return Workload(name, shape, batch=batch, canvas=canvas, steps=steps,
                    prefix_len=prefix_len, prefix_cap=prefix_cap, **kw)


# ----------------------------------------------------------------------------
# storage format helpers (data layout only)
# ----------------------------------------------------------------------------

def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(seed: int, stream: str) -> np.random.Generator:
    return np.random.default_rng([int(seed), _STREAM[stream]])


def _normal(seed, stream, shape, std, dtype):
    a = _rng(seed, stream).standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return to_bf16_bits(a) if dtype == "bf16" else a


def make_weights(shape: ModelShape, seed: int = 0) -> Dict[str, np.ndarray]:
    """Random-init weights, row-major, out-features by in-features.

    bf16 shapes return uint16 bit patterns, the f32 shape returns float32.
    """
    d, V = shape.d_model, shape.vocab
    return {
        "emb": _normal(seed, "emb", (V, d), 1.0, shape.dtype),
        "w_q": _normal(seed, "w_q", (shape.q_dim, d), 0.02, shape.dtype),
        "w_k": _normal(seed, "w_k", (shape.kv_dim, d), 0.02, shape.dtype),
        "w_v": _normal(seed, "w_v", (shape.kv_dim, d), 0.02, shape.dtype),
        "w_o": _normal(seed, "w_o", (d, shape.q_dim), 0.02, shape.dtype),
        "w_lm": _normal(seed, "w_lm", (V, d), 0.02, shape.dtype),
    }


def make_prefix(wl: Workload, seed: Optional[int] = None):
    """Prefix of every canvas.

    Returns ``(lens, tokens, k, v)``: ``lens`` int32[B]; for ``prefix_kind ==
    'tokens'`` a list of int32 arrays (one per canvas) and ``k = v = None``;
    for ``'kv'`` ``tokens = None`` and ``k, v`` of shape [B][Hkv][max_len][Dh]
    (bf16 bits or float32), of which only the first ``lens[b]`` positions of
    canvas b are meaningful.
    """
    seed = wl.seed if seed is None else seed
    lo, hi = wl.prefix_len
    B = wl.batch
    if lo == hi:
        lens = np.full(B, lo, dtype=np.int32)
    else:
        lens = _rng(seed, "prefix_len").integers(lo, hi + 1, size=B).astype(np.int32)
    sh = wl.shape
    if wl.prefix_kind == "tokens":
        r = _rng(seed, "prefix_tok")
        toks = [r.integers(0, sh.vocab, size=int(n)).astype(np.int32) for n in lens]
        return lens, toks, None, None
    L = int(lens.max())
    shp = (B, sh.n_kv_heads, L, sh.head_dim)
    k = _normal(seed, "prefix_k", shp, 1.0, sh.dtype)
    v = _normal(seed, "prefix_v", shp, 1.0, sh.dtype)
    return lens, None, k, v


def make_eos_plant(wl: Workload, seed: Optional[int] = None) -> List[Tuple[int, int]]:
    """(canvas, slot) pairs at which the EOS id is pre-committed."""
    seed = wl.seed if seed is None else seed
    if wl.eos_frac <= 0.0:
        return []
    r = _rng(seed, "eos")
    pick = r.random(wl.batch) < wl.eos_frac
    slots = r.integers(0, wl.canvas, size=wl.batch)
    return [(int(b), int(slots[b])) for b in range(wl.batch) if pick[b]]
