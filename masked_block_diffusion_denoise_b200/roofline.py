"""Roofline arithmetic for the denoise step.

Two parts:

* the course "Diffusion LLMs" illustrative model (sections 1, 10 and 11):
  a weight-read bound and an ideal-arithmetic bound per model call, for an
  autoregressive step and for a diffusion pass over a canvas of N positions;
* the algorithmic bytes and flops of one denoise step of this library's
  kernels, per stage, which ``bench.py`` divides by measured kernel times.

Algorithmic bytes count every weight once per step, the prefix K/V once per
(sequence, KV head), activations once in and once out; full logits are never
stored, so they are not counted.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Sequence


# ---------------------------------------------------------------------------
# course model (course "Diffusion LLMs", sections 1, 10, 11)
# ---------------------------------------------------------------------------

def ar_bounds(params: float, weight_bytes: float, mem_bw: float, flops: float) -> Dict[str, float]:
    """One autoregressive step at batch 1: reading every weight once versus
    the ideal 2P arithmetic."""
    t_mem = weight_bytes / mem_bw
    t_compute = 2.0 * params / flops
    return {"t_mem_s": t_mem, "t_compute_s": t_compute,
            "compute_share": t_compute / t_mem,
            "tokens_per_s": 1.0 / max(t_mem, t_compute)}


def diffusion_pass(params: float, canvas: int, weight_bytes: float, mem_bw: float,
                   flops: float) -> Dict[str, float]:
    """One model call over a canvas of N positions: 2PN flops against one
    read of the weights; the pass takes the larger of the two."""
    work = 2.0 * params * canvas
    t_compute = work / flops
    t_mem = weight_bytes / mem_bw
    return {"flop": work, "t_compute_s": t_compute, "t_mem_s": t_mem,
            "t_pass_s": max(t_compute, t_mem),
            "bound": "compute" if t_compute >= t_mem else "memory"}


def diffusion_tokens_per_s(canvas: int, steps: int, t_pass_s: float) -> float:
    """Q <= N / (S * t_pass)."""
    return canvas / (steps * t_pass_s)


def parity_steps(canvas: int, t_pass_s: float, ar_tokens_per_s: float) -> float:
    """Step count S* at which the diffusion bound equals the AR bound."""
    return canvas / (t_pass_s * ar_tokens_per_s)


# ---------------------------------------------------------------------------
# this library's step
# ---------------------------------------------------------------------------

@dataclass(frozen=True)
class StepShape:
    d_model: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    vocab: int
    elem_bytes: int          # 2 for bf16, 4 for fp32
    canvas: int
    prefix_lens: Sequence[int]   # per active sequence

    @property
    def rows(self) -> int:
        return self.canvas * len(self.prefix_lens)


def step_work(s: StepShape, lm_tile: int = 128, part_bytes: int = 24,
              lm_elem_bytes: int = 0, lm_nvfp4: bool = False) -> Dict[str, Dict[str, float]]:
    """Algorithmic bytes and flops of each stage of one denoise step.
    lm_elem_bytes = 1: the e4m3 LM head (one-byte weights and input rows, a
    float32 scale per vocabulary row and per input row, and the quantisation
    of the input rows); lm_nvfp4: the NVFP4 head (half a byte per element,
    one e4m3 scale per 16 elements, a float32 scale per row, for weights and
    input rows, and the quantisation of the input rows); otherwise the head
    in the model's element type."""
    e = s.elem_bytes
    M, d, V = s.rows, s.d_model, s.vocab
    qd, kvd = s.n_heads * s.head_dim, s.n_kv_heads * s.head_dim
    nqkv = qd + 2 * kvd
    keys = sum(L + s.canvas for L in s.prefix_lens)
    ntiles = -(-V // lm_tile)
    out = {
        "embed": {"bytes": 2.0 * M * d * e + 4.0 * M, "flop": 0.0},
        "qkv": {"bytes": float(nqkv * d * e + M * d * e + M * nqkv * e),
                "flop": 2.0 * M * d * nqkv},
        # every key/value of the prefix plus the canvas, once per KV head;
        # queries in, attention output out
        "attention": {"bytes": float(2 * keys * kvd * e + 2 * M * qd * e),
                      "flop": 4.0 * keys * s.canvas * s.n_heads * s.head_dim},
        "wo": {"bytes": float(d * qd * e + M * qd * e + 2 * M * d * e),
               "flop": 2.0 * M * qd * d},
        "lm_head": {"bytes": float(V * d * e + M * d * e + M * ntiles * part_bytes),
                    "flop": 2.0 * M * d * V},
        "quantize": {"bytes": 0.0, "flop": 0.0},
        "reduce": {"bytes": float(M * ntiles * part_bytes + 12 * M), "flop": 0.0},
        "commit": {"bytes": float(M * (4 + 1 + 4 + 4 + 4) * 2), "flop": 0.0},
    }
    if lm_nvfp4:
        q4 = lambda rows: rows * d / 2 + rows * d / 16 + 4 * rows
        out["lm_head"]["bytes"] = float(q4(V) + q4(M) + M * ntiles * part_bytes)
        out["quantize"]["bytes"] = float(M * d * e + q4(M))
    elif lm_elem_bytes == 1:
        out["lm_head"]["bytes"] = float(V * d + M * d + 4 * V + 4 * M + M * ntiles * part_bytes)
        out["quantize"]["bytes"] = float(M * d * e + M * d + 4 * M)
    out["step"] = {"bytes": sum(v["bytes"] for v in out.values()),
                   "flop": sum(v["flop"] for v in out.values())}
    return out
