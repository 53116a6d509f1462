"""Convenience layer over the C ABI: uploads weights with torch, owns a
library context and a set of canvas tensors, and reads results back.

No arithmetic of the method happens here; every step runs in the library's
kernels through the functions of this package.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np
import torch

from . import (DLM_BF16, DLM_F32, DLM_MASK, DLM_UNIFORM, dlm_canvas, dlm_canvas_init,
               dlm_canvas_stats, dlm_check, dlm_commit, dlm_create, dlm_debug_buffer,
               dlm_debug_logits, dlm_decode_block, dlm_decode_block_host, dlm_denoise_step, dlm_generate,
               dlm_destroy, dlm_kv_append, dlm_model_desc, dlm_sampler_params, dlm_weights)

_TORCH = {"f32": torch.float32, "bf16": torch.bfloat16}
_NP_TYPESTR = {torch.float32: "<f4", torch.bfloat16: "<u2", torch.int32: "<i4",
               torch.uint8: "|u1"}


class _DevArray:
    """Zero-copy view of library-owned device memory for torch.as_tensor."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 2}


def host_to_device(a: np.ndarray, dtype: str, device) -> torch.Tensor:
    """numpy weights (bf16 bit patterns as uint16, or float32) -> device tensor."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(device)


@dataclass
class Canvas:
    tokens: torch.Tensor
    committed: torch.Tensor
    step: torch.Tensor
    done: torch.Tensor
    eos_pos: torch.Tensor
    stats: torch.Tensor      # int32 [B][6]
    prev_cand: torch.Tensor  # int32 [B][C], adaptive stopping
    stable: torch.Tensor     # int32 [B], adaptive stopping

    @property
    def c(self) -> dlm_canvas:
        return dlm_canvas(self.tokens.data_ptr(), self.committed.data_ptr(),
                          self.step.data_ptr(), self.done.data_ptr(), self.eos_pos.data_ptr(),
                          self.prev_cand.data_ptr(), self.stable.data_ptr())

    def numpy(self) -> Dict[str, np.ndarray]:
        return {"tokens": self.tokens.cpu().numpy().astype(np.int64),
                "committed": self.committed.cpu().numpy().astype(bool),
                "step": self.step.cpu().numpy().astype(np.int64),
                "done": self.done.cpu().numpy().astype(bool),
                "eos_pos": self.eos_pos.cpu().numpy().astype(np.int64),
                "prev_cand": self.prev_cand.cpu().numpy().astype(np.int64),
                "stable": self.stable.cpu().numpy().astype(np.int64),
                "stats": self.stats.cpu().numpy()}

    def load(self, tokens, committed, step, done, eos_pos, prev_cand=None, stable=None) -> None:
        self.tokens.copy_(torch.as_tensor(np.asarray(tokens, dtype=np.int32)))
        self.committed.copy_(torch.as_tensor(np.asarray(committed, dtype=np.uint8)))
        self.step.copy_(torch.as_tensor(np.asarray(step, dtype=np.int32)))
        self.done.copy_(torch.as_tensor(np.asarray(done, dtype=np.uint8)))
        self.eos_pos.copy_(torch.as_tensor(np.asarray(eos_pos, dtype=np.int32)))
        if prev_cand is None:
            self.prev_cand.fill_(-1)
        else:
            self.prev_cand.copy_(torch.as_tensor(np.asarray(prev_cand, dtype=np.int32)))
        if stable is None:
            self.stable.zero_()
        else:
            self.stable.copy_(torch.as_tensor(np.asarray(stable, dtype=np.int32)))


def sampler_params(canvas: int, steps: int, threshold: float = 0.9, quota: int = 0,
                   corruption: str = "mask", entropy_bound: float = -1.0,
                   temperature: float = 0.0, t_max: float = 0.8, t_min: float = 0.4,
                   seed: int = 0, stability_steps: int = 1, stop_entropy: float = -1.0,
                   editing: int = 0, editing_threshold: float = 0.9) -> dlm_sampler_params:
    return dlm_sampler_params(canvas, steps, threshold, quota,
                              DLM_UNIFORM if corruption == "uniform" else DLM_MASK, editing,
                              entropy_bound, temperature, t_max, t_min, seed, stability_steps,
                              stop_entropy, editing_threshold)


class Session:
    """One library context for a model shape and its weights."""

    def __init__(self, shape, weights: Dict[str, np.ndarray], *, max_batch: int,
                 max_prefix: int, max_canvas: int, device="cuda:0", upload=None):
        self.shape = shape
        self.device = torch.device(device)
        self.dtype = _TORCH[shape.dtype]
        if upload is None:
            self.w = {k: host_to_device(v, shape.dtype, self.device) for k, v in weights.items()}
        else:
            self.w = upload
        desc = dlm_model_desc(shape.d_model, shape.n_heads, shape.n_kv_heads, shape.head_dim,
                              shape.vocab, DLM_BF16 if shape.dtype == "bf16" else DLM_F32,
                              float(shape.rope_theta), shape.mask_id, shape.eos_id,
                              max_batch, max_prefix, max_canvas,
                              2 if getattr(shape, "lm_nvfp4", False)
                              else (1 if getattr(shape, "lm_fp8", False) else 0))
        wts = dlm_weights(*(self.w[k].data_ptr() for k in
                            ("emb", "w_q", "w_k", "w_v", "w_o", "w_lm")))
        torch.cuda.synchronize(self.device)
        self.ctx = dlm_create(desc, wts)
        self.max_batch, self.max_prefix, self.max_canvas = max_batch, max_prefix, max_canvas

    def close(self) -> None:
        if getattr(self, "ctx", None):
            dlm_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- prefix -------------------------------------------------------------
    def kv_append_tokens(self, seq: int, tokens: np.ndarray, stream=None) -> None:
        t = torch.as_tensor(np.asarray(tokens, dtype=np.int32)).to(self.device)
        dlm_kv_append(self.ctx, seq, int(t.numel()), tokens=t, stream=stream)
        torch.cuda.synchronize(self.device)

    def kv_append_kv(self, seq: int, k: np.ndarray, v: np.ndarray, stream=None) -> None:
        """k, v: [Hkv][n][Dh] as bf16 bit patterns (uint16) or float32."""
        kt = host_to_device(k, self.shape.dtype, self.device)
        vt = host_to_device(v, self.shape.dtype, self.device)
        dlm_kv_append(self.ctx, seq, int(k.shape[1]), k=kt, v=vt, stream=stream)
        torch.cuda.synchronize(self.device)

    # -- canvas ---------------------------------------------------------------
    def new_canvas(self, batch: int, C: int) -> Canvas:
        dev = self.device
        return Canvas(torch.zeros((batch, C), dtype=torch.int32, device=dev),
                      torch.zeros((batch, C), dtype=torch.uint8, device=dev),
                      torch.zeros(batch, dtype=torch.int32, device=dev),
                      torch.zeros(batch, dtype=torch.uint8, device=dev),
                      torch.full((batch,), -1, dtype=torch.int32, device=dev),
                      torch.zeros((batch, 6), dtype=torch.int32, device=dev),
                      torch.full((batch, C), -1, dtype=torch.int32, device=dev),
                      torch.zeros(batch, dtype=torch.int32, device=dev))

    def init(self, cv: Canvas, p: dlm_sampler_params, stream=None) -> None:
        dlm_canvas_init(self.ctx, cv.c, cv.tokens.shape[0], p, stream=stream)

    def step(self, cv: Canvas, p: dlm_sampler_params, stream=None) -> None:
        dlm_denoise_step(self.ctx, cv.c, cv.tokens.shape[0], p, stats=cv.stats, stream=stream)

    def block(self, cv: Canvas, p: dlm_sampler_params, stream=None) -> None:
        dlm_decode_block(self.ctx, cv.c, cv.tokens.shape[0], p, stats=cv.stats, stream=stream)

    def commit(self, cv: Canvas, p: dlm_sampler_params, cand, conf, ent, stream=None) -> None:
        dlm_commit(self.ctx, cv.c, cv.tokens.shape[0], p, cand, conf, ent, stats=cv.stats,
                   stream=stream)

    def generate(self, cv: Canvas, p: dlm_sampler_params, n_blocks: int,
                 eos_early_stop: bool = True, stream=None) -> tuple:
        """(tokens [B][n_blocks*C] int32 on the device, blocks decoded)."""
        B, C = cv.tokens.shape
        out = torch.zeros((B, n_blocks * C), dtype=torch.int32, device=self.device)
        n = dlm_generate(self.ctx, cv.c, B, p, n_blocks, out, eos_early_stop=eos_early_stop,
                         stats=cv.stats, stream=stream)
        return out, n

    def check(self, stream=None) -> None:
        dlm_check(self.ctx, stream)

    # -- inspection ---------------------------------------------------------
    def buffer(self, which: int, shape, dtype: torch.dtype) -> torch.Tensor:
        ptr, nbytes = dlm_debug_buffer(self.ctx, which)
        n = int(np.prod(shape))
        assert n * torch.tensor([], dtype=dtype).element_size() <= nbytes
        t = torch.as_tensor(_DevArray(ptr, (n,), _NP_TYPESTR[dtype]), device=self.device)
        if dtype == torch.bfloat16:
            t = t.view(torch.bfloat16)
        return t.view(*shape)

    def logits(self, batch: int, C: int) -> torch.Tensor:
        out = torch.empty((batch * C, self.shape.vocab), dtype=torch.float32, device=self.device)
        dlm_debug_logits(self.ctx, batch, C, out)
        return out
