"""Python binding of the masked block-diffusion denoise-step library.

Argument marshalling only: every function forwards to the C ABI of
``libdlm.so`` (declared in ``include/dlm.h``) under the same name; all work
runs in the library's CUDA kernels.  PyTorch supplies device memory and
streams.  Importing this package does not load the library; the first call
does, and raises if ``libdlm.so`` has not been built (there is no fallback).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "DLM_OK", "DLM_EINVAL", "DLM_ENOMEM", "DLM_ECUDA", "DLM_ECAP", "DLM_ETIMEOUT",
    "DLM_EBOUNDS", "DLM_ESTATE", "DLM_F32", "DLM_BF16", "DLM_MASK", "DLM_UNIFORM",
    "DLM_BUF_X", "DLM_BUF_Q", "DLM_BUF_O", "DLM_BUF_Y", "DLM_BUF_CAND", "DLM_BUF_CONF",
    "DLM_BUF_ENTROPY", "DLM_BUF_K_CACHE", "DLM_BUF_V_CACHE", "DLM_BUF_LM_Q", "DLM_BUF_LM_SCALE",
    "DLM_BUF_Y_Q", "DLM_BUF_Y_SCALE", "DLM_BUF_LM_SF", "DLM_BUF_Y_SF", "DLM_LM_MODEL",
    "DLM_LM_E4M3", "DLM_LM_NVFP4",
    "dlm_model_desc", "dlm_weights", "dlm_sampler_params", "dlm_canvas", "dlm_canvas_stats",
    "DlmError", "lib", "library_path", "dlm_create", "dlm_destroy", "dlm_kv_append",
    "dlm_reset_kv", "dlm_kv_length", "dlm_canvas_init", "dlm_denoise_step",
    "dlm_decode_block", "dlm_decode_block_host", "dlm_commit", "dlm_generate", "dlm_debug_buffer",
    "dlm_debug_logits", "dlm_check", "dlm_launches_per_step", "dlm_last_error",
    "EXPORTED_SYMBOLS", "dlm_set_stage_events", "DLM_STAGE_EMBED", "DLM_STAGE_QKV",
    "DLM_STAGE_ATTENTION", "DLM_STAGE_WO", "DLM_STAGE_LM_HEAD", "DLM_STAGE_COMMIT",
    "DLM_NUM_STAGES", "dlm_attention_noalloc", "dlm_attention_noalloc_check",
    "dlm_trace_layout", "dlm_trace_read", "dlm_trace_clear", "dlm_decode_steps",
    "dlm_attention_plan", "dlm_test_withhold_loads", "dlm_test_exp2",
]

DLM_OK, DLM_EINVAL, DLM_ENOMEM, DLM_ECUDA, DLM_ECAP, DLM_ETIMEOUT, DLM_EBOUNDS, DLM_ESTATE = \
    0, -1, -2, -3, -4, -5, -6, -7
DLM_F32, DLM_BF16 = 0, 1
DLM_MASK, DLM_UNIFORM = 0, 1
(DLM_BUF_X, DLM_BUF_Q, DLM_BUF_O, DLM_BUF_Y, DLM_BUF_CAND, DLM_BUF_CONF, DLM_BUF_ENTROPY,
 DLM_BUF_K_CACHE, DLM_BUF_V_CACHE, DLM_BUF_LM_Q, DLM_BUF_LM_SCALE, DLM_BUF_Y_Q,
 DLM_BUF_Y_SCALE, DLM_BUF_LM_SF, DLM_BUF_Y_SF) = range(15)
DLM_LM_MODEL, DLM_LM_E4M3, DLM_LM_NVFP4 = 0, 1, 2

(DLM_STAGE_EMBED, DLM_STAGE_QKV, DLM_STAGE_ATTENTION, DLM_STAGE_WO, DLM_STAGE_LM_HEAD,
 DLM_STAGE_COMMIT, DLM_NUM_STAGES) = range(7)

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.environ.get("DLM_LIBRARY", os.path.join(_HERE, "libdlm.so"))


class dlm_model_desc(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("n_heads", ctypes.c_int),
                ("n_kv_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
                ("vocab", ctypes.c_int), ("dtype", ctypes.c_int),
                ("rope_theta", ctypes.c_float), ("mask_id", ctypes.c_int),
                ("eos_id", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("max_prefix", ctypes.c_int), ("max_canvas", ctypes.c_int),
                ("lm_quant", ctypes.c_int)]


class dlm_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("emb", "w_q", "w_k", "w_v", "w_o", "w_lm")]


class dlm_sampler_params(ctypes.Structure):
    _fields_ = [("canvas", ctypes.c_int), ("steps", ctypes.c_int),
                ("threshold", ctypes.c_float), ("quota", ctypes.c_int),
                ("corruption", ctypes.c_int), ("editing", ctypes.c_int),
                ("entropy_bound", ctypes.c_float), ("temperature", ctypes.c_float),
                ("t_max", ctypes.c_float), ("t_min", ctypes.c_float),
                ("seed", ctypes.c_ulonglong), ("stability_steps", ctypes.c_int),
                ("stop_entropy", ctypes.c_float), ("editing_threshold", ctypes.c_float)]


class dlm_canvas(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("tokens", "committed", "step", "done", "eos_pos",
                                                  "prev_cand", "stable")]


class dlm_canvas_stats(ctypes.Structure):
    _fields_ = [("steps_used", ctypes.c_int32), ("committed_by_sampler", ctypes.c_int32),
                ("forced_at_budget", ctypes.c_int32), ("eos_autofill", ctypes.c_int32),
                ("frozen", ctypes.c_int32), ("edited", ctypes.c_int32)]


class DlmError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__("dlm error %d: %s" % (code, msg))
        self.code = code


_P = ctypes.c_void_p
_I = ctypes.c_int
_SIGS = {
    "dlm_create": (_I, [ctypes.POINTER(dlm_model_desc), ctypes.POINTER(dlm_weights),
                        ctypes.POINTER(_P)]),
    "dlm_destroy": (None, [_P]),
    "dlm_kv_append": (_I, [_P, _I, _I, _P, _P, _P, _P]),
    "dlm_reset_kv": (_I, [_P, _I]),
    "dlm_kv_length": (_I, [_P, _I]),
    "dlm_canvas_init": (_I, [_P, ctypes.POINTER(dlm_canvas), _I,
                             ctypes.POINTER(dlm_sampler_params), _P]),
    "dlm_denoise_step": (_I, [_P, ctypes.POINTER(dlm_canvas), _I,
                              ctypes.POINTER(dlm_sampler_params), _P, _P]),
    "dlm_decode_block": (_I, [_P, ctypes.POINTER(dlm_canvas), _I,
                              ctypes.POINTER(dlm_sampler_params), _P, _P]),
    "dlm_decode_steps": (_I, [_P, ctypes.POINTER(dlm_canvas), _I,
                              ctypes.POINTER(dlm_sampler_params), _I, _P, _P]),
    "dlm_attention_plan": (_I, [_P, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I),
                                ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "dlm_decode_block_host": (_I, [_P, _P, _P, _P, _P, _P, _I,
                                   ctypes.POINTER(dlm_sampler_params), _P, _P]),
    "dlm_commit": (_I, [_P, ctypes.POINTER(dlm_canvas), _I, ctypes.POINTER(dlm_sampler_params),
                        _P, _P, _P, _P, _P]),
    "dlm_generate": (_I, [_P, ctypes.POINTER(dlm_canvas), _I, ctypes.POINTER(dlm_sampler_params),
                          _I, _I, _P, _P, ctypes.POINTER(_I), _P]),
    "dlm_debug_buffer": (_I, [_P, _I, ctypes.POINTER(_P), ctypes.POINTER(ctypes.c_size_t)]),
    "dlm_debug_logits": (_I, [_P, _I, _I, _P, _P]),
    "dlm_set_stage_events": (_I, [_P, _I, ctypes.POINTER(_P), _I]),
    "dlm_attention_noalloc": (_I, [_P, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _P]),
    "dlm_attention_noalloc_check": (_I, [_P]),
    "dlm_check": (_I, [_P, _P]),
    "dlm_launches_per_step": (_I, [_P]),
    "dlm_test_withhold_loads": (_I, [_P, _I]),
    "dlm_test_exp2": (_I, [_P, _P, _I, _P]),
    "dlm_trace_layout": (_I, [ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "dlm_trace_read": (_I, [ctypes.POINTER(ctypes.c_ulonglong), ctypes.c_size_t]),
    "dlm_trace_clear": (_I, []),
    "dlm_last_error": (ctypes.c_char_p, [_P]),
}
EXPORTED_SYMBOLS = tuple(_SIGS)

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libdlm.so once; raise if it is missing."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError("libdlm.so not built (%s); run python -m "
                               "masked_block_diffusion_denoise_b200.build" % path)
        L = ctypes.CDLL(path)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(x) -> Optional[int]:
    """Device/host address of a torch tensor, an int, or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(ctx, rc: int) -> int:
    if rc < 0:
        raise DlmError(rc, lib().dlm_last_error(ctx).decode())
    return rc


def dlm_last_error(ctx) -> str:
    return lib().dlm_last_error(ctx).decode()


def dlm_create(desc: dlm_model_desc, weights: dlm_weights) -> int:
    out = ctypes.c_void_p()
    rc = lib().dlm_create(ctypes.byref(desc), ctypes.byref(weights), ctypes.byref(out))
    if rc != DLM_OK:
        raise DlmError(rc, lib().dlm_last_error(None).decode())
    return out.value


def dlm_destroy(ctx) -> None:
    lib().dlm_destroy(ctx)


def dlm_kv_append(ctx, seq: int, n: int, tokens=None, k=None, v=None, stream=None) -> int:
    return _check(ctx, lib().dlm_kv_append(ctx, seq, n, _ptr(tokens), _ptr(k), _ptr(v),
                                           _stream(stream)))


def dlm_reset_kv(ctx, seq: int) -> int:
    return _check(ctx, lib().dlm_reset_kv(ctx, seq))


def dlm_kv_length(ctx, seq: int) -> int:
    return _check(ctx, lib().dlm_kv_length(ctx, seq))


def dlm_canvas_init(ctx, canvas: dlm_canvas, batch: int, params: dlm_sampler_params,
                    stream=None) -> int:
    return _check(ctx, lib().dlm_canvas_init(ctx, ctypes.byref(canvas), batch,
                                             ctypes.byref(params), _stream(stream)))


def dlm_denoise_step(ctx, canvas: dlm_canvas, batch: int, params: dlm_sampler_params,
                     stats=None, stream=None) -> int:
    return _check(ctx, lib().dlm_denoise_step(ctx, ctypes.byref(canvas), batch,
                                              ctypes.byref(params), _ptr(stats),
                                              _stream(stream)))


def dlm_decode_block(ctx, canvas: dlm_canvas, batch: int, params: dlm_sampler_params,
                     stats=None, stream=None) -> int:
    return _check(ctx, lib().dlm_decode_block(ctx, ctypes.byref(canvas), batch,
                                              ctypes.byref(params), _ptr(stats),
                                              _stream(stream)))


def dlm_decode_steps(ctx, canvas: dlm_canvas, batch: int, params: dlm_sampler_params,
                     n_steps: int, stats=None, stream=None) -> int:
    return _check(ctx, lib().dlm_decode_steps(ctx, ctypes.byref(canvas), batch,
                                              ctypes.byref(params), n_steps, _ptr(stats),
                                              _stream(stream)))


def dlm_attention_plan(ctx, batch: int, canvas: int) -> dict:
    """The attention split plan for the context's current prefix lengths."""
    ns, ch, cl, rows = _I(), _I(), _I(), _I()
    _check(ctx, lib().dlm_attention_plan(ctx, batch, canvas, ctypes.byref(ns), ctypes.byref(ch),
                                         ctypes.byref(cl), ctypes.byref(rows)))
    return {"nsplit": ns.value, "chunk": ch.value, "cluster": cl.value,
            "rows_per_cta": rows.value}


def dlm_decode_block_host(ctx, tokens, committed, step, done, eos_pos, batch: int,
                          params: dlm_sampler_params, stats=None, stream=None) -> int:
    """Host (CPU, ideally pinned) tensors in, results copied back in place."""
    return _check(ctx, lib().dlm_decode_block_host(
        ctx, _ptr(tokens), _ptr(committed), _ptr(step), _ptr(done), _ptr(eos_pos), batch,
        ctypes.byref(params), _ptr(stats), _stream(stream)))


def dlm_commit(ctx, canvas: dlm_canvas, batch: int, params: dlm_sampler_params, cand, conf,
               entropy, stats=None, stream=None) -> int:
    return _check(ctx, lib().dlm_commit(ctx, ctypes.byref(canvas), batch, ctypes.byref(params),
                                        _ptr(cand), _ptr(conf), _ptr(entropy), _ptr(stats),
                                        _stream(stream)))


def dlm_generate(ctx, canvas: dlm_canvas, batch: int, params: dlm_sampler_params,
                 n_blocks: int, out_tokens, eos_early_stop: bool = True, stats=None,
                 stream=None) -> int:
    """Decodes up to n_blocks blocks; returns how many were decoded."""
    n = ctypes.c_int(0)
    _check(ctx, lib().dlm_generate(ctx, ctypes.byref(canvas), batch, ctypes.byref(params),
                                   n_blocks, 1 if eos_early_stop else 0, _ptr(out_tokens),
                                   _ptr(stats), ctypes.byref(n), _stream(stream)))
    return n.value


def dlm_debug_buffer(ctx, which: int):
    """(device address, size in bytes) of one of the context's buffers."""
    p = ctypes.c_void_p()
    n = ctypes.c_size_t()
    _check(ctx, lib().dlm_debug_buffer(ctx, which, ctypes.byref(p), ctypes.byref(n)))
    return p.value, n.value


def dlm_debug_logits(ctx, batch: int, canvas: int, logits, stream=None) -> int:
    return _check(ctx, lib().dlm_debug_logits(ctx, batch, canvas, _ptr(logits),
                                              _stream(stream)))


def dlm_set_stage_events(ctx, stage: int, events) -> int:
    """events: a flat list of cudaEvent_t handles (ints), two per step slot."""
    n = len(events)
    arr = (ctypes.c_void_p * max(n, 1))(*events)
    return _check(ctx, lib().dlm_set_stage_events(ctx, stage, arr if n else None, n // 2))


def dlm_attention_noalloc(q, k_cache, v_cache, lens, max_len: int, o, batch: int, canvas: int,
                          n_heads: int, n_kv_heads: int, head_dim: int, kv_batch: int,
                          kv_capacity: int, stream=None) -> int:
    """Canvas attention with no device allocation (see include/dlm.h)."""
    rc = lib().dlm_attention_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(lens), max_len,
                                     _ptr(o), batch, canvas, n_heads, n_kv_heads, head_dim,
                                     kv_batch, kv_capacity, _stream(stream))
    if rc != DLM_OK:
        raise DlmError(rc, lib().dlm_last_error(None).decode())
    return rc


def dlm_attention_noalloc_check(stream=None) -> int:
    """Read and clear the device error word of dlm_attention_noalloc; raises
    DlmError(DLM_ETIMEOUT / DLM_EBOUNDS) when a kernel recorded one."""
    rc = lib().dlm_attention_noalloc_check(_stream(stream))
    if rc != DLM_OK:
        raise DlmError(rc, lib().dlm_last_error(None).decode())
    return rc


def dlm_check(ctx, stream=None) -> int:
    return _check(ctx, lib().dlm_check(ctx, _stream(stream)))


def dlm_launches_per_step(ctx) -> int:
    return _check(ctx, lib().dlm_launches_per_step(ctx))


def dlm_test_exp2(x, out, n: int, stream=None) -> int:
    """out = 2^x by the attention kernels' polynomial exponential (test hook)."""
    rc = lib().dlm_test_exp2(_ptr(x), _ptr(out), n, _stream(stream))
    if rc != DLM_OK:
        raise DlmError(rc, lib().dlm_last_error(None).decode())
    return rc


def dlm_test_withhold_loads(ctx, n_launches: int) -> int:
    """Failure-detection test hook: the next n GEMM launches issue no loads,
    so their bounded waits run out and DLM_ETIMEOUT is recorded."""
    return _check(ctx, lib().dlm_test_withhold_loads(ctx, n_launches))


def dlm_trace_layout():
    """(kinds, ctas, slots) of the device timeline; DlmError(DLM_ESTATE)
    unless the library is the DLM_TRACE build (see include/dlm.h)."""
    k, c, s = _I(), _I(), _I()
    _check(None, lib().dlm_trace_layout(ctypes.byref(k), ctypes.byref(c), ctypes.byref(s)))
    return k.value, c.value, s.value


def dlm_trace_read():
    """The device timeline as a uint64 array [kinds][ctas][slots] (ns)."""
    import numpy as np
    k, c, s = dlm_trace_layout()
    t = np.zeros(k * c * s, dtype=np.uint64)
    _check(None, lib().dlm_trace_read(t.ctypes.data_as(ctypes.POINTER(ctypes.c_ulonglong)),
                                      t.size))
    return t.reshape(k, c, s)


def dlm_trace_clear() -> int:
    return _check(None, lib().dlm_trace_clear())
