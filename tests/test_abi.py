"""The C ABI library loads, exports every function include/dlm.h declares,
and rejects invalid arguments on the host before touching a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "dlm.h")


def _library():
    import masked_block_diffusion_denoise_b200 as dlm
    if not os.path.exists(dlm.library_path()):
        from masked_block_diffusion_denoise_b200 import build
        build.build()
    return dlm


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dlm_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ("dlm_kv_append", "dlm_denoise_step", "dlm_decode_block", "dlm_create",
                 "dlm_destroy", "dlm_canvas_init", "dlm_commit", "dlm_last_error"):
        assert name in fns


def test_library_exports_every_declared_symbol():
    dlm = _library()
    out = subprocess.run(["nm", "-D", "--defined-only", dlm.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(dlm_\w+)", out))
    missing = [f for f in header_functions() if f not in exported]
    assert not missing, missing
    assert sorted(dlm.EXPORTED_SYMBOLS) == header_functions()
    L = dlm.lib()
    for f in header_functions():
        assert getattr(L, f) is not None


def test_struct_layouts_match_header_sizes():
    dlm = _library()
    # sizes of the C structs compiled by the host compiler from the header itself
    code = r'''
#include <stdio.h>
#include "dlm.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu\n", sizeof(dlm_model_desc), sizeof(dlm_weights),
         sizeof(dlm_sampler_params), sizeof(dlm_canvas), sizeof(dlm_canvas_stats));
  return 0;
}
'''
    import tempfile
    with tempfile.TemporaryDirectory() as td:
        c = os.path.join(td, "s.c")
        exe = os.path.join(td, "s")
        open(c, "w").write(code)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        sizes = list(map(int, subprocess.run([exe], capture_output=True, text=True,
                                             check=True).stdout.split()))
    assert sizes == [ctypes.sizeof(dlm.dlm_model_desc), ctypes.sizeof(dlm.dlm_weights),
                     ctypes.sizeof(dlm.dlm_sampler_params), ctypes.sizeof(dlm.dlm_canvas),
                     ctypes.sizeof(dlm.dlm_canvas_stats)]


def test_enum_values_match_header():
    """Every DLM_* enumerator of the header has the binding's value."""
    dlm = _library()
    header = open(os.path.join(ROOT, "include", "dlm.h")).read()
    names = sorted(set(re.findall(r"\b(DLM_[A-Z0-9_]+)\s*=", header)))
    code = "#include <stdio.h>\n#include \"dlm.h\"\nint main(void) {\n"
    code += "".join('  printf("%%d\\n", (int)%s);\n' % n for n in names)
    code += "  return 0;\n}\n"
    import tempfile
    with tempfile.TemporaryDirectory() as td:
        c = os.path.join(td, "e.c")
        exe = os.path.join(td, "e")
        open(c, "w").write(code)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe], check=True)
        vals = list(map(int, subprocess.run([exe], capture_output=True, text=True,
                                            check=True).stdout.split()))
    assert len(names) > 20
    for n, v in zip(names, vals):
        assert getattr(dlm, n) == v, n


def _desc(dlm, **kw):
    base = dict(d_model=256, n_heads=4, n_kv_heads=2, head_dim=128, vocab=1000,
                dtype=dlm.DLM_BF16, rope_theta=1e6, mask_id=100, eos_id=11, max_batch=2,
                max_prefix=64, max_canvas=32)
    base.update(kw)
    return dlm.dlm_model_desc(**base)


@pytest.mark.parametrize("bad", [
    dict(n_heads=3),                      # not a multiple of n_kv_heads
    dict(head_dim=64),                    # bf16 attention needs head_dim 128
    dict(d_model=200),                    # bf16 needs d_model % 64 == 0
    dict(mask_id=1000),                   # mask id outside the vocabulary
    dict(max_canvas=2048),                # canvas above the commit kernel's 1024
    dict(max_batch=0),
    dict(dtype=7),
    dict(dtype=0, head_dim=48),           # fp32 head_dim not supported
])
def test_create_rejects_invalid_descriptors(bad):
    dlm = _library()
    w = dlm.dlm_weights(1, 1, 1, 1, 1, 1)    # never dereferenced: validation comes first
    with pytest.raises(dlm.DlmError) as e:
        dlm.dlm_create(_desc(dlm, **bad), w)
    assert e.value.code == dlm.DLM_EINVAL
    assert dlm.dlm_last_error(None)


def test_create_rejects_null_weights():
    dlm = _library()
    with pytest.raises(dlm.DlmError) as e:
        dlm.dlm_create(_desc(dlm), dlm.dlm_weights(1, 0, 1, 1, 1, 1))
    assert e.value.code == dlm.DLM_EINVAL


def test_null_context_is_rejected():
    dlm = _library()
    L = dlm.lib()
    assert L.dlm_kv_append(None, 0, 1, None, None, None, None) == dlm.DLM_EINVAL
    assert L.dlm_kv_length(None, 0) == dlm.DLM_EINVAL
    assert L.dlm_launches_per_step(None) == dlm.DLM_EINVAL
    L.dlm_destroy(None)
