"""The attention kernels compute part of every key tile's exponentials on the
FMA pipe (dlm_test_exp2 runs the same device function): Cody-Waite range
reduction and a cubic for 2^f on [-1/2, 1/2].  Checked against 2^x in float64
over the arguments the softmax produces (x <= 8): maximum relative error
below 1e-4 (the fit's 7.5e-5; a bf16 P is rounded by up to 2^-9 anyway),
exact integer powers within the same bound, and 0 for masked keys."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # pragma: no cover - collected on CPU-only hosts
    pytest.skip("needs a CUDA device", allow_module_level=True)

from masked_block_diffusion_denoise_b200 import dlm_test_exp2


def _run(x: np.ndarray) -> np.ndarray:
    xd = torch.as_tensor(x.astype(np.float32)).cuda()
    out = torch.empty_like(xd)
    dlm_test_exp2(xd, out, xd.numel())
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


def test_polynomial_exp2_relative_error():
    r = np.random.default_rng(5)
    x = np.concatenate([np.linspace(-125.0, 8.0, 200001), r.uniform(-30, 8, 100000),
                        np.arange(-125, 9, dtype=np.float64),                  # integers
                        np.arange(-125, 8, dtype=np.float64) + 0.5]).astype(np.float32)
    got = _run(x)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1e-4, float(rel.max())


def test_polynomial_exp2_masked_keys_are_zero():
    x = np.array([-np.inf, -1e30, -126.0, -125.5, -200.0], dtype=np.float32)
    assert np.array_equal(_run(x), np.zeros(5))
