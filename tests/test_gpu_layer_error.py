"""GPU layer-error sweep against the oracle: err(k) = ||Y_RAC(k) - X What^T||
/ ||X What^T|| of one dense layer (QUADS, gist.science/it 2.2 B and section 2),
over RAC channel counts and outlier strengths, both RAC operand forms.

The GPU's Y_RAC and reference each carry only binary32 accumulation error
(below 1e-6 of ||Y||), so its err(k) agrees with the oracle's binary64 value
to within 1e-5 absolute plus 1e-3 relative."""
import numpy as np
import pytest
import torch

from oracle.layer_error import rac_layer_error
from quantization_nvfp4_quantize_b200 import workloads as wl
from quantization_nvfp4_quantize_b200.sweep import LayerErrorProbe, rac_channels

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("alpha", [1.0, 20.0])
@pytest.mark.parametrize("mode", ["bf16", "nvfp4"])
def test_layer_error_matches_oracle(cuda, alpha, mode):
    T, K, N = 384, 2048, 256
    x = wl.outlier_activations(T, K, alpha, 7).to(cuda)
    w = wl.dense_weight(N, K, 7).to(cuda)
    ks = [rac_channels(p, K) for p in (0, 1, 10, 50, 100)]
    got = LayerErrorProbe(w, T).errors(x, ks, mode)
    want = rac_layer_error(_bits(x), _bits(w), ks, mode)
    for k, g, e in zip(ks, got, want):
        assert abs(g - e) <= 1e-5 + 1e-3 * e, (k, g, e)
    # more compensated channels, less error (up to the rounding of rho)
    assert got[-1] < got[2] < got[0]


def test_layer_error_reference_is_exact_product(cuda):
    """The reference X What^T from the BF16 GEMM of e2m1*sf matches the
    oracle's binary64 product to binary32 accumulation accuracy."""
    import oracle
    T, K, N = 200, 1024, 512
    x = wl.outlier_activations(T, K, 5.0, 2).to(cuda)
    w = wl.dense_weight(N, K, 2).to(cuda)
    yref = LayerErrorProbe(w, T).reference(x).cpu().numpy()
    want = oracle.bf16_to_f32(_bits(x)).astype(np.float64) @ oracle.quantize(_bits(w)).xhat.astype(np.float64).T
    assert np.linalg.norm(yref - want) <= 1e-6 * np.linalg.norm(want)
