"""nvfp4_quantize_noalloc, the entry point for callers that cannot allocate
device memory when they call in (it keeps its scratch in a fixed array inside
the library), must give the same results as nvfp4_quantize with a caller
workspace.  Two calls in a row, the first with a larger tensor maximum than
the second, so that scratch left over from the first call would show up in
the second.  This file is collected last on purpose."""
import numpy as np
import pytest
import torch

from quantization_nvfp4_quantize_b200 import _lib, api

pytestmark = pytest.mark.gpu

SCORE_RTOL = 5.5e-7     # the tolerance the quantize parity tests use


def _noalloc(x, rac_k, rac_ld, dev):
    lib = _lib.load()
    M, K = x.shape
    out = api.Quantized(codes=torch.empty(M, K // 2, dtype=torch.uint8, device=dev),
                        scales=torch.empty(api.scale_bytes(M, K), dtype=torch.uint8, device=dev),
                        s_t=torch.empty(1, dtype=torch.float32, device=dev),
                        score=torch.empty(K, dtype=torch.float64, device=dev),
                        sel=torch.empty(rac_k, dtype=torch.int32, device=dev),
                        r_sel=torch.empty(M, rac_ld, dtype=torch.bfloat16, device=dev))
    p = api._p
    st = lib.nvfp4_quantize_noalloc(p(x), M, K, x.stride(0), None, None, None, p(out.s_t), None, 1, M, p(out.codes),
                                    p(out.scales), p(out.score), rac_k, rac_ld, p(out.sel), p(out.r_sel), None,
                                    api._stream(dev))
    _lib.check(st)
    return out


def _valid_scales(buf, M, K):
    """Scale bytes of rows < M, read through the tensor-core scale layout
    (512-byte atoms of 128 rows x 4 scale columns)."""
    r = np.arange(M)[:, None]
    c = np.arange(K // 16)[None, :]
    off = ((r // 128) * (K // 64) + c // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + c % 4
    return buf.cpu().numpy()[off]


def test_noalloc_matches_workspace_entry_point_twice(cuda):
    lib = _lib.load()
    assert lib.nvfp4_quantize_noalloc_max_scratch() >= lib.nvfp4_quantize_workspace_size(16384, 4096)
    g = torch.Generator().manual_seed(2024)
    cases = [(1000, 2048, 64, 30.0), (300, 768, 32, 1.0)]
    for M, K, k, outlier in cases:
        x = torch.randn(M, K, generator=g)
        x[:, 5] *= outlier
        x = x.to(torch.bfloat16).to(cuda)
        got = _noalloc(x, k, 64, cuda)
        ref = api.quantize(x, rac_k=k, rac_ld=64, want_score=True)
        torch.cuda.synchronize()
        assert got.s_t.item() == ref.s_t.item()
        assert torch.equal(got.codes, ref.codes)
        # only the M real rows are defined; padding rows up to 128 are never written
        assert np.array_equal(_valid_scales(got.scales, M, K), _valid_scales(ref.scales, M, K))
        np.testing.assert_allclose(got.score.cpu().numpy(), ref.score.cpu().numpy(), rtol=SCORE_RTOL, atol=0)
        assert torch.equal(got.sel, ref.sel[:k])
        assert torch.equal(got.r_sel.view(torch.int16), ref.r_sel.view(torch.int16))
