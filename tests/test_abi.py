"""The C-ABI library builds, loads, exports every symbol its header declares,
and rejects bad arguments synchronously (no GPU needed)."""
import ctypes
import os
import re

import pytest

from quantization_nvfp4_quantize_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)
    return names


def test_header_declares_entry_points():
    names = declared_symbols()
    for n in ["nvfp4_quantize", "nvfp4_qdq_weights", "moe_w4a4_grouped_gemm_rac", "moe_route",
              "nvfp4_gather_weight_channels"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert name in _lib.SIGNATURES, f"binding lacks {name}"


def test_version_and_workspace_sizes():
    lib = _lib.load()
    assert lib.nvfp4_version() >= 100
    assert lib.nvfp4_quantize_workspace_size(4096, 2048) > 2048 * 8
    assert lib.nvfp4_quantize_workspace_size(-1, 64) == 0
    assert lib.moe_route_workspace_size(16, 128) >= 512


def _status(fn, *args):
    return fn(*args)


def test_argument_errors_are_synchronous():
    lib = _lib.load()
    # null input
    st = lib.nvfp4_quantize(None, 4, 64, 64, None, None, None, None, None, 1, 4, None, None, None, 0, 0, None, None,
                            None, None, 0, None)
    assert st == 1 and b"required" in lib.nvfp4_last_error_string()
    fake = ctypes.c_void_p(0x10000)          # never dereferenced: rejected before any launch
    # K not a multiple of 64
    st = lib.nvfp4_quantize(fake, 4, 48, 48, None, None, None, fake, None, 1, 4, fake, fake, None, 0, 0, None, None,
                            None, fake, 1 << 20, None)
    assert st == 3
    # misaligned pointer
    st = lib.nvfp4_quantize(ctypes.c_void_p(0x10008), 4, 64, 64, None, None, None, fake, None, 1, 4, fake, fake, None,
                            0, 0, None, None, None, fake, 1 << 20, None)
    assert st == 2
    # rac_k too large
    st = lib.nvfp4_quantize(fake, 4, 64, 64, None, None, None, fake, None, 1, 4, fake, fake, fake, 65, 128, fake, fake,
                            None, fake, 1 << 20, None)
    assert st == 3
    # GEMM shape errors
    args = [fake, fake, fake, 128, fake, fake, fake, 256, 256, 1, fake, 128, 0, None, None, 0, fake, fake, fake, 256,
            None, None, None]
    bad_k = list(args)
    bad_k[8] = 320
    assert lib.moe_w4a4_grouped_gemm_rac(*bad_k) == 3
    bad_e = list(args)
    bad_e[9] = 300
    assert lib.moe_w4a4_grouped_gemm_rac(*bad_e) == 3
    bad_epi = list(args)
    bad_epi[15] = 7
    assert lib.moe_w4a4_grouped_gemm_rac(*bad_epi) == 1
    bad_align = list(args)
    bad_align[11] = 64
    assert lib.moe_w4a4_grouped_gemm_rac(*bad_align) == 1
    pair_rows = list(args)
    pair_rows[11] = 256                      # M_pad_max (128) is not a multiple of 256
    assert lib.moe_w4a4_grouped_gemm_rac(*pair_rows) == 3
    # BF16 grouped GEMM (W4A16) and the bf16 row gather
    bargs = [fake, 256, 128, fake, 256, 256, 1, fake, 128, 0, fake, None, fake, 256, None, None, None]
    bad = list(bargs)
    bad[5] = 96                              # K not a multiple of 64
    assert lib.moe_bf16_grouped_gemm(*bad) == 3
    bad = list(bargs)
    bad[1] = 100                             # lda not a multiple of 8
    assert lib.moe_bf16_grouped_gemm(*bad) == 2
    bad = list(bargs)
    bad[9] = 2                               # scatter-add without row_gate
    assert lib.moe_bf16_grouped_gemm(*bad) == 1
    assert lib.moe_gather_rows_bf16(fake, 4, 64, 64, fake, 0, fake, 64, 16, None) == 1
    assert lib.moe_gather_rows_bf16(fake, 4, 60, 64, fake, 2, fake, 64, 16, None) == 2
    # routing
    assert lib.moe_route(fake, 16, 300, 2, fake, fake, 128, fake, fake, fake, fake, 1 << 20, fake, 4096, None) == 3
    assert lib.moe_route(fake, 16, 8, 2, fake, fake, 128, fake, fake, fake, fake, 128, fake, 4096, None) == 1
    assert lib.moe_route(fake, 16, 8, 2, fake, fake, 100, fake, fake, fake, fake, 1 << 20, fake, 4096, None) == 1


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        _lib.load()


def test_api_rejects_non_cuda_tensors():
    """The binding has no CPU path: host tensors are refused with a clear error."""
    import torch
    from quantization_nvfp4_quantize_b200 import api
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA tensors only"):
        api.quantize(x)
