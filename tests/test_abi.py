"""The C-ABI library loads and exports every entry point include/mxfp8.h
declares (CPU only: no compute call is made); host-side size helpers agree
with the layout definition."""
import ctypes
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(mxfp8_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    from mxfp8_grouped_gemm_quantize_b200 import build
    build.build()
    import mxfp8_grouped_gemm_quantize_b200 as m
    return m.lib()


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("mxfp8_quantize_rowwise", "mxfp8_quantize_colwise", "mxfp8_grouped_gemm_fwd",
              "mxfp8_grouped_gemm_dgrad", "mxfp8_grouped_gemm_wgrad", "mxfp8_get_status"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_python_binding_names_match_the_header():
    import mxfp8_grouped_gemm_quantize_b200 as m
    assert set(m.EXPORTED) == set(_declared())


@pytest.mark.parametrize("R,C,G", [(0, 32, 1), (64, 256, 4), (49152, 2048, 64), (16384, 7168, 32), (1, 32, 1)])
def test_size_helpers_agree_with_the_layout_definition(lib, R, C, G):
    import mxfp8_grouped_gemm_quantize_b200 as m
    assert m.mxfp8_colwise_ld(R, G) == oracle.colwise_ld(R, G)
    assert m.mxfp8_colwise_pitch(R, G) == oracle.colwise_pitch(R, G)
    assert m.mxfp8_rowwise_scale_bytes(R, C, G) == oracle.rowwise_scale_bytes(R, C, G)
    assert m.mxfp8_colwise_scale_bytes(R, C, G) == oracle.colwise_scale_bytes(R, C, G)


def test_status_strings(lib):
    import mxfp8_grouped_gemm_quantize_b200 as m
    for code in range(7):
        assert m.lib().mxfp8_status_string(code)


def test_no_cpu_fallback_without_a_gpu_tensor():
    """The binding only marshals device pointers: host tensors are refused
    loudly, and nothing falls back to a CPU computation."""
    import torch
    import mxfp8_grouped_gemm_quantize_b200 as mx
    x = torch.zeros((64, 64), dtype=torch.bfloat16)
    with pytest.raises(AssertionError, match="CUDA"):
        mx.mxfp8_quantize_rowwise(x)
    with pytest.raises(AssertionError, match="CUDA"):
        mx.mxfp8_quantize_dual(x)


def test_missing_library_is_an_error(monkeypatch, tmp_path):
    import mxfp8_grouped_gemm_quantize_b200 as mx
    monkeypatch.setattr(mx, "_LIB", None)
    monkeypatch.setattr(mx, "LIB_PATH", str(tmp_path / "libmxfp8.so"))
    with pytest.raises(RuntimeError, match="missing"):
        mx.lib()


@pytest.mark.parametrize("C", [32, 64, 96, 1408, 2048, 7168])
def test_ep_record_size_agrees_with_the_format(lib, C):
    import mxfp8_grouped_gemm_quantize_b200 as m
    assert m.mxfp8_ep_record_bytes(C) == oracle.ep_record_bytes(C)
    assert m.mxfp8_ep_record_bytes(C) % 16 == 0 and m.mxfp8_ep_record_bytes(C) >= C + C // 32
    assert lib.mxfp8_ep_record_bytes(0) == 0 and lib.mxfp8_ep_record_bytes(48) == 0   # cols % 32 != 0


def test_ep_plan_workspace_grows_with_tokens_and_ranks(lib):
    w = lib.mxfp8_ep_plan_workspace_bytes
    assert w(0, 1) > 0 and w(0, 1) % 16 == 0
    assert w(4096, 8) >= w(2048, 8) >= w(2048, 2)
    assert w(10, 0) == 0 and w(10, 257) == 0 and w(-1, 2) == 0


def test_tiling_switch_accepts_the_documented_values_only(lib):
    try:
        for cta_pair in (-1, 0, 1):
            for stage_k in (-1, 1, 2):
                assert lib.mxfp8_set_gemm_tiling(cta_pair, stage_k) == 0
        for bad in ((2, -1), (-2, -1), (0, 0), (0, 3), (1, -2)):
            assert lib.mxfp8_set_gemm_tiling(*bad) == 1   # MXF8_ERR_INVALID_ARG
    finally:
        lib.mxfp8_set_gemm_tiling(-1, -1)


def test_argument_errors_are_reported_before_any_device_call(lib):
    """Host-side validation needs no GPU: invalid sizes and null pointers are
    rejected with MXF8_ERR_INVALID_ARG before the library touches a device."""
    assert lib.mxfp8_quantize_rowwise(None, 4, 48, None, 1, None, None, 0, None) == 1      # cols % 32
    assert lib.mxfp8_moe_plan(None, 4, 0, 8, None, None, None, None, 0, None) == 1           # top_k < 1
    assert lib.mxfp8_ep_plan(None, 4, 2, 5, 2, None, None, None, None, None, None, 0, None) == 1   # E % P
    assert lib.mxfp8_ep_pack(None, 4, 48, None, 1, None, None) == 1                            # cols % 32
    assert lib.mxfp8_gather_rows(None, 4, 24, None, 1, None, None) == 1                        # row bytes % 16
