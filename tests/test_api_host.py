"""Host-side tests of the C-ABI library: it loads, exports every symbol the
header declares, and its argument validation refuses bad calls before any
launch (no GPU needed: every call here fails validation or is a no-op)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "vlaq.h")
GOLDEN = os.path.join(ROOT, "tests", "golden", "k3420_rejection.txt")


@pytest.fixture(scope="module")
def vq():
    from conftest import build_library
    build_library()
    import vlaq_quantize_act_b200 as vq
    return vq


def _declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"VLAQ_API\s+[\w\s\*]+?\b(vlaq_\w+)\s*\(", text)))


def test_header_declares_entry_points():
    names = _declared_symbols()
    for required in ("vlaq_quantize_weight_nvfp4", "vlaq_quantize_act_nvfp4", "vlaq_linear_nvfp4",
                     "vlaq_linear_fp8", "vlaq_quantize_weight_fp8", "vlaq_quantize_act_fp8"):
        assert required in names


def test_library_exports_every_declared_symbol(vq):
    lib = ctypes.CDLL(vq.LIB_PATH)
    for name in _declared_symbols():
        assert hasattr(lib, name), name


def test_version_and_size_helpers(vq):
    assert vq.vlaq_version() >= 100
    assert vq.vlaq_nvfp4_code_pitch(3584) == 1792
    assert vq.vlaq_nvfp4_code_pitch(3424) == 54 * 32
    assert vq.vlaq_nvfp4_scale_bytes(1, 3584) == 128 * 224
    assert vq.vlaq_nvfp4_scale_bytes(1024, 18944) == 1024 * 1184
    assert vq.vlaq_nvfp4_scale_bytes(130, 336) == 256 * 24


FAKE = 0x10000  # never dereferenced: validation fails (or M == 0) before any use


def test_k3420_rejected_with_page_arithmetic(vq):
    rec = {}
    for line in open(GOLDEN):
        if line.strip() and not line.startswith("#"):
            k, v = line.strip().split(" ", 1)
            rec[k] = v
    K = int(rec["K"])
    for call in (
        lambda: vq.vlaq_quantize_act_nvfp4(FAKE, 4, K, None, 1e-6, 0, FAKE, FAKE, FAKE),
        lambda: vq.vlaq_quantize_weight_nvfp4(FAKE, 64, K, 0, FAKE, FAKE, FAKE),
        lambda: vq.vlaq_linear_nvfp4(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 64, K),
    ):
        with pytest.raises(vq.VlaqError) as ei:
            call()
        assert ei.value.status == 2  # VLAQ_ERR_SHAPE
        assert rec["message_contains"] in ei.value.message
    assert rec["message_contains"] in vq.vlaq_last_error()


def test_fp8_k_rejections(vq):
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_act_fp8(FAKE, 4, 100, None, 1e-6, 0, FAKE, FAKE)
    assert ei.value.status == 2 and "100 / 16 = 6.25" in ei.value.message
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_linear_fp8(FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 64, 8)
    assert ei.value.status == 2


def test_hadamard_needs_k_multiple_of_64(vq):
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_act_nvfp4(FAKE, 4, 336, None, 1e-6, vq.F_HADAMARD64, FAKE, FAKE, FAKE)
    assert ei.value.status == 2 and "336 / 64 = 5.25" in ei.value.message


def test_null_and_misaligned_pointers(vq):
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_act_nvfp4(None, 4, 256, None, 1e-6, 0, FAKE, FAKE, FAKE)
    assert ei.value.status == 1
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_act_nvfp4(FAKE + 8, 4, 256, None, 1e-6, 0, FAKE, FAKE, FAKE)
    assert ei.value.status == 3
    with pytest.raises(vq.VlaqError) as ei:  # RMSNorm without a gain
        vq.vlaq_quantize_act_nvfp4(FAKE, 4, 256, None, 1e-6, vq.F_RMSNORM, FAKE, FAKE, FAKE)
    assert ei.value.status == 1
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_linear_nvfp4(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE, 4, 64, 256)
    assert ei.value.status == 3


def test_bad_flags_and_sizes(vq):
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_act_nvfp4(FAKE, 4, 256, None, 1e-6, 0x80, FAKE, FAKE, FAKE)
    assert ei.value.status == 1
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_act_nvfp4(FAKE, -1, 256, None, 1e-6, 0, FAKE, FAKE, FAKE)
    assert ei.value.status == 1
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_act_nvfp4(FAKE, 4, 65536, None, 1e-6, 0, FAKE, FAKE, FAKE)
    assert ei.value.status == 2
    with pytest.raises(vq.VlaqError) as ei:  # N not a multiple of 8
        vq.vlaq_linear_nvfp4(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 60, 256)
    assert ei.value.status == 2
    with pytest.raises(vq.VlaqError) as ei:  # weight rows must be >= 1
        vq.vlaq_quantize_weight_nvfp4(FAKE, 0, 256, 0, FAKE, FAKE, FAKE)
    assert ei.value.status == 2


def test_m_zero_is_a_noop(vq):
    vq.vlaq_quantize_act_nvfp4(None, 0, 256, None, 1e-6, 0, None, None, None)
    vq.vlaq_quantize_act_fp8(None, 0, 256, None, 1e-6, 0, None, None)
    vq.vlaq_linear_nvfp4(None, None, None, None, None, None, None, None, 0, 64, 256)
    vq.vlaq_linear_fp8(None, None, None, None, None, None, 0, 64, 256)
    assert vq.vlaq_last_error() == ""


def test_no_device_is_an_error_not_a_fallback(vq):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_act_nvfp4(FAKE, 4, 256, None, 1e-6, 0, FAKE, FAKE, FAKE)
    assert ei.value.status in (4, 5)


def test_scales_to_rowmajor_refuses_bad_k(vq):
    with pytest.raises(vq.VlaqError) as ei:
        vq._check(vq._lib.vlaq_scales_to_rowmajor(16, 16, 4, 3420, None))
    assert ei.value.status == 2 and "3420 / 16 = 213.75" in ei.value.message


@pytest.mark.parametrize("g", [0.0, -1.0, float("nan"), float("inf"), -0.0])
def test_static_scale_must_be_finite_and_positive(vq, g):
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_act_nvfp4_static(FAKE, 4, 256, None, None, 1e-6, 0, g, FAKE, FAKE, FAKE)
    assert ei.value.status == 1 and "g_static" in ei.value.message


def test_static_smoothing_flags_need_factors(vq):
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_act_nvfp4_static(FAKE, 4, 256, None, None, 1e-6, vq.F_SMOOTH_MUL, 1.0, FAKE, FAKE, FAKE)
    assert ei.value.status == 1


def test_int8_entry_points_validate_before_the_device(vq):
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_act_int8(FAKE, 4, 3420, None, 1e-6, 0, FAKE, FAKE)
    assert ei.value.status == 2
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_quantize_weight_int8(FAKE, 4, 96, vq.F_HADAMARD64, FAKE, FAKE)
    assert ei.value.status == 2
    with pytest.raises(vq.VlaqError) as ei:
        vq.vlaq_linear_int8(FAKE, FAKE, FAKE, FAKE, None, FAKE, 4, 60, 256)
    assert ei.value.status == 2
    vq.vlaq_quantize_act_int8(None, 0, 256, None, 1e-6, 0, None, None)
    vq.vlaq_linear_int8(None, None, None, None, None, None, 0, 64, 256)
    assert vq.vlaq_last_error() == ""
