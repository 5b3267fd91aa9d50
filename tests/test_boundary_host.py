"""Host-only tests of the C ABI: the library loads without a GPU, exports every
entry point include/bsq.h declares, validates before it launches, and passes
an already row-wise FP8 weight through untouched with no GPU work
(dispatch_proj_rowwise.rs, its passthrough unit tests).  No GPU needed: every
call here is rejected (or passed through) before any CUDA call."""
import ctypes
import os
import re

import pytest

import int8_gemm_gemv_b200 as bsq
from int8_gemm_gemv_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# fake, never dereferenced device addresses
A16 = 0x7F0000000000
A16b = 0x7F0000100000
A16c = 0x7F0000200000
A16d = 0x7F0000300000
A16e = 0x7F0000400000
ODD = 0x7F0000000001


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "bsq.h")).read()
    return re.findall(r"^BSQ_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)


def test_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 15
    L = ctypes.CDLL(bsq.library_path())
    for n in names:
        assert hasattr(L, n), n


def test_status_strings():
    assert bsq.status_string(0) == "BSQ_OK"
    for s in range(1, 5):
        assert bsq.status_string(s).startswith("BSQ_ERR_")
    assert "unknown" in bsq.status_string(99)


def _status(fn, *args):
    return getattr(bsq.lib(), fn)(*args)


def test_validation_launches_nothing():
    n0 = bsq.debug_launch_count()
    L = bsq.lib
    cases = [
        # (expected, fn, args)
        (1, "quantize_bf16_to_nvfp4", (A16, A16b, A16c, 1.0, 4, 24, 0)),        # k % 16
        (1, "quantize_bf16_to_nvfp4", (A16, A16b, A16c, 0.0, 4, 32, 0)),        # scale2 <= 0
        (1, "quantize_bf16_to_nvfp4", (A16, A16b, A16c, float("inf"), 4, 32, 0)),
        (1, "quantize_bf16_to_nvfp4", (None, A16b, A16c, 1.0, 4, 32, 0)),       # NULL
        (1, "quantize_bf16_to_nvfp4", (A16, A16b, A16c, 1.0, -1, 32, 0)),       # m < 0
        (2, "quantize_bf16_to_nvfp4", (ODD, A16b, A16c, 1.0, 4, 32, 0)),        # misaligned
        (0, "quantize_bf16_to_nvfp4", (None, None, None, 1.0, 0, 32, 0)),       # empty
        (1, "quantize_bf16_to_nvfp4_devscale", (A16, A16b, A16c, None, None, 4, 32, 0)),   # amax NULL
        (1, "quantize_bf16_to_nvfp4_devscale", (A16, A16b, A16c, A16d, None, 4, 24, 0)),   # k % 16
        (2, "quantize_bf16_to_nvfp4_devscale", (A16, A16b, A16c, ODD, None, 4, 32, 0)),    # amax odd
        (0, "quantize_bf16_to_nvfp4_devscale", (None, None, None, None, None, 0, 32, 0)),  # empty
        (1, "w4a4_gemm_devscale", (A16, A16b, A16c, A16d, A16e, 1.0, None, 16, 16, 256, 0)),
        (2, "w4a4_gemm_devscale", (A16, A16b, A16c, A16d, A16e, 1.0, ODD, 16, 16, 256, 0)),
        (3, "w4a4_gemm_devscale", (A16, A16b, A16c, A16d, A16e, 1.0, A16, 16, 16, 272, 0)),
        (0, "w4a4_gemm_devscale", (A16, A16b, A16c, A16d, A16e, 1.0, None, 0, 16, 256, 0)),
        (1, "w4a4_gemm", (A16, A16b, A16c, A16d, A16e, 1.0, 1.0, 16, 16, 40, 0)),
        (3, "w4a4_gemm", (A16, A16b, A16c, A16d, A16e, 1.0, 1.0, 16, 16, 272, 0)),  # k % 256
        (2, "w4a4_gemm", (A16, A16b, A16c, A16d, ODD, 1.0, 1.0, 16, 16, 256, 0)),
        (1, "w4a4_gemm", (A16, A16b, A16c, A16d, A16e, float("nan"), 1.0, 16, 16, 256, 0)),
        (0, "w4a4_gemm", (A16, A16b, A16c, A16d, A16e, 1.0, 1.0, 0, 16, 256, 0)),
        (1, "fp8_gemv_rowscale", (A16, A16b, A16c, A16d, 0, 64, 64, 0)),         # m = 0
        (1, "fp8_gemv_rowscale", (A16, A16b, A16c, A16d, 17, 64, 64, 0)),        # m = 17
        (1, "fp8_gemv_rowscale", (A16, A16b, A16c, A16d, 8, 64, 72, 0)),         # k % 16
        (2, "fp8_gemv_rowscale", (A16, ODD, A16c, A16d, 8, 64, 64, 0)),
        (0, "fp8_gemv_rowscale", (A16, A16b, A16c, A16d, 8, 0, 64, 0)),
        (1, "fp8_gemv_blockscaled", (A16, A16b, A16c, A16d, 0, 128, 128, 0)),   # m = 0
        (1, "fp8_gemv_blockscaled", (A16, A16b, A16c, A16d, 4, 128, 120, 0)),   # k % 16
        (3, "fp8_gemv_blockscaled", (A16, A16b, A16c, A16d, 4, 100, 128, 0)),   # n % 128
        (3, "fp8_gemv_blockscaled", (A16, A16b, A16c, A16d, 4, 128, 144, 0)),   # k % 128
        (2, "fp8_gemv_blockscaled", (A16, A16b, A16c, ODD, 4, 128, 128, 0)),    # out odd
        (0, "fp8_gemv_blockscaled", (A16, A16b, A16c, A16d, 4, 0, 128, 0)),
        (1, "quant_rowwise_fp8", (A16, A16b, A16c, 4, 40, 0)),
        (1, "quant_blockfp8", (A16, A16b, A16c, 100, 128, 0)),
        (1, "requant_w_nvfp4_int8", (A16, A16b, 1.0, A16c, A16d, 4, 48, 0)),
        (1, "requant_w_nvfp4_int8", (A16, A16b, -1.0, A16c, A16d, 4, 64, 0)),
        (1, "quant_act_int8_per32", (A16, A16b, A16c, 4, 48, 0)),
        (1, "int8_blockscaled_gemm", (A16, A16b, A16c, A16d, A16e, 4, 4, 48, 0)),
        (3, "int8_blockscaled_gemm", (A16, A16b, A16c, A16d, A16e, 4, 4, 96, 0)),  # k % 128
        (2, "int8_blockscaled_gemm", (A16, A16b, A16c, A16d, ODD, 4, 4, 128, 0)),
        (3, "int8_w4a8_prefill", (A16, A16b, A16c, A16d, A16e, A16, 4, 4, 96, 0)),
        (1, "fp8_gemm_rowscale", (A16, A16b, A16c, A16d, A16e, 4, 4, 24, 0)),
        (2, "fp8_gemm_rowscale", (ODD, A16b, A16c, A16d, A16e, 4, 4, 32, 0)),
        (0, "fp8_gemm_rowscale", (A16, A16b, A16c, A16d, A16e, 4, 0, 32, 0)),
        (1, "bsq_amax_bf16", (A16, 10, None, 0)),
    ]
    for expected, fn, args in cases:
        assert _status(fn, *args) == expected, (fn, args)
    assert bsq.debug_launch_count() == n0


def _requant(tag, w, s, n, k, wo, so):
    wu, su = ctypes.c_void_p(), ctypes.c_void_p()
    st = bsq.lib().requant_blockfp8_to_rowwise(tag, w, s, n, k, wo, so, ctypes.byref(wu), ctypes.byref(su), 0)
    return st, wu.value, su.value


def test_rowwise_weight_passes_through_verbatim():
    """An already row-wise FP8 weight comes back as its own pointers, with no
    launch and no output written (w_out/scale_out may even be NULL)."""
    n0 = bsq.debug_launch_count()
    st, wu, su = _requant(bsq.BSQ_FP8_PER_ROW, 0xBEEF0, 0x5CA1E0, 4096, 5120, None, None)
    assert st == bsq.BSQ_OK and (wu, su) == (0xBEEF0, 0x5CA1E0)
    # the binding returns the same pair
    assert bsq.requant_blockfp8_to_rowwise(bsq.BSQ_FP8_PER_ROW, 0xBEEF0, 0x5CA1E0, 4096, 5120, None, None,
                                           stream=0) == (0xBEEF0, 0x5CA1E0)
    assert bsq.debug_launch_count() == n0


def test_other_formats_are_not_passed_through():
    n0 = bsq.debug_launch_count()
    for tag in (bsq.BSQ_FP8_SINGLE_SCALE, bsq.BSQ_BF16, bsq.BSQ_NVFP4):
        st, wu, su = _requant(tag, A16, A16b, 256, 256, A16c, A16d)
        assert st == bsq.BSQ_ERR_UNSUPPORTED and wu is None and su is None
    st, _, _ = _requant(77, A16, A16b, 256, 256, A16c, A16d)
    assert st == bsq.BSQ_ERR_INVALID_ARG
    # block-scaled with a grid the shape does not fit: rejected before launch
    st, wu, _ = _requant(bsq.BSQ_FP8_BLOCK_SCALED, A16, A16b, 200, 256, A16c, A16d)
    assert st == bsq.BSQ_ERR_INVALID_ARG and wu is None
    st, _, _ = _requant(bsq.BSQ_FP8_BLOCK_SCALED, A16, A16b, 256, 256, ODD, A16d)
    assert st == bsq.BSQ_ERR_MISALIGNED
    assert bsq.debug_launch_count() == n0


def test_binding_raises_on_error_status():
    with pytest.raises(bsq.BsqError) as e:
        bsq.fp8_gemv_rowscale(A16, A16b, A16c, A16d, 0, 64, 64, stream=0)
    assert e.value.status == bsq.BSQ_ERR_INVALID_ARG


def test_binding_rejects_host_tensors():
    torch = pytest.importorskip("torch")
    with pytest.raises(ValueError):
        bsq.quant_rowwise_fp8(torch.zeros(4, 16, dtype=torch.bfloat16), A16, A16b, 4, 16, stream=0)


def test_int8_ws_validation():
    L = bsq.lib()
    n0 = bsq.debug_launch_count()
    # NULL workspace, misaligned workspace; nothing launches
    assert L.int8_blockscaled_gemm_ws(A16, A16b, A16c, A16d, A16e, None, 1 << 24, 128, 128, 128, None) == \
        bsq.BSQ_ERR_INVALID_ARG
    assert L.int8_blockscaled_gemm_ws(A16, A16b, A16c, A16d, A16e, A16 + 8, 1 << 24, 128, 128, 128, None) == \
        bsq.BSQ_ERR_MISALIGNED
    # the shape checks of the plain call come first
    assert L.int8_blockscaled_gemm_ws(A16, A16b, A16c, A16d, A16e, A16, 1 << 24, 128, 128, 96, None) == \
        bsq.BSQ_ERR_UNSUPPORTED
    assert L.int8_blockscaled_gemm_ws(A16, A16b, A16c, A16d, A16e, A16, 1 << 24, 0, 128, 128, None) == bsq.BSQ_OK
    assert bsq.debug_launch_count() == n0


def test_int8_workspace_bytes_matches_the_device():
    """One 64 KB piece of FP32 sums plus a 4-byte counter per SM of the
    current device; 0 where there is no device, and the workspace call then
    reports the CUDA failure instead of launching."""
    torch = pytest.importorskip("torch")
    L = bsq.lib()
    got = bsq.int8_gemm_workspace_bytes()
    if torch.cuda.is_available():
        sms = torch.cuda.get_device_properties(0).multi_processor_count
        assert got == sms * (512 * 32 * 4 + 4)
        return
    assert got == 0
    n0 = bsq.debug_launch_count()
    assert L.int8_blockscaled_gemm_ws(A16, A16b, A16c, A16d, A16e, A16, 1 << 24, 128, 128, 128, None) == \
        bsq.BSQ_ERR_CUDA
    assert bsq.debug_launch_count() == n0


def test_noalloc_validation():
    """int8_w4a8_prefill_noalloc checks the shape (including the fixed
    scratch's limit of 41,943,040 activation codes), then its pointers,
    before any CUDA call; nothing launches."""
    fn = bsq.lib().int8_w4a8_prefill_noalloc
    n0 = bsq.debug_launch_count()
    assert fn(A16, A16b, A16c, A16d, -1, 128, 128, None) == bsq.BSQ_ERR_INVALID_ARG
    assert fn(A16, A16b, A16c, A16d, 128, 128, 48, None) == bsq.BSQ_ERR_INVALID_ARG  # K not a multiple of 32
    assert fn(A16, A16b, A16c, A16d, 128, 128, 96, None) == bsq.BSQ_ERR_UNSUPPORTED  # nor of 128
    assert fn(A16, A16b, A16c, A16d, 40961, 8, 1024, None) == bsq.BSQ_ERR_UNSUPPORTED  # one row past the scratch
    # exactly at the limit the size passes, so the NULL input is what fails
    assert fn(None, A16b, A16c, A16d, 40960, 8, 1024, None) == bsq.BSQ_ERR_INVALID_ARG
    assert fn(A16, A16b, A16c, A16d, 0, 128, 128, None) == bsq.BSQ_OK
    assert fn(A16, A16b, A16c, None, 128, 128, 128, None) == bsq.BSQ_ERR_INVALID_ARG
    assert fn(ODD, A16b, A16c, A16d, 128, 128, 128, None) == bsq.BSQ_ERR_MISALIGNED
    assert fn(A16, A16b, A16c + 4, A16d, 128, 128, 128, None) == bsq.BSQ_ERR_MISALIGNED
    assert bsq.debug_launch_count() == n0


def test_stream_read_validation():
    """The plain-read probe behind the benchmark's floor rows: mode 0 or 1,
    whole 16-byte units, a 16-byte aligned source and a 4-byte aligned sink."""
    fn = bsq.lib().bsq_debug_stream_read
    n0 = bsq.debug_launch_count()
    assert fn(A16, 1024, A16b, 2, None) == bsq.BSQ_ERR_INVALID_ARG
    assert fn(A16, 1000, A16b, 0, None) == bsq.BSQ_ERR_INVALID_ARG
    assert fn(A16, 0, A16b, 0, None) == bsq.BSQ_OK
    assert fn(None, 1024, A16b, 0, None) == bsq.BSQ_ERR_INVALID_ARG
    assert fn(A16, 1024, None, 1, None) == bsq.BSQ_ERR_INVALID_ARG
    assert fn(A16 + 8, 1024, A16b, 0, None) == bsq.BSQ_ERR_MISALIGNED
    assert fn(A16, 1024, A16b + 2, 0, None) == bsq.BSQ_ERR_MISALIGNED
    assert bsq.debug_launch_count() == n0
