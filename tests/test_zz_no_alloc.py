"""The allocation-free W4A8 prefill entry point.

int8_w4a8_prefill_noalloc serves callers that cannot allocate device memory
(their device memory belongs to another allocator, or they may not call
cudaMalloc on this path), so it keeps the activation scratch in a fixed
array inside the library instead of taking scratch buffers.  This test calls
it through the C ABI twice in a row, with different shapes so that contents
left in the shared array by the first call would show in the second, and
checks each result against the scratch-taking entry point int8_w4a8_prefill
within the tolerance the parity tests use.  The file is named to be
collected last; it passes alone in a fresh process and after the other
tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import int8_gemm_gemv_b200 as bsq
import oracle
from int8_gemm_gemv_b200 import synth
from gpu_helpers import bf16_out, check_tol, empty, host, to_dev

pytestmark = pytest.mark.gpu


def _inputs(m, n, k, seed):
    a_bf, _ = synth.w4a8_inputs(m, n, k, seed=seed)
    w = synth.uniform_int8((n, k), seed, 50)
    sw = synth.uniform_f32((n, k // 32), seed, 51, 1e-4, 1e-3)
    return a_bf, w, sw


def _with_scratch(a, w, sw, m, n, k):
    out = bf16_out((m, n))
    bsq.int8_w4a8_prefill(a, w, sw, empty((m, k), torch.int8), empty((m, k // 32), torch.float32), out, m, n, k)
    return out


def _noalloc_c_abi(a, w, sw, m, n, k):
    out = bf16_out((m, n))
    fn = bsq.lib().int8_w4a8_prefill_noalloc
    st = fn(ctypes.c_void_p(a.data_ptr()), ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(sw.data_ptr()),
            ctypes.c_void_p(out.data_ptr()), m, n, k, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == bsq.BSQ_OK, bsq.status_string(st)
    return out


def test_noalloc_prefill_matches_scratch_prefill_two_calls():
    for (m, n, k, seed) in ((96, 256, 512, 7), (40, 136, 1024, 8)):
        a_bf, w, sw = _inputs(m, n, k, seed)
        a, wd, swd = to_dev(a_bf), to_dev(w), to_dev(sw)
        ref = _with_scratch(a, wd, swd, m, n, k)
        got = _noalloc_c_abi(a, wd, swd, m, n, k)
        torch.cuda.synchronize()
        # the tolerance reference magnitude sum|a*w| comes from the oracle
        aq, sa = oracle.quant_act_int8_per32(a_bf)
        _, _, abssum = oracle.int8_blockscaled_gemm(aq, w, sa, sw)
        check_tol(host(got, np.uint16), host(ref, np.uint16), abssum, f"noalloc prefill {m}x{n}x{k}")
    assert bsq.debug_take_timeouts() == 0


def test_noalloc_prefill_rejects_sizes_beyond_its_scratch():
    n0 = bsq.debug_launch_count()
    fn = bsq.lib().int8_w4a8_prefill_noalloc
    big_m, k = 40961, 1024  # m * k = 41,944,064 > 41,943,040
    st = fn(ctypes.c_void_p(16), ctypes.c_void_p(32), ctypes.c_void_p(48), ctypes.c_void_p(64), big_m, 8, k,
            ctypes.c_void_p(0))
    assert st == bsq.BSQ_ERR_UNSUPPORTED
    assert bsq.debug_launch_count() == n0
