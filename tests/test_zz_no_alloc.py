"""The allocation-free W4A8 prefill entry point.

int8_w4a8_prefill_noalloc serves callers that cannot allocate device memory:
code whose device memory all belongs to another allocator (a framework's
caching allocator, a fixed arena), plug-ins with no allocation API at hand,
and latency-critical paths that must not call cudaMalloc, which can
synchronise the device.  It keeps the activation scratch in a fixed array
inside the library instead of taking scratch buffers.

The test calls it through the C ABI twice in a row, with different shapes so
that contents left in the shared array by the first call would show in the
second.  Each result must be bit-identical to the scratch-taking entry point
int8_w4a8_prefill (both run the same two kernels on the same inputs), and
within the product tolerance of the CPU oracle evaluated on the oracle's own
per-32 activation codes.  Free device memory must not change across a call
(the first call, which loads the array's module and looks up its address,
comes before the measured one).  The file is named to be collected last; it
passes alone in a fresh process and after the other tests.
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


def _noalloc_c_abi(a, w, sw, out, m, n, k):
    fn = bsq.lib().int8_w4a8_prefill_noalloc
    st = fn(ctypes.c_void_p(a.data_ptr()), ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(sw.data_ptr()),
            ctypes.c_void_p(out.data_ptr()), m, n, k, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == bsq.BSQ_OK, bsq.status_string(st)


def test_noalloc_prefill_matches_scratch_prefill_two_calls():
    shapes = ((96, 256, 512, 7), (40, 136, 1024, 8))
    # a first call loads the scratch array's module and looks up its device
    # address; the calls checked below then must not change free memory
    a0, w0, sw0 = (to_dev(x) for x in _inputs(8, 128, 128, 9))
    _noalloc_c_abi(a0, w0, sw0, bf16_out((8, 128)), 8, 128, 128)
    torch.cuda.synchronize()
    for (m, n, k, seed) in shapes:
        a_bf, w, sw = _inputs(m, n, k, seed)
        a, wd, swd = to_dev(a_bf), to_dev(w), to_dev(sw)
        ref = _with_scratch(a, wd, swd, m, n, k)
        got = bf16_out((m, n))
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        _noalloc_c_abi(a, wd, swd, got, m, n, k)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free0, "the no-alloc call changed free device memory"
        g, r = host(got, np.uint16), host(ref, np.uint16)
        assert np.array_equal(g, r), f"noalloc differs from int8_w4a8_prefill at {m}x{n}x{k}"
        aq, sa = oracle.quant_act_int8_per32(a_bf)
        ob, _, abssum = oracle.int8_blockscaled_gemm(aq, w, sa, sw)
        check_tol(g, ob, abssum, f"noalloc prefill {m}x{n}x{k}")
    assert bsq.debug_take_timeouts() == 0


def test_noalloc_prefill_rejects_sizes_beyond_its_scratch():
    n0 = bsq.debug_launch_count()
    fn = bsq.lib().int8_w4a8_prefill_noalloc
    big_m, k = 40961, 1024  # m * k = 41,944,064 > 41,943,040
    st = fn(ctypes.c_void_p(16), ctypes.c_void_p(32), ctypes.c_void_p(48), ctypes.c_void_p(64), big_m, 8, k,
            ctypes.c_void_p(0))
    assert st == bsq.BSQ_ERR_UNSUPPORTED
    assert bsq.debug_launch_count() == n0
