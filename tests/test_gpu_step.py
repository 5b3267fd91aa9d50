"""The W4A4 linear layer's step exactly as the benchmark launches it, at the
benchmark's shape: quantize_bf16_to_nvfp4 of the BF16 activations into
device buffers, then w4a4_gemm on the same stream (gemm_fp4.rs, the
`quantize_bf16_to_nvfp4` launcher followed by `w4a4_gemm`), inputs already on
the device.  Two steps run back to back, so the second quantiser also follows
a GEMM.  The activation codes and scales must equal the oracle's bit for bit;
sampled output rows must be within the product tolerance of the oracle on
those codes."""
import numpy as np
import pytest
import torch

import int8_gemm_gemv_b200 as bsq
import oracle
from int8_gemm_gemv_b200 import synth
from gpu_helpers import bf16_out, check_tol, empty, host, to_dev

pytestmark = pytest.mark.gpu


def test_w4a4_step_launch_sequence_full_size():
    m, n, k = 4096, 17408, 5120
    a_bf, w_bf = synth.w4a4_inputs(m, n, k, seed=0, heavy_tailed=True)
    a2_bf = synth.student_t_bf16((m, k), 4.0, 1, 1, outlier_frac=0.01, outlier_scale=20.0)
    sb2 = float(np.float32(oracle.amax_bf16(w_bf)) / np.float32(6 * 448))
    wp, wsf = oracle.quant_nvfp4(w_bf, sb2)
    wpd, wsfd = to_dev(wp), to_dev(wsf)
    stream = torch.cuda.current_stream()
    ins = [to_dev(a_bf), to_dev(a2_bf)]
    aps = [empty((m, k // 2), torch.uint8) for _ in ins]
    asfs = [empty((m, k // 16), torch.uint8) for _ in ins]
    outs = [bf16_out((m, n)) for _ in ins]
    torch.cuda.synchronize()
    n0 = bsq.debug_launch_count()
    for a, ap, asf, out in zip(ins, aps, asfs, outs):
        bsq.quantize_bf16_to_nvfp4(a, ap, asf, 1.0, m, k, stream)
        bsq.w4a4_gemm(ap, asf, wpd, wsfd, out, 1.0, sb2, m, n, k, stream)
    torch.cuda.synchronize()
    assert bsq.debug_launch_count() - n0 == 4
    assert bsq.debug_take_timeouts() == 0
    g = np.random.default_rng(7)
    for src, ap, asf, out in zip((a_bf, a2_bf), aps, asfs, outs):
        op, osf = oracle.quant_nvfp4(src, 1.0)
        assert np.array_equal(host(ap), op) and np.array_equal(host(asf), osf)
        rows = np.unique(np.concatenate([[0, 255, 256, m - 1], g.integers(0, m, 8)]))
        ob, _, ab = oracle.w4a4_gemm(op, osf, wp, wsf, 1.0, sb2, rows=rows)
        check_tol(host(out, np.uint16)[rows], ob, ab, "w4a4 step 4096x17408x5120")
