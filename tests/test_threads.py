"""Entry points called from several host threads at once.

The library keeps per-device caches (SM count, kernel attributes, the cluster
occupancy of the W4A4 kernel) and a launch counter; each is set under a lock
or atomically, so concurrent first calls from different threads must neither
fail nor disturb one another.  The CPU test drives the validation paths from
eight threads; the GPU test makes the first calls of one fresh process from
eight threads at once, on separate streams, and checks every result against
the same call made alone."""
import os
import subprocess
import sys
import threading

import pytest

import int8_gemm_gemv_b200 as bsq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
A16 = 0x7F0000000000


def test_validation_from_eight_threads():
    L = bsq.lib()
    n0 = bsq.debug_launch_count()
    errors = []

    def work(tid):
        try:
            for i in range(2000):
                # m outside 1..16, k not a multiple of 16, K % 256 != 0, bad tag
                assert L.fp8_gemv_rowscale(A16, A16, A16, A16, 17, 64, 64, None) == bsq.BSQ_ERR_INVALID_ARG
                assert L.quantize_bf16_to_nvfp4(A16, A16, A16, 1.0, 4, 24, None) == bsq.BSQ_ERR_INVALID_ARG
                assert L.w4a4_gemm(A16, A16, A16, A16, A16, 1.0, 1.0, 256, 256, 272, None) == \
                    bsq.BSQ_ERR_UNSUPPORTED
                assert L.int8_blockscaled_gemm(A16 + 1, A16, A16, A16, A16, 64, 64, 128, None) == \
                    bsq.BSQ_ERR_MISALIGNED
        except AssertionError as e:  # pragma: no cover - reported below
            errors.append((tid, repr(e)))

    ts = [threading.Thread(target=work, args=(t,)) for t in range(8)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors, errors[:3]
    assert bsq.debug_launch_count() == n0


_CHILD = r"""
import sys, threading
import numpy as np, torch
sys.path.insert(0, sys.argv[1])
import int8_gemm_gemv_b200 as bsq

torch.cuda.init()
g = torch.Generator(device="cuda"); g.manual_seed(0)
def u8(shape, lo=0, hi=256):
    return torch.randint(lo, hi, shape, dtype=torch.uint8, device="cuda", generator=g)
m, n, k = 300, 768, 1024
jobs = []
for t in range(8):
    kind = t % 4
    if kind == 0:   # W4A4, CTA pairs
        ap, asf, wp, wsf = u8((m, k // 2)), u8((m, k // 16), 0x30, 0x40), u8((n, k // 2)), u8((n, k // 16), 0x30, 0x40)
        out = torch.empty((m, n), dtype=torch.int16, device="cuda")
        jobs.append((lambda s, ap=ap, asf=asf, wp=wp, wsf=wsf, out=out:
                     bsq.w4a4_gemm(ap, asf, wp, wsf, out, 1.0, 1.0, m, n, k, s), out))
    elif kind == 1:  # FP8 GEMV
        x = (torch.randn((4, k), device="cuda", generator=g)).to(torch.bfloat16)
        w, rs = u8((n, k), 0, 0x7F), torch.rand(n, device="cuda", generator=g)
        out = torch.empty((4, n), dtype=torch.int16, device="cuda")
        jobs.append((lambda s, x=x, w=w, rs=rs, out=out: bsq.fp8_gemv_rowscale(x, w, rs, out, 4, n, k, s), out))
    elif kind == 2:  # int8 per-32 GEMM
        a = torch.randint(-127, 128, (m, k), dtype=torch.int8, device="cuda", generator=g)
        w = torch.randint(-127, 128, (n, k), dtype=torch.int8, device="cuda", generator=g)
        sa, sw = torch.rand(m, k // 32, device="cuda", generator=g), torch.rand(n, k // 32, device="cuda", generator=g)
        out = torch.empty((m, n), dtype=torch.int16, device="cuda")
        jobs.append((lambda s, a=a, w=w, sa=sa, sw=sw, out=out:
                     bsq.int8_blockscaled_gemm(a, w, sa, sw, out, m, n, k, s), out))
    else:            # FP8 GEMM
        a, w = u8((m, k), 0, 0x7F), u8((n, k), 0, 0x7F)
        sa, sw = torch.rand(m, device="cuda", generator=g), torch.rand(n, device="cuda", generator=g)
        out = torch.empty((m, n), dtype=torch.int16, device="cuda")
        jobs.append((lambda s, a=a, sa=sa, w=w, sw=sw, out=out:
                     bsq.fp8_gemm_rowscale(a, sa, w, sw, out, m, n, k, s), out))
torch.cuda.synchronize()
streams = [torch.cuda.Stream() for _ in jobs]
start = threading.Barrier(len(jobs))
errs = []
def run(i):
    try:
        start.wait()
        with torch.cuda.stream(streams[i]):
            jobs[i][0](streams[i])
    except Exception as e:
        errs.append(repr(e))
ts = [threading.Thread(target=run, args=(i,)) for i in range(len(jobs))]
for t in ts: t.start()
for t in ts: t.join()
torch.cuda.synchronize()
assert not errs, errs
first = [j[1].clone() for j in jobs]
for i, (fn, out) in enumerate(jobs):   # the same calls again, one at a time
    out.fill_(-1)
    fn(torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert torch.equal(out, first[i]), i
assert bsq.debug_take_timeouts() == 0
print("threads ok")
"""


@pytest.mark.gpu
def test_first_calls_from_eight_threads():
    r = subprocess.run([sys.executable, "-c", _CHILD, ROOT], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "threads ok" in r.stdout, r.stdout + r.stderr
