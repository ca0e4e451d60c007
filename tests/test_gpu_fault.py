"""Failure detection on the GPU without a fault: a bounded wait on an mbarrier
that nothing arrives at gives up after its limit, the kernel records the
fault bit and returns, the host reads the status, and the context keeps
working (the next quantize + GEMM still matches the oracle)."""
import time

import pytest
import torch

from parity import bits, gemm_check, norms, upload

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_context_stays_usable(orc):
    from nvfp4_w4a4_quantized_elem_b200 import build, nvfp4, workloads as wl
    build.build()
    assert nvfp4.read_fault() == 0
    t0 = time.perf_counter()
    nvfp4.selftest_wait_timeout(5_000_000)      # 5 ms
    fault = nvfp4.read_fault()
    elapsed = time.perf_counter() - t0
    assert fault == 256, fault
    assert 0.005 <= elapsed < 5.0
    assert nvfp4.read_fault() == 0              # read_fault cleared the word
    cfg = wl.tiny()
    x, w = cfg.x(), cfg.w()
    qx, qw = orc.quantize(bits(x)), orc.quantize(bits(w))
    y = nvfp4.gemm(nvfp4.quantize(x.cuda()), upload(qw))
    torch.cuda.synchronize()
    gemm_check(y, orc.gemm(qx, qw), norms(orc, qx), norms(orc, qw), "after timeout")
    assert nvfp4.read_fault() == 0
