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


@pytest.mark.parametrize("m,n,k", [
    (256, 256, 4096),     # paired kernel: the producer waits for the stalled stage again
    (512, 512, 512),      # paired kernel, 4 pairs: the producer finishes first, others time out
    (16, 256, 512),       # few-token kernel, stream-K split over many CTAs
    (16, 15360, 4096),    # few-token kernel, whole tiles longer than its ring
])
def test_gemm_kernel_stall_gives_up_and_context_stays_usable(orc, m, n, k):
    """The GEMM kernels' own abort path: with the first ring stage never
    filled, every role's bounded wait (1 ms here) runs out or sees the abort,
    copies and tensor-core work in flight are drained, tensor memory is
    freed and the kernel returns. The host reads NVFP4_ERR_TIMEOUT with only
    that kernel's role bits, and the next GEMM still matches the oracle."""
    import numpy as np
    from nvfp4_w4a4_quantized_elem_b200 import build, nvfp4
    build.build()
    assert nvfp4.read_fault() == 0
    g = torch.Generator().manual_seed(m + n + k)
    x = torch.randn((m, k), generator=g).to(torch.bfloat16)
    w = (torch.randn((n, k), generator=g) * 0.02).to(torch.bfloat16)
    qx, qw = orc.quantize(bits(x)), orc.quantize(bits(w))
    A, W = upload(qx), upload(qw)
    nb = nvfp4.gemm_workspace_bytes(m, n, k)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda") if nb else None
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    nvfp4.selftest_gemm_stall(A, W, limit_ns=1_000_000, workspace=ws)
    fault = nvfp4.read_fault()
    elapsed = time.perf_counter() - t0
    roles = 0xF if m > 64 else 0xF0
    assert fault != 0 and (fault & roles) == fault, hex(fault)
    assert elapsed < 5.0
    assert nvfp4.read_fault() == 0
    y = nvfp4.gemm(A, W, workspace=ws)
    torch.cuda.synchronize()
    rows = np.arange(min(m, 64))
    gemm_check(y[:len(rows)], orc.gemm(qx, qw, a_rows=rows), norms(orc, qx, rows),
               norms(orc, qw), "after stall")
    assert nvfp4.read_fault() == 0
