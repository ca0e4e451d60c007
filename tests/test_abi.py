"""The C-ABI library loads, exports every symbol include/nvfp4.h declares, and
rejects bad arguments on the host (no GPU needed: argument checks return a
status before anything touches CUDA)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")

OK, INVALID, UNSUPPORTED, MISALIGNED = 0, 1, 2, 3


@pytest.fixture(scope="module")
def L():
    from nvfp4_w4a4_quantized_elem_b200 import build, nvfp4
    build.build()
    return nvfp4.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for f in ("nvfp4_quantize", "nvfp4_gemm", "nvfp4_fuse_group_scales"):
        assert f in names


def test_binding_constants_match_the_header():
    """Constants the binding mirrors from include/nvfp4.h."""
    from nvfp4_w4a4_quantized_elem_b200 import nvfp4
    text = open(HEADER).read()
    m = re.search(r"#define NVFP4_ONE_PASS_MAX_BYTES (\d+)", text)
    assert m and int(m.group(1)) == nvfp4.ONE_PASS_MAX_BYTES
    m = re.search(r"#define NVFP4_LINEAR_IN_KERNEL_MAX_TOKENS (\d+)", text)
    assert m and int(m.group(1)) == nvfp4.LINEAR_IN_KERNEL_MAX_TOKENS


def test_library_exports_every_declared_symbol(L):
    from nvfp4_w4a4_quantized_elem_b200 import nvfp4
    names = declared_functions()
    assert sorted(nvfp4.EXPORTS) == names
    for name in names:
        assert hasattr(L, name), name


def test_status_strings(L):
    for code, name in [(0, b"NVFP4_OK"), (1, b"NVFP4_ERR_INVALID_ARG"), (5, b"NVFP4_ERR_TIMEOUT")]:
        assert L.nvfp4_status_string(code) == name


def test_sf_bytes(L):
    assert L.nvfp4_sf_bytes(64, 256) == 128 * 16
    assert L.nvfp4_sf_bytes(12384, 5120) == 12416 * 320
    assert L.nvfp4_sf_bytes(1, 16) == 128 * 4
    assert L.nvfp4_sf_bytes(0, 16) == 0
    assert L.nvfp4_sf_bytes(4, 24) == 0     # k % 16 != 0
    assert L.nvfp4_sf_bytes(-1, 16) == 0


def test_sf_bytes_matches_oracle(L, orc):
    for rows, k in [(1, 16), (130, 80), (8192, 5120), (48, 5120), (32768, 17408)]:
        assert L.nvfp4_sf_bytes(rows, k) == orc.sf_bytes(rows, k)


P = ctypes.c_void_p
FAKE = 1 << 20  # an aligned, never-dereferenced address (checks fail first)


def q(L, x=FAKE, rows=4, k=32, ldx=32, gin=None, codes=FAKE, sf=FAKE, gout=FAKE,
      ws=FAKE, wsb=1 << 16):
    return L.nvfp4_quantize(P(x), rows, k, ldx, P(gin), P(codes), P(sf), P(gout), P(ws), wsb, None)


def test_quantize_argument_checks(L):
    assert q(L, k=24) == UNSUPPORTED
    assert q(L, k=0) == INVALID
    assert q(L, rows=-1) == INVALID
    assert q(L, x=None) == INVALID
    assert q(L, gout=None) == INVALID
    assert q(L, ldx=16) == INVALID           # ldx < k
    assert q(L, ldx=36) == MISALIGNED        # ldx % 8
    assert q(L, x=FAKE + 8) == MISALIGNED
    assert q(L, sf=FAKE + 4) == MISALIGNED
    assert q(L, codes=FAKE + 2) == MISALIGNED
    assert q(L, ws=None) == INVALID          # dynamic mode needs workspace
    assert q(L, wsb=16) == INVALID


def g(L, a=FAKE, asf=FAKE, ag=FAKE, b=FAKE, bsf=FAKE, bg=FAKE, y=FAKE, yd=0, ldy=64,
      m=8, n=64, k=64):
    return L.nvfp4_gemm(P(a), P(asf), P(ag), P(b), P(bsf), P(bg), P(y), yd, ldy, m, n, k,
                        None, 0, None)


def test_gemm_argument_checks(L):
    assert g(L, k=48) == UNSUPPORTED         # k % 32
    assert g(L, m=0) == INVALID
    assert g(L, yd=2) == INVALID
    assert g(L, ldy=32) == INVALID           # ldy < n
    assert g(L, n=60, ldy=60) == MISALIGNED  # 120-byte row pitch
    assert g(L, a=FAKE + 8) == MISALIGNED
    assert g(L, bsf=FAKE + 4) == MISALIGNED
    assert g(L, ag=None) == INVALID


def test_fuse_argument_checks(L):
    rows = (ctypes.c_int64 * 2)(48, 48)
    ptrs = (ctypes.c_void_p * 2)(FAKE, FAKE + (1 << 16))
    f = L.nvfp4_fuse_group_scales
    cast = lambda a: ctypes.cast(a, P)
    assert f(0, cast(rows), 64, cast(ptrs), P(FAKE), P(FAKE * 4), P(FAKE * 8), None) == INVALID
    assert f(17, cast(rows), 64, cast(ptrs), P(FAKE), P(FAKE * 4), P(FAKE * 8), None) == INVALID
    assert f(2, cast(rows), 40, cast(ptrs), P(FAKE), P(FAKE * 4), P(FAKE * 8), None) == UNSUPPORTED
    # output overlapping an input scale buffer (in place) is refused
    assert f(2, cast(rows), 64, cast(ptrs), P(FAKE * 2), P(FAKE), P(FAKE * 8), None) == INVALID
    # g* written over one of the input globals is refused
    assert f(2, cast(rows), 64, cast(ptrs), P(FAKE * 2), P(FAKE * 4), P(FAKE * 2 + 4), None) == INVALID


def test_silu_argument_checks(L):
    f = L.nvfp4_silu_mul
    assert f(P(FAKE), 4, 12, 24, P(FAKE), 16, None) == UNSUPPORTED  # n % 8
    assert f(P(FAKE), 4, 16, 16, P(FAKE), 16, None) == INVALID      # ldy < 2n
    assert f(P(FAKE + 2), 4, 16, 32, P(FAKE), 16, None) == MISALIGNED


def test_interleave_gate_up_permutation():
    import torch
    from nvfp4_w4a4_quantized_elem_b200 import nvfp4
    ffn, k = 384, 4
    w = torch.arange(2 * ffn, dtype=torch.float32)[:, None].expand(2 * ffn, k).contiguous()
    wi = nvfp4.interleave_gate_up(w)[:, 0].long()
    for b in range(ffn // 128):
        assert torch.equal(wi[256 * b:256 * b + 128], torch.arange(128 * b, 128 * b + 128))
        assert torch.equal(wi[256 * b + 128:256 * b + 256],
                           torch.arange(ffn + 128 * b, ffn + 128 * b + 128))


def test_swiglu_quant_argument_checks(L):
    f = L.nvfp4_gemm_swiglu_quant
    args = lambda ffn=256, k=512, h=FAKE: (P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE),
                                           P(FAKE), P(h), P(FAKE), 8, ffn, k, None)
    assert f(*args(ffn=200)) == UNSUPPORTED      # ffn % 128
    assert f(*args(k=48)) == UNSUPPORTED
    assert f(*args(h=FAKE + 8)) == MISALIGNED
    assert f(*args(h=None)) == INVALID


def test_swiglu_quant_dynamic_argument_checks(L):
    f = L.nvfp4_gemm_swiglu_quant_dynamic
    need = L.nvfp4_gemm_swiglu_quant_dynamic_workspace_bytes(8, 256)
    assert need >= 8 * 256 * 2 + 4 * 148
    assert L.nvfp4_gemm_swiglu_quant_dynamic_workspace_bytes(0, 256) == 0

    def args(ffn=256, k=512, hg=FAKE, ws=FAKE, wsb=need):
        return (P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(hg),
                8, ffn, k, P(ws), wsb, None)
    assert f(*args(ffn=200, wsb=1 << 24)) == UNSUPPORTED   # ffn % 128
    assert f(*args(k=48)) == UNSUPPORTED
    assert f(*args(hg=None)) == INVALID
    assert f(*args(ws=None)) == INVALID
    assert f(*args(ws=FAKE + 16)) == MISALIGNED           # workspace: 256-byte alignment
    assert f(*args(hg=FAKE + 2)) == MISALIGNED
    assert f(*args(wsb=need - 1)) == INVALID                # short workspace


def lin(L, x=FAKE, m=8, k=64, ldx=64, xg=None, wc=FAKE, wsf=FAKE, wg=FAKE, n=64, y=FAKE, yd=0,
        ldy=64, ws=FAKE, wsb=1 << 24):
    return L.nvfp4_linear(P(x), m, k, ldx, P(xg), P(wc), P(wsf), P(wg), n, P(y), yd, ldy, P(ws),
                          wsb, None)


def test_linear_argument_checks(L):
    assert lin(L, x=None) == INVALID
    assert lin(L, ws=None) == INVALID
    assert lin(L, m=0) == INVALID
    assert lin(L, ldx=32) == INVALID         # ldx < k
    assert lin(L, yd=2) == INVALID
    assert lin(L, k=48, ldx=48) == UNSUPPORTED
    assert lin(L, ws=FAKE + 16) == MISALIGNED  # workspace needs 256-byte alignment
    assert lin(L, x=FAKE + 8) == MISALIGNED
    assert lin(L, ldx=68) == MISALIGNED      # row pitch of x: 8 elements
    assert lin(L, xg=FAKE + 2) == MISALIGNED
    assert lin(L, wsb=16) == INVALID         # short workspace


def test_linear_workspace_bytes(L):
    f = L.nvfp4_linear_workspace_bytes
    assert f(0, 64, 64) == 0 and f(8, 0, 64) == 0 and f(8, 64, 48) == 0
    m, n, k = 8, 1000, 2048
    # quantized activations + partial maxima + (few tokens) counters and 9 slabs per tile
    w_tiles = -(-n // 128)
    slabs = w_tiles * 9 * m * 128 * 4
    assert f(m, n, k) >= m * k // 2 + L.nvfp4_sf_bytes(m, k) + 16384 + slabs
    assert f(65, n, k) < f(64, n, k)         # no split workspace above 64 tokens
    # the split counters' region (n only: at least 64 tiles x 16 counters) + slabs
    assert L.nvfp4_gemm_workspace_bytes(m, n, k) == 4096 + slabs
    assert L.nvfp4_gemm_workspace_bytes(65, n, k) == 0


def test_selftest_limit_checks(L):
    f = L.nvfp4_selftest_wait_timeout
    assert f(0, None) == INVALID
    assert f(999, None) == INVALID
    assert f(20_000_000_000, None) == INVALID
    g = L.nvfp4_selftest_gemm_stall
    args = lambda lim: (P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), 256, 256,
                        512, lim, None, 0, None)
    assert g(*args(999)) == INVALID
    assert g(*args(20_000_000_000)) == INVALID
