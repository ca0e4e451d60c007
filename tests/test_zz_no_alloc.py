"""nvfp4_quantize_noalloc against nvfp4_quantize.

The allocation-free entry point serves callers that are handed only their
input and output buffers and may not call cudaMalloc (a plugin inside a
framework whose allocator owns the device memory, or a runtime that forbids
device allocation after start-up). It keeps the amax pass's partial maxima in
a fixed device array inside the library instead of a caller workspace, so its
output must equal the workspace entry point's — bit for bit, which is the
tolerance every quantization test here uses — on consecutive calls that
reuse that array.

This file is collected last, so a run that stops at the first failure has
already run every other test.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


def _equal(a, b):
    return (torch.equal(a.codes, b.codes) and torch.equal(a.sf, b.sf)
            and torch.equal(a.global_scale, b.global_scale))


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    from nvfp4_w4a4_quantized_elem_b200 import build, nvfp4
    build.build()
    gen = torch.Generator(device="cpu").manual_seed(11)
    shapes = [(8192, 5120), (300, 1040)]   # many amax CTAs, then few
    xs = [(torch.randn(s, generator=gen) * (3.0 if i else 0.5)).to(torch.bfloat16).cuda()
          for i, s in enumerate(shapes)]
    xs[0][:, 7] *= 50.0                     # an outlier channel moves the global
    for x in xs:                            # two calls in a row share the array
        ref = nvfp4.quantize(x)             # existing entry point, caller workspace
        out = nvfp4.NVFP4Tensor.empty(x.shape[0], x.shape[1])
        nvfp4.quantize_noalloc(x, out)
        torch.cuda.synchronize()
        assert _equal(out, ref)
    # static global: no scratch used at all
    g = torch.tensor([37.0], device="cuda")
    ref = nvfp4.quantize(xs[1], global_scale=g)
    out = nvfp4.NVFP4Tensor.empty(*xs[1].shape)
    nvfp4.quantize_noalloc(xs[1], out, global_scale=g)
    torch.cuda.synchronize()
    assert _equal(out, ref)
    assert nvfp4.read_fault() == 0


def test_noalloc_calls_leave_free_device_memory_unchanged():
    """The property the entry point exists for: once its first call in the
    context has looked up the scratch array, further calls allocate no
    device memory. Outputs are allocated up front; torch's caching allocator
    is then untouched, so any drop in the device's free memory would come
    from the library."""
    from nvfp4_w4a4_quantized_elem_b200 import build, nvfp4
    build.build()
    gen = torch.Generator(device="cpu").manual_seed(12)
    x = (torch.randn(4096, 5120, generator=gen)).to(torch.bfloat16).cuda()
    out = nvfp4.NVFP4Tensor.empty(*x.shape)
    nvfp4.quantize_noalloc(x, out)           # first call: address look-up
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(5):
        nvfp4.quantize_noalloc(x, out)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    ref = nvfp4.quantize(x)
    torch.cuda.synchronize()
    assert _equal(out, ref)
    assert nvfp4.read_fault() == 0
