"""The NF4 quantiser entry point that allocates nothing (lst_k_nf4_quantize_noalloc).

It exists for callers that cannot allocate device memory: code whose GPU memory is all held by
its own caching allocator, or code that must not cause the device-wide synchronisation of
cudaMalloc / cudaFree while other streams are running. Its output must be the same bytes as the
allocating entry point's, call after call, although every call reuses one fixed scratch array.
This file is collected last so that, if it fails, every other test has already run.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
lst = pytest.importorskip("layer_streamed_qlora_streaming_b200")

MAX_ELEMS = 1 << 26


def _buffers(n, device):
    return (torch.empty(n // 2, dtype=torch.uint8, device=device),
            torch.empty(n // 64, dtype=torch.int8, device=device),
            torch.empty((n // 64 + 255) // 256, dtype=torch.float32, device=device),
            torch.empty(1, dtype=torch.float32, device=device))


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(4096, 1024), (688, 256), (14336, 4096)])
def test_noalloc_quantize_equals_allocating_quantize_twice(shape):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    n = shape[0] * shape[1]
    g = torch.Generator(device="cuda")
    g.manual_seed(n)
    outs = []
    for call in range(3):
        w = torch.randn(n, generator=g, device="cuda", dtype=torch.float32) * 0.02
        ref = _buffers(n, "cuda")
        lst.k_nf4_quantize(w, *ref)
        # two calls in a row on the same scratch; the second must not see the first's leftovers
        for _ in range(2):
            got = _buffers(n, "cuda")
            lst.k_nf4_quantize_noalloc(w, *got)
            torch.cuda.synchronize()
            for a, b in zip(got, ref):
                # bytes and codes: compared exactly (the tolerance for integer work is zero)
                assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
        outs.append(got[0].sum().item())
    assert len(set(outs)) > 1   # different inputs really went through


@pytest.mark.gpu
def test_noalloc_quantize_rejects_oversize():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    w = torch.zeros(64, device="cuda")
    bufs = _buffers(64, "cuda")
    with pytest.raises(lst.LstError) as e:
        lst.k_nf4_quantize_noalloc(w, *bufs, n=MAX_ELEMS + 64)   # rejected before any launch
    assert e.value.status == 1
    lst.k_nf4_quantize_noalloc(w, *bufs)                        # still usable afterwards
    torch.cuda.synchronize()
