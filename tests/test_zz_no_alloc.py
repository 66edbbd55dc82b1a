"""The allocation-free quantiser entry point (GPU).

nf4_quantize_tensor_noalloc serves callers that cannot allocate device memory: it
keeps its scratch in a fixed device array inside the library.  These checks call it
through the C ABI twice in a row and compare each result with nf4_quantize_tensor,
which takes a caller-provided scratch buffer: the bytes must be identical (the
quantiser's own tolerance is exact).  Sizes above the fixed maximum are refused.
This file is collected last so that a failure here cannot hide the other results.
"""
import ctypes

import pytest
import torch

from nf4_layer_streamed_b200 import api, binding as B, synth

pytestmark = pytest.mark.gpu


def _noalloc(w: torch.Tensor) -> dict:
    n = w.numel()
    packed = torch.empty(n // 2, dtype=torch.uint8, device="cuda")
    q8 = torch.empty(n // 64, dtype=torch.uint8, device="cuda")
    nested = torch.empty((n // 64 + 255) // 256, dtype=torch.float32, device="cuda")
    offset = torch.empty(1, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    B.call("nf4_quantize_tensor_noalloc", ctypes.c_void_p(w.data_ptr()), n, ctypes.c_void_p(packed.data_ptr()),
           ctypes.c_void_p(q8.data_ptr()), ctypes.c_void_p(nested.data_ptr()), ctypes.c_void_p(offset.data_ptr()),
           stream)
    return {"packed": packed, "q8": q8, "nested": nested, "offset": offset}


def test_noalloc_quantizer_matches_scratch_quantizer_on_two_calls():
    shapes = [(4096, 1024), (257, 64)]   # a large tensor, then a small one with a partial nested group
    for i, shape in enumerate(shapes):
        w = synth.tensor_values(shape, seed=100 + i, scale=0.02, device="cuda")
        got = _noalloc(w)
        ref = api.nf4_quantize_tensor(w)
        torch.cuda.synchronize()
        for k in ("packed", "q8", "nested", "offset"):
            assert torch.equal(got[k], ref[k]), (shape, k)
    st, err = api.device_error()
    assert st == 0, err


def test_noalloc_quantizer_rejects_sizes_beyond_its_scratch():
    mx = B.lib().nf4ls_quantize_noalloc_max_elems()
    assert mx == 1 << 28
    st = B.call_status("nf4_quantize_tensor_noalloc", ctypes.c_void_p(256), mx + 64, ctypes.c_void_p(256),
                       ctypes.c_void_p(256), ctypes.c_void_p(256), ctypes.c_void_p(256), None)
    assert st == -1 and "exceeds the fixed scratch" in B.last_error()
