"""fp4_nvfp4_quantize_noalloc: the NVFP4 quantiser for callers that cannot
allocate device memory (for example an inference-engine plugin's execute
callback, or a service whose device memory was all reserved up front).  It
keeps its workspace in a __device__ array inside the library instead of
taking one from the caller.

Checked through the C ABI against fp4_nvfp4_quantize (which takes a caller
workspace): packed codes, scale bytes, global scale and status must be
identical, bit for bit, on two calls in a row -- the second on a different
tensor, so that whatever the first call left in the shared array cannot
leak into the second -- and inside a CUDA graph: a call captured once and
replayed on new inputs copied into the captured input buffer.  The file
sorts last so that a run stopping at the first failure has run every other
test already; it also passes alone.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_scaled_fp4_reduce_b200 as fp4
import workloads

pytestmark = pytest.mark.gpu


def _regular(x):
    q = fp4.nvfp4_quantize(x)
    return q.packed, q.scales, q.global_scale, q.status


def _outputs(x):
    R, C = x.shape
    return (torch.empty((R, C // 2), dtype=torch.uint8, device=x.device),
            torch.empty((R, C // 16), dtype=torch.uint8, device=x.device),
            torch.empty(1, dtype=torch.float32, device=x.device),
            torch.zeros(1, dtype=torch.int32, device=x.device))


def _noalloc(x, out=None):
    R, C = x.shape
    packed, scales, g, st = out if out is not None else _outputs(x)
    rc = fp4.lib().fp4_nvfp4_quantize_noalloc(
        ctypes.c_void_p(x.data_ptr()), fp4._dtype_code(x), R, C, ctypes.c_void_p(packed.data_ptr()),
        ctypes.c_void_p(scales.data_ptr()), ctypes.c_void_p(g.data_ptr()), ctypes.c_void_p(st.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == fp4.OK, fp4.lib().fp4_status_string(rc)
    return packed, scales, g, st


def test_noalloc_matches_the_workspace_entry_point_on_two_calls_in_a_row():
    first = workloads.generate(workloads.ACT_8K).cuda()                       # 8192 x 14336 bf16
    second = workloads.generate(workloads.with_shape(workloads.TINY_F32, 96, 1024, seed_offset=5)).cuda()
    for x in (first, second):
        want = _regular(x)
        got = _noalloc(x)
        torch.cuda.synchronize()
        for a, b, what in zip(got, want, ("packed", "scales", "global scale", "status")):
            assert torch.equal(a, b), what
        assert int(got[3].item()) == fp4.OK


def test_noalloc_rejects_bad_arguments_without_launching():
    L = fp4.lib()
    P = 1 << 20
    assert L.fp4_nvfp4_quantize_noalloc(P, fp4.BF16, 4, 24, P, P, P, P, None) == fp4.ERR_SHAPE
    assert L.fp4_nvfp4_quantize_noalloc(P + 4, fp4.BF16, 4, 32, P, P, P, P, None) == fp4.ERR_ALIGN
    assert L.fp4_nvfp4_quantize_noalloc(P, fp4.BF16, 4, 32, P, P, None, P, None) == fp4.ERR_INVALID_ARG


def test_noalloc_captured_in_a_cuda_graph_and_replayed():
    inputs = [workloads.generate(workloads.with_shape(workloads.WEIGHT_4K, 256, 4096, seed_offset=k)).cuda()
              for k in (11, 12, 13)]
    x = inputs[0].clone()
    out = _outputs(x)
    _noalloc(x, out)  # the first call in this context, before the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        _noalloc(x, out)
    for new in inputs[1:]:
        x.copy_(new)
        out[3].zero_()
        graph.replay()
        want = _regular(new)
        torch.cuda.synchronize()
        for a, b, what in zip(out, want, ("packed", "scales", "global scale", "status")):
            assert torch.equal(a, b), what
        assert int(out[3].item()) == fp4.OK
    del graph
