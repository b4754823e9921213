"""mx_quantize_noalloc, the entry point for callers that cannot allocate
device memory (no allocator handle, inside a graph capture, HBM reserved up
front): called through the C ABI, it must reproduce mx_quantize's outputs --
codes, scales, tensor scale and fidelity statistics -- on two calls in a row
sharing its built-in scratch array.  Collected last on purpose."""
import ctypes as C

import numpy as np
import pytest
import torch

from microscaling_block_quantization_b200 import inputs

pytestmark = pytest.mark.gpu

REL = 1e-4


@pytest.fixture(scope="module")
def mx():
    from microscaling_block_quantization_b200 import build
    build.build()
    import microscaling_block_quantization_b200 as m
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return m


def _noalloc(mx, cfg, x):
    rows, cols = x.shape
    q = mx.alloc_outputs(cfg, rows, cols, x.device, stats=True)
    p = lambda t: None if t is None else C.c_void_p(t.data_ptr())
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = mx.mx_quantize_noalloc(cfg, p(x), mx.DT_BF16 if x.dtype == torch.bfloat16 else mx.DT_FP32,
                                rows, cols, p(q.codes), p(q.scales), p(q.tensor_scale), p(q.macro),
                                p(q.offsets), p(q.stats), stream)
    assert rc == 0, mx.mx_strerror(rc)
    return q


def _same(mx, a, b):
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes)
    assert torch.equal(a.scales, b.scales)
    assert torch.equal(a.tensor_scale, b.tensor_scale)
    sa, sb = a.stats.cpu().numpy(), b.stats.cpu().numpy()
    for i in (0, 1, 5, 6):
        assert abs(sa[i] - sb[i]) <= REL * abs(sb[i])
    assert abs(sa[7] - sb[7]) <= 1e-3
    assert sa[3] == sb[3] and sa[4] == sb[4] and sa[10] == sb[10]


@pytest.mark.parametrize("name", ["mxfp4", "nvfp4", "sr_fp32", "nvfp4_mse"])
def test_noalloc_matches_mx_quantize_twice(mx, name):
    if name == "mxfp4":
        cfg = mx.MXFP4
        x = inputs.laplace_outlier_cols(1024, 2048, seed=4).cuda()
    elif name == "nvfp4":
        cfg = mx.NVFP4
        x = inputs.normal(512, 4096, sigma=0.02, seed=2).cuda()
    elif name == "nvfp4_mse":
        # the heaviest scratch user: four global-step reductions through the
        # records and the ticket, and the per-round tensor scales kept in the
        # control words, which the call clears for the next one
        cfg = mx.Config(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_MSE, tensor_scale=mx.TS_COMPUTE)
        x = inputs.normal(512, 2048, sigma=0.02, seed=3).cuda()
    else:
        cfg = mx.Config(round=mx.ROUND_STOCHASTIC, seed=9)
        x = inputs.gradient_like(256, 4096, seed=5).cuda()
    ref = mx.quantize(x, cfg)
    first = _noalloc(mx, cfg, x)
    second = _noalloc(mx, cfg, x)
    _same(mx, first, ref)
    _same(mx, second, ref)


def test_noalloc_rejections_leave_the_array_usable(mx):
    """The two configurations the no-alloc entry does not take -- a rotation,
    and an amax handed in through a caller's workspace -- are refused with
    MX_ERR_UNSUPPORTED before anything is queued, and a following call still
    reproduces mx_quantize."""
    x = inputs.normal(256, 1024, sigma=0.02, seed=2).cuda()
    P = lambda t: C.c_void_p(t.data_ptr())
    q = mx.alloc_outputs(mx.NVFP4, 256, 1024, x.device, stats=True)
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    for cfg in (mx.Config(hadamard=32), mx.Config(hadamard=16, block=16),
                mx.Config(block=16, scale_fmt=mx.SCALE_UE4M3, rule=mx.RULE_NEAREST, tensor_scale=mx.TS_AMAX)):
        rc = mx.mx_quantize_noalloc(cfg, P(x), mx.DT_BF16, 256, 1024, P(q.codes), P(q.scales),
                                    P(q.tensor_scale), None, None, P(q.stats), stream)
        assert rc == -2, mx.mx_strerror(rc)
    _same(mx, _noalloc(mx, mx.NVFP4, x), mx.quantize(x, mx.NVFP4))
