"""moe_ffn_forward_static: the MoE forward for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc where they run the layer (an engine's enqueue
hook that must not allocate, a runtime that reserved all device memory up front),
so this entry point takes its scratch from an array built into the library.  The
checks go through the C ABI: two calls in a row must give the output of
moe_ffn_forward with a caller-provided workspace, within the parity tolerance,
and a size beyond the built-in array must be refused before anything runs.
This file is collected last on purpose.
"""
import dataclasses

import numpy as np
import pytest

from synth import workloads
from tests.gpu_helpers import assert_close_output, bf16_dev_to_f64, need_cuda
from tests.helpers import quantize_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    need_cuda()


def _layer(shape, seed):
    from int4_group_affine_b200.layer import DeviceLayer
    t = quantize_layer(workloads.moe_weights(shape, seed=seed))
    return DeviceLayer.from_host(shape, t)


def _reference(d, xd, aid, T):
    """moe_ffn_forward with a workspace the caller allocated."""
    import int4_group_affine_b200 as m
    ws, nb = d.workspace(T)
    y = torch.empty_like(xd)
    m.moe_ffn_forward(d.L, xd, aid, T, y, ws, nb)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("shape,T", [(workloads.TINY, 4),
                                     (dataclasses.replace(workloads.TINY, n_adapters=3, random_adapters=True), 37)])
def test_static_forward_matches_workspace_forward_twice(shape, T):
    import int4_group_affine_b200 as m
    from int4_group_affine_b200.layer import to_device
    d = _layer(shape, seed=900 + T)
    x, aid = workloads.moe_inputs(shape, seed=900 + T, T=T)
    xd = to_device(x)
    ad = None if aid is None else to_device(aid)
    ref = bf16_dev_to_f64(_reference(d, xd, ad, T))
    for call in range(2):  # the shared array keeps the previous call's contents
        y = torch.full_like(xd, -1)
        m.moe_ffn_forward_static(d.L, xd, ad, T, y)
        torch.cuda.synchronize()
        assert_close_output(bf16_dev_to_f64(y), ref, "static call %d" % call)


def test_static_forward_follows_a_different_shape():
    # A small call after a larger one still starts from a clean header.
    import int4_group_affine_b200 as m
    from int4_group_affine_b200.layer import to_device
    shape = workloads.TINY
    d = _layer(shape, seed=910)
    for T in (70, 3):
        x, _ = workloads.moe_inputs(shape, seed=910 + T, T=T)
        xd = to_device(x)
        y = torch.empty_like(xd)
        m.moe_ffn_forward_static(d.L, xd, None, T, y)
        torch.cuda.synchronize()
        assert_close_output(bf16_dev_to_f64(y), bf16_dev_to_f64(_reference(d, xd, None, T)), "T=%d" % T)


def test_static_status_word_reports_device_errors():
    """The built-in array's status word: MOE_OK after a clean call, MOE_ERR_DEVICE_INDEX
    (5) after a call with an adapter id out of range, and cleared by the read."""
    import int4_group_affine_b200 as m
    from int4_group_affine_b200.layer import to_device
    shape = dataclasses.replace(workloads.TINY, n_adapters=2)
    d = _layer(shape, seed=930)
    x, _ = workloads.moe_inputs(shape, seed=930, T=4)
    xd = to_device(x)
    y = torch.empty_like(xd)
    m.moe_ffn_forward_static(d.L, xd, to_device(np.array([0, 1, -1, 0], np.int32)), 4, y)
    assert m.moe_ffn_static_device_status() == 0
    m.moe_ffn_forward_static(d.L, xd, to_device(np.array([0, 7, 1, -1], np.int32)), 4, y)
    assert m.moe_ffn_static_device_status() == 5
    assert m.moe_ffn_static_device_status() == 0  # read and cleared


def test_static_forward_refuses_oversize():
    import int4_group_affine_b200 as m
    from int4_group_affine_b200 import MoeError
    from int4_group_affine_b200._lib import lib
    shape = workloads.TINY
    d = _layer(shape, seed=920)
    limit = 16 * 1024 * 1024
    T = 1
    while m.moe_ffn_workspace_bytes(d.L, T) <= limit:
        T *= 2
    x = torch.zeros((1, shape.H), dtype=torch.int16, device="cuda")
    y = torch.zeros_like(x)
    with pytest.raises(MoeError) as ei:
        m.moe_ffn_forward_static(d.L, x, None, T, y)
    assert ei.value.status == 4
    assert lib().moe_status_string(4) == b"workspace missing, misaligned or too small"
    torch.cuda.synchronize()
    assert int(y.abs().sum().item()) == 0  # nothing was enqueued
