"""GPU parity of the EdgeRazor mixed layer in weight-activation form (8-bit activations;
"EDGERAZOR 深度解读" section 2.1 矩阵乘法分解 and the W/A table of section 3.1): the
activation codes and scales bit-exact, the integer-dot outputs within fp32 rounding of
the oracle's, and the MLP and residual block within the method's output tolerance."""
import numpy as np
import pytest

import oracle
import synth
from synth import workloads
from tests.gpu_helpers import assert_close_output, bf16_dev_to_f64, need_cuda
from tests.helpers import rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    need_cuda()


def _mods():
    import int4_group_affine_b200 as m
    from int4_group_affine_b200 import layer as ly
    return m, ly


@pytest.fixture(scope="module")
def mixed():
    s = workloads.MIXED_B1
    W = workloads.mixed_weights(s, seed=8)
    return s, W, {n: oracle.quant_mixed(W[n], s.rho) for n in W}


@pytest.mark.parametrize("T,n", [(1, 1024), (7, 1024), (16, 3072), (3, 64)])
def test_act8_codes_bit_exact(T, n):
    m, ly = _mods()
    x = synth.bf16(synth.normal(800 + T, "a8", (T, n)) * np.linspace(0.01, 3.0, T, dtype=np.float32)[:, None])
    x[0, :8] = 0  # a few zeros
    q = torch.empty((T, n), dtype=torch.int8, device="cuda")
    sc = torch.empty(T, dtype=torch.float32, device="cuda")
    m.moe_act8_quant(ly.to_device(x), T, n, q, sc)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quant_act8(synth.bf16_to_f32(x))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy(), s_ref)


@pytest.mark.parametrize("T,which", [(1, "gate"), (5, "gate"), (16, "down"), (20, "up")])
def test_linear_a8(mixed, T, which):
    m, ly = _mods()
    s, W, q = mixed
    out, in_ = (s.H, s.I) if which == "down" else (s.I, s.H)
    dm = ly.DeviceMixed.from_host(out, in_, s.rho, *q[which])
    x = synth.bf16(synth.normal(810 + T, "a8x", (T, in_)))
    nb = m.moe_mixed_linear_a8_workspace_bytes(in_, T)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    y = torch.empty((T, out), dtype=torch.float32, device="cuda")
    m.moe_mixed_linear_a8(dm.T, ly.to_device(x), T, y, ws, nb)
    torch.cuda.synchronize()
    ref = oracle.mixed_linear_a8(q[which][0], q[which][1], out, in_, s.rho, x)
    # exact integer sums times two fp32 scales: a few fp32 roundings
    assert np.max(np.abs(y.cpu().numpy() - ref) / np.maximum(np.abs(ref), 1e-30)) < 1e-6 or \
        rel_l2(y.cpu().numpy(), ref) < 1e-6


@pytest.mark.parametrize("T,residual", [(1, 0), (16, 0), (1, 1), (16, 1), (3, 1)])
def test_mlp_a8(mixed, T, residual):
    m, ly = _mods()
    s, W, q = mixed
    x = workloads.mixed_inputs(s, seed=820 + T, T=T)
    dg = ly.DeviceMixed.from_host(s.I, s.H, s.rho, *q["gate"])
    du = ly.DeviceMixed.from_host(s.I, s.H, s.rho, *q["up"])
    dd = ly.DeviceMixed.from_host(s.H, s.I, s.rho, *q["down"])
    nb = m.moe_mixed_mlp_a8_workspace_bytes(s.H, s.I, T)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    xd = ly.to_device(x)
    y = torch.empty_like(xd)
    m.moe_mixed_mlp_forward_a8(dg.T, du.T, dd.T, xd, T, residual, 1e-6, y, ws, nb)
    torch.cuda.synchronize()
    out = bf16_dev_to_f64(y)
    if residual:
        ref = synth.bf16_to_f32(oracle.mixed_block_a8(q["gate"], q["up"], q["down"], s.H, s.I, s.rho, x))
        xs = synth.bf16_to_f32(x).astype(np.float64)
        ref = ref.astype(np.float64)
        tol = np.abs(ref) * 2.0 ** -7 + 1e-2 * np.max(np.abs(ref - xs))
        assert np.all(np.abs(out - ref) <= tol)
    else:
        ref = oracle.mixed_mlp_a8(q["gate"], q["up"], q["down"], s.H, s.I, s.rho, x)
        assert_close_output(out, ref, "mlp a8")
