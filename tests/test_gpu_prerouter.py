"""GPU parity of the prerouter head and of the forward routed by a given expert set
("Edge0 项目推荐" review, 亮点一): head logits against the oracle, the predicted top-K
bit-exact outside near ties, the select forward on every path, and the double shift
(layer N's head at token t gives the set layer N+1 runs at token t+1)."""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from synth import workloads
from tests.gpu_helpers import (TIE_GAP, assert_close_output, bf16_dev_to_f64, check_routing, check_weights,
                               forward_with_record, need_cuda, path_ran)
from tests.helpers import oracle_layer, quantize_layer

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    need_cuda()


def _mods():
    import int4_group_affine_b200 as m
    from int4_group_affine_b200 import layer as ly
    return m, ly


class DevHead:
    """One prerouter head's fp16 weights on the device and its descriptor."""

    def __init__(self, shape, w):
        m, ly = _mods()
        self.t = {k: ly.to_device(v) for k, v in w.items() if v is not None}
        P = m.Prerouter()
        P.hidden, P.n_experts, P.top_k, P.head_dim = shape.H, shape.E, shape.K, shape.D
        for k in ("w1", "b1", "w2", "b2", "wl", "bl"):
            setattr(P, k, self.t[k].data_ptr() if k in self.t else None)
        self.P = P
        self.shape = shape

    def forward(self, h, ex, pv):
        m, ly = _mods()
        T = h.shape[0]
        nb = m.moe_prerouter_workspace_bytes(self.P, T)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        m.moe_workspace_init(ws, nb)
        z = torch.empty((T, self.shape.E), dtype=torch.float32, device="cuda")
        idx = torch.empty((T, self.shape.K), dtype=torch.int32, device="cuda")
        m.moe_prerouter_forward(self.P, ly.to_device(h), ly.to_device(ex), None if pv is None else ly.to_device(pv),
                                T, z, idx, ws, nb)
        torch.cuda.synchronize()
        return z.cpu().numpy().astype(np.float64), idx.cpu().numpy(), m.moe_get_device_status(ws)


@pytest.fixture(scope="module")
def head():
    s = workloads.PREROUTER
    return s, workloads.prerouter_weights(s, seed=0)


@pytest.mark.parametrize("T,prev", [(1, True), (3, True), (17, True), (64, True), (2, False)])
def test_head_logits_and_prediction(head, T, prev):
    s, w = head
    h, ex, pv = workloads.prerouter_inputs(s, seed=700 + T, T=T)
    if not prev:
        pv = None
    z, idx, st = DevHead(s, w).forward(h, ex, pv)
    assert st == 0
    z_ref = oracle.prerouter(s.H, s.E, s.K, s.D, w, h, ex, pv)
    # fp32 sums of fp16 x bf16 products: far inside the near-tie margin
    assert np.max(np.abs(z - z_ref)) < 0.2 * TIE_GAP
    idx_ref, _ = oracle.topk(z_ref, s.K)
    check_routing(idx, idx_ref, z_ref, s.K)


def test_head_tiny_duplicates_and_bad_entries():
    s = workloads.PREROUTER_TINY
    w = workloads.prerouter_weights(s, seed=9)
    h, ex, pv = workloads.prerouter_inputs(s, seed=9)
    ex = ex.copy()
    ex[1] = [3, 3]  # an expert listed twice sets one one
    z, _, st = DevHead(s, w).forward(h, ex, pv)
    assert st == 0
    assert np.max(np.abs(z - oracle.prerouter(s.H, s.E, s.K, s.D, w, h, ex, pv))) < 1e-5
    bad = ex.copy()
    bad[2, 0] = s.E  # out of range: contributes nothing, flagged
    z2, _, st2 = DevHead(s, w).forward(h, bad, pv)
    assert st2 == 5
    fixed = bad.copy()
    fixed[2, 0] = bad[2, 1]  # the oracle with that entry dropped (a repeat sets nothing new)
    assert np.max(np.abs(z2 - oracle.prerouter(s.H, s.E, s.K, s.D, w, h, fixed, pv))) < 1e-5


@pytest.fixture(scope="module")
def layer():
    shape = dataclasses.replace(workloads.DECODE_K4, n_adapters=2, random_adapters=True)
    t = quantize_layer(workloads.moe_weights(shape, seed=11))
    return shape, t


def _select_forward(shape, t, x, aid, sel):
    m, ly = _mods()
    d = ly.DeviceLayer.from_host(shape, t)
    T = x.shape[0]
    ws, nb = d.workspace(T)
    xd = ly.to_device(x)
    y = torch.empty_like(xd)
    idx = torch.empty((T, shape.K), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, shape.K), dtype=torch.float32, device="cuda")
    m.moe_timing_enable(True)
    try:
        m.moe_ffn_forward_select(d.L, xd, None if aid is None else ly.to_device(aid), ly.to_device(sel), T, y, ws, nb)
        m.moe_ffn_routing(d.L, T, ws, nb, idx, wts)
        torch.cuda.synchronize()
        kinds = set(m.moe_timing_collect())
    finally:
        m.moe_timing_enable(False)
    return bf16_dev_to_f64(y), idx.cpu().numpy(), wts.cpu().numpy(), kinds, m.moe_get_device_status(ws)


@pytest.mark.parametrize("T,path", [(1, "cluster"), (2, "chain"), (3, None), (6, "cuda_core"), (20, "tensor_core")])
def test_select_forward_every_path(layer, T, path):
    shape, t = layer
    x, aid = workloads.moe_inputs(shape, seed=720 + T, T=T)
    # a given set that is not the router's top-K: random distinct experts per token
    sel = np.argsort(synth.uniform(720 + T, "sel", (T, shape.E)), axis=1, kind="stable")[:, :shape.K].astype(np.int32)
    y, idx, wts, kinds, st = _select_forward(shape, t, x, aid, sel)
    assert st == 0 and (path is None or path_ran(path, kinds)), kinds
    assert np.array_equal(idx, sel)
    y_ref, _, w_ref, _, _ = oracle_layer(shape, t).ffn(x, aid, select=sel)
    assert np.allclose(wts, w_ref, rtol=2e-5, atol=1e-6)
    assert_close_output(y, y_ref, "select T=%d" % T)


@pytest.fixture(scope="module")
def layer8():
    shape = dataclasses.replace(workloads.DECODE_K4, K=8, n_adapters=2, random_adapters=True)
    t = quantize_layer(workloads.moe_weights(shape, seed=12))
    return shape, t


def test_select_forward_top8_cluster(layer8):
    """One token at top-8 with a given set: the cluster kernel's lean layout, whose routed
    rows are copied after the cluster's logits as on the router path (the set itself is
    repaired in the kernel's prologue); one entry repeated."""
    shape, t = layer8
    x, aid = workloads.moe_inputs(shape, seed=740, T=1)
    sel = np.argsort(synth.uniform(740, "sel", (1, shape.E)), axis=1, kind="stable")[:, :shape.K].astype(np.int32)
    y, idx, wts, kinds, st = _select_forward(shape, t, x, aid, sel)
    assert st == 0 and path_ran("cluster", kinds), kinds
    assert np.array_equal(idx, sel)
    y_ref, _, w_ref, _, _ = oracle_layer(shape, t).ffn(x, aid, select=sel)
    assert np.allclose(wts, w_ref, rtol=2e-5, atol=1e-6)
    assert_close_output(y, y_ref, "select top-8 T=1")
    bad = sel.copy()
    bad[0, 5] = bad[0, 2]  # a repeat: replaced by the lowest expert not in the set
    y2, idx2, _, _, st2 = _select_forward(shape, t, x, aid, bad)
    want = bad.copy()
    want[0, 5] = min(set(range(shape.E)) - set(int(v) for v in bad[0]))
    assert st2 == 5 and np.array_equal(idx2, want)
    assert_close_output(y2, oracle_layer(shape, t).ffn(x, aid, select=want)[0], "repaired select top-8")


@pytest.mark.parametrize("T", [1, 6])
def test_select_repairs_bad_entries(layer, T):
    shape, t = layer
    x, aid = workloads.moe_inputs(shape, seed=730 + T, T=T)
    sel = np.tile(np.array([[9, 9, 300, 2]], np.int32), (T, 1))  # a repeat and an entry out of range
    y, idx, _, _, st = _select_forward(shape, t, x, aid, sel)
    assert st == 5
    assert np.array_equal(idx, np.tile(np.array([[9, 0, 1, 2]], np.int32), (T, 1)))
    y_ref = oracle_layer(shape, t).ffn(x, aid, select=idx)[0]
    assert_close_output(y, y_ref, "repaired select")


def test_double_shift_prediction_is_the_routing(layer, head):
    """Layer N runs tokens t-1 and t with its own routing; its head predicts from token t's
    input and the executed sets of tokens t and t-1; layer N+1 runs token t+1 on exactly
    that prediction.  Every step on the GPU against the same chain in the oracle."""
    m, ly = _mods()
    shape, t = layer
    hs, w = head
    tN1 = quantize_layer(workloads.moe_weights(shape, seed=12))
    x, aid = workloads.moe_inputs(shape, seed=740, T=3)  # layer N inputs of tokens t-1, t; layer N+1 input of t+1
    dN = ly.DeviceLayer.from_host(shape, t)
    ws, nb = dN.workspace(2)
    y, idx_g, _, _ = forward_with_record(m, dN, ly.to_device(x[:2]), ly.to_device(aid[:2]), 2, ws, nb)
    LN = oracle_layer(shape, t)
    _, idx_r, _, _, z_r = LN.ffn(x[:2], aid[:2])
    check_routing(idx_g, idx_r, z_r, shape.K)
    ex, pv = idx_g[1:2], idx_g[0:1]
    z, pred, st = DevHead(hs, w).forward(x[1:2], ex, pv)
    assert st == 0
    z_ref = oracle.prerouter(hs.H, hs.E, hs.K, hs.D, w, x[1:2], ex, pv)
    pred_ref, _ = oracle.topk(z_ref, hs.K)
    check_routing(pred, pred_ref, z_ref, hs.K)
    y1, idx1, _, kinds, st1 = _select_forward(shape, tN1, x[2:3], aid[2:3], pred)
    assert st1 == 0 and np.array_equal(idx1, pred) and path_ran("cluster", kinds)
    assert_close_output(y1, oracle_layer(shape, tN1).ffn(x[2:3], aid[2:3], select=pred)[0], "layer N+1 on the prediction")
