"""GPU parity of the expert-parallel building blocks: the dispatch (a stable rank-major
partition of the routed jobs, bit-exact), the experts-only forward against the oracle,
the combine, a G-rank expert-parallel forward simulated on one GPU (the all-to-alls done
by copying the row ranges), and ep_forward over a one-rank NCCL group."""
import dataclasses
import os
import socket

import numpy as np
import pytest

import oracle
import synth
from synth import workloads
from tests.gpu_helpers import assert_close_output, bf16_dev_to_f64, need_cuda
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


def _np_partition(idx, E, G):
    owner = idx.reshape(-1) // (E // G)
    order = np.argsort(owner, kind="stable")
    pos = np.empty(idx.size, np.int64)
    pos[order] = np.arange(idx.size)
    return pos.reshape(idx.shape), np.bincount(owner, minlength=G), order


@pytest.mark.parametrize("T,K,E,G", [(64, 4, 256, 8), (5, 2, 8, 2), (3, 4, 256, 1), (1500, 8, 256, 4)])
def test_dispatch_bit_exact(T, K, E, G):
    m, ly = _mods()
    H = 64
    z = synth.normal(40 + T, "ep/z", (T, E)).astype(np.float64)
    idx, _ = oracle.topk(z, K)
    aid = synth.randint(41, "ep/a", (T,), -1, 2)
    x = synth.bf16(synth.normal(42, "ep/x", (T, H)))
    pos = torch.empty((T, K), dtype=torch.int32, device="cuda")
    counts = torch.empty(G, dtype=torch.int32, device="cuda")
    sx = torch.empty((T * K, H), dtype=torch.int16, device="cuda")
    meta = torch.empty((T * K, 2), dtype=torch.int32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.moe_ep_dispatch(ly.to_device(x), ly.to_device(idx), ly.to_device(aid), 3, T, K, H, E, G, pos, counts, sx, meta,
                      st)
    torch.cuda.synchronize()
    p_ref, c_ref, order = _np_partition(idx, E, G)
    assert np.array_equal(pos.cpu().numpy(), p_ref)
    assert np.array_equal(counts.cpu().numpy(), c_ref)
    tok = np.repeat(np.arange(T), K)
    assert np.array_equal(ly.to_host(sx, np.uint16), x[tok[order]])
    assert np.array_equal(meta.cpu().numpy(), np.stack([idx.reshape(-1)[order], aid[tok[order]]], axis=1))
    assert int(st.item()) == 0


@pytest.fixture(scope="module")
def layer():
    shape = dataclasses.replace(workloads.DECODE_K4, n_adapters=2, random_adapters=True)
    return shape, quantize_layer(workloads.moe_weights(shape, seed=21))


def _experts_only_oracle(shape, t):
    tx = dict(t)
    for k in ("s_gate", "s_up", "s_down", "sgate"):
        for suf in ("_p", "_s", "_b"):
            tx[k + suf] = None
    return oracle.OracleLayer(shape.H, shape.E, 1, shape.I, 0, tx, rank=shape.rank, alpha=shape.alpha)


@pytest.mark.parametrize("N", [3, 40])
def test_experts_forward_against_oracle(layer, N):
    m, ly = _mods()
    shape, t = layer
    d = ly.DeviceLayer.from_host(shape, t)
    x = synth.bf16(synth.normal(50 + N, "ep/rows", (N, shape.H)))
    e = synth.randint(51 + N, "ep/e", (N,), 0, shape.E - 1)
    a = synth.randint(52 + N, "ep/ad", (N,), -1, 1)
    nb = m.moe_experts_workspace_bytes(d.L, N)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    m.moe_workspace_init(ws, nb)
    y = torch.empty((N, shape.H), dtype=torch.int16, device="cuda")
    m.moe_experts_forward(d.L, ly.to_device(x), ly.to_device(e), ly.to_device(a), N, y, ws, nb)
    torch.cuda.synchronize()
    assert m.moe_get_device_status(ws) == 0
    Lx = _experts_only_oracle(shape, t)
    ref = np.stack([Lx.ffn(x[n:n + 1], a[n:n + 1], select=e[n:n + 1, None])[0][0] for n in range(N)])
    assert_close_output(bf16_dev_to_f64(y), ref, "experts N=%d" % N)


def _simulated_ep(m, ly, d, shape, xs, aids, G):
    """G ranks on one GPU: each routes and dispatches its tokens; the all-to-alls are row
    range copies; each owner runs its experts; each rank combines."""
    from int4_group_affine_b200.ep import CudaBackend
    bes = [CudaBackend(d, g, G) for g in range(G)]
    st = []
    for g in range(G):
        T = xs[g].shape[0]
        idx, w, sg = bes[g].route(xs[g], T)
        pos, counts, sx, meta = bes[g].dispatch(xs[g], idx, aids[g], T)
        st.append((idx, w, sg, pos, counts, sx, meta))
    offs = [np.concatenate([[0], np.cumsum(s[4])]) for s in st]
    outs = []
    for dst in range(G):  # owner dst receives, from every source in rank order, its row range
        rows = torch.cat([st[g][5][offs[g][dst]:offs[g][dst + 1]] for g in range(G)])
        meta = torch.cat([st[g][6][offs[g][dst]:offs[g][dst + 1]] for g in range(G)])
        outs.append(bes[dst].experts(rows, meta, rows.shape[0]))
    ys = []
    for g in range(G):  # the outputs back to their source, in its send order
        parts, k = [], 0
        for dst in range(G):
            n_before = sum(st[s][4][dst] for s in range(g))
            parts.append(outs[dst][n_before:n_before + st[g][4][dst]])
        ret = torch.cat(parts)
        idx, w, sg, pos = st[g][:4]
        sh = bes[g].shared(xs[g], aids[g], xs[g].shape[0])
        ys.append(bes[g].combine(ret, pos, w, sh, sg, xs[g].shape[0]))
    return ys


@pytest.mark.parametrize("G", [1, 2, 8])
def test_simulated_expert_parallel_forward(layer, G):
    m, ly = _mods()
    shape, t = layer
    d = ly.DeviceLayer.from_host(shape, t)
    L = oracle_layer(shape, t)
    xs_h, aids_h = [], []
    for g in range(G):
        x, aid = workloads.moe_inputs(shape, seed=60 + g, T=3 + 2 * g)
        xs_h.append(x)
        aids_h.append(aid)
    ys = _simulated_ep(m, ly, d, shape, [ly.to_device(x) for x in xs_h], [ly.to_device(a) for a in aids_h], G)
    torch.cuda.synchronize()
    for g in range(G):
        y_ref = L.ffn(xs_h[g], aids_h[g])[0]
        assert_close_output(bf16_dev_to_f64(ys[g]), y_ref, "EP G=%d rank %d" % (G, g))


def test_ep_forward_one_rank_nccl_group(layer):
    """ep_forward itself (the NCCL all-to-alls included) in a one-rank group against the
    single-GPU forward."""
    import torch.distributed as dist
    from int4_group_affine_b200.ep import CudaBackend, ep_forward
    m, ly = _mods()
    shape, t = layer
    d = ly.DeviceLayer.from_host(shape, t)
    x, aid = workloads.moe_inputs(shape, seed=70, T=6)
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0, world_size=1)
    try:
        y = ep_forward(CudaBackend(d, 0, 1), None, ly.to_device(x), ly.to_device(aid), 6)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    y_ref = oracle_layer(shape, t).ffn(x, aid)[0]
    assert_close_output(bf16_dev_to_f64(y), y_ref, "ep_forward world 1")
