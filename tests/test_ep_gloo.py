"""Expert parallelism's exchange logic with two gloo ranks on the CPU.

ep.ep_forward runs unchanged; its steps come from a backend written here from the
definitions (routing and experts by the oracle, the stable rank-major dispatch and the
fixed-order combine in numpy).  Each rank owns half of the experts and routes its own
tokens; the result must equal the oracle's single-process forward of those tokens."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _shape():
    from synth import workloads
    import dataclasses
    return dataclasses.replace(workloads.TINY, n_adapters=2, random_adapters=True)


class OracleBackend:
    """The steps of the expert-parallel forward on the CPU, from their definitions."""

    def __init__(self, shape, t, rank, world):
        import torch
        from tests.helpers import oracle_layer
        import oracle
        self.torch, self.oracle = torch, oracle
        self.shape, self.rank, self.world = shape, rank, world
        self.per = shape.E // world
        self.lo = rank * self.per
        self.full = oracle_layer(shape, t)
        # experts only (no shared expert, top-1) and the shared expert alone
        tx = dict(t)
        for k in ("s_gate", "s_up", "s_down", "sgate"):
            for suf in ("_p", "_s", "_b"):
                tx[k + suf] = None
        self.experts_layer = oracle.OracleLayer(shape.H, shape.E, 1, shape.I, 0, tx, rank=shape.rank,
                                                alpha=shape.alpha, group=shape.group)
        self.comm_device = torch.device("cpu")

    def rows(self, n):
        return self.torch.empty((n, self.shape.H), dtype=self.torch.float64)

    def meta(self, n):
        return self.torch.empty((n, 2), dtype=self.torch.int32)

    def route(self, x, T):
        y, idx, w, sg, z = self.full.ffn(x, self.aid)
        self.y_ref = y
        return idx, w, sg

    def dispatch(self, x, idx, adapter_id, T):
        K = idx.shape[1]
        owner = idx.reshape(-1) // self.per
        order = np.argsort(owner, kind="stable")  # rank-major, job order within a rank
        pos = np.empty(T * K, np.int64)
        pos[order] = np.arange(T * K)
        counts = [int(np.sum(owner == g)) for g in range(self.world)]
        tok = np.repeat(np.arange(T), K)
        xs = __import__("synth").bf16_to_f32(x).astype(np.float64)
        send_x = self.torch.from_numpy(xs[tok[order]])
        aid = adapter_id if adapter_id is not None else np.zeros(T, np.int32)
        meta = np.stack([idx.reshape(-1)[order], aid[tok[order]]], axis=1).astype(np.int32)
        return pos.reshape(T, K), counts, send_x, self.torch.from_numpy(meta)

    def experts(self, rows, meta, n):
        out = self.rows(n)
        import synth
        for i in range(n):
            e, a = int(meta[i, 0]), int(meta[i, 1])
            assert self.lo <= e < self.lo + self.per  # only owned experts arrive here
            xb = synth.bf16(rows[i].numpy().astype(np.float32))[None]
            out[i] = self.torch.from_numpy(self.experts_layer.ffn(xb, np.array([a], np.int32),
                                                                 select=np.array([[e]], np.int32))[0][0])
        return out

    def shared(self, x, adapter_id, T):
        return None  # folded into the combine below from the full forward

    def combine(self, ret, pos, w, shared, sg, T):
        r = ret.numpy()
        y = np.zeros((T, self.shape.H))
        for t in range(T):
            for k in range(w.shape[1]):
                y[t] += w[t, k] * r[pos[t, k]]
        return y


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from synth import workloads
        from tests.helpers import quantize_layer
        from int4_group_affine_b200.ep import ep_forward
        oracle.build()
        shape = _shape()
        t = quantize_layer(workloads.moe_weights(shape, seed=31))
        x, aid = workloads.moe_inputs(shape, seed=32 + rank, T=6 + rank)
        be = OracleBackend(shape, t, rank, world)
        be.aid = aid
        y_routed = ep_forward(be, None, x, aid, x.shape[0])
        # the routed part of the oracle's own forward: its output less the gated shared expert
        full_y, idx, w, sg, _ = be.full.ffn(x, aid)
        tx = dict(t)
        for k in ("s_gate", "s_up", "s_down"):
            for suf in ("_p", "_s", "_b"):
                tx[k + suf] = None
        routed_only = oracle.OracleLayer(shape.H, shape.E, shape.K, shape.I, 0, tx, rank=shape.rank,
                                         alpha=shape.alpha).ffn(x, aid)[0]
        err = float(np.max(np.abs(y_routed - routed_only)) / np.max(np.abs(routed_only)))
        q.put((rank, err))
    finally:
        dist.destroy_process_group()


def test_ep_exchange_two_gloo_ranks():
    import torch.multiprocessing as mp
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ps = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
    assert all(p.exitcode == 0 for p in ps), [p.exitcode for p in ps]
    res = dict(q.get() for _ in range(2))
    assert set(res) == {0, 1}
    for r, err in res.items():
        assert err < 1e-12, (r, err)
