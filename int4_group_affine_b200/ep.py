"""Expert parallelism of the MoE layer over a torch.distributed group (one process per GPU).

Rank g of G owns experts [g E/G, (g+1) E/G) of each layer; the router and the shared
expert are replicated on every rank.  A forward of a rank's own tokens:

  1. route them (router GEMV, softmax, top-K: libmoeq's router kernels),
  2. put their routed jobs in send order, rank-major (libmoeq's dispatch kernel),
  3. exchange the row counts, then the rows and their {expert, adapter} (all-to-all),
  4. run the owned experts on the rows received (libmoeq's expert kernels),
  5. send the outputs back (the reverse all-to-all),
  6. run the shared expert on the own tokens and combine, in fixed order, the routed
     outputs weighted by their routing weights plus the gated shared output.

The collectives are NCCL's through torch.distributed; every step of the arithmetic
runs in libmoeq's kernels (``CudaBackend``).  The orchestration takes the backend as
an argument, so that the exchange logic can be exercised with any implementation of
the same steps.  The expert outputs cross the all-to-all as bf16 (the single-GPU
forward keeps them in fp32 until its combine).
"""
from __future__ import annotations

import ctypes

import torch

from . import (Layer, moe_ep_combine, moe_ep_dispatch, moe_experts_forward, moe_experts_workspace_bytes,
               moe_router_topk, moe_workspace_init)


def ep_forward(backend, group, x, adapter_id, T: int):
    """The expert-parallel forward of this rank's T tokens (x [T, H]); returns y [T, H]."""
    import torch.distributed as dist
    idx, w, sg = backend.route(x, T)
    pos, counts, send_x, send_meta = backend.dispatch(x, idx, adapter_id, T)
    dev = backend.comm_device
    cnt = torch.tensor(counts, dtype=torch.int64, device=dev)
    rcnt = torch.empty_like(cnt)
    dist.all_to_all_single(rcnt, cnt, group=group)
    recv_counts = [int(v) for v in rcnt.tolist()]
    n_send, n_recv = sum(counts), sum(recv_counts)
    recv_x = backend.rows(n_recv)
    dist.all_to_all_single(recv_x, send_x[:n_send], output_split_sizes=recv_counts, input_split_sizes=counts,
                           group=group)
    recv_meta = backend.meta(n_recv)
    dist.all_to_all_single(recv_meta, send_meta[:n_send], output_split_sizes=recv_counts,
                           input_split_sizes=counts, group=group)
    y_rows = backend.experts(recv_x, recv_meta, n_recv)
    ret = backend.rows(n_send)
    dist.all_to_all_single(ret, y_rows, output_split_sizes=counts, input_split_sizes=recv_counts, group=group)
    shared = backend.shared(x, adapter_id, T)
    return backend.combine(ret, pos, w, shared, sg, T)


def _slice_q(q, lo: int, n: int):
    """View of experts [lo, lo + n) of an expert-stacked affine tensor descriptor."""
    from . import QTensor
    s = QTensor()
    words = q.out * q.in_ * q.bits // 32
    groups = q.out * (q.in_ // q.group)
    s.packed = q.packed + lo * words * 4
    s.scales = q.scales + lo * groups * 2
    s.biases = q.biases + lo * groups * 2
    s.n, s.out, s.in_, s.bits, s.group = n, q.out, q.in_, q.bits, q.group
    return s


class CudaBackend:
    """Every step of the expert-parallel forward in libmoeq's kernels on the current device.

    ``layer`` is a DeviceLayer holding the whole layer; only the descriptor of the owned
    slice of experts and the replicated router and shared expert are used (a rank that
    holds only its slice can build the same descriptors over its own tensors)."""

    def __init__(self, layer, rank: int, world: int):
        L = layer.L
        self.H, self.E, self.K = L.hidden, L.n_experts, L.top_k
        if self.E % world:
            raise ValueError("experts must split evenly over the ranks")
        self.world, self.rank = world, rank
        self.per = self.E // world
        self.lo = rank * self.per
        self.layer = layer
        self.full = L
        self.comm_device = torch.device("cuda", torch.cuda.current_device())
        # the owned slice: experts [lo, lo + per), their LoRA factors, the full router
        sl = Layer()
        ctypes.memmove(ctypes.byref(sl), ctypes.byref(L), ctypes.sizeof(Layer))
        sl.n_experts = self.per
        sl.top_k = 1
        sl.gate, sl.up, sl.down = (_slice_q(L.gate, self.lo, self.per), _slice_q(L.up, self.lo, self.per),
                                   _slice_q(L.down, self.lo, self.per))
        sl.router = _slice_q(L.router, 0, 1)  # the first rows of the router: never read by this forward
        sl.router.out = self.per
        r = L.rank
        for a in range(L.n_adapters):
            for proj, (out, in_) in (("gate", (L.inter, L.hidden)), ("up", (L.inter, L.hidden)),
                                     ("down", (L.hidden, L.inter))):
                src = getattr(L.lora[a], proj)
                dst = getattr(sl.lora[a], proj)
                if src.A and src.B:
                    dst.A = src.A + self.lo * r * in_ * 2
                    dst.B = src.B + self.lo * out * r * 2
        self.slice = sl
        # the shared expert as the only routed expert of a one-expert layer
        self.shared_layer = None
        if L.s_gate.packed:
            sh = Layer()
            ctypes.memmove(ctypes.byref(sh), ctypes.byref(L), ctypes.sizeof(Layer))
            sh.n_experts, sh.top_k, sh.inter = 1, 1, L.shared_inter
            sh.gate, sh.up, sh.down = L.s_gate, L.s_up, L.s_down
            sh.router = L.shared_gate if L.shared_gate.packed else _slice_q(L.router, 0, 1)
            if not L.shared_gate.packed:
                sh.router.out = 1
            for a in range(L.n_adapters):
                for proj in ("gate", "up", "down"):
                    setattr(sh.lora[a], proj, getattr(L.lora[a], "s_" + proj))
            self.shared_layer = sh

    # ------------------------------------------------------------ buffers
    def rows(self, n):
        return torch.empty((n, self.H), dtype=torch.bfloat16, device=self.comm_device)

    def meta(self, n):
        return torch.empty((n, 2), dtype=torch.int32, device=self.comm_device)

    def _ws(self, layer, n):
        nb = moe_experts_workspace_bytes(layer, n)
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=self.comm_device)
        moe_workspace_init(ws, ws.numel())
        return ws, nb

    # ------------------------------------------------------------ steps
    def route(self, x, T):
        L = self.full
        dev = self.comm_device
        idx = torch.empty((T, self.K), dtype=torch.int32, device=dev)
        w = torch.empty((T, self.K), dtype=torch.float32, device=dev)
        sg = torch.empty(T, dtype=torch.float32, device=dev)
        logits = torch.empty((T, self.E), dtype=torch.float32, device=dev)
        lb = self.layer.t.get("logit_bias")
        moe_router_topk(x, L.router, L.shared_gate if L.shared_gate.packed else None, lb, T, self.H, self.E,
                        self.K, idx, w, sg, logits)
        return idx, w, sg

    def dispatch(self, x, idx, adapter_id, T):
        dev = self.comm_device
        J = T * self.K
        pos = torch.empty((T, self.K), dtype=torch.int32, device=dev)
        counts = torch.zeros(self.world, dtype=torch.int32, device=dev)
        send_x = torch.empty((max(J, 1), self.H), dtype=torch.bfloat16, device=dev)
        send_meta = torch.empty((max(J, 1), 2), dtype=torch.int32, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        moe_ep_dispatch(x, idx, adapter_id, self.full.n_adapters, T, self.K, self.H, self.E, self.world, pos,
                        counts, send_x, send_meta, status)
        self.status = status
        return pos, [int(v) for v in counts.tolist()], send_x, send_meta

    def experts(self, rows, meta, n):
        out = self.rows(n)
        if n == 0:
            return out
        local = (meta[:, 0] - self.lo).contiguous()
        aid = meta[:, 1].contiguous()
        ws, nb = self._ws(self.slice, n)
        moe_experts_forward(self.slice, rows, local, aid, n, out, ws, nb)
        return out

    def shared(self, x, adapter_id, T):
        if self.shared_layer is None:
            return None
        out = self.rows(T)
        zero = torch.zeros(T, dtype=torch.int32, device=self.comm_device)
        ws, nb = self._ws(self.shared_layer, T)
        moe_experts_forward(self.shared_layer, x, zero, adapter_id, T, out, ws, nb)
        return out

    def combine(self, ret, pos, w, shared, sg, T):
        y = torch.empty((T, self.H), dtype=torch.int16, device=self.comm_device)
        moe_ep_combine(ret, pos, w, shared, sg if shared is not None else None, T, self.K, self.H, y)
        return y
