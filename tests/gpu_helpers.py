"""Shared pieces of the GPU parity tests: device upload, tolerances, near-tie handling."""
from __future__ import annotations

import contextlib
import itertools

import numpy as np
import pytest

import oracle
import synth
from tests.helpers import oracle_layer, quantize_layer, rel_l2

torch = pytest.importorskip("torch")

# Output tolerance of the method: relative L2 <= 5e-3 and max |diff| <= 1e-2 max |y_ref|.
REL_L2 = 5e-3
MAX_ABS_FRAC = 1e-2
# Routing decisions closer than this (K-th vs (K+1)-th logit) may legitimately differ.
TIE_GAP = 1e-4


def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from int4_group_affine_b200 import build
    build.build()


def assert_close_output(y_gpu, y_ref, what=""):
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    r = rel_l2(y_gpu, y_ref)
    m = float(np.max(np.abs(y_gpu - y_ref))) if y_ref.size else 0.0
    bound = MAX_ABS_FRAC * float(np.max(np.abs(y_ref))) if y_ref.size else 0.0
    assert r <= REL_L2, "%s rel-L2 %.3e > %.1e" % (what, r, REL_L2)
    assert m <= bound, "%s max-abs %.3e > %.3e" % (what, m, bound)
    return r, m


def bf16_dev_to_f64(t):
    from int4_group_affine_b200.layer import to_host
    return synth.bf16_to_f32(to_host(t, np.uint16)).astype(np.float64)


def near_tie_tokens(logits: np.ndarray, K: int) -> np.ndarray:
    """Tokens whose K-th and (K+1)-th largest oracle logits are closer than TIE_GAP."""
    if logits.shape[1] <= K:
        return np.zeros(logits.shape[0], bool)
    s = -np.sort(-logits, axis=1)
    return (s[:, K - 1] - s[:, K]) < TIE_GAP


def alternative_sets(z: np.ndarray, K: int):
    """Every top-K expert set consistent with the oracle logits z up to TIE_GAP ties."""
    order = sorted(range(len(z)), key=lambda e: (-z[e], e))
    zk = z[order[K - 1]]
    sure = [e for e in order if z[e] > zk + TIE_GAP]
    window = [e for e in order if abs(z[e] - zk) <= TIE_GAP]
    need = K - len(sure)
    out = []
    for comb in itertools.combinations(window, need):
        s = sure + list(comb)
        out.append(sorted(s, key=lambda e: (-z[e], e)))
    return out


def check_routing(idx_gpu, idx_ref, logits_ref, K):
    """Routing indices against the oracle's, bit-exact outside near ties.

    A token whose K-th and (K+1)-th oracle logits are closer than TIE_GAP may take any
    top-K set those logits allow.  Every other token must pick exactly the oracle's set,
    in the oracle's order, except that two picks whose oracle logits are within TIE_GAP
    of each other may come in either order.  Returns the boundary-tie mask."""
    idx_gpu = np.asarray(idx_gpu)
    ties = near_tie_tokens(logits_ref, K)
    for t in range(idx_gpu.shape[0]):
        got = idx_gpu[t].tolist()
        if ties[t]:
            alts = [sorted(a) for a in alternative_sets(logits_ref[t], K)]
            assert sorted(got) in alts, (t, got)
            continue
        ref = idx_ref[t].tolist()
        assert sorted(got) == sorted(ref), (t, got, ref)
        for k in range(K):
            if got[k] != ref[k]:
                assert abs(logits_ref[t][got[k]] - logits_ref[t][ref[k]]) < TIE_GAP, (t, got, ref)
    return ties


def check_weights(idx_gpu, w_gpu, idx_ref, w_ref, ties, rtol=2e-5, atol=1e-6):
    """Renormalised routing weights of the tokens outside near ties, matched by expert
    (a weight depends on the chosen set, not on the order of the picks)."""
    for t in np.nonzero(~ties)[0]:
        g = dict(zip(np.asarray(idx_gpu[t]).tolist(), np.asarray(w_gpu[t], np.float64).tolist()))
        r = dict(zip(np.asarray(idx_ref[t]).tolist(), np.asarray(w_ref[t], np.float64).tolist()))
        assert g.keys() == r.keys(), t
        for e in r:
            assert abs(g[e] - r[e]) <= atol + rtol * abs(r[e]), (t, e, g[e], r[e])


@contextlib.contextmanager
def decode_path(m, path):
    """Runs the block with the single-kernel decode choice set to `path` (None: unchanged)."""
    old = m.moe_decode_path()
    if path is not None:
        m.moe_set_decode_path(path)
    try:
        yield
    finally:
        m.moe_set_decode_path(old)


def forward_with_record(m, d, xd, ad, T, ws, nb, block_eps=None, decode=None):
    """One forward through the C ABI with the library's launch record on: returns the
    routing the call used (from moe_ffn_routing) and the kernel kinds it launched.
    `decode` forces one single-kernel decode (m.DECODE_CHAIN / m.DECODE_BARRIER)."""
    K = d.K
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    y = torch.empty_like(xd)
    m.moe_timing_enable(True)
    try:
        if decode is not None:
            m.moe_set_decode_path(decode)
        if block_eps is None:
            m.moe_ffn_forward(d.L, xd, ad, T, y, ws, nb)
        else:
            m.moe_block_forward(d.L, xd, ad, T, block_eps, y, ws, nb)
        m.moe_ffn_routing(d.L, T, ws, nb, idx, w)
        torch.cuda.synchronize()
        kinds = set(m.moe_timing_collect())
    finally:
        m.moe_timing_enable(False)
        m.moe_set_decode_path(m.DECODE_AUTO)
    assert m.moe_get_device_status(ws) == 0
    return y, idx.cpu().numpy(), w.cpu().numpy(), kinds


# kernel kinds that identify each execution path of the forward: "chain", "fused" and
# "cluster" are the single-kernel decode paths (chain, barrier and cluster kernels),
# "decode" any of them
PATH_KINDS = {"chain": {"decode_chain"}, "fused": {"decode_fused"}, "cluster": {"decode_cluster"},
              "cuda_core": {"gate_up", "down"},
              "tensor_core": {"tc_gate_up", "tc_down"}}


def path_ran(path, kinds):
    if path == "decode":
        return bool({"decode_chain", "decode_fused", "decode_cluster"} & kinds)
    return PATH_KINDS[path] <= kinds


def oracle_for_gpu_routing(L, x, aid, idx_gpu, logits_ref, y_ref):
    """Oracle output per token, re-evaluated (from oracle-derived alternatives) where the
    GPU resolved a near tie differently."""
    K = idx_gpu.shape[1]
    y = y_ref.copy()
    ties = near_tie_tokens(logits_ref, K)
    for t in np.nonzero(ties)[0]:
        for alt in alternative_sets(logits_ref[t], K):
            if sorted(alt) == sorted(idx_gpu[t].tolist()):
                sel = np.array([alt], np.int32)
                a = None if aid is None else aid[t:t + 1]
                y[t] = L.ffn(x[t:t + 1], a, select=sel)[0][0]
    return y
