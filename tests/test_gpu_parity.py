"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the same seeded inputs.

Integer work (packing, codes, routing indices, job lists) must be bit-exact;
floating-point outputs must meet rel-L2 <= 5e-3 and max-abs <= 1e-2 max|y_ref|.
"""
import dataclasses

import numpy as np
import pytest

import oracle
import synth
from synth import workloads
from tests.gpu_helpers import (PATH_KINDS, REL_L2, TIE_GAP, path_ran, assert_close_output, bf16_dev_to_f64, check_routing,
                               check_weights, forward_with_record, need_cuda, near_tie_tokens,
                               oracle_for_gpu_routing)
from tests.helpers import oracle_layer, quantize_layer, rel_l2

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    need_cuda()


def _mods():
    import int4_group_affine_b200 as m
    from int4_group_affine_b200 import layer as ly
    return m, ly


# ------------------------------------------------------------------ packing
def _special_rows(W):
    W = W.copy()
    W[0, :64] = 0.0            # zero group
    W[1, 64:128] = 0.5         # constant bf16-exact group
    W[2, :64] = 0.0123         # constant, not bf16-exact
    W[3, :32] = -0.0
    W[3, 32:64] = 0.0          # signed zeros mixed
    return W


@pytest.mark.parametrize("bits,group", [(4, 64), (8, 64), (4, 32), (8, 32)])
def test_pack_affine_bit_exact(bits, group):
    m, ly = _mods()
    W = _special_rows(synth.normal(100 + bits, "pack", (37, 512), std=0.02, outlier_prob=1e-2, outlier_factor=20.0))
    p, s, b = oracle.quant_affine(W, bits, group)
    Wd = ly.to_device(W)
    pd = torch.empty((37, 512 * bits // 32), dtype=torch.int32, device="cuda")
    sd = torch.empty((37, 512 // group), dtype=torch.int16, device="cuda")
    bd = torch.empty_like(sd)
    m.moe_quant_pack(m.FMT_AFFINE_INT4 if bits == 4 else m.FMT_AFFINE_INT8, Wd, 37, 512, group, 0.0, pd, sd, bd)
    torch.cuda.synchronize()
    assert np.array_equal(ly.to_host(pd, np.uint32), p)
    assert np.array_equal(ly.to_host(sd, np.uint16), s)
    assert np.array_equal(ly.to_host(bd, np.uint16), b)


@pytest.mark.parametrize("bits", [4, 8])
def test_dequant_bit_exact_zero_error(bits):
    m, ly = _mods()
    W = synth.normal(110 + bits, "deq", (3, 5, 256), std=0.02, outlier_prob=1e-2, outlier_factor=20.0)
    p, s, b = oracle.quant_affine(W, bits, 64)
    ref = oracle.dequant_affine(p, s, b, 256, bits, 64)
    t = m.QTensor()
    pd, sd, bd = ly.to_device(p), ly.to_device(s), ly.to_device(b)
    t.packed, t.scales, t.biases = pd.data_ptr(), sd.data_ptr(), bd.data_ptr()
    t.n, t.out, t.in_, t.bits, t.group = 3, 5, 256, bits, 64
    out = torch.empty((3, 5, 256), dtype=torch.float32, device="cuda")
    m.moe_dequant(t, out)
    torch.cuda.synchronize()
    assert np.max(np.abs(out.cpu().numpy() - ref)) == 0.0


@pytest.mark.parametrize("rho", [0.25, 0.5, 1 / 3, 0.0, 1.0, 0.125])
def test_pack_mixed_bit_exact(rho):
    m, ly = _mods()
    W = synth.normal(120, "mpack", (37, 192), std=0.02, outlier_prob=1e-2, outlier_factor=20.0)
    p, s = oracle.quant_mixed(W, rho)
    dm = ly.DeviceMixed.from_fp32(ly.to_device(W), rho)
    torch.cuda.synchronize()
    assert np.array_equal(ly.to_host(dm.packed, np.uint32), p)
    assert np.array_equal(ly.to_host(dm.scales, np.uint16), s)
    out = torch.empty((37, 192), dtype=torch.float32, device="cuda")
    m.moe_mixed_dequant(dm.T, out)
    torch.cuda.synchronize()
    assert np.max(np.abs(out.cpu().numpy() - oracle.dequant_mixed(p, s, 37, 192, rho))) == 0.0


# ------------------------------------------------------------------ router
def _router_case(shape, seed, T):
    w = workloads.moe_weights(shape, seed=seed)
    t = quantize_layer(w)
    L = oracle_layer(shape, t)
    x, aid = workloads.moe_inputs(shape, seed=seed, T=T)
    return t, L, x, aid


def _gpu_router(t, shape, x, T):
    m, ly = _mods()
    d = ly.DeviceLayer.from_host(shape, t)
    xd = ly.to_device(x)
    E, K = shape.E, shape.K
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    sg = torch.empty(T, dtype=torch.float32, device="cuda")
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    lb = d.t.get("logit_bias")
    m.moe_router_topk(xd, d.L.router, d.L.shared_gate, lb, T, shape.H, E, K, idx, w, sg, logits)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy(), sg.cpu().numpy(), logits.cpu().numpy()


@pytest.mark.parametrize("shape,T", [(workloads.TINY, 4), (workloads.TINY, 37),
                                     (dataclasses.replace(workloads.TINY, K=1), 9),
                                     (dataclasses.replace(workloads.TINY, K=8), 9),
                                     (dataclasses.replace(workloads.TINY, logit_bias_std=1.0), 40)])
def test_router_topk_tiny(shape, T):
    t, L, x, _ = _router_case(shape, 200, T)
    idx, w, sg, logits = _gpu_router(t, shape, x, T)
    y, idx_r, w_r, sg_r, logits_r = L.ffn(x)
    assert np.allclose(logits, logits_r, rtol=1e-5, atol=1e-5)
    ties = check_routing(idx, idx_r, logits_r, shape.K)
    assert np.allclose(w[~ties], w_r[~ties], rtol=1e-5, atol=1e-6)
    assert np.allclose(sg, sg_r, rtol=1e-6, atol=1e-6)


def test_router_equal_logits_take_lower_index():
    m, ly = _mods()
    shape = dataclasses.replace(workloads.TINY, K=3)
    w = workloads.moe_weights(shape, seed=201)
    w["router"][:] = 0.0
    t = quantize_layer(w)
    x, _ = workloads.moe_inputs(shape, seed=201, T=5)
    idx, wts, _, _ = _gpu_router(t, shape, x, 5)
    assert np.all(idx == np.array([0, 1, 2]))
    assert np.allclose(wts, 1 / 3, rtol=1e-6)


# ------------------------------------------------------------------ index build
@pytest.mark.parametrize("T,K,E,na", [(1, 4, 256, 1), (5, 2, 8, 0), (37, 4, 16, 4), (100, 8, 64, 2),
                                      (64, 4, 256, 4), (2048, 4, 256, 1)])
def test_index_build_bit_exact(T, K, E, na):
    m, ly = _mods()
    z = synth.normal(300 + T, "ib/z", (T, E)).astype(np.float64)
    idx, _ = oracle.topk(z, K)
    aid = synth.randint(300 + T, "ib/a", (T,), -1, na - 1) if na > 1 else None
    counts, offsets, perm = oracle.index_build(idx, aid, E, na)
    nbytes = m.moe_index_workspace_bytes(T, K, E, na)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    c = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    o = torch.empty(E + 2, dtype=torch.int32, device="cuda")
    p = torch.empty((T * (K + 1), 4), dtype=torch.int32, device="cuda")
    ad = None if aid is None else ly.to_device(aid)
    m.moe_index_build(ly.to_device(idx), ad, T, K, E, na, c, o, p, ws, nbytes)
    torch.cuda.synchronize()
    assert np.array_equal(c.cpu().numpy(), counts)
    assert np.array_equal(o.cpu().numpy(), offsets)
    assert np.array_equal(p.cpu().numpy(), perm)
    assert m.moe_get_device_status(ws) == 0


def test_index_build_flags_out_of_range():
    m, ly = _mods()
    T, K, E = 6, 2, 8
    idx = np.array([[0, 1]] * T, np.int32)
    idx[2, 1] = 9   # expert out of range
    aid = np.array([0, 0, 0, 5, 0, 0], np.int32)  # adapter out of range
    nbytes = m.moe_index_workspace_bytes(T, K, E, 1)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    c = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    o = torch.empty(E + 2, dtype=torch.int32, device="cuda")
    p = torch.empty((T * (K + 1), 4), dtype=torch.int32, device="cuda")
    m.moe_index_build(ly.to_device(idx), ly.to_device(aid), T, K, E, 1, c, o, p, ws, nbytes)
    assert m.moe_get_device_status(ws) == 5
    assert m.moe_get_device_status(ws) == 0  # read-and-clear
    assert int(o.cpu().numpy()[-1]) == T * (K + 1)


# ------------------------------------------------------------------ FFN tiny
def _gpu_ffn(d, x, aid=None, block_eps=None):
    m, ly = _mods()
    T = x.shape[0]
    xd = ly.to_device(x)
    ad = None if aid is None else ly.to_device(aid)
    ws, nb = d.workspace(T)
    y = torch.empty_like(xd)
    if block_eps is None:
        m.moe_ffn_forward(d.L, xd, ad, T, y, ws, nb)
    else:
        m.moe_block_forward(d.L, xd, ad, T, block_eps, y, ws, nb)
    torch.cuda.synchronize()
    assert m.moe_get_device_status(ws) == 0
    return y


def _ffn_case(shape, seed, T=None, n_adapters=None, lora_zero_B=False):
    w = workloads.moe_weights(shape, seed=seed, lora_zero_B=lora_zero_B)
    t = quantize_layer(w)
    x, aid = workloads.moe_inputs(shape, seed=seed, T=T)
    return t, x, aid


def _check_ffn(shape, t, x, aid, n_adapters=None, what="", path=None, decode=None):
    """The forward against the oracle: the routing the forward itself used (bit-exact
    outside near ties, weights within fp32 rounding), then the output, with near ties
    resolved by the forward's own choice.  `path` names the kernels the call must run;
    `decode` forces one of the single-kernel decodes."""
    m, ly = _mods()
    L = oracle_layer(shape, t, n_adapters=n_adapters)
    d = ly.DeviceLayer.from_host(shape, t, n_adapters=n_adapters)
    T = x.shape[0]
    ws, nb = d.workspace(T)
    yd, idx_g, w_g, kinds = forward_with_record(m, d, ly.to_device(x), None if aid is None else ly.to_device(aid),
                                                T, ws, nb, decode=decode)
    if path is not None:
        assert path_ran(path, kinds), (what, path, kinds)
    y = bf16_dev_to_f64(yd)
    y_ref, idx_r, w_r, _, logits_r = L.ffn(x, aid)
    ties = check_routing(idx_g, idx_r, logits_r, shape.K)
    check_weights(idx_g, w_g, idx_r, w_r, ties)
    if ties.any():
        y_ref = oracle_for_gpu_routing(L, x, aid, idx_g, logits_r, y_ref)
    return assert_close_output(y, y_ref, what), y, y_ref


@pytest.mark.parametrize("T", [4, 1, 12, 37, 70])
def test_ffn_tiny(T):
    """One token: the cluster decode kernel by default, then the barrier and chain kernels
    forced; up to four tokens at top-2: the barrier kernel by default, then the chain
    kernel forced; more tokens: the tensor-core path."""
    m, _ = _mods()
    shape = workloads.TINY
    t, x, aid = _ffn_case(shape, 400, T=T)
    auto = "cluster" if T == 1 else "fused" if T <= 4 else "tensor_core"
    _check_ffn(shape, t, x, aid, what="tiny T=%d" % T, path=auto)
    if T <= 4:
        _check_ffn(shape, t, x, aid, what="tiny T=%d chain" % T, path="chain", decode=m.DECODE_CHAIN)
    if T == 1:
        _check_ffn(shape, t, x, aid, what="tiny T=1 barrier", path="fused", decode=m.DECODE_BARRIER)


@pytest.mark.parametrize("T", [5, 6])
def test_ffn_tiny_fused_decode_path(T):
    """Five to eight tokens with at most 32 jobs: the older fused decode kernel (grid
    barriers, dedicated LoRA-A CTAs), which takes what the chain kernel does not."""
    shape = workloads.TINY
    t, x, aid = _ffn_case(shape, 405, T=T)
    _check_ffn(shape, t, x, aid, what="tiny T=%d" % T, path="fused")


@pytest.mark.parametrize("variant,T", [("kE", 4), ("kE", 8), ("rank64", 3), ("rank64", 8)])
def test_ffn_tiny_cuda_core_path(variant, T):
    """Calls the fused decode kernel declines (more than 32 jobs, or a LoRA rank above
    32) with fewer tokens than the tensor-core path takes: the multi-kernel CUDA-core
    path (router, top-K, index build, LoRA-A, gate/up, down, combine kernels)."""
    shape = workloads.TINY
    if variant == "kE":
        shape = dataclasses.replace(shape, K=shape.E)
    else:
        shape = dataclasses.replace(shape, rank=64, n_adapters=2, random_adapters=True)
    t, x, aid = _ffn_case(shape, 415, T=T)
    _check_ffn(shape, t, x, aid, what="%s T=%d" % (variant, T), path="cuda_core")


@pytest.mark.parametrize("variant", ["k1", "kE", "no_lora", "no_shared", "no_sgate", "multi_adapter", "bias",
                                     "group32", "group32_decode", "rank24", "rank64", "k1_chain", "no_lora_chain",
                                     "no_shared_chain", "no_sgate_chain", "multi_adapter_chain", "bias_chain",
                                     "rank24_chain", "k1_cluster", "kE_cluster", "no_lora_cluster",
                                     "no_shared_cluster", "no_sgate_cluster", "multi_adapter_cluster", "bias_cluster",
                                     "rank24_cluster", "group32_cluster"])
def test_ffn_tiny_variants(variant):
    """Layer variants on the tensor-core path (19 tokens), for the _chain ones on the
    chain decode kernel (3 tokens) and for the _cluster ones on the cluster decode kernel
    (one token)."""
    m, _ = _mods()
    chain = variant.endswith("_chain")
    cluster = variant.endswith("_cluster")
    variant = variant[:-6] if chain else variant[:-8] if cluster else variant
    shape = workloads.TINY
    na = None
    if variant == "k1":
        shape = dataclasses.replace(shape, K=1)
    elif variant == "kE":
        shape = dataclasses.replace(shape, K=shape.E)
    elif variant == "multi_adapter":
        shape = dataclasses.replace(shape, n_adapters=3, random_adapters=True)
    elif variant == "bias":
        shape = dataclasses.replace(shape, logit_bias_std=1.0)
    elif variant in ("group32", "group32_decode"):
        shape = dataclasses.replace(shape, group=32)
    elif variant in ("rank24", "rank64"):  # LoRA-A products wider than one 32-column warp group
        shape = dataclasses.replace(shape, rank=int(variant[4:]), n_adapters=2, random_adapters=True)
    t, x, aid = _ffn_case(shape, 410, T=1 if cluster else 3 if (variant == "group32_decode" or chain) else 19)
    if variant in ("group32", "group32_decode"):
        w = workloads.moe_weights(shape, seed=410)
        t = quantize_layer(w, group=32)
    if variant == "no_lora":
        na = 0
    if variant == "no_shared":
        for k in ("s_gate", "s_up", "s_down"):
            for suf in ("_p", "_s", "_b"):
                t[k + suf] = None
    if variant == "no_sgate":
        for suf in ("_p", "_s", "_b"):
            t["sgate" + suf] = None
    if variant == "multi_adapter":
        aid = aid.copy()
        aid[::5] = -1  # some tokens with the base only
    if variant == "multi_adapter" and cluster:
        aid = np.array([2], np.int32)  # (one token: an adapter other than the first)
    _check_ffn(shape, t, x, aid, n_adapters=na,
               what=variant + (" (chain)" if chain else " (cluster)" if cluster else ""),
               path="chain" if chain else "cluster" if cluster else ("decode" if variant == "group32_decode" else None),
               decode=m.DECODE_CHAIN if chain else m.DECODE_CLUSTER if cluster else None)


def test_zero_B_equals_base_bitwise():
    _, ly = _mods()
    shape = workloads.TINY
    t, x, _ = _ffn_case(shape, 420, T=9, lora_zero_B=True)
    y0 = _gpu_ffn(ly.DeviceLayer.from_host(shape, t), x)
    yb = _gpu_ffn(ly.DeviceLayer.from_host(shape, t, n_adapters=0), x)
    assert torch.equal(y0, yb)


def test_planted_swap_is_caught():
    # The tolerance separates the method from its most likely wiring mistake:
    # the GPU output must be far from an oracle with SiLU on the up branch.
    _, ly = _mods()
    shape = workloads.TINY
    t, x, aid = _ffn_case(shape, 430, T=8)
    d = ly.DeviceLayer.from_host(shape, t)
    y = bf16_dev_to_f64(_gpu_ffn(d, x))
    L = oracle_layer(shape, t)
    oracle.set_mutation(oracle.MUTATION_SWAP_GATE_UP)
    try:
        ym = L.ffn(x)[0]
    finally:
        oracle.set_mutation(oracle.MUTATION_NONE)
    assert rel_l2(y, ym) > 20 * REL_L2


def test_bad_adapter_flags_status_and_falls_back_to_base():
    m, ly = _mods()
    shape = dataclasses.replace(workloads.TINY, n_adapters=2)
    t, x, _ = _ffn_case(shape, 440, T=4)
    aid = np.array([0, 7, 1, -1], np.int32)
    d = ly.DeviceLayer.from_host(shape, t)
    xd = ly.to_device(x)
    ws, nb = d.workspace(4)
    y = torch.empty_like(xd)
    m.moe_ffn_forward(d.L, xd, ly.to_device(aid), 4, y, ws, nb)
    assert m.moe_get_device_status(ws) == 5
    aid_ok = aid.copy()
    aid_ok[1] = -1
    y2 = torch.empty_like(xd)
    m.moe_ffn_forward(d.L, xd, ly.to_device(aid_ok), 4, y2, ws, nb)
    torch.cuda.synchronize()
    assert m.moe_get_device_status(ws) == 0
    assert torch.equal(y, y2)


@pytest.mark.parametrize("T,kernel", [(3, "chain"), (1, "chain"), (1, "cluster")])
def test_block_tiny_single_kernel(T, kernel):
    """The pre-norm residual block on the chain and cluster decode kernels (RMSNorm inside)."""
    m, ly = _mods()
    shape = workloads.TINY
    t, x, aid = _ffn_case(shape, 455, T=T)
    L = oracle_layer(shape, t)
    d = ly.DeviceLayer.from_host(shape, t)
    ws, nb = d.workspace(T)
    yd, idx_g, _, kinds = forward_with_record(m, d, ly.to_device(x), None, T, ws, nb, block_eps=1e-6,
                                              decode=m.DECODE_CHAIN if kernel == "chain" else m.DECODE_CLUSTER)
    assert path_ran(kernel, kinds), kinds
    ref = synth.bf16_to_f32(L.block(x, eps=1e-6)).astype(np.float64)
    assert_close_block(bf16_dev_to_f64(yd), ref, synth.bf16_to_f32(x).astype(np.float64))


def test_bounded_wait_runs_out_and_reports_timeout():
    """A bounded device wait that cannot be satisfied gives up, reports MOE_ERR_TIMEOUT and
    leaves the context usable.  The chain decode kernel's ticket counter (the first word of
    its region, right after the 256-byte workspace header) is set to 1 instead of a multiple
    of the grid, so one CTA takes a different epoch from the others and waits for words and
    counts that never come; with a 2 ms wait limit it gives up.  After re-initialising the
    workspace the same call runs normally."""
    m, ly = _mods()
    shape = workloads.TINY
    t, x, aid = _ffn_case(shape, 470, T=1)
    d = ly.DeviceLayer.from_host(shape, t)
    ws, nb = d.workspace(1)
    xd = ly.to_device(x)
    y = torch.zeros_like(xd)
    ws.view(torch.int64)[32] = 1
    m.moe_set_wait_limit_ns(2_000_000)
    m.moe_set_decode_path(m.DECODE_CHAIN)
    try:
        m.moe_timing_enable(True)
        m.moe_ffn_forward(d.L, xd, None, 1, y, ws, nb)
        torch.cuda.synchronize()
        kinds = set(m.moe_timing_collect())
    finally:
        m.moe_timing_enable(False)
        m.moe_set_wait_limit_ns(0)
        m.moe_set_decode_path(m.DECODE_AUTO)
    assert "decode_chain" in kinds
    assert m.moe_get_device_status(ws) == 6
    m.moe_workspace_init(ws, nb)
    yd, _, _, kinds = forward_with_record(m, d, xd, None, 1, ws, nb, decode=m.DECODE_CHAIN)
    assert path_ran("chain", kinds)
    y_ref = oracle_layer(shape, t).ffn(x)[0]
    assert_close_output(bf16_dev_to_f64(yd), y_ref, "after a timeout")


def _cluster_ticket_word(E, K, I, Is, r):
    """Index (in 8-byte words) of the cluster decode kernel's ticket counter in a forward
    workspace: the 256-byte header, then the chain kernel's region (its size formula), each
    rounded up to 256 bytes."""
    Tm = min(4, 16 // K)
    rr, Jm, Imx = max(r, 1), Tm * (K + 1), max(I, Is)
    chain = 8 + Tm * E + Tm * 2 * rr + Tm * K * 2 * rr + Tm * K + (Jm * Imx + 1) // 2 + (256 * 3 * Tm * rr + 1) // 2 + 2
    return (256 + (chain * 8 + 255) // 256 * 256) // 8


def test_bounded_wait_runs_out_on_the_cluster_kernel():
    """The cluster kernel's grid-wide exchange of h gives up as the chain kernel's does: its
    ticket counter set to 1 puts one CTA in another epoch, whose h words the others never
    see (nor it theirs); every CTA still passes every cluster barrier, the call reports
    MOE_ERR_TIMEOUT and the next call on a re-initialised workspace is correct."""
    m, ly = _mods()
    shape = workloads.TINY
    t, x, aid = _ffn_case(shape, 475, T=1)
    d = ly.DeviceLayer.from_host(shape, t)
    ws, nb = d.workspace(1)
    xd = ly.to_device(x)
    y = torch.zeros_like(xd)
    ws.view(torch.int64)[_cluster_ticket_word(shape.E, shape.K, shape.I, shape.Is, shape.rank)] = 1
    m.moe_set_wait_limit_ns(2_000_000)
    m.moe_set_decode_path(m.DECODE_CLUSTER)
    try:
        m.moe_timing_enable(True)
        m.moe_ffn_forward(d.L, xd, None, 1, y, ws, nb)
        torch.cuda.synchronize()
        kinds = set(m.moe_timing_collect())
    finally:
        m.moe_timing_enable(False)
        m.moe_set_wait_limit_ns(0)
        m.moe_set_decode_path(m.DECODE_AUTO)
    assert "decode_cluster" in kinds
    assert m.moe_get_device_status(ws) == 6
    m.moe_workspace_init(ws, nb)
    yd, _, _, kinds = forward_with_record(m, d, xd, None, 1, ws, nb, decode=m.DECODE_CLUSTER)
    assert path_ran("cluster", kinds)
    y_ref = oracle_layer(shape, t).ffn(x)[0]
    assert_close_output(bf16_dev_to_f64(yd), y_ref, "after a timeout")


def test_block_tiny():
    _, ly = _mods()
    shape = workloads.TINY
    t, x, aid = _ffn_case(shape, 450, T=11)
    L = oracle_layer(shape, t)
    d = ly.DeviceLayer.from_host(shape, t)
    out = bf16_dev_to_f64(_gpu_ffn(d, x, block_eps=1e-6))
    ref = synth.bf16_to_f32(L.block(x, eps=1e-6)).astype(np.float64)
    assert_close_block(out, ref, synth.bf16_to_f32(x).astype(np.float64))
    # RMSNorm alone: bf16 results equal except where fp32 and fp64 round differently
    m, _ = _mods()
    xd = ly.to_device(x)
    xn = torch.empty_like(xd)
    m.moe_rmsnorm(xd, x.shape[0], shape.H, 1e-6, xn)
    torch.cuda.synchronize()
    got = ly.to_host(xn, np.uint16)
    exp = oracle.rmsnorm_bf16(x, shape.H, 1e-6)
    assert np.mean(got == exp) > 0.99
    assert np.max(np.abs(synth.bf16_to_f32(got).astype(np.float64) - synth.bf16_to_f32(exp))) <= \
        np.max(np.abs(synth.bf16_to_f32(exp))) * 2.0 ** -7


def _offset_copy(t):
    """A copy of t whose data starts 2 bytes past an aligned allocation."""
    flat = torch.empty(t.numel() + 1, dtype=t.dtype, device=t.device)
    v = flat[1:].view(t.shape)
    v.copy_(t)
    return v


def test_buffers_two_bytes_off_take_the_element_wise_paths():
    """The API asks only 2-byte alignment of these buffers: a router input, an RMSNorm input and
    output, and an FFN output 2 bytes past a 16-byte boundary go through the kernels that read
    and write element by element, with the same results."""
    m, ly = _mods()
    shape, T = workloads.TINY, 20  # enough tokens for the tensor-core path of the aligned case
    t, L, x, _ = _router_case(shape, 205, T)
    d = ly.DeviceLayer.from_host(shape, t)
    xd = ly.to_device(x)
    xo = _offset_copy(xd)
    assert xo.data_ptr() % 16 == 2
    E, K = shape.E, shape.K
    idx = torch.empty((T, K), dtype=torch.int32, device="cuda")
    w = torch.empty((T, K), dtype=torch.float32, device="cuda")
    sg = torch.empty(T, dtype=torch.float32, device="cuda")
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    m.moe_router_topk(xo, d.L.router, d.L.shared_gate, d.t.get("logit_bias"), T, shape.H, E, K, idx, w, sg, logits)
    torch.cuda.synchronize()
    y_r, idx_r, w_r, sg_r, logits_r = L.ffn(x)
    assert np.allclose(logits.cpu().numpy(), logits_r, rtol=1e-5, atol=1e-5)
    ties = check_routing(idx.cpu().numpy(), idx_r, logits_r, K)
    assert np.allclose(w.cpu().numpy()[~ties], w_r[~ties], rtol=1e-5, atol=1e-6)
    assert np.allclose(sg.cpu().numpy(), sg_r, rtol=1e-6, atol=1e-6)
    # RMSNorm, input and output both off
    xn = _offset_copy(torch.zeros_like(xd))
    m.moe_rmsnorm(xo, T, shape.H, 1e-6, xn)
    torch.cuda.synchronize()
    got = ly.to_host(xn.contiguous(), np.uint16)
    exp = oracle.rmsnorm_bf16(x, shape.H, 1e-6)
    assert np.mean(got == exp) > 0.99
    assert np.max(np.abs(synth.bf16_to_f32(got).astype(np.float64) - synth.bf16_to_f32(exp))) <= \
        np.max(np.abs(synth.bf16_to_f32(exp))) * 2.0 ** -7
    # the FFN output off (x itself must be 16-byte aligned)
    ws, nb = d.workspace(T)
    y = _offset_copy(torch.zeros_like(xd))
    m.moe_ffn_forward(d.L, xd, None, T, y, ws, nb)
    torch.cuda.synchronize()
    assert m.moe_get_device_status(ws) == 0
    y_ref = y_r
    near = near_tie_tokens(logits_r, K)
    if near.any():
        y_ref = oracle_for_gpu_routing(L, x, None, idx.cpu().numpy(), logits_r, y_r)
    assert_close_output(bf16_dev_to_f64(y.contiguous()), y_ref, "ffn, output 2 bytes off")


def assert_close_block(out, ref, x):
    """Block outputs are bf16(x + y): equal up to one bf16 step of the sum plus the FFN tolerance."""
    y = ref - x
    tol = np.abs(ref) * 2.0 ** -7 + 1e-2 * np.max(np.abs(y))
    assert np.all(np.abs(out - ref) <= tol)
    assert np.mean(out == ref) > 0.8


# ------------------------------------------------------------------ full-size layers
@pytest.fixture(scope="module")
def full_layer():
    """The Edge0-35B-shaped layer (seed 0) with 4 adapters and a logit bias, packed by the oracle."""
    shape = workloads.MULTI_TENANT
    w = workloads.moe_weights(shape, seed=0)
    t = quantize_layer(w)
    return shape, w, t


def test_full_size_pack_bit_exact(full_layer):
    m, ly = _mods()
    shape, w, t = full_layer
    weights = {k: ly.to_device(w[k]) for k in ("router", "sgate", "gate", "up", "down", "s_gate", "s_up", "s_down")}
    d = ly.DeviceLayer.from_fp32(shape, weights)
    torch.cuda.synchronize()
    for name in ("router", "sgate", "gate", "up", "down", "s_gate", "s_up", "s_down"):
        for suf, dt in (("_p", np.uint32), ("_s", np.uint16), ("_b", np.uint16)):
            got = ly.to_host(d.t[name + suf], dt)
            assert got.size == t[name + suf].size, name + suf
            assert np.array_equal(got.ravel(), t[name + suf].ravel()), name + suf


@pytest.mark.parametrize("K,T,kernel,path", [(4, 1, "auto", "cluster"), (4, 1, "chain", "chain"),
                                             (4, 1, "barrier", "fused"), (8, 1, "auto", "cluster"),
                                             (8, 1, "cluster", "cluster"),
                                             (8, 1, "chain", "chain"), (8, 1, "barrier", "fused"),
                                             (4, 2, "auto", "fused"), (4, 2, "chain", "chain"),
                                             (4, 3, "auto", "decode"), (4, 6, "auto", None)])
def test_full_size_decode(full_layer, K, T, kernel, path):
    """The Edge0 layer at decode sizes: the default choice among the single-kernel decodes
    (cluster kernel for one token — at top-8 in its lean shared-memory layout —, barrier
    kernel for more at top-4) and each one forced."""
    m, _ = _mods()
    shape0, w, t = full_layer
    shape = dataclasses.replace(workloads.DECODE_K4, K=K)
    tt = dict(t)
    tt["logit_bias"] = None
    x, _ = workloads.moe_inputs(shape, seed=500 + K, T=T)
    force = {"auto": None, "chain": m.DECODE_CHAIN, "barrier": m.DECODE_BARRIER, "cluster": m.DECODE_CLUSTER}[kernel]
    _check_ffn(shape, tt, x, None, n_adapters=1, what="decode K=%d T=%d %s" % (K, T, kernel), path=path,
               decode=force)


@pytest.mark.parametrize("T", [4, 5, 8])
def test_full_size_cuda_core_top8(full_layer, T):
    """Top-8 (the Edge0 config's K) at 4-8 tokens: 36-72 jobs, more than the fused decode
    kernel takes and fewer tokens than the tensor-core path takes, so the CUDA-core
    kernels run it; the routing comes from the CUDA-core router and top-K kernels."""
    shape0, w, t = full_layer
    shape = workloads.DECODE_K8
    tt = dict(t)
    tt["logit_bias"] = None
    x, _ = workloads.moe_inputs(shape, seed=530 + T, T=T)
    _check_ffn(shape, tt, x, None, n_adapters=1, what="top-8 T=%d" % T, path="cuda_core")


@pytest.fixture(scope="module")
def full_layer_rank64():
    """The Edge0-shaped layer with one rank-64 adapter set (alpha 128)."""
    shape = dataclasses.replace(workloads.DECODE_K4, rank=64, alpha=128.0)
    w = workloads.moe_weights(shape, seed=3)
    return shape, quantize_layer(w)


@pytest.mark.parametrize("T", [1, 2, 8])
def test_full_size_cuda_core_rank64(full_layer_rank64, T):
    """A LoRA rank above the fused decode kernel's 32 at decode sizes: CUDA-core path."""
    shape, t = full_layer_rank64
    x, _ = workloads.moe_inputs(shape, seed=540 + T, T=T)
    _check_ffn(shape, t, x, None, what="rank 64 T=%d" % T, path="cuda_core")


@pytest.mark.parametrize("T", [5, 2048])
def test_full_size_router_topk_entry(full_layer, T):
    """moe_router_topk at the Edge0 shape: the CUDA-core router kernel (5 tokens) and the
    tensor-core router (2048 tokens); indices bit-exact outside near ties."""
    shape0, w, t = full_layer
    shape = workloads.PREFILL
    tt = dict(t)
    tt["logit_bias"] = None
    L = oracle_layer(shape, tt, n_adapters=1)
    x, _ = workloads.moe_inputs(shape, seed=550 + T, T=T)
    idx, wts, sg, logits = _gpu_router(tt, shape, x, T)
    z_ref, gs_ref = L.router(x)
    idx_r, w_r = oracle.topk(z_ref, shape.K)
    # logit error well inside the near-tie margin, which is what makes the tie exclusion sound
    assert np.max(np.abs(logits - z_ref)) < 0.5 * TIE_GAP
    ties = check_routing(idx, idx_r, z_ref, shape.K)
    check_weights(idx, wts, idx_r, w_r, ties)
    assert np.allclose(sg, 1.0 / (1.0 + np.exp(-gs_ref)), rtol=1e-6, atol=1e-6)


@pytest.mark.parametrize("case", ["decode", "multi_tenant"])
def test_full_size_group32(full_layer, case):
    """The same Edge0-shaped weights packed at group 32 (twice the scales and biases): one
    token through the fused decode kernel, 64 multi-tenant tokens through the tensor cores."""
    shape0, w, _ = full_layer
    t = quantize_layer(w, group=32)
    if case == "decode":
        shape = dataclasses.replace(workloads.DECODE_K4, group=32)
        t["logit_bias"] = None
        x, aid = workloads.moe_inputs(shape, seed=520, T=1)
        _check_ffn(shape, t, x, None, n_adapters=1, what="group 32 decode", path="decode")
    else:
        shape = dataclasses.replace(shape0, group=32)
        x, aid = workloads.moe_inputs(shape, seed=521)
        _check_ffn(shape, t, x, aid, what="group 32 multi-tenant")


def test_full_size_multi_tenant(full_layer):
    shape, w, t = full_layer
    x, aid = workloads.moe_inputs(shape, seed=0)
    assert aid is not None and len(np.unique(aid)) == 4
    _check_ffn(shape, t, x, aid, what="multi-tenant T=64")


def _chunk_sample(T, seed, n):
    """First and last token of every 32-token chunk, topped up with random tokens to n."""
    edges = np.unique(np.concatenate([np.arange(0, T, 32), np.minimum(np.arange(31, T + 31, 32), T - 1)]))
    rest = np.setdiff1d(np.arange(T), edges)
    pick = synth.randint(seed, "sample", (len(rest),), 0, 1 << 30)
    extra = rest[np.argsort(pick, kind="stable")[:max(0, n - len(edges))]]
    return np.sort(np.concatenate([edges, extra]))


def test_full_size_prefill_layer(full_layer):
    """All 2048 tokens on the GPU (tensor-core path).  The routing the forward used is
    checked for every token against the oracle's router; the outputs of 256+ tokens (the
    first and last of each 32-token chunk and a random sample) are recomputed one by one."""
    m, ly = _mods()
    shape0, w, t = full_layer
    shape = workloads.PREFILL
    tt = dict(t)
    tt["logit_bias"] = None
    x, _ = workloads.moe_inputs(shape, seed=510)
    d = ly.DeviceLayer.from_host(shape, tt, n_adapters=1)
    ws, nb = d.workspace(shape.T)
    yd, idx_g, w_g, kinds = forward_with_record(m, d, ly.to_device(x), None, shape.T, ws, nb)
    assert PATH_KINDS["tensor_core"] <= kinds and "tc_router" in kinds, kinds
    y = bf16_dev_to_f64(yd)
    assert np.all(np.isfinite(y))
    L = oracle_layer(shape, tt, n_adapters=1)
    z_ref, _ = L.router(x)
    idx_r, w_r = oracle.topk(z_ref, shape.K)
    ties = check_routing(idx_g, idx_r, z_ref, shape.K)
    check_weights(idx_g, w_g, idx_r, w_r, ties)
    sample = _chunk_sample(shape.T, 510, 256)
    assert len(sample) == 256
    y_ref, _, _, _, logits_r = L.ffn(x[sample])
    if ties[sample].any():
        y_ref = oracle_for_gpu_routing(L, x[sample], None, idx_g[sample], logits_r, y_ref)
    assert_close_output(y[sample], y_ref, "prefill sample")


@pytest.fixture(scope="module")
def stack_layers():
    """Three distinct Edge0-shaped layers (one adapter set each), packed by the oracle."""
    shape = workloads.PREFILL
    out = []
    for l in range(3):
        t = quantize_layer(workloads.moe_weights(shape, seed=7, layer=l))
        t["logit_bias"] = None
        t["lora"] = t["lora"][:1]
        out.append(t)
    return shape, out


def test_full_size_prefill_stack_teacher_forced(stack_layers):
    """The 2048-token prefill stack, block by block (RMSNorm, FFN, residual): each GPU block
    output is compared with the oracle's block run on that block's GPU input (teacher
    forcing) for 256+ sampled tokens.  Then 40 blocks (the three layers in turn) run on the
    GPU and 16 tokens go through the same 40 blocks in the oracle, free-running: the
    end-to-end drift is printed, not gated."""
    m, ly = _mods()
    shape, ts = stack_layers
    T = shape.T
    x0, _ = workloads.moe_inputs(shape, seed=560)
    devs = [ly.DeviceLayer.from_host(shape, t) for t in ts]
    Ls = [oracle_layer(shape, t) for t in ts]
    ws, nb = devs[0].workspace(T)
    sample = _chunk_sample(T, 560, 256)
    xd = ly.to_device(x0)
    for l, (d, L) in enumerate(zip(devs, Ls)):
        yd, idx_g, _, kinds = forward_with_record(m, d, xd, None, T, ws, nb, block_eps=1e-6)
        assert "rmsnorm" in kinds and PATH_KINDS["tensor_core"] <= kinds, kinds
        x_in = ly.to_host(xd, np.uint16)
        out = bf16_dev_to_f64(yd)
        ref = synth.bf16_to_f32(L.block(x_in[sample], eps=1e-6)).astype(np.float64)
        # tokens whose normalised input sits at a routing near tie: the oracle block with
        # the forward's own routing
        xn = oracle.rmsnorm_bf16(x_in[sample], shape.H, 1e-6)
        y_ref, _, _, _, logits_r = L.ffn(xn)
        ties = near_tie_tokens(logits_r, shape.K)
        if ties.any():
            y_alt = oracle_for_gpu_routing(L, xn, None, idx_g[sample], logits_r, y_ref)
            xs = synth.bf16_to_f32(x_in[sample]).astype(np.float64)
            ref[ties] = synth.bf16_to_f32(synth.bf16((xs + y_alt)[ties])).astype(np.float64)
        assert_close_block(out[sample], ref, synth.bf16_to_f32(x_in[sample]).astype(np.float64))
        xd = yd
    # free-running drift over 40 blocks
    n_layers = shape.layers
    xa = ly.to_device(x0)
    xb = torch.empty_like(xa)
    for l in range(n_layers):
        m.moe_block_forward(devs[l % 3].L, xa, None, T, 1e-6, xb, ws, nb)
        xa, xb = xb, xa
    torch.cuda.synchronize()
    assert m.moe_get_device_status(ws) == 0
    g = bf16_dev_to_f64(xa)
    few = sample[:16]
    xr = x0[few]
    for l in range(n_layers):
        xr = Ls[l % 3].block(xr, eps=1e-6)
    r = synth.bf16_to_f32(xr).astype(np.float64)
    assert np.all(np.isfinite(g))
    print("40-block drift over %d tokens: rel-L2 %.3e, max-abs %.3e (max |x| %.2f)" % (
        len(few), rel_l2(g[few], r), np.max(np.abs(g[few] - r)), np.max(np.abs(r))))


# ------------------------------------------------------------------ mixed layout
@pytest.fixture(scope="module")
def mixed_layer():
    s = workloads.MIXED_B1
    W = workloads.mixed_weights(s, seed=0)
    q = {n: oracle.quant_mixed(W[n], s.rho) for n in W}
    return s, W, q


@pytest.mark.parametrize("T", [1, 2, 5, 9, 16, 20])
def test_mixed_linear_full_size(mixed_layer, T):
    m, ly = _mods()
    s, W, q = mixed_layer
    x = workloads.mixed_inputs(s, seed=600 + T, T=T)
    dm = ly.DeviceMixed.from_host(s.I, s.H, s.rho, *q["gate"])
    y = torch.empty((T, s.I), dtype=torch.float32, device="cuda")
    m.moe_mixed_linear(dm.T, ly.to_device(x), T, y)
    torch.cuda.synchronize()
    ref = oracle.mixed_linear(q["gate"][0], q["gate"][1], s.I, s.H, s.rho, x)
    assert rel_l2(y.cpu().numpy(), ref) < 1e-5


@pytest.mark.parametrize("T,residual", [(1, 0), (16, 0), (1, 1), (16, 1), (3, 1)])
def test_mixed_mlp_full_size(mixed_layer, T, residual):
    m, ly = _mods()
    s, W, q = mixed_layer
    x = workloads.mixed_inputs(s, seed=610 + T, T=T)
    dg = ly.DeviceMixed.from_host(s.I, s.H, s.rho, *q["gate"])
    du = ly.DeviceMixed.from_host(s.I, s.H, s.rho, *q["up"])
    dd = ly.DeviceMixed.from_host(s.H, s.I, s.rho, *q["down"])
    nb = m.moe_mixed_mlp_workspace_bytes(s.H, s.I, T)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    xd = ly.to_device(x)
    y = torch.empty_like(xd)
    m.moe_mixed_mlp_forward(dg.T, du.T, dd.T, xd, T, residual, 1e-6, y, ws, nb)
    torch.cuda.synchronize()
    out = bf16_dev_to_f64(y)
    if residual:
        ref = synth.bf16_to_f32(oracle.mixed_block(q["gate"], q["up"], q["down"], s.H, s.I, s.rho, x)).astype(np.float64)
        assert_close_block(out, ref, synth.bf16_to_f32(x).astype(np.float64))
    else:
        ref = oracle.mixed_mlp(q["gate"], q["up"], q["down"], s.H, s.I, s.rho, x)
        assert_close_output(out, ref, "mixed mlp")


@pytest.mark.parametrize("T", [1, 4])
def test_host_buffers_forward_matches_device_forward(T):
    """moe_ffn_forward_host with x and y in pinned host memory: one token through the cluster
    kernel reading and writing across the bus, four tokens staged through the workspace; each
    bit-for-bit the device forward's output, and the oracle's within tolerance."""
    m, ly = _mods()
    shape = workloads.TINY
    t, x, aid = _ffn_case(shape, 480 + T, T=T)
    d = ly.DeviceLayer.from_host(shape, t)
    ws, nb = d.workspace(T)
    xd = ly.to_device(x)
    yd = torch.empty_like(xd)
    m.moe_ffn_forward(d.L, xd, None, T, yd, ws, nb)
    torch.cuda.synchronize()
    assert m.moe_get_device_status(ws) == 0
    hx = torch.from_numpy(x.view(np.int16).copy()).pin_memory()
    hy = torch.zeros((T, shape.H), dtype=torch.int16).pin_memory()
    m.moe_workspace_init(ws, nb)
    m.moe_timing_enable(True)
    try:
        m.moe_ffn_forward_host(d.L, hx, None, T, hy, ws, nb)
        torch.cuda.synchronize()
        kinds = set(m.moe_timing_collect())
    finally:
        m.moe_timing_enable(False)
    assert m.moe_get_device_status(ws) == 0
    assert path_ran("cluster" if T == 1 else "decode", kinds), kinds
    assert np.array_equal(hy.numpy(), yd.cpu().numpy())
    y_ref = oracle_layer(shape, t).ffn(x)[0]
    assert_close_output(synth.bf16_to_f32(hy.numpy().view(np.uint16)).astype(np.float64), y_ref, "host buffers")


def test_full_size_host_buffers_forward(full_layer):
    """The Edge0 layer, one token, x and y in pinned host memory: the device forward's output."""
    m, ly = _mods()
    shape0, w, t = full_layer
    shape = workloads.DECODE_K4
    tt = dict(t)
    tt["logit_bias"] = None
    x, _ = workloads.moe_inputs(shape, seed=530, T=1)
    d = ly.DeviceLayer.from_host(shape, tt, n_adapters=1)
    ws, nb = d.workspace(1)
    xd = ly.to_device(x)
    yd = torch.empty_like(xd)
    m.moe_ffn_forward(d.L, xd, None, 1, yd, ws, nb)
    hx = torch.from_numpy(x.view(np.int16).copy()).pin_memory()
    hy = torch.zeros((1, shape.H), dtype=torch.int16).pin_memory()
    m.moe_ffn_forward_host(d.L, hx, None, 1, hy, ws, nb)
    torch.cuda.synchronize()
    assert m.moe_get_device_status(ws) == 0
    assert np.array_equal(hy.numpy(), yd.cpu().numpy())
