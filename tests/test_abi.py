"""The C ABI library loads, exports every declared symbol, and validates on the host (no GPU)."""
import ctypes
import os
import re

import pytest

import oracle
from int4_group_affine_b200 import _lib
from int4_group_affine_b200 import (Layer, LoraPtrs, MoeError, lora_set_adapters, moe_ffn_forward,
                                    moe_ffn_workspace_bytes, moe_index_workspace_bytes, moe_mixed_mlp_workspace_bytes,
                                    moe_mixed_words)

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if not h.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", h)).read()
        names += re.findall(r"^MOEQ_API\s+[\w\s\*]+?\b(\w+)\(", src, flags=re.M)
    return names


@pytest.fixture(scope="module", autouse=True)
def built():
    from int4_group_affine_b200 import build
    build.build()


def test_every_declared_symbol_is_exported():
    names = _declared()
    assert len(names) >= 19
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), set(names) ^ set(_lib.SIGNATURES)


def test_internal_symbols_hidden():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if l.strip()}
    assert not any("launch_" in s for s in exported)


def test_version():
    assert _lib.lib().moe_version() == 1
    assert _lib.lib().moe_status_string(4) == b"workspace missing, misaligned or too small"


@pytest.mark.parametrize("out,in_,rho", [(3072, 1024, 0.25), (1024, 3072, 0.25), (10, 96, 0.25), (8, 64, 0.0),
                                         (8, 64, 1.0), (24, 128, 1 / 3), (16, 64, 0.125)])
def test_mixed_words_matches_oracle(out, in_, rho):
    assert moe_mixed_words(out, in_, rho) == oracle.mixed_words(out, in_, rho)


def _fake_layer(H=256, E=8, K=2, I=128, Is=128, group=64):
    """A layer descriptor with aligned fake device addresses (host validation only)."""
    L = Layer()
    L.hidden, L.n_experts, L.top_k, L.inter, L.shared_inter = H, E, K, I, Is
    base = [0x10000000]

    def q(n, out, in_, bits):
        from int4_group_affine_b200 import QTensor
        t = QTensor()
        t.packed, t.scales, t.biases = base[0], base[0] + 0x1000000, base[0] + 0x2000000
        base[0] += 0x4000000
        t.n, t.out, t.in_, t.bits, t.group = n, out, in_, bits, group
        return t

    L.router = q(1, E, H, 8)
    L.shared_gate = q(1, 1, H, 8)
    L.gate, L.up, L.down = q(E, I, H, 4), q(E, I, H, 4), q(E, H, I, 4)
    L.s_gate, L.s_up, L.s_down = q(1, Is, H, 4), q(1, Is, H, 4), q(1, H, Is, 4)
    return L


def test_workspace_bytes_host_only():
    L = _fake_layer()
    n4 = moe_ffn_workspace_bytes(L, 4)
    n64 = moe_ffn_workspace_bytes(L, 64)
    assert n4 > 0 and n64 > n4 and n4 % 256 == 0
    assert moe_ffn_workspace_bytes(L, 0) > 0
    bad = _fake_layer()
    bad.top_k = 9  # K > E
    assert moe_ffn_workspace_bytes(bad, 4) == 0
    assert moe_index_workspace_bytes(2048, 4, 256, 1) > 0
    assert moe_mixed_mlp_workspace_bytes(1024, 3072, 16) > 0


@pytest.mark.parametrize("mutate,status", [
    (lambda L: setattr(L, "top_k", 0), 1),
    (lambda L: setattr(L, "top_k", 17), 2),
    (lambda L: setattr(L, "n_experts", 513), 2),
    (lambda L: setattr(L.gate, "group", 48), 1),
    (lambda L: setattr(L.gate, "out", 64), 1),
    (lambda L: setattr(L.router, "bits", 4), 1),
    (lambda L: setattr(L.down, "packed", 0x10000004), 1),   # misaligned packed words
    (lambda L: setattr(L, "hidden", 250), 1),
])
def test_forward_rejects_bad_layer_before_any_launch(mutate, status):
    L = _fake_layer()
    mutate(L)
    with pytest.raises(MoeError) as ei:
        moe_ffn_forward(L, 0x20000000, None, 4, 0x30000000, 0x40000000, 1 << 30, stream=0)
    assert ei.value.status == status


def test_forward_rejects_small_or_misaligned_workspace():
    L = _fake_layer()
    need = moe_ffn_workspace_bytes(L, 4)
    with pytest.raises(MoeError) as ei:
        moe_ffn_forward(L, 0x20000000, None, 4, 0x30000000, 0x40000000, need - 1, stream=0)
    assert ei.value.status == 4
    with pytest.raises(MoeError) as ei:
        moe_ffn_forward(L, 0x20000000, None, 4, 0x30000000, 0x40000010, need, stream=0)
    assert ei.value.status == 4


def test_zero_tokens_is_a_no_op():
    L = _fake_layer()
    need = moe_ffn_workspace_bytes(L, 0)
    moe_ffn_forward(L, 0x20000000, None, 0, 0x30000000, 0x40000000, need, stream=0)


def test_lora_set_adapters_host_rules():
    L = _fake_layer()
    sets = [LoraPtrs() for _ in range(3)]
    for s in sets:
        s.gate.A, s.gate.B = 0x50000000, 0x51000000
    lora_set_adapters(L, 3, 16, 32.0, sets)
    assert L.n_adapters == 3 and L.rank == 16 and L.alpha == 32.0
    assert L.lora[2].gate.A == 0x50000000 and not L.lora[3].gate.A
    with pytest.raises(MoeError):
        lora_set_adapters(L, 17, 16, 32.0, [LoraPtrs()] * 17)
    with pytest.raises(MoeError):
        lora_set_adapters(L, 1, 65, 32.0, sets[:1])
    half = LoraPtrs()
    half.up.A = 0x50000000  # A without B
    with pytest.raises(MoeError):
        lora_set_adapters(L, 1, 16, 32.0, [half])
    lora_set_adapters(L, 0, 0, 0.0, [])
    assert L.n_adapters == 0


def _edge0_fake_layer(n_adapters):
    L = _fake_layer(H=2048, E=256, K=4, I=512, Is=512)
    if n_adapters:
        sets = [LoraPtrs() for _ in range(n_adapters)]
        for st in sets:
            for p in ("gate", "up", "down", "s_gate", "s_up", "s_down"):
                lp = getattr(st, p)
                lp.A, lp.B = 0x50000000, 0x51000000
        lora_set_adapters(L, n_adapters, 16, 32.0, sets)
    return L


@pytest.mark.parametrize("n_adapters", [0, 1, 4])
def test_static_array_holds_256_tokens_of_the_edge0_layer(n_adapters):
    """The documented guarantee of moe_ffn_forward_static: 256 tokens of the Edge0-shaped
    layer fit the built-in 16 MiB array."""
    L = _edge0_fake_layer(n_adapters)
    assert 0 < moe_ffn_workspace_bytes(L, 256) <= 16 * 1024 * 1024


@pytest.mark.parametrize("mutate", [lambda L: setattr(L, "top_k", 17), lambda L: setattr(L, "n_experts", 513),
                                    lambda L: setattr(L.gate, "group", 48), lambda L: setattr(L, "hidden", 250)])
def test_static_forward_rejects_like_forward(mutate):
    """The static entry point returns moe_ffn_forward's own status for a bad layer, before
    it touches the device."""
    from int4_group_affine_b200 import moe_ffn_forward_static
    L = _fake_layer()
    mutate(L)
    with pytest.raises(MoeError) as e1:
        moe_ffn_forward(L, 0x20000000, None, 4, 0x30000000, 0x40000000, 1 << 30, stream=0)
    with pytest.raises(MoeError) as e2:
        moe_ffn_forward_static(L, 0x20000000, None, 4, 0x30000000, stream=0)
    assert e1.value.status == e2.value.status


def test_static_forward_checks_x_and_y_first():
    from int4_group_affine_b200 import moe_ffn_forward_static
    L = _fake_layer()
    for x, y in ((0x20000000, 0x20000000), (0x20000008, 0x30000000), (0, 0x30000000)):
        with pytest.raises(MoeError) as ei:
            moe_ffn_forward_static(L, x, None, 4, y, stream=0)
        assert ei.value.status == 1


def test_wait_limit_setting():
    from int4_group_affine_b200 import moe_set_wait_limit_ns, moe_wait_limit_ns
    assert moe_wait_limit_ns() == 1000000000
    moe_set_wait_limit_ns(2000000)
    try:
        assert moe_wait_limit_ns() == 2000000
    finally:
        moe_set_wait_limit_ns(0)
    assert moe_wait_limit_ns() == 1000000000


def test_decode_path_setting():
    from int4_group_affine_b200 import (DECODE_AUTO, DECODE_BARRIER, DECODE_CHAIN, DECODE_CLUSTER, MoeError,
                                        moe_decode_path, moe_set_decode_path)
    assert moe_decode_path() == DECODE_AUTO
    try:
        for p in (DECODE_CHAIN, DECODE_BARRIER, DECODE_CLUSTER, DECODE_AUTO):
            moe_set_decode_path(p)
            assert moe_decode_path() == p
        with pytest.raises(MoeError) as ei:
            moe_set_decode_path(4)
        assert ei.value.status == 1
        assert moe_decode_path() == DECODE_AUTO
    finally:
        moe_set_decode_path(DECODE_AUTO)


def test_host_forward_takes_decode_sizes_only():
    """moe_ffn_forward_host: the forward's own checks first (x == y, misaligned), then more
    than 8 tokens is UNSUPPORTED; all before any CUDA call."""
    from int4_group_affine_b200 import moe_ffn_forward_host
    L = _fake_layer()
    for x, y, T, code in ((0x20000000, 0x20000000, 4, 1), (0x20000008, 0x30000000, 4, 1),
                          (0x20000000, 0x30000000, 9, 2)):
        with pytest.raises(MoeError) as ei:
            moe_ffn_forward_host(L, x, None, T, y, 0x40000000, 1 << 30, stream=0)
        assert ei.value.status == code
