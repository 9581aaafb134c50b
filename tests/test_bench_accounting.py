"""Host-side accounting of bench.py (no GPU): per-launch times and the workload table."""
import pytest

import bench
from synth import workloads


def test_launch_times_add_up_to_the_graph_time():
    kt = {"a": (10.0, 2), "b": (4.0, 2)}  # summed event intervals 14 ms over 4 launches
    lt = bench.launch_times(kt, 12.0)
    assert lt["a"] == (4.5, 2) and lt["b"] == (1.5, 2)
    assert sum(t * c for t, c in lt.values()) == pytest.approx(12.0)


def test_single_launch_step_gets_the_step_time():
    lt = bench.launch_times({"decode_fused": (0.8, 20)}, 0.7)
    assert lt["decode_fused"][0] == pytest.approx(0.7 / 20)


def test_every_moe_workload_has_a_shape_and_step_count():
    for w in bench.MOE_WORKLOADS:
        assert w in workloads.MOE_SHAPES
        assert bench.default_steps(w) > 0
    assert workloads.MOE_SHAPES["decode_k4_g32"].group == 32


def test_group_32_bytes():
    # 2048 x 512 int4 with bf16 scale and bias per 32: 2048*256 + 2048*16*4 bytes
    gu, d = bench.expert_bytes(2048, 512, 32)
    assert d == 2048 * (256 + 16 * 4)
    assert gu == 2 * 512 * (1024 + 64 * 4)


def test_every_single_kernel_decode_kind_has_a_unit():
    """The fused decode kernels are a whole layer call each: their bytes are the layer's."""
    for kind in ("decode_fused", "decode_chain", "decode_cluster"):
        assert bench.KIND_UNIT[kind] == "layer"
    from int4_group_affine_b200 import _lib
    names = {_lib.lib().moe_timing_kind_name(k).decode() for k in range(_lib.lib().moe_timing_kinds())}
    assert {"decode_fused", "decode_chain", "decode_cluster", "tc_gate_up", "gate_up"} <= names
