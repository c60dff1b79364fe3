"""Host-side checks of the algorithmic work counts and the stream/column sharding (CPU)."""
import pytest

from weight_linear_attention_ttt_b200 import inputs as inp
from weight_linear_attention_ttt_b200 import metrics
from weight_linear_attention_ttt_b200.shard import split_range


@pytest.mark.parametrize("name,flops,mbytes,bound", [
    ("dual_bf16_B8H12T2048_d64C16", 5.637e9, 104.6, "hbm"),
    ("dual_bf16_B2H32T32768_d64C16", 60.13e9, 1084.0, "hbm"),
    ("assoc_bf16_B4H16T65536_d128C64", 412.3e9, 4316.0, "hbm"),
    ("inplace_bf16_T32768_Dff9728_D2560_C1024", 3.264e12, 1122.5, "tensor"),
    ("assoc_bwd_bf16_B4H16T65536_d128C64", 1.2370e12, 7558.1, "hbm"),
    ("dual_bwd_bf16_B8H12T2048_d64C16", 13.287e9, 182.45, "hbm"),
    ("dual_bf16_B1H4T262144_d64C16", 30.065e9, 541.2, "hbm"),
    ("dual_seg_bf16_B1H4T262144_d64C16", 30.065e9, 541.2, "hbm"),
    ("dual_bwd_bf16_B1H4T262144_d64C16", 70.867e9, 948.1, "hbm"),
    ("dual_seg_bwd_bf16_B1H4T262144_d64C16", 70.867e9, 948.1, "hbm"),
    ("assoc_momentum_bf16_B4H16T65536_d128C64", 824.6e9, 4328.5, "hbm"),
    ("inplace_lm_bf16_T32768_Dff9728_D2560_Dm2560_C1024", 3.6943e12, 1135.6, "tensor"),
])
def test_algorithmic_counts(name, flops, mbytes, bound):
    w = inp.WORKLOADS[name]
    a = metrics.algorithmic(w)
    assert a["flops"] == pytest.approx(flops, rel=2e-3)
    assert a["bytes"] / 1e6 == pytest.approx(mbytes, rel=2e-3)
    t, b = metrics.roofline_seconds(w, 6472.4, 1696.1)
    assert b == bound


def test_dual_counts_by_hand():
    # one stream, one chunk: 6 d^2 + 4 C d flops per token; 4 d bf16 elements + eta per token
    w = inp.Workload("x", "dual", 0, B=1, H=1, T=16, d=64, C=16)
    a = metrics.algorithmic(w)
    assert a["flops"] == 16 * (6 * 64 * 64 + 4 * 16 * 64)
    assert a["bytes"] == 16 * (4 * 64 * 2 + 4) + 2 * 64 * 64 * 4
    assert a["tokens"] == 16


@pytest.mark.parametrize("n,world", [(96, 1), (96, 2), (96, 8), (7, 3), (2, 4), (0, 2)])
def test_split_range_partitions(n, world):
    spans = [split_range(n, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        split_range(n, world, world)
