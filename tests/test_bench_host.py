"""Host-side figures of bench.py: the per-token FLOPs and per-expert bytes
behind the roofline are the unit figures of the layer, and the bytes equal
the library's own packed buffers."""
import pytest

import bench
import quantized_moe_expert_warp_b200 as mq
import synth
from quantized_moe_expert_warp_b200 import build as mqbuild


def test_flops_per_token_a3b():
    # routed: k experts x (gate, up, down) x 2 H I; router 2 H E; shared expert and its gate
    assert bench.flops_per_token(synth.get_config("a3b_t512")) == 57_675_776


@pytest.mark.parametrize("name,want", [("a3b_t512", 1_622_016), ("a3b_t4096_q4k", 1_769_472),
                                       ("a3b_t512_asym", 1_671_168)])
def test_expert_bytes_unit_figures(name, want):
    gu, dn = bench.expert_bytes(synth.get_config(name))
    assert gu + dn == want and gu == 2 * dn


@pytest.mark.parametrize("name", ["a3b_t512", "a3b_t4096_q4k", "a3b_t512_asym", "tiny_t64"])
def test_expert_bytes_equal_packed_buffers(name):
    mqbuild.build()
    cfg = synth.get_config(name)
    sizes = mq.moe_packed_sizes(cfg)
    et = cfg.E_total
    gu, dn = bench.expert_bytes(cfg)
    assert (sizes[0] + sizes[1]) == et * gu
    assert (sizes[2] + sizes[3]) == et * dn
