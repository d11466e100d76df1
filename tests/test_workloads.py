"""Host-side workload bookkeeping: shapes, output sizes and algorithmic work,
pinned to the figures recomputed from the pages' shapes (tests/golden)."""
import json
import os

from depthwise_convolution_fp32_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_work_counts_match_golden(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "output_sizes.json")))
    d = wl.DENSE_5X9
    assert (d.P, d.Q) == (508, 504)
    assert (d.P, d.Q) == (oracle_mod.out_extent(512, 5, 1, 0, 1), oracle_mod.out_extent(512, 9, 1, 0, 1))
    assert d.n_out == g["work"]["dense_5x9_outputs"]
    assert d.macs == g["work"]["dense_5x9_macs"]
    assert d.N * d.C * d.H * d.W == g["work"]["dense_5x9_input_floats"]
    c = wl.FUSED_CHAIN.conv
    assert (c.P, c.Q) == (254, 254)
    assert c.macs == g["work"]["fused_chain_conv_macs"]
    assert (c.K // wl.FUSED_CHAIN.gn_groups) * c.P * c.Q == g["work"]["fused_chain_gn_group_elements"]
    dw = wl.DEPTHWISE
    assert (dw.P, dw.Q) == (56, 56)
    # x + y + w of the depthwise workload: 2 * 4*144*56*56 + 144*9 floats
    assert dw.bytes == (2 * 4 * 144 * 56 * 56 + 144 * 9) * 4


def test_sweep80_shapes():
    shapes = wl.sweep80()
    assert len(shapes) == 80 and len(set(shapes)) == 80
    for s in shapes:
        assert (s.R, s.S, s.stride, s.pad, s.dil) == (3, 3, 1, 1, 1)
        assert s.K == s.C and s.cpg in (1, 2, 4, 8) and s.H == s.W
        assert s.N in (1, 4, 16, 32) and s.C in (32, 64, 128, 256, 512) and s.H in (14, 28, 56, 112)
        assert (s.P, s.Q) == (s.H, s.W)
    # the permutation spreads batch sizes (a nested-order prefix would only hold N=1)
    assert len({s.N for s in shapes}) == 4
    assert len({s.cpg for s in shapes}) == 4
    saved = json.load(open(os.path.join(os.path.dirname(wl.__file__), "sweep80.json")))
    assert [list(x) for x in saved["shapes"]] == [[s.N, s.C, s.cpg, s.H] for s in shapes]


def test_stored_traffic_matches_kernel_sources():
    """The DRAM traffic the benchmark reports (`roofline.traffic`) comes from
    committed ncu captures keyed to a hash of the kernel sources; after a
    kernel change the figure is withheld until it is captured again.  Fails
    when a page workload's stored figure no longer matches the sources."""
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import bench
    for name in ("depthwise", "dense_5x9", "fused_chain"):
        t = bench.stored_traffic(name)
        assert t is not None and t > 0, f"{name}: stored traffic missing or captured from other sources"
