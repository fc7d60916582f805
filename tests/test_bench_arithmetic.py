"""The bench's roofline arithmetic against counts done by hand from the
workload shapes (no GPU): algorithmic bytes and nominal flops per launch."""
import dataclasses

import bench
from sparse_spd_selected_b200 import inputs

W = inputs.WORKLOADS


def test_chain_selinv_bytes_and_flops():
    w = W["chain_4096x64_b16"]
    # D and B read, G_diag and G_lower written (2 b^2 per block and edge each), plus r and x
    blocks, edges = 4096 * 64, 4096 * 63
    assert bench.algorithmic_bytes(w, 8, 4096) == 8 * (2 * 256 * blocks + 2 * 256 * edges + 2 * 16 * blocks)
    assert bench.algorithmic_bytes(w, 8, 4096) == 2197815296
    assert bench.algorithmic_flops(w, 4096) == 7 * 16 ** 3 * blocks


def test_tree_and_grid():
    w = W["forest_8x32768_b16"]
    n = 8 * 32768
    assert bench.algorithmic_bytes(w, 8, 8) == 8 * 256 * (2 * n + 2 * (n - 8))
    g = W["grid_256x128_b128"]
    assert bench.algorithmic_flops(g, 256) == 7 * 128 ** 3 * 256 * 128 == 481036337152


def test_draw_backward_bidiag():
    w = W["chain_4096x64_b16"]
    blocks, edges = 4096 * 64, 4096 * 63
    # a draw reads D, B, r, z and writes eta; 7/3 b^3 flops (the collect only)
    assert bench.algorithmic_bytes(w, 8, 4096, "sample") == 8 * (256 * blocks + 256 * edges + 3 * 16 * blocks)
    assert abs(bench.algorithmic_flops(w, 4096, "sample") - 7 / 3 * 16 ** 3 * blocks) < 1
    # the backward reads D, G_diag, Gb_diag, B, G_lower, Gb_lower and writes Db, Bb; 73/3 b^3 flops
    assert bench.algorithmic_bytes(w, 8, 4096, "backward") == 8 * 4 * 256 * (blocks + edges)
    assert abs(bench.algorithmic_flops(w, 4096, "backward") - 73 / 3 * 16 ** 3 * blocks) < 1
    # the non-symmetric chain reads M_ii, M_{i+1,i} and writes G_ii, G_{i+1,i}
    assert bench.algorithmic_bytes(w, 8, 4096, "bidiag") == 8 * 2 * 256 * (blocks + edges)
    t = W["forest_8x32768_b16"]
    n = 8 * 32768
    assert bench.algorithmic_bytes(t, 8, 8, "sample") == 8 * (256 * n + 256 * (n - 8) + 2 * 16 * n)


def test_oracle_stand_ins_stay_small():
    """The dense-definition oracles time stand-ins of at most 512 unknowns."""
    for name, op in [("chain_4096x64_b16", "backward"), ("forest_8x32768_b16", "backward"),
                     ("chain_4096x64_b16", "bidiag"), ("lattice_64x1024_b8", "selinv")]:
        w, note = bench.oracle_workload(W[name], op)
        assert w.L * w.b <= 512 and note
    w, note = bench.oracle_workload(W["chain_4096x64_b16"], "selinv")
    assert w == W["chain_4096x64_b16"] and note == ""
    assert dataclasses.replace(W["chain_1x8_b4"]) == W["chain_1x8_b4"]


def test_l2_rule_per_workload():
    # workloads whose inputs stay in L2 are flushed before every timed step; the rest
    # are larger than L2 (126 MB) by more than twice
    small = {n for n, w in inputs.WORKLOADS.items() if bench.fits_l2(w)}
    assert "chain_1x8_b4" in small and "lattice_64x1024_b8" in small
    for n, w in inputs.WORKLOADS.items():
        cfg = bench.config_dict(w, w.batch, 1, "selinv", True)
        if n in small:
            assert "flushes L2" in cfg["l2"]
        else:
            assert w.L * w.batch * w.b * w.b * 8 > 2 * 126e6
            assert cfg["l2"].startswith("inputs larger than L2")
