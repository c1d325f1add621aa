"""Host-side accounting of bench.py (CPU): the algorithmic bytes behind the
roofline fractions and the L2 timing policy."""
import pytest

import bench
from structured_state_space_mamba_b200 import binding
from structured_state_space_mamba_b200.inputs import WORKLOADS

MB = 1e6


def layout(cfg):
    d = binding.make_dims(cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"], cfg["dstate"],
                          cfg["ngroups"], cfg["dtype"])
    return binding.workspace_layout(d, cfg["chunk_len"])


def test_scan_bytes_of_the_sweep_layer_by_hand():
    """Four-kernel sequence (few (batch, head pair) chains with short ranges):
    the chunk-wide scan reads x, B, C, l, g and the bf16 s_in, and writes y."""
    cfg = dict(WORKLOADS["sweep_N128_Q256"])
    lay = layout(cfg)
    assert lay.single_pass == 0
    wm = bench.work_model(cfg, False, lay)
    B, T, H, P, N, G, Q = 2, 8192, 32, 64, 128, 1, 256
    nc = T // Q
    x = B * T * H * P * 2
    bc = 2 * B * T * G * N * 2
    l_g = B * H * nc * Q * 4 + B * H * nc * (Q + 4) * 4
    s_in = B * nc * H * P * N * 2
    assert wm["per_kernel_bytes"]["ssd_chunk_scan"] == 2 * x + bc + l_g + s_in + H * 4
    assert wm["stages"] == ("ssd_chunk_cumsum", "ssd_chunk_state", "ssd_state_passing", "ssd_chunk_scan")


def test_presolved_bytes_of_the_long_context_layer_by_hand():
    """The long grouped layer runs the presolved single pass: the range states
    read x, B (once per head pair), w and alpha; the single pass moves the
    compulsory bytes plus l and g and the ranges' entering states."""
    cfg = dict(WORKLOADS["long_g8"])
    lay = layout(cfg)
    assert lay.single_pass == 1 and lay.launches == 5
    wm = bench.work_model(cfg, True, lay)
    B, T, H, P, N, G, Q = 1, 65536, 32, 64, 128, 8, 256
    nc = T // Q
    x = B * T * H * P * 2
    bc = 2 * B * T * G * N * 2
    comp = 2 * x + bc + B * T * H * 4 + 2 * H * 4 + 2 * B * H * P * N * 4  # h0 and final
    assert wm["bytes"] == comp
    assert wm["stages"] == ("ssd_chunk_cumsum", "ssd_range_states", None, "ssd_chunk_fused")
    assert wm["per_kernel_comp"]["ssd_chunk_fused"] == 2 * x + bc + H * 4 + 2 * B * H * P * N * 4


def test_single_pass_bytes_of_the_2p7b_layer_by_hand():
    """The 2.7B-shaped layer runs the single-pass kernel: it moves the compulsory
    bytes (x, B, C in; y, final state out) plus the cumsum's l and g."""
    cfg = dict(WORKLOADS["mamba2_2p7b"])
    lay = layout(cfg)
    assert lay.single_pass == 1 and lay.launches == 3
    assert binding.SCAN_ENGINES[lay.scan_engine] == "single_pass"
    wm = bench.work_model(cfg, True, lay)
    B, T, H, P, N, Q = 4, 4096, 80, 64, 128, 256
    nc = T // Q
    x = B * T * H * P * 2
    bc = 2 * B * T * N * 2
    fin = B * H * P * N * 4
    comp = 2 * x + bc + B * T * H * 4 + 2 * H * 4 + fin
    assert wm["bytes"] == comp
    assert wm["per_kernel_comp"]["ssd_chunk_fused"] == 2 * x + bc + H * 4 + fin
    l_g = B * H * nc * Q * 4 + B * H * nc * (Q + 4) * 4
    assert wm["per_kernel_bytes"]["ssd_chunk_fused"] == wm["per_kernel_comp"]["ssd_chunk_fused"] + l_g
    assert wm["stages"][1] == "ssd_chunk_fused" and wm["stages"][2] is None


def test_fused_layout_has_no_state_passing_traffic():
    # the 130M-shaped layer at dstate 32 (not a single-pass size): one wave of
    # (batch, head pair) units
    cfg = dict(WORKLOADS["mamba2_130m"], dstate=32)
    lay = layout(cfg)
    assert lay.fused_state == 1 and lay.single_pass == 0
    wm = bench.work_model(cfg, True, lay)
    assert wm["per_kernel_bytes"]["ssd_state_passing"] == 0


def test_flops_count_the_causal_products_once():
    cfg = dict(WORKLOADS["mamba2_2p7b"])
    wm = bench.work_model(cfg, True, layout(cfg))
    B, T, H, P, N, G, Q = 4, 4096, 80, 64, 128, 1, 256
    nc = T // Q
    per_bch = Q * (Q + 1) * P + 4 * Q * N * P
    per_bcg = Q * (Q + 1) * N
    assert wm["flops"] == B * nc * (H * per_bch + G * per_bcg)


@pytest.mark.parametrize("name, flush", [("mamba2_2p7b", False), ("long_g8", False),
                                         ("mamba2_130m", True), ("tiny_f32", True)])
def test_l2_policy(name, flush):
    got, note = bench.l2_policy(WORKLOADS[name], 126 * 1024 * 1024)
    assert got is flush
    assert ("flushed" in note) is flush


def test_traffic_figure_only_for_the_captured_kernel_and_build():
    for (wl, kern, ver), traffic in bench.NCU_TRAFFIC.items():
        # a capture moves at least the kernel's compulsory bytes and, with L2
        # hits, at most somewhat more than its workspace-inclusive bytes
        assert wl in WORKLOADS
        w = bench.work_model(dict(WORKLOADS[wl]), True, layout(dict(WORKLOADS[wl])))
        assert 0.8 * w["per_kernel_comp"][kern] < traffic <= 1.2 * w["per_kernel_bytes"][kern]
    # a build the capture was not taken from reports no traffic figure
    assert bench.NCU_TRAFFIC.get(("mamba2_2p7b", "ssd_chunk_fused", "some other build")) is None


def test_kernel_roofline_counts_compulsory_bytes_only():
    """A scan's roofline bytes are the compulsory bytes it moves itself (x in,
    y out, B, C and D in); the chunk states it reads are not among them."""
    cfg = dict(WORKLOADS["sweep_N128_Q256"])
    wm = bench.work_model(cfg, True, layout(cfg))
    B, T, H, P, N, G = 2, 8192, 32, 64, 128, 1
    x = B * T * H * P * 2
    bc = 2 * B * T * G * N * 2
    assert wm["per_kernel_comp"]["ssd_chunk_scan"] == 2 * x + bc + H * 4
    assert wm["per_kernel_comp"]["ssd_chunk_cumsum"] == B * T * H * 4 + H * 4
    assert wm["per_kernel_comp"]["ssd_chunk_scan"] < wm["per_kernel_bytes"]["ssd_chunk_scan"]


def test_both_arms_build_the_same_config_block():
    """The reference arm and the GPU arm describe one workload with one config
    block when they see the same L2 size."""
    cfg = dict(WORKLOADS["mamba2_2p7b"])
    cfg.setdefault("final_state", True)
    l2 = 133 * 1000 * 1000
    a = bench.config_block(cfg, "mamba2_2p7b", bench.l2_policy(cfg, l2)[1])
    b = bench.config_block(cfg, "mamba2_2p7b", bench.l2_policy(cfg, l2)[1])
    assert a == b
    # without a GPU the helper falls back to the nominal L2 size
    assert bench.device_l2_bytes() > 0


def test_backward_launch_count_by_hand():
    """The launches one ssd_backward call makes on the 2.7B-shaped layer (bf16,
    no initial state): prep_k, prep_t and three fp32 copies (x, B, C); the
    transposed dfinal; the scans of K and h (4 launches each); the transposed
    scans, two 64-wide dstate slices each on the bf16 tensor-core plan (4
    launches each); and the five finishing kernels -- 35, the count of the
    ncu launch list of that layer (175 launches over 5 calls)."""
    from structured_state_space_mamba_b200.inputs import make_workload
    assert bench.backward_launches(make_workload("mamba2_2p7b")) == 5 + 1 + 2 * 4 + 2 * 2 * 4 + 5


def test_presolved_layout_recognised_with_a_ragged_tail():
    """A presolved single-pass layout keeps its accounting when the length
    leaves a ragged tail (one more launch, the tail kernel)."""
    cfg = dict(WORKLOADS["long_g8"])
    cfg["seqlen"] = cfg["seqlen"] - 100
    lay = layout(cfg)
    assert lay.single_pass == 1 and lay.launches == 6
    wm = bench.work_model(cfg, True, lay)
    assert wm["stages"] == ("ssd_chunk_cumsum", "ssd_range_states", None, "ssd_chunk_fused")
