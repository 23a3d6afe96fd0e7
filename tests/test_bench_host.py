"""Host-side logic of bench.py (CPU only): the stage folding that turns the
timed forward's six stage slots into the stages the plan runs, the committed
traffic figures being used only for the GEMM sources they were taken on, and
the workload description of the JSON line."""
import os
import shutil

import pytest

import bench
from nvfp4_moe_expert_topk_b200 import workloads as W


class _Plan:
    """A Workload's plan without the device (fold() reads only the plan)."""

    def __init__(self, fused, pair_mode=0):
        self.fused = fused
        self.pair_mode = pair_mode


STAGE_MS = {"global_scale": 0.01, "route": 0.02, "quantize_permute": 0.04,
            "l1_gate_up_swiglu_quant": 2.0, "l2_down": 1.0, "combine": 0.07}


def test_fold_fused_plan():
    d = bench.Workload.fold(_Plan(True), STAGE_MS)
    assert set(d) == {bench.FRONT_STAGE, bench.FUSED_STAGE, "combine"}
    assert d[bench.FRONT_STAGE] == pytest.approx(0.07)
    assert d[bench.FUSED_STAGE] == pytest.approx(3.0)
    assert sum(d.values()) == pytest.approx(sum(STAGE_MS.values()))


def test_fold_two_launch_plan():
    d = bench.Workload.fold(_Plan(False), STAGE_MS)
    assert set(d) == {bench.FRONT_STAGE, "l1_gate_up_swiglu_quant", "l2_down", "combine"}
    assert d["l2_down"] == 1.0


def test_fold_split_plan_and_its_bytes():
    """Pair mode 1: the fused pair launch and the fused 1-CTA launch are two
    stages; each stage's algorithmic bytes read the experts it touches once
    (an expert with an odd number of m-tiles is read by both).  The tile
    split follows the plan's rule."""
    import numpy as np
    d = bench.Workload.fold(_Plan(True, 1), STAGE_MS)
    assert set(d) == {bench.FRONT_STAGE, bench.PAIRS_STAGE, bench.LIGHT_STAGE, "combine"}
    assert d[bench.PAIRS_STAGE] == 2.0 and d[bench.LIGHT_STAGE] == 1.0
    cfg = W.MoeConfig("t", E=4, k=2, T=400, H=256, I=128, routing="softmax", outliers=False, warmup_T=8)
    counts = np.array([300, 256, 44, 200])          # m-tiles 3, 2, 1, 2
    pair_rows, light_rows = bench.tile_split(counts, 1)
    assert list(pair_rows) == [256, 256, 0, 200] and list(light_rows) == [44, 0, 44, 0]
    assert list(bench.tile_split(counts, 2)[0]) == [300, 256, 44, 200]
    assert list(bench.tile_split(counts, 0)[1]) == [300, 256, 44, 200]
    split = bench.stage_bytes(cfg, counts, True, 1)
    whole = bench.stage_bytes(cfg, counts, True, 0)
    w_expert = 3 * cfg.H * cfg.I * bench.FP4_BYTES
    # the pairs and the light launch read expert 0's weights each; the rest once
    assert split[bench.PAIRS_STAGE] + split[bench.LIGHT_STAGE] == pytest.approx(whole[bench.FUSED_STAGE] + w_expert)
    assert bench.launches_per_step(True, 0) == 3 and bench.launches_per_step(True, 1) == 4
    assert bench.launches_per_step(False, 2) == 4 and bench.launches_per_step(False, 0) == 4


def _copy_tree(tmp_path):
    root = tmp_path / "repo"
    csrc = root / "nvfp4_moe_expert_topk_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.GEMM_SOURCES:
        shutil.copy(os.path.join(bench.ROOT, "nvfp4_moe_expert_topk_b200", "csrc", name), csrc / name)
    (root / "profiles").mkdir()
    return root, csrc


def test_source_hash_ignores_comments_not_code(tmp_path, monkeypatch):
    root, csrc = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    h0 = bench.gemm_source_sha()
    assert h0 == bench.gemm_source_sha()
    g = csrc / "gemm.cu"
    text = g.read_text()
    g.write_text("// a new comment line\n/* and a block\n   comment */\n" + text.replace("\n", "\n\n", 3))
    assert bench.gemm_source_sha() == h0                  # comments and blank lines only
    g.write_text(text.replace("kBM = 128", "kBM = 64", 1))
    assert "kBM = 64" in g.read_text()
    assert bench.gemm_source_sha() != h0                  # a code change


def test_traffic_used_only_for_matching_sources(tmp_path, monkeypatch):
    root, csrc = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    prof = root / "profiles" / "ncu_traffic.txt"
    assert bench.ncu_traffic("l1_l2_fused", "decode") is None            # no summary
    prof.write_text(f"# comment\nsource_sha: {bench.gemm_source_sha()}\n"
                    "decode.l1_l2_fused.dram_bytes_per_launch: 1809793536\n")
    assert bench.ncu_traffic("l1_l2_fused", "decode") == 1809793536.0
    assert bench.ncu_traffic("l1_l2_fused", "prefill") is None           # not captured
    prof.write_text("source_sha: 0123456789abcdef\ndecode.l1_l2_fused.dram_bytes_per_launch: 1\n")
    assert bench.ncu_traffic("l1_l2_fused", "decode") is None            # taken on other sources


def test_config_block_names_the_workload():
    c = bench.config_block(W.MOE_CONFIGS["prefill"], 8)
    assert c["workload"] == "prefill_moe_E384_k6_T4096_H7168_I3072_zipf1.1_16empty"
    assert c["global_batch"] == 8 * 4096 and c["tokens_per_gpu"] == 4096
    assert c["parallelism"].startswith("dp8")
    c1 = bench.config_block(W.MOE_CONFIGS["decode_shared"], 1)
    assert c1["workload"] == "decode_shared_moe_E49_k7_T64_H7168_I3072"
    assert c1["parallelism"] == "replicas"


def test_clock_regions_summarise_only_their_samples():
    c = bench.Clocks(device=None)
    c.source = "test"
    cap, hw = bench.Clocks.REASONS["sw_power_cap"], bench.Clocks.REASONS["hw_slowdown"]
    # (monotonic s, SM MHz, max MHz, power W, reason bits)
    c.samples = [(1.0, 1965.0, 1965.0, 400.0, 0), (2.0, 1400.0, 1965.0, 990.0, cap),
                 (2.1, 1420.0, 1965.0, 995.0, cap), (3.0, 1000.0, 1965.0, 500.0, hw)]
    c.regions = {"a": (1.5, 2.5), "b": (2.9, 3.1), "empty": (5.0, 6.0)}
    a = c.summary(["a"])
    assert a["sm_mhz"] == 1410.0 and a["samples"] == 2 and a["reasons"] == ["sw_power_cap"]
    assert c.summary(["b"])["reasons"] == ["hw_slowdown"]
    assert c.summary(["empty"])["samples"] == 0 and c.mhz("empty") is None
    both = c.summary()
    assert both["samples"] == 3 and both["sm_max_mhz"] == 1965.0
    t = bench.compact({"x": 3.14159265, "y": [2.718281828], "z": "s", "n": 7})
    assert t == {"x": 3.142, "y": [2.718], "z": "s", "n": 7}



def test_source_hash_ignores_other_declarations_not_gemm_args(tmp_path, monkeypatch):
    """Of internal.h only the GemmArgs struct the kernels take counts: a new
    declaration of another kernel keeps the key, a GemmArgs field changes it."""
    root, csrc = _copy_tree(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    h0 = bench.gemm_source_sha()
    ih = csrc / "internal.h"
    text = ih.read_text()
    assert "struct GemmArgs {" in text
    ih.write_text(text.replace("namespace nvfp4 {", "namespace nvfp4 {\nint another_kernel_launch(int n);", 1))
    assert bench.gemm_source_sha() == h0
    ih.write_text(text.replace("struct GemmArgs {", "struct GemmArgs {\n    int extra_field;", 1))
    assert bench.gemm_source_sha() != h0
