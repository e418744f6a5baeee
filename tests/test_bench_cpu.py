"""The benchmark's work model on the CPU: the algorithmic bytes and FLOPs behind every
roofline fraction, against the layer's sizes written out by hand."""
import synth

import bench

SHAPE = synth.Shape(T=8, H=2816, E=128, k=8, I=704, D=2112)


def test_flops_per_token_of_the_layer():
    # 2 k 3 I H (routed experts) + 2 3 D H (dense MLP) + 2 E H (router) per token
    a = bench.algorithmic(SHAPE, used_experts=50)
    per_token = a["flops"] / SHAPE.T
    assert per_token == 2 * 8 * 3 * 704 * 2816 + 2 * 3 * 2112 * 2816 + 2 * 128 * 2816
    assert abs(per_token / 1e6 - 131.56) < 0.01


def test_bytes_count_the_used_experts_and_the_weight_type():
    H, E, I, D, T = 2816, 128, 704, 2112, 8
    fixed = 3 * D * H * 2 + E * H * 2 + 6 * H * 2 + E * 2 + 2 * T * H * 2
    for u in (1, 54, 128):
        assert bench.algorithmic(SHAPE, u)["bytes"] == u * 3 * I * H * 2 + fixed
        # 8-bit experts (int8 or E4M3): one byte per weight plus an fp32 scale per row
        assert bench.algorithmic(SHAPE, u, True)["bytes"] == \
            u * (3 * I * H + (2 * I + H) * 4) + fixed
        # NVFP4 experts: half a byte per weight, an E4M3 scale per 16 weights, an fp32
        # scale per matrix (two matrices per expert)
        assert bench.algorithmic(SHAPE, u, nvfp4=True)["bytes"] == \
            u * (3 * I * H * (0.5 + 1 / 16) + 2 * 4) + fixed
    assert bench.algorithmic(SHAPE, 54, nvfp4=True)["gate_up_bytes"] == \
        (54 * (2 * I * H * (0.5 + 1 / 16) + 4) + 2 * D * H * 2 + (T * 8 + T) * H * 2
         + (T * 8 * I + T * D) * 2)
    # the gate_up launch alone: its weights, token rows in, h out
    g = bench.algorithmic(SHAPE, 54)
    assert g["gate_up_bytes"] == (54 * 2 * I * H * 2 + 2 * D * H * 2 + (T * 8 + T) * H * 2
                                  + (T * 8 * I + T * D) * 2)
    assert g["gate_up_flops"] == T * (2 * 8 * 2 * I * H + 2 * 2 * D * H)


def test_clock_record_keeps_every_throttle_reason():
    """A throttle reason seen Active in any sample is reported (a run with hw or thermal
    slowdown must be recognisable); the SM clock is the median; bad lines are skipped."""
    txt = "\n".join([
        "1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "1500, 1965, 998.0, 0x4, Not Active, Not Active, Not Active, Active",
        "1400, 1965, 999.0, 0x8, Active, Not Active, Not Active, Active",
        "garbage line",
        "N/A, 1965, 1.0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ])
    r = bench.parse_clock_samples(txt)
    assert r == {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0,
                 "reasons": ["hw_slowdown", "sw_power_cap"], "samples": 3}
    assert bench.parse_clock_samples("") is None


def test_traffic_record_follows_the_kernel_code(tmp_path, monkeypatch):
    """The ncu DRAM traffic of a summary is used only while the GEMM's code (comments
    aside) still hashes to the value recorded with it."""
    monkeypatch.setattr(bench, "PROFILES", str(tmp_path))
    (tmp_path / "k.md").write_text(
        "notes\n\n    traffic_bytes_per_launch: 123456\n"
        f"    source_sha256: {bench.kernel_sha()}\n")
    assert bench.ncu_traffic("k.md") == 123456
    (tmp_path / "s.md").write_text(
        "    traffic_bytes_per_launch: 123456\n    source_sha256: " + "0" * 64 + "\n")
    assert bench.ncu_traffic("s.md") is None
    assert bench.ncu_traffic("missing.md") is None
