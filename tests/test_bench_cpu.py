"""bench.py's host-side accounting and its CPU reference arm for the codec workload (no GPU).

The byte counts are the codec's algorithmic traffic ("quantization_mxfp4" (KerasFormers),
Primitives: one 16-byte block of e2m1 pairs and one e8m0 scale byte per 32 values), and
the per-expert packed size is the 120B-shaped expert set's (4.25 bits per weight)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_codec_leg_bytes_closed_forms():
    # one row of one 32-value block: 128 B of fp32, 16 B of blocks, 1 scale byte
    b = bench.codec_leg_bytes(1, 32)
    assert b == {"quantize": 128 + 16 + 1, "dequantize_bf16": 16 + 1 + 64, "dequantize_f32": 16 + 1 + 128}
    # the full sweep: 128 experts x (5760 + 2880) rows x 2880 values
    n = 128 * 8640 * 2880
    full = bench.codec_leg_bytes(128 * 8640, 2880)
    assert full["quantize"] == 4 * n + n // 2 + n // 32
    assert full["dequantize_f32"] == full["quantize"]
    assert full["dequantize_bf16"] == n // 2 + n // 32 + 2 * n


def test_per_expert_packed_bytes():
    # gate_up 8,294,400 B of blocks + 518,400 B of scales, down half of each
    assert bench.PER_EXPERT_PACKED(2880, 2880) == 8_812_800 + 4_406_400 == 13_219_200


def test_codec_reference_arm_runs_on_cpu_and_only_on_rank_0():
    class A:
        workload, steps, warmup, ref_step_s, codec_experts = "codec", 1, 3, 0.0, 128

    assert bench.run_reference_codec(A(), world=2, rank=1) is None
    res = bench.run_reference_codec(A(), world=1, rank=0)
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "config", "cpu_baseline", "e2e"):
        assert key in res
    assert res["impl"] == "reference" and res["metric"] == bench.CODEC_METRIC and res["unit"] == "GB/s"
    assert res["value"] > 0 and res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["e2e"]["d2h_bytes_per_step"] == 0


def test_ncu_traffic_reads_the_matching_block_and_drops_stale_sources(tmp_path, monkeypatch):
    import hashlib
    (tmp_path / "profiles").mkdir()
    src = tmp_path / "k.cu"
    src.write_text("kernel source\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles" / "p.md").write_text(
        "# summary\n\n"
        "- workload: prefill\n- kernel: gate_up\n- traffic_bytes_per_launch: 123\n"
        f"- source: k.cu sha256 prefix {digest}\n\n"
        "- workload: prefill\n- kernel: down\n- traffic_bytes_per_launch: 45\n"
        f"- source: k.cu sha256 prefix {digest}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.ncu_traffic("prefill", "gate_up") == 123
    assert bench.ncu_traffic("prefill", "down") == 45
    assert bench.ncu_traffic("decode1", "gate_up") is None
    src.write_text("kernel source, edited\n")          # the counters no longer describe it
    assert bench.ncu_traffic("prefill", "gate_up") is None


def test_step_roofline_against_both_bounds():
    pk = {"hbm_gbs": 6538.6, "bf16_tflops": 1628.9, "bf16_tflops_sustained": 1376.3}
    # the 120B prefill step: 1,744,404,480 B and 818,392,596,480 FLOP
    r = bench.step_roofline(1_744_404_480, 818_392_596_480, 0.85, pk, fp8=True, fp8_peak=2500.0)
    m, n = r["measured"], r["nominal"]
    assert m["bound"] == "tensor" and abs(m["t_bound_ms"] - 818.392596480 / 2500.0) < 1e-5
    # without a probe figure: twice the measured bf16 burst peak
    r2 = bench.step_roofline(1_744_404_480, 818_392_596_480, 0.85, pk, fp8=True)
    assert r2["measured"]["tensor_tflops"] == 2 * 1628.9
    assert abs(m["frac"] - m["t_bound_ms"] / 0.85) < 1e-4
    # nominal: 218 us of bytes at 8 TB/s against 182 us of FP8 FLOPs at 4.5 PF
    assert n["bound"] == "hbm" and abs(n["t_bound_ms"] - 0.2180506) < 1e-6
    # bf16 activations take the bf16 peaks
    b = bench.step_roofline(1_744_404_480, 818_392_596_480, 1.52, pk, fp8=False)
    assert b["measured"]["tensor_tflops"] == 1628.9 and b["nominal"]["tensor_tflops"] == 2250.0
    assert b["nominal"]["bound"] == "tensor"


def test_cpulist_and_numa_fallback(monkeypatch):
    assert bench._cpulist("0-3,8-11,16\n") == {0, 1, 2, 3, 8, 9, 10, 11, 16}
    assert bench._cpulist("5") == {5}

    class Props:   # a device whose PCI node file does not exist: no placement, no error
        pci_domain_id, pci_bus_id, pci_device_id = 0xFFFF, 0xFF, 0x1F

    monkeypatch.setattr(bench.torch.cuda, "get_device_properties", lambda dev: Props())
    assert bench.gpu_numa_cpus(0) == (None, None)


def test_one_token_oracle_figure_on_cpu_tensors():
    from helpers import pack, to_device
    from mxfp4_block_scaled_moe_b200 import inputs
    lay = inputs.small_layer(E=8, k=2, T=2, H=128, I=128, seed=1)
    d = to_device(pack(lay), device="cpu")
    r = bench.oracle_one_token(lay, d, None)
    assert r["cores"] == 1 and r["kind"] == "oracle" and r["value"] > 0 and lay.name in r["sample"]
