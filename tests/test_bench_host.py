"""Host logic of bench.py (CPU only): the traffic record's source key (comments
and blank lines do not change it, code does) and the algorithmic counts the
roofline uses."""
import bench


def test_source_hash_ignores_comments_only(tmp_path):
    a = tmp_path / "a.cu"
    a.write_text("// header\n__global__ void k(int *p) {\n    p[0] = 1;  // store\n}\n")
    b = tmp_path / "b.cu"
    b.write_text("/* a block\n   comment */\n__global__ void k(int *p) {\n\n    p[0] = 1;\n}\n// tail\n")
    c = tmp_path / "c.cu"
    c.write_text("__global__ void k(int *p) {\n    p[0] = 2;\n}\n")
    assert bench.source_hash(str(a)) == bench.source_hash(str(b))
    assert bench.source_hash(str(a)) != bench.source_hash(str(c))



def test_algorithmic_counts_bf16_and_fp8():
    """Layer FLOPs and bytes as the roofline uses them: expert FLOPs on kept
    rows; x + y + W_r + the weights of experts that kept a row (e4m3 experts:
    one byte per weight and a 4-byte scale per output channel)."""
    import numpy as np
    from mixture_experts_layer_49_b200 import synthetic as syn
    wl = syn.Workload("c", T=64, d_model=32, E=4, d_ff=16, top_k=2)          # SwiGLU, bf16
    kept = np.array([40, 0, 50, 38])
    flops, b, rows = bench.algorithmic_counts(wl, kept, kept)
    assert rows == 128
    assert flops == 2 * 128 * 32 * 16 * 3
    xy = 2 * 64 * 32 * 2
    wr = 32 * 4 * 4
    assert b == xy + wr + 3 * (3 * 32 * 16 * 2)                              # three touched experts
    _, b8, _ = bench.algorithmic_counts(wl, kept, kept, fp8=True)
    assert b8 == xy + wr + 3 * (3 * 32 * 16 * 1) + 3 * 4 * (2 * 16 + 32)


def test_tensor_peak_follows_the_runs_clock_record():
    import bench
    peaks = {"hbm_gbs": 6557.0, "bf16_tflops": 1667.1, "bf16_tflops_sustained": 1408.6}
    assert bench.tensor_peak(peaks, {"reasons": []})[0] == 1667.1
    assert bench.tensor_peak(peaks, {"reasons": ["sw_power_cap"]})[0] == 1408.6
    assert bench.tensor_peak(peaks, {"reasons": None})[0] == 1667.1


def test_roofline_fields_use_the_chosen_peak():
    import numpy as np
    import bench
    peaks = {"hbm_gbs": 6557.0, "bf16_tflops": 1667.1, "bf16_tflops_sustained": 1408.6}
    r = dict(flops=1.2e12, ms=1.3, bound="tensor", layer_roof_ms=1.2e12 / 1667.1e9, layer_roof_burst_ms=0.72,
             layer_roof_sust_ms=0.85, alg_bytes=1.3e9, peaks=peaks, peak_src="measured", peak_t=1667.1,
             peak_which="burst", ffn_tflops=1100.0, traffic=None, stage_avg={"grouped_ffn": 1.0},
             kept_rows=100, n_dropped=0, loss=1.0, counts=np.array([1, 2]))
    f = bench.roofline_fields(r, fp8=False)
    assert abs(f["roofline"]["frac"] - 1100.0 / 1667.1) < 1e-12
    assert abs(f["roofline"]["frac_sustained"] - 1100.0 / 1408.6) < 1e-12
    assert f["layer_roofline"]["frac"] == r["layer_roof_ms"] / 1.3
    assert "of measured" in f["roofline"]["peak_note"]
