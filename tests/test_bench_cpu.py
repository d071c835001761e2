"""Host-side pieces of the benchmark (no GPU): the compact summary that ends
the JSON line, and the lookup of ncu traffic figures tied to a source hash."""
import hashlib
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _fake_out():
    k = {"frac_of_measured_pipe": 0.5}
    b = {"o_proj_topk_w2a8_4096x4096x4096": {"gemm_frac_of_pipe": 0.6, "topk_frac_hbm": 0.3},
         "down_proj_relu2_w2a8_4096x11008x4096": {"gemm_frac_of_pipe": 0.7, "relu2_quant_frac_hbm": 0.74},
         "decode_llama7b_layer": {"weight_bytes": 1, **{f"batch{n}": {"weight_frac_hbm": 0.4, "gemv_sum_us": 20.0}
                                                        for n in (1, 4, 8, 64)}},
         "kv_quant_3bit_2x4096x32x128": {"frac_hbm": 0.56},
         "kv_attention_3bit_4096x32x128": {"queries1": {"frac_hbm": 0.09}, "queries8": {"frac_hbm": 0.05}}}
    return {"value": 2400.0, "roofline": {"frac": 0.62}, "tensor_pipe_peaks_TOPS": {"i8_pair": 4500.0},
            "kernels": {n: dict(k) for n in bench.GEMM_NAMES}, "breakdown": b,
            "e2e": {"value": 87.0}, "cpu_baseline": {"value": 0.05, "single_thread": {"value": 0.01}}}


def test_summary_is_short_and_complete():
    sm = bench.summary(_fake_out())
    text = json.dumps({"summary": sm})
    assert len(text) < 1400  # fits in the tail of a log that keeps 1500 characters
    assert set(sm["decode_weight_frac_hbm"]) == {"batch1", "batch4", "batch8", "batch64"}
    assert set(sm["gemm_frac_of_pipe"]) == set(bench.GEMM_NAMES) | {"o_proj", "down_proj"}
    assert sm["kv_attn_frac_hbm"] == {"queries1": 0.09, "queries8": 0.05}
    assert sm["cpu_TOPS"] == {"all_cores": 0.05, "one_core": 0.01}


def test_traffic_lookup_follows_the_source_hash(tmp_path, monkeypatch):
    src = os.path.join(bench.CSRC, "gemm.cu")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps({"k_ok": {"source": "gemm.cu", "source_sha256": h, "dram_bytes_per_launch": 123.0},
                             "k_old": {"source": "gemm.cu", "source_sha256": "0" * 64,
                                       "dram_bytes_per_launch": 9.0}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.read_traffic("k_ok") == (123.0, "ncu")
    assert bench.read_traffic("k_old")[0] is None
    assert bench.read_traffic("missing")[0] is None
