"""Host-side parts of bench.py that run without a GPU: the reference arm (the
oracle timed on the host cores) prints one JSON line with the contract's keys,
the traffic lookup is tied to the kernels' current sources, and the kernel
count per step follows the launch sequence of the library."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0", "--ref-tokens", "16"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT, check=True).stdout
    line = json.loads(out.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "relu_ffn_layer_1.5b"
    # the step time is what was measured for the sampled tokens, not scaled up
    assert line["config"]["tokens_per_step"] == 16
    assert line["ms_per_step"] <= 1e3 * line["total_timed_s"] * 1.0001
    assert abs(line["value"] - 16 / (line["ms_per_step"] * 1e-3)) < 1e-6 * line["value"]


def test_cpu_baseline_reports_all_cores_one_core_and_the_packer():
    import twell_synth as S
    L = S.tiny_relu(0)
    cb = bench._cpu_baseline(L, seconds=0.2, sample_tokens=32)
    assert cb["kind"] == "oracle" and cb["value"] > 0 and cb["cores"] >= 1
    assert cb["value_1core"] is None or cb["value_1core"] > 0
    assert cb["pack_tokens_s"] > 0 and "pack" in cb["sample_pack"]


def test_median():
    assert bench._median([3.0, 1.0, 2.0]) == 2.0
    assert bench._median([4.0, 1.0, 2.0, 3.0]) == 2.5


def test_traffic_lookup_follows_the_kernel_source(monkeypatch, tmp_path):
    src = tmp_path / "activation_sparse_ffn_twell_b200" / "csrc"
    src.mkdir(parents=True)
    (src / "k_demo.cu").write_text("// kernel v1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench._kernel_source_hash(os.path.join("activation_sparse_ffn_twell_b200", "csrc", "k_demo.cu"))
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"w": {"k_demo": {"source": "k_demo.cu", "source_sha256_16": h, "dram_bytes_per_launch": 123}}}))
    assert bench._ncu_traffic("k_demo", "w") == 123.0
    assert bench._ncu_traffic("k_demo", "other") is None
    (src / "k_demo.cu").write_text("// kernel v2\n")            # the kernel changed: no figure
    assert bench._ncu_traffic("k_demo", "w") is None


def test_kernels_per_step():
    # reset, producer, backup scan, scatter + block pass, gather, tensor-core kernel
    assert bench._kernels_per_step("auto", False, 2048) == 7
    # the 2:4 path (sparse mode only): prep, decision, 2:4 kernel, dense kernel
    assert bench._kernels_per_step("auto", False, 2048, True) == 7
    assert bench._kernels_per_step("sparse", False, 2048, True) == 8
    # + block pass (split counters) and the tensor-core kernel
    assert bench._kernels_per_step("mma", False, 2048) == 6
    assert bench._kernels_per_step("mma", False, 256) == 5
    assert bench._kernels_per_step("gather", False, 2048) == 5
    # decode-size: the split-K down kernel alone; up to 256 tokens the backup scan
    # and scatter are one kernel
    assert bench._kernels_per_step("auto", True, 4096) == 5
    assert bench._kernels_per_step("auto", True, 4096, False, True) == 6   # + k_dec_touch
    assert bench._kernels_per_step("auto", True, 4096, False, False, 128) == 4
    assert bench._kernels_per_step("auto", True, 4096, False, True, 32) == 5


def test_decode_touched_rule(monkeypatch):
    """The bench's restatement of the library's choice of the touched-unit decode
    kernel: up to 32 tokens by default, never with TWELL_DECODE_TOUCHED=0, every
    decode-size batch whose stage ring allows it with =all."""
    monkeypatch.delenv("TWELL_DECODE_TOUCHED", raising=False)
    assert bench._decode_touched(32, 16384) and not bench._decode_touched(33, 16384)
    assert not bench._decode_touched(32, 131072)            # d_ff above 65536
    monkeypatch.setenv("TWELL_DECODE_TOUCHED", "0")
    assert not bench._decode_touched(1, 16384)
    monkeypatch.setenv("TWELL_DECODE_TOUCHED", "all")
    assert bench._decode_touched(128, 16384) and not bench._decode_touched(256, 16384)
