"""Host-side logic of bench.py that runs without a GPU: traffic figures are
taken from a committed ncu summary only while its source hash matches, the
clock sampler's summary reads nvidia-smi CSV rows, peaks come from the
measured file, and the reference arm prints its JSON line from the oracle."""

import json
import os

import bench


def test_profile_traffic_requires_matching_source(tmp_path):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1")
    prof = tmp_path / "p.json"
    prof.write_text(json.dumps({"source_sha256": bench.sources_sha256([str(src)]), "dram_bytes_per_launch": 123.0}))
    assert bench.profile_traffic(str(prof), [str(src)]) == 123.0
    src.write_text("kernel v2")  # the kernel changed after the capture: no traffic figure
    assert bench.profile_traffic(str(prof), [str(src)]) is None
    assert bench.profile_traffic(str(tmp_path / "missing.json"), [str(src)]) is None


def test_committed_profiles_are_keyed_to_sources():
    # every summary the bench reads names the sources it was taken on and its command; a summary that
    # is not there (yet) gives a null traffic figure, never a stale one
    found = 0
    for name, (prof, sources) in list(bench.ROW_PROFILES.items()) + [("headline", (bench.GEMM_PROFILE,
                                                                                    bench.GEMM_SOURCES))]:
        assert all(os.path.exists(s) for s in sources)
        if not os.path.exists(prof):
            assert bench.profile_traffic(prof, sources) is None
            continue
        found += 1
        d = json.load(open(prof))
        assert len(d["source_sha256"]) == 64 and d["dram_bytes_per_launch"] > 0 and "ncu" in d["command"]
    assert found >= 1


def test_profile_traffic_per_workload(tmp_path):
    src = tmp_path / "k.cu"
    src.write_text("kernel")
    prof = tmp_path / "p.json"
    prof.write_text(json.dumps({"source_sha256": bench.sources_sha256([str(src)]),
                                "per_workload": {"a": {"dram_bytes_per_launch": 7.0}}}))
    assert bench.profile_traffic(str(prof), [str(src)], workload="a") == 7.0
    assert bench.profile_traffic(str(prof), [str(src)], workload="b") is None  # not captured: no figure
    src.write_text("kernel v2")
    assert bench.profile_traffic(str(prof), [str(src)], workload="a") is None


def test_few_token_profiles_cover_the_kernel_each_shape_runs():
    # the text-encoder shapes: 21 tokens and 130 x 2560 -> 2560 run the few-token kernel, 130 x 2560 -> 9728
    # the CTA-pair kernel (76 weight tiles x a split of 2 would need 152 SMs); each summary holds the
    # shapes its kernel serves
    sms = 148
    assert bench.few_token_gemm(21, 9728, sms) == "small"
    assert bench.few_token_gemm(21, 2560, sms) == "small"
    assert bench.few_token_gemm(130, 9728, sms) == "pair"
    assert bench.few_token_gemm(130, 2560, sms) == "small"
    assert bench.few_token_gemm(128, 1 << 20, sms) == "small"  # up to 128 tokens whatever N
    assert bench.few_token_gemm(257, 256, sms) == "pair"
    for kern, names in (("small", ["text_enc_up_21", "text_enc_down_21", "text_enc_down_130"]),
                        ("pair", ["text_enc_up_130"])):
        prof, sources = bench.FEW_TOKEN_PROFILES[kern]
        d = json.load(open(prof))
        assert len(d["source_sha256"]) == 64 and "ncu" in d["command"]
        for n in names:
            assert d["per_workload"][n]["dram_bytes_per_launch"] > 0


def test_clock_summary_parses_nvidia_smi_rows(tmp_path):
    c = bench.ClockSampler("GPU-test")
    c.proc = object()  # as if a sampler had run
    c.path = str(tmp_path / "clocks.csv")
    rows = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 980.3, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 345, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active",  # idle sample
        "garbage line",
    ]
    open(c.path, "w").write("\n".join(rows) + "\n")
    s = c.summary()
    assert s["sm_max_mhz"] == 1965.0
    assert s["sm_mhz"] == 1957.5  # median of the loaded samples
    assert s["reasons"] == ["sw_power_cap"]
    assert s["samples"] == 3


def test_peaks_come_from_the_measured_file():
    peaks, kind = bench.load_peaks()
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        assert kind == "measured" and peaks["bf16_tflops"] > 0 and peaks["hbm_gbs"] > 0
    else:
        assert kind == "fallback"


def test_reference_arm_prints_one_json_line(capsys, monkeypatch):
    # the oracle arm on the tiny workload, one step: the line carries the contract's keys
    monkeypatch.delenv("RANK", raising=False)
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    args = bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0", "--workload", "tiny"])
    assert bench.step_layers("tiny") == ("tiny",) and bench.step_layers("dit_mlp") == ("dit_mlp_up", "dit_mlp_down")
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["impl"] == "reference" and line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    cpu = line["cpu_baseline"]
    assert cpu["cores"] >= 1 and cpu["nproc"] >= 1 and cpu["cpu_model"]
