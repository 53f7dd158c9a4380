"""Host logic of bench.py: the algorithmic work it divides by, the roofline it reports and the
gating of stored DRAM-traffic records.  No GPU.

The per-call work follows the store layout of [LLA §3 eq. (4)]: a decode call reads every cached
token's latents once, (r_k + r_v) bf16 values per head (one row for all heads in LLA-2D), and the
compression ratio is rho = 2 T d_head / (r_k + r_v) (2 T H d_head / (r_k + r_v) for LLA-2D).
"""

import json

import pytest

import bench
import lla_synth as syn


@pytest.mark.parametrize("name,rho", [("tiny_d16_t4", 32 / 3), ("ouro_rho4_b32_n4096", 4.0),
                                      ("ouro_rho21_b768_n4096", 64 / 3), ("ouro_2d_b256_n8192", 256 / 3),
                                      ("huginn_t32_b16_n32768", 32.0)])
def test_compression_ratio_of_each_workload(name, rho):
    assert bench.rho_of(syn.CONFIGS[name]) == pytest.approx(rho, rel=1e-12)


def test_algorithmic_bytes_and_flops_per_call():
    # batch 768 x 4096 tokens x 16 heads x (16 + 32) bf16 latents
    assert bench.bytes_per_call(syn.CONFIGS["ouro_rho21_b768_n4096"]) == 768 * 4096 * 16 * 48 * 2 == 4_831_838_208
    # LLA-2D: one (64 + 128)-wide row per token for all heads
    c2d = syn.CONFIGS["ouro_2d_b256_n8192"]
    assert bench.bytes_per_call(c2d) == 256 * 8192 * 192 * 2 == 805_306_368
    # key reconstruction [tokens x r_k] . [r_k x H d]: 2 flops per multiply-add
    assert bench.flops_per_call(c2d) == 2 * 256 * 8192 * 16 * 128 * 64
    assert bench.flops_per_call(c2d) == pytest.approx(0.550e12, rel=1e-3)


def test_roofline_against_the_measured_peaks():
    cfg = syn.CONFIGS["ouro_rho21_b768_n4096"]
    hbm, kind = bench.measured_peak("hbm_gbs")
    r = bench.roofline(cfg, "tc", [1.0, 1.0, 1.0], "ouro_rho21_b768_n4096")
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(4831.838208, rel=1e-9)  # bytes per call over 1 ms
    assert r["frac"] == pytest.approx(r["achieved"] / hbm) and r["peak"] == hbm
    assert r["peak_source"].startswith(kind)
    r2 = bench.roofline(syn.CONFIGS["ouro_2d_b256_n8192"], "tc", [2.0], "ouro_2d_b256_n8192")
    tf, _ = bench.measured_peak("bf16_tflops_sustained")
    assert r2["bound"] == "tensor" and r2["unit"] == "TFLOP/s" and r2["peak"] == tf
    assert r2["achieved"] == pytest.approx(2 * 256 * 8192 * 16 * 128 * 64 / 2e-3 / 1e12)


def test_traffic_record_only_for_current_sources(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    rec = {"kernel": "k", "workload": "w", "source_sha256": "abc", "dram_bytes_per_launch": 1234}
    (tmp_path / "profiles" / "traffic_tc_w.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_sha", lambda kernel: "abc")
    assert bench.traffic_record("tc", "w") == 1234
    monkeypatch.setattr(bench, "kernel_sha", lambda kernel: "changed")
    assert bench.traffic_record("tc", "w") is None  # the kernel changed since the counters were taken
    assert bench.traffic_record("tc", "other") is None


def test_committed_traffic_records_name_their_sources():
    for w in ("ouro_rho21_b768_n4096", "ouro_rho4_b32_n4096", "ouro_2d_b256_n8192", "huginn_t32_b16_n32768"):
        with open(f"{bench.ROOT}/profiles/traffic_tc_{w}.json") as f:
            j = json.load(f)
        assert j["workload"] == w and len(j["source_sha256"]) == 64
        # traffic at or a little above the latents the call must read
        assert bench.bytes_per_call(syn.CONFIGS[w]) <= j["dram_bytes_per_launch"] <= 1.2 * bench.bytes_per_call(
            syn.CONFIGS[w])


def test_defaults(monkeypatch):
    monkeypatch.setattr("sys.argv", ["bench.py"])
    a = bench.parse()
    assert a.gpus == 1 and a.steps >= 1 and a.warmup >= 3 and a.kernel_sample >= 1
    assert a.workload == "ouro_rho21_b768_n4096"


def test_kernel_sha_ignores_comments_only():
    """A traffic record stays valid across comment-only edits of its kernel's sources, and not
    across code edits (string literals count as code)."""
    base = 'int a = 1; // note\n/* block\n comment */ f("// kept");\n'
    assert bench._code_only(base) == bench._code_only(base.replace("// note", "// another note"))
    assert bench._code_only(base) == bench._code_only(base.replace("block", "longer block"))
    assert bench._code_only(base) != bench._code_only(base.replace("a = 1", "a = 2"))
    assert bench._code_only(base) != bench._code_only(base.replace('"// kept"', '"// changed"'))


@pytest.mark.parametrize("numel,ncalls", [(604 * 2**20, 96), (7, 96), (96, 96), (1000, 7), (0, 4)])
def test_stack_upload_pieces_cover_the_stacks_once(numel, ncalls):
    """The e2e step's new-token stacks go up in one piece per call: together the pieces cover
    every element exactly once, in order."""
    pieces = bench.upload_pieces(numel, ncalls)
    assert len(pieces) == ncalls
    pos = 0
    for a, b in pieces:
        assert a == pos and b >= a
        pos = b
    assert pos == numel
