"""CPU checks of the benchmark's host-side arithmetic: the byte counts behind `value` and `roofline`,
and the rule that ties `roofline.traffic` to the sources an ncu capture was taken on."""
import os

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_of_the_bench_workload():
    # B=16 sequences of 32768 tokens, one shard of g=2: 256 latent columns + the 64-wide RoPE key,
    # bf16 -> 640 bytes per token; the queries add B * H * 320 * 2 bytes
    spec = bench.workload_spec("tpla_g2_dsv3_b16_32k")
    cache, total = bench.algorithmic_bytes(spec, 16 * 32768, "shard")
    assert cache == 16 * 32768 * 640 == 335_544_320
    assert total - cache == 16 * 128 * 320 * 2
    # all shards: the whole latent (512) plus one RoPE key per token
    cache_full, _ = bench.algorithmic_bytes(spec, 16 * 32768, "full")
    assert cache_full == 16 * 32768 * (512 + 64) * 2


@pytest.mark.parametrize("name,per_token", [
    ("tpla_g4_kimi_b8_32k", (128 + 64) * 2),
    ("mla_g1_dsv3_b1_4k", (512 + 64) * 2),
])
def test_bytes_per_token_follow_the_shard_width(name, per_token):
    spec = bench.workload_spec(name)
    cache, _ = bench.algorithmic_bytes(spec, 1000, spec["mode"])
    assert cache == 1000 * per_token


def test_profiled_traffic_needs_matching_sources(tmp_path, monkeypatch):
    # the committed summary is read only while the digest of the kernel's sources matches it
    summary = os.path.join(ROOT, "profiles", "attn_sm100_tpla_g2_dsv3_b16_32k.txt")
    if not os.path.exists(summary):
        pytest.skip("no committed summary")
    vals = dict(ln.split(":", 1) for ln in open(summary) if ":" in ln)
    stored = vals["source_digest"].strip()
    got = bench.profiled_traffic("attn_sm100", "tpla_g2_dsv3_b16_32k")
    if stored == bench.source_digest("attn_sm100"):
        assert got == float(vals["dram_bytes_per_launch"])
    else:
        assert got is None
    # a summary whose digest differs from the sources yields no traffic figure
    fake_root = tmp_path
    os.makedirs(fake_root / "profiles")
    with open(fake_root / "profiles" / "attn_sm100_w.txt", "w") as f:
        f.write("source_digest: 0000000000000000\ndram_bytes_per_launch: 123\n")
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    monkeypatch.setattr(bench, "source_digest", lambda kernel=None: "ffffffffffffffff")
    assert bench.profiled_traffic("attn_sm100", "w") is None
    monkeypatch.setattr(bench, "source_digest", lambda kernel=None: "0000000000000000")
    assert bench.profiled_traffic("attn_sm100", "w") == 123.0


def test_kernel_digest_covers_only_its_sources():
    # the attention digest is computed from the files that decide one attention launch
    assert set(bench.KERNEL_SOURCES["attn_sm100"]) == {"attn_sm100.cu", "sm100_ptx.cuh", "tpla_internal.cuh", "api.cu"}
    assert bench.source_digest("attn_sm100") != bench.source_digest()
