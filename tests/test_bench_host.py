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


def _included(csrc, name, seen):
    # the file and every local header it includes, transitively
    if name in seen or not os.path.exists(os.path.join(csrc, name)):
        return seen
    seen.add(name)
    for ln in open(os.path.join(csrc, name)):
        if ln.startswith('#include "') and not ln.startswith('#include "../'):
            _included(csrc, ln.split('"')[1], seen)
    return seen


@pytest.mark.parametrize("kernel", ["attn_sm100", "attn_sm100_wide"])
def test_kernel_digest_covers_only_its_sources(kernel):
    # the attention digest is computed from the files that decide one attention launch: the
    # kernel's file, every header it includes, and the host-side plan (api.cu)
    csrc = os.path.join(ROOT, "latent_attention_decode_tpla_b200", "csrc")
    want = _included(csrc, kernel + ".cu", set()) | {"api.cu"}
    assert set(bench.KERNEL_SOURCES[kernel]) == want
    assert bench.source_digest(kernel) != bench.source_digest()


def test_cache_replicas_defeat_l2():
    # a step that reads more than twice the L2 needs no replica; a smaller cache is rotated over an
    # even number of replicas whose bytes together exceed twice the L2
    assert bench.cache_replicas(335_544_320) == 1
    for per_step in (21_000_000, 4_718_592, 100_663_296, 1):
        n = bench.cache_replicas(per_step)
        assert n % 2 == 0 and n * per_step > 2 * bench.L2_BYTES
        assert (n - 2) * per_step <= 2 * bench.L2_BYTES          # not more than needed (+1 for evenness)
    assert "rotated" in bench.l2_note(14, 21_000_000) and "no flush" in bench.l2_note(1, 335_544_320)


def test_percentile_interpolates():
    assert bench.percentile([3.0, 1.0, 2.0], 0.5) == 2.0
    assert bench.percentile([1.0, 2.0, 3.0, 4.0, 5.0, 6.0, 7.0, 8.0, 9.0, 10.0], 0.9) == pytest.approx(9.1)
    assert bench.percentile([5.0], 0.9) == 5.0
