"""GPU parity: the CUDA path through the C ABI against the float64 oracle.

Inputs are seeded and identical on both sides (bf16 values).  Tolerances on
the fp32 outputs: max-abs <= 2e-2 and relative RMS <= 1e-3.  Small cases span
several 64-token tiles, ragged tails and empty sequences; the benchmark
configurations run at full size, every sequence compared with the oracle.
"""

import math

import numpy as np
import pytest
import torch

import gpu_harness as hx
from oracle import tpla_ref as ref
from latent_attention_decode_tpla_b200 import inputs as gen
from latent_attention_decode_tpla_b200 import tpla

pytestmark = pytest.mark.gpu

KERNELS = ["simt", "sm100"]


def _kernel_or_skip(d, kernel, tile=0):
    if kernel == "sm100" and not hx.sm100_available(d):
        pytest.skip("no tcgen05 variant for this shape")
    if tile and (kernel != "sm100" or d["L"] // d["g"] > 256):
        pytest.skip("the tile size is an option of the tcgen05 kernel for L/g <= 256 only")


TILES = [0, 64]      # the library default and one-page tiles (two-page tiles when the default is 64)


def _case(B, H, L, R, dv, g, lens, seed, transform=None, **kw):
    d = gen.make_workload(B=B, H=H, L=L, R=R, dv=dv, g=g, seq_lens=lens, seed=seed, extra_pages=5,
                          cache_values="none" if transform is not None else "normal", **kw)
    if transform is not None:
        Rd = gen.random_orthogonal(L, seed) if transform == ref.TRANSFORM_DENSE else None
        hx.oracle_fill_cache(d, transform, Rd)
    return d


# ------------------------------------------------------------------ tiny TPLA decode (H8 L64 R16 dv32, g=2, 128 tokens)

@pytest.mark.parametrize("kernel", KERNELS)
def test_tiny_g2_hadamard(kernel):
    spec = gen.WORKLOADS["tiny_g2"]
    d = _case(spec["B"], spec["H"], spec["L"], spec["R"], spec["dv"], spec["g"], [spec["T"]], 0,
              transform=ref.TRANSFORM_HADAMARD, **spec["stds"])
    _kernel_or_skip(d, kernel)
    scale = gen.softmax_scale(spec)
    hx.assert_close(hx.run_gpu(d, scale, kernel=kernel), hx.run_oracle(d, scale), "tiny out")
    hx.assert_close(hx.run_gpu(d, scale, with_wuv=False, kernel=kernel),
                    hx.run_oracle(d, scale, with_wuv=False), "tiny latent")
    tot = 0
    for s in range(2):
        got = hx.run_gpu(d, scale, mode="shard", shard=s, kernel=kernel)
        hx.assert_close(got, hx.run_oracle(d, scale, mode="shard", shard=s), "tiny shard %d" % s)
        tot = tot + got
        hx.assert_close(hx.run_gpu(d, scale, mode="shard", shard=s, with_wuv=False, kernel=kernel),
                        hx.run_oracle(d, scale, mode="shard", shard=s, with_wuv=False), "tiny shard latent")
    # the sum of the per-rank terms is the full result (fp32 reassociation only)
    np.testing.assert_allclose(tot, hx.run_gpu(d, scale, kernel=kernel), rtol=0, atol=1e-5)


# ------------------------------------------------------------------ ragged small cases

RAGGED = [0, 1, 63, 64, 65, 200, 7, 129]


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("H,L,R,dv,g", [
    (8, 64, 16, 32, 2), (128, 512, 64, 128, 1), (128, 512, 64, 128, 2), (64, 512, 64, 128, 4),
    (100, 512, 64, 128, 2), (128, 512, 64, 128, 8), (16, 256, 32, 64, 2), (64, 128, 16, 32, 4),
    (32, 512, 64, 128, 2), (64, 512, 64, 128, 8), (48, 512, 64, 128, 2),
])
def test_ragged_batch(kernel, H, L, R, dv, g, tile):
    d = _case(len(RAGGED), H, L, R, dv, g, RAGGED, seed=3 + H + g)
    _kernel_or_skip(d, kernel, tile)
    with hx.tile_tokens(tile):
        _ragged_batch(d, kernel, H, L, R, dv, g)


def _ragged_batch(d, kernel, H, L, R, dv, g):
    scale = 1 / math.sqrt(128 + R)
    want = hx.run_oracle(d, scale)
    hx.assert_close(hx.run_gpu(d, scale, kernel=kernel), want, "out")
    assert np.all(hx.run_gpu(d, scale, kernel=kernel)[0] == 0.0)          # empty sequence
    hx.assert_close(hx.run_gpu(d, scale, with_wuv=False, kernel=kernel), hx.run_oracle(d, scale, with_wuv=False),
                    "latent")
    s = g - 1
    hx.assert_close(hx.run_gpu(d, scale, mode="shard", shard=s, kernel=kernel),
                    hx.run_oracle(d, scale, mode="shard", shard=s), "shard")
    # identity page layout (block_table = NULL) on an unshuffled cache
    d2 = gen.make_workload(B=3, H=H, L=L, R=R, dv=dv, g=g, seq_lens=[70, 0, 130], seed=9, shuffle=False)
    hx.assert_close(hx.run_gpu(d2, scale, block_table=False, kernel=kernel), hx.run_oracle(d2, scale),
                    "identity layout")


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("g", [2, 1])
@pytest.mark.parametrize("workers", [1, 2, 3, 7, 0])
def test_split_schedule_invariance(kernel, g, workers, tile):
    """Any number of split-KV workers gives the same result (segments cross workers and sequences)."""
    d = _case(5, 128, 512, 64, 128, g, [300, 1, 0, 640, 65], seed=17)
    _kernel_or_skip(d, kernel, tile)
    scale = 1 / math.sqrt(192)
    old = tpla.get_option(tpla.OPT_MAX_WORKERS)
    tpla.set_option(tpla.OPT_MAX_WORKERS, workers)
    try:
        tpla.set_option(tpla.OPT_TILE_TOKENS, tile)
        got = hx.run_gpu(d, scale, kernel=kernel)
        got_s = hx.run_gpu(d, scale, mode="shard", shard=g - 1, kernel=kernel)
    finally:
        tpla.set_option(tpla.OPT_MAX_WORKERS, old)
        tpla.set_option(tpla.OPT_TILE_TOKENS, 0)
    hx.assert_close(got, hx.run_oracle(d, scale), "workers=%d" % workers)
    hx.assert_close(got_s, hx.run_oracle(d, scale, mode="shard", shard=g - 1), "shard workers=%d" % workers)


# ------------------------------------------------------------------ benchmark configurations, full size

@pytest.mark.parametrize("kernel", KERNELS)
def test_mla_g1_dsv3_4k(kernel):
    spec = gen.WORKLOADS["mla_g1_dsv3_b1_4k"]
    d = _case(1, 128, 512, 64, 128, 1, [4096], 1, transform=ref.TRANSFORM_HADAMARD)
    _kernel_or_skip(d, kernel)
    scale = gen.softmax_scale(spec)
    want = hx.run_oracle(d, scale)
    hx.assert_close(hx.run_gpu(d, scale, mode="mla", kernel=kernel), want, "mla_decode")
    hx.assert_close(hx.run_gpu(d, scale, mode="full", kernel=kernel), want, "tpla_decode g=1")


@pytest.mark.parametrize("kernel", KERNELS)
def test_tpla_g2_dsv3_b1_32k(kernel):
    spec = gen.WORKLOADS["tpla_g2_dsv3_b1_32k"]
    d = _case(1, 128, 512, 64, 128, 2, [32768], 2)
    _kernel_or_skip(d, kernel)
    scale = gen.softmax_scale(spec)
    hx.assert_close(hx.run_gpu(d, scale, mode="shard", shard=0, kernel=kernel),
                    hx.run_oracle(d, scale, mode="shard", shard=0), "shard 0")
    hx.assert_close(hx.run_gpu(d, scale, kernel=kernel), hx.run_oracle(d, scale), "all shards")


def _every_sequence(d, scale, kernel, modes=("shard", "full"), chunk=4, dev=None):
    """Every sequence of a full-size case against the oracle (the oracle runs a few sequences at
    a time so that its float64 copy of the cache stays small)."""
    for mode in modes:
        got = hx.run_gpu(d, scale, mode=mode, shard=0, kernel=kernel, dev=dev)
        for b0 in range(0, d["B"], chunk):
            batch = list(range(b0, min(d["B"], b0 + chunk)))
            want = hx.run_oracle(d, scale, mode=mode, shard=0, batch=batch)
            hx.assert_close(got[batch], want, "%s sequences %d..%d" % (mode, batch[0], batch[-1]))


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("kernel", KERNELS)
def test_tpla_g2_dsv3_b16_32k(kernel, tile):
    """DeepSeek-V3 shape, g = 2, 16 x 32768 tokens; the cache is the oracle's append of seeded raw
    latents through the Hadamard transform and sliced RMSNorm."""
    spec = gen.WORKLOADS["tpla_g2_dsv3_b16_32k"]
    d = _case(16, 128, 512, 64, 128, 2, [32768] * 16, 3, transform=ref.TRANSFORM_HADAMARD)
    _kernel_or_skip(d, kernel, tile)
    with hx.tile_tokens(tile):
        _every_sequence(d, gen.softmax_scale(spec), kernel)


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("kernel", KERNELS)
def test_tpla_g4_kimi_b8_32k(kernel, tile):
    """Kimi-K2 shape, g = 4, 8 x 32768 tokens; the cache is the oracle's append through the seeded
    random orthogonal transform (the PCA stand-in) and sliced RMSNorm."""
    spec = gen.WORKLOADS["tpla_g4_kimi_b8_32k"]
    d = _case(8, 64, 512, 64, 128, 4, [32768] * 8, 4, transform=ref.TRANSFORM_DENSE)
    _kernel_or_skip(d, kernel, tile)
    with hx.tile_tokens(tile):
        _every_sequence(d, gen.softmax_scale(spec), kernel)


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("kernel", KERNELS)
def test_mixed_b64_paged_with_append(kernel, tile):
    """DeepSeek-V3 shape, g=2: 64 sequences of 1K..64K tokens on a shuffled page table, plus one appended token each."""
    spec = gen.WORKLOADS["tpla_g2_dsv3_b64_mixed"]
    lens = gen.workload_seq_lens(spec, seed=0)
    d = gen.make_workload(B=64, H=128, L=512, R=64, dv=128, g=2, seq_lens=lens, seed=5)
    _kernel_or_skip(d, kernel, tile)
    with hx.tile_tokens(tile):
        _mixed_b64(d, kernel, spec, lens)


def _mixed_b64(d, kernel, spec, lens):
    scale = gen.softmax_scale(spec)
    dev = hx.to_device(d)
    dims = hx.dims_of(d, scale)
    tpla.append_kv(dims, dev["x_new"], dev["kpe_new"], tpla.TRANSFORM_HADAMARD, None, None, 1e-6,
                   dev["seq_lens"], dev["block_table"], dev["ckv"], dev["kpe"])
    torch.cuda.synchronize()
    assert tpla.check_device_status() == tpla.TPLA_OK
    # the oracle appends the same tokens into its own copy of the cache
    batch = [int(lens.argmax()), int(lens.argmin()), 17]
    ckv = hx.to64(d["ckv"])
    kpe = hx.to64(d["kpe"])
    bt = d["block_table"].numpy()
    ref.append_kv(hx.to64(d["x_new"]), hx.to64(d["kpe_new"]), lens.numpy(), bt, ckv, kpe, g=2,
                  max_pages_per_seq=d["max_pages_per_seq"], transform=ref.TRANSFORM_HADAMARD, eps=1e-6)
    d_or = dict(d)
    d_or["ckv"] = torch.from_numpy(ckv).to(torch.bfloat16)
    d_or["kpe"] = torch.from_numpy(kpe).to(torch.bfloat16)
    d_or["seq_lens"] = lens + 1
    dev["seq_lens"] = (lens + 1).cuda()
    # appended rows agree with the oracle's within one bf16 ulp
    for b in batch:
        page, slot = bt[b, int(lens[b]) // 64], int(lens[b]) % 64
        g_row = dev["ckv"][page, :, slot].cpu().to(torch.float64).numpy()
        o_row = ckv[page, :, slot]
        assert np.all(np.abs(g_row - o_row) <= np.abs(o_row) * 2.0 ** -7 + 1e-30)
    # end to end: GPU append + GPU decode against oracle append + oracle decode, every sequence
    _every_sequence(d_or, scale, kernel, modes=("full", "shard"), chunk=8, dev=dev)


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("g", [2, 1])
def test_pv_precision_modes_at_the_length_boundary(kernel, g, tile):
    """Sequences just below 8192 tokens run PV in fp16, from 8192 on in bf16; both meet the tolerance."""
    d = _case(4, 128, 512, 64, 128, g, [8191, 8192, 8193, 100], seed=23)
    _kernel_or_skip(d, kernel, tile)
    scale = 1 / math.sqrt(192)
    with hx.tile_tokens(tile):
        hx.assert_close(hx.run_gpu(d, scale, kernel=kernel), hx.run_oracle(d, scale), "all shards")
        hx.assert_close(hx.run_gpu(d, scale, mode="shard", shard=g - 1, kernel=kernel),
                        hx.run_oracle(d, scale, mode="shard", shard=g - 1), "shard %d" % (g - 1))


@pytest.mark.parametrize("kernel", KERNELS)
def test_mla_g1_dsv3_b8_32k(kernel):
    """MLA (g = 1) at batch 8 x 32768 tokens, DeepSeek-V3 shape; the cache is the oracle's append
    through the Hadamard transform and RMSNorm; every sequence against the oracle."""
    spec = gen.WORKLOADS["mla_g1_dsv3_b8_32k"]
    d = _case(8, 128, 512, 64, 128, 1, [32768] * 8, 6, transform=ref.TRANSFORM_HADAMARD)
    _kernel_or_skip(d, kernel)
    scale = gen.softmax_scale(spec)
    got = hx.run_gpu(d, scale, mode="mla", kernel=kernel)
    for b0 in range(0, 8, 4):
        batch = list(range(b0, b0 + 4))
        hx.assert_close(got[batch], hx.run_oracle(d, scale, batch=batch), "mla sequences %d.." % b0)


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("g", [2, 1])
@pytest.mark.parametrize("scale", [-1 / math.sqrt(192), 0.0, 0.5])
def test_softmax_scale_sign_and_size(kernel, scale, g, tile):
    """A negative scale (the kernel folds its sign into the query), a zero scale (uniform
    weights over the valid tokens, ragged tails included) and a large one (the row maximum
    grows by more than the lazy-rescale threshold across tiles)."""
    d = _case(4, 128, 512, 64, 128, g, [300, 1, 129, 1000], seed=23)
    _kernel_or_skip(d, kernel, tile)
    with hx.tile_tokens(tile):
        _scale_case(d, kernel, scale)


def _scale_case(d, kernel, scale):
    hx.assert_close(hx.run_gpu(d, scale, kernel=kernel), hx.run_oracle(d, scale), "scale %g" % scale)
    hx.assert_close(hx.run_gpu(d, scale, mode="shard", shard=0, with_wuv=False, kernel=kernel),
                    hx.run_oracle(d, scale, mode="shard", shard=0, with_wuv=False), "scale %g shard latent" % scale)


# cache magnitudes at fp16's limits (sequences shorter than 8192 tokens run PV on fp16 tiles, scaled
# by a power of two where a tile's largest |value| lies outside [2^-10, 65280], and on bf16 tiles
# where it lies outside [2^-18, 2^23)): name -> (scale of the selected token rows, which rows, scale
# of the query, rel-RMS bound)
RANGE_CASES = {
    "tiny": (2.0 ** -16, "all", 2.0 ** 16, hx.REL_RMS),          # fp16 subnormal range: scaled up by 2^4
    "huge": (5.0e4, "all", 1.0 / 5.0e4, hx.REL_RMS),              # up to ~2.5e5 > 65504: scaled down by 2^-2
    "near_max": (1.2e4, "all", 1.0 / 1.2e4, hx.REL_RMS),          # up to ~5.4e4: fits fp16 as it is
    "mixed_tiny": (2.0 ** -20, "every5", 1.0, hx.REL_RMS),        # a few subnormal rows inside fp16 tiles
    "mixed_huge": (1.0e5, "every97", 1.0e-5, hx.REL_RMS),         # a few large rows: those tiles scaled down
    # beyond what a power-of-two shift brings into fp16: bf16 tiles, whose 8-bit P costs about 1e-3
    # relative error on sequences this short (the documented bound for such caches is 2e-3)
    "beyond_tiny": (2.0 ** -26, "all", 2.0 ** 26, 2e-3),
    "beyond_huge": (1.0e9, "all", 1.0e-9, 2e-3),
}


@pytest.mark.parametrize("tile", TILES)
@pytest.mark.parametrize("kernel", KERNELS)
@pytest.mark.parametrize("g", [2, 1])
@pytest.mark.parametrize("case", sorted(RANGE_CASES))
def test_pv_fp16_range_limits(kernel, g, case, tile):
    """Latent values whose magnitude fp16 cannot hold (or holds only as subnormals), on sequences
    short enough for fp16 PV tiles.  Scores are kept ordinary by scaling the query the other way;
    outputs scale with the cache, so both sides are divided by the row scale before comparing."""
    d = _case(4, 128, 512, 64, 128, g, [300, 1000, 129, 4000], seed=29)
    _kernel_or_skip(d, kernel, tile)
    with hx.tile_tokens(tile):
        _range_case(d, kernel, g, case)


def _range_case(d, kernel, g, case):
    row_scale, which, q_scale, rel_bound = RANGE_CASES[case]
    ckv = d["ckv"].to(torch.float32)
    if which == "all":
        ckv = ckv * row_scale
    else:
        step = int(which[len("every"):])
        ckv[:, :, ::step, :] *= row_scale                 # every step-th slot of every page
    d["ckv"] = ckv.to(torch.bfloat16)
    d["q"] = (d["q"].to(torch.float32) * q_scale).to(torch.bfloat16)
    scale = 1 / math.sqrt(192)
    norm = row_scale if which == "all" or row_scale > 1 else 1.0
    for mode, with_wuv in (("full", True), ("shard", False)):
        got = hx.run_gpu(d, scale, mode=mode, shard=g - 1, with_wuv=with_wuv, kernel=kernel)
        want = hx.run_oracle(d, scale, mode=mode, shard=g - 1, with_wuv=with_wuv)
        hx.assert_close(got / norm, want / norm, "%s %s" % (case, mode), rel_rms=rel_bound)


# ------------------------------------------------------------------ GLA-style decode (heads split with the latent)

@pytest.mark.parametrize("H,g", [(128, 2), (64, 4), (128, 1)])
def test_gla_style_decode(H, g):
    """Head group s attends to latent shard s only (the contrast on the TPLA pages): the library's
    kernels per group against the oracle's GLA-style decode, with and without W_UV."""
    from latent_attention_decode_tpla_b200 import gla
    d = _case(len(RAGGED), H, 512, 64, 128, g, RAGGED, seed=61 + g)
    scale = 1 / math.sqrt(192)
    dev = hx.to_device(d)
    dims = hx.dims_of(d, scale)
    bt = d["block_table"].numpy()
    kw = dict(max_pages_per_seq=d["max_pages_per_seq"])
    f = lambda t: hx.to64(t)
    for with_wuv in (True, False):
        cols = 128 if with_wuv else 512 // g
        out = torch.full((len(RAGGED), H, cols), float("nan"), dtype=torch.float32, device="cuda")
        gla.gla_decode(dims, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], dev["block_table"], dev["seq_lens"],
                       dev["w_uv"] if with_wuv else None, out)
        torch.cuda.synchronize()
        assert tpla.check_device_status() == tpla.TPLA_OK
        want = ref.gla_decode(f(d["q"]), f(d["q_pe"]), f(d["ckv"]), f(d["kpe"]), bt, d["seq_lens"].numpy(), scale,
                              w_uv=f(d["w_uv"]) if with_wuv else None, **kw)
        hx.assert_close(hx.to64(out), want, "gla H=%d g=%d w_uv=%s" % (H, g, with_wuv))
