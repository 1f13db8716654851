"""tpla_decode_static: decode for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (code inside an allocator or memory-pool
callback, frameworks that own all device memory, loops where an allocation
may block), so they cannot pass a workspace.  The static entry point keeps
its scratch in the library's fixed device array.  This test compares it with
tpla_decode, through the C ABI, on two calls in a row (the array keeps the
previous call's contents, which must not leak into the next result).  It sits
in a file of its own that pytest collects last.
"""

import math

import numpy as np
import pytest
import torch

import gpu_harness as hx
from latent_attention_decode_tpla_b200 import inputs as gen
from latent_attention_decode_tpla_b200 import tpla

pytestmark = pytest.mark.gpu


def _decode_both(d, scale):
    dev = hx.to_device(d)
    dims = hx.dims_of(d, scale)
    B, H, dv = d["B"], d["H"], d["dv"]
    ref_out = torch.empty(B, H, dv, dtype=torch.float32, device="cuda")
    ws = tpla.alloc_workspace(dims)
    tpla.decode(dims, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], dev["block_table"], dev["seq_lens"],
                dev["w_uv"], ref_out, ws)
    outs = []
    for _ in range(2):
        out = torch.full((B, H, dv), float("nan"), dtype=torch.float32, device="cuda")
        tpla.decode_static(dims, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], dev["block_table"],
                           dev["seq_lens"], dev["w_uv"], out)
        outs.append(out)
    torch.cuda.synchronize()
    assert tpla.check_device_status() == tpla.TPLA_OK
    return hx.to64(ref_out), [hx.to64(o) for o in outs]


@pytest.mark.parametrize("B,H,g,lens", [
    (5, 128, 2, [300, 1, 0, 640, 65]),
    (3, 64, 4, [2000, 129, 64]),
    (16, 128, 2, [4096] * 16),
])
def test_static_scratch_matches_workspace_entry(B, H, g, lens):
    d = gen.make_workload(B=B, H=H, L=512, R=64, dv=128, g=g, seq_lens=lens, seed=31 + B, extra_pages=2)
    scale = 1 / math.sqrt(192)
    want, outs = _decode_both(d, scale)
    for o in outs:
        hx.assert_close(o, want, "static scratch vs workspace")


def test_static_scratch_second_call_with_other_sizes():
    # a larger call first, then a smaller one: stale contents of the shared array must not matter
    scale = 1 / math.sqrt(192)
    big = gen.make_workload(B=8, H=128, L=512, R=64, dv=128, g=2, seq_lens=[3000] * 8, seed=5)
    small = gen.make_workload(B=2, H=128, L=512, R=64, dv=128, g=2, seq_lens=[70, 5], seed=6)
    for d in (big, small):
        want, outs = _decode_both(d, scale)
        for o in outs:
            hx.assert_close(o, want, "static scratch after another call")


def test_static_scratch_with_fewer_workers_near_its_limit():
    # 100 sequences x 2 shards: 200 per-sequence partial slots of 128 x 256 fp32 (128 KiB each) plus
    # the header leave room for only 54 split-KV workers in the 32 MiB array, fewer than the SM
    # count tpla_decode uses: the result must not change
    lens = gen.seq_lengths(100, 1, 600, seed=8)
    d = gen.make_workload(B=100, H=128, L=512, R=64, dv=128, g=2, seq_lens=lens, seed=8, extra_pages=3)
    want, outs = _decode_both(d, 1 / math.sqrt(192))
    for o in outs:
        hx.assert_close(o, want, "static scratch, clamped worker count")


def test_static_scratch_kernel_choice_follows_the_options():
    # the static entry chooses its attention kernel as tpla_decode does: a forced tcgen05 kernel on a
    # shape without one is rejected, and the kernel that ran is reported
    d = gen.make_workload(B=2, H=16, L=256, R=32, dv=64, g=2, seq_lens=[100, 7], seed=12)
    dev = hx.to_device(d)
    dims = hx.dims_of(d, 0.2)
    out = torch.zeros(2, 16, 64, dtype=torch.float32, device="cuda")
    old = tpla.get_option(tpla.OPT_ATTENTION_KERNEL)
    try:
        tpla.set_option(tpla.OPT_ATTENTION_KERNEL, 2)
        with pytest.raises(tpla.TplaError) as e:
            tpla.decode_static(dims, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], dev["block_table"],
                               dev["seq_lens"], dev["w_uv"], out)
        assert e.value.status == tpla.TPLA_ERR_UNSUPPORTED
        tpla.set_option(tpla.OPT_ATTENTION_KERNEL, 1)
        tpla.decode_static(dims, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], dev["block_table"],
                           dev["seq_lens"], dev["w_uv"], out)
        torch.cuda.synchronize()
        assert tpla.get_option(tpla.OPT_LAST_ATTENTION_KERNEL) == 1
    finally:
        tpla.set_option(tpla.OPT_ATTENTION_KERNEL, old)
    assert tpla.check_device_status() == tpla.TPLA_OK


def test_static_scratch_rejects_sizes_beyond_its_limit():
    # 1024 sequences x 2 shards of 128 x 256 fp32 partials need 256 MiB > 32 MiB
    d = tpla.make_dims(B=1024, H=128, L=512, R=64, dv=128, g=2, max_pages_per_seq=1, num_pages=1024,
                       softmax_scale=0.1)
    t = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    lens = torch.zeros(1024, dtype=torch.int32, device="cuda")
    out = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(tpla.TplaError) as e:
        tpla.decode_static(d, t, t, t, t, None, lens, None, out)
    assert e.value.status == tpla.TPLA_ERR_WORKSPACE
