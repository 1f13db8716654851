"""Device-side failure reporting, without faulting or hanging the GPU.

Out-of-range indices are skipped and recorded; a pipeline wait that runs
out (forced with a barrier nothing signals and a 20 ms limit) returns
TPLA_ERR_TIMEOUT and leaves the context usable.
"""

import math

import numpy as np
import pytest
import torch

import gpu_harness as hx
from latent_attention_decode_tpla_b200 import inputs as gen
from latent_attention_decode_tpla_b200 import tpla

pytestmark = pytest.mark.gpu


def _small(g):
    # g = 2: the 128-token-tile tcgen05 kernel; g = 1 (512 latent columns per shard): the CTA-pair one
    return gen.make_workload(B=3, H=128, L=512, R=64, dv=128, g=g, seq_lens=[100, 64, 300], seed=2, extra_pages=4)


@pytest.mark.parametrize("g", [2, 1])
@pytest.mark.parametrize("kernel", ["simt", "sm100"])
def test_bad_page_and_length_are_reported(kernel, g):
    d = _small(g)
    if kernel == "sm100" and not hx.sm100_available(d):
        pytest.skip("no tcgen05 variant")
    scale = 1 / math.sqrt(192)
    dev = hx.to_device(d)
    dims = hx.dims_of(d, scale)
    ws = tpla.alloc_workspace(dims)
    out = torch.empty(3, 128, 128, dtype=torch.float32, device="cuda")
    old = tpla.get_option(tpla.OPT_ATTENTION_KERNEL)
    tpla.set_option(tpla.OPT_ATTENTION_KERNEL, hx.KERNELS[kernel])
    try:
        bt = dev["block_table"].clone()
        bt[1, 0] = d["num_pages"] + 3                      # outside the cache
        tpla.decode(dims, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], bt, dev["seq_lens"], dev["w_uv"], out, ws)
        assert tpla.check_device_status() == tpla.TPLA_ERR_INDEX
        assert torch.isfinite(out).all()
        lens = dev["seq_lens"].clone()
        lens[2] = d["max_pages_per_seq"] * 64 + 1         # longer than its pages
        tpla.decode(dims, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], dev["block_table"], lens, dev["w_uv"],
                    out, ws)
        assert tpla.check_device_status() == tpla.TPLA_ERR_INDEX
        assert tpla.check_device_status() == tpla.TPLA_OK
    finally:
        tpla.set_option(tpla.OPT_ATTENTION_KERNEL, old)


@pytest.mark.parametrize("g", [2, 1])
def test_bounded_wait_times_out_and_context_survives(g):
    d = _small(g)
    if not hx.sm100_available(d):
        pytest.skip("no tcgen05 variant")
    scale = 1 / math.sqrt(192)
    dev = hx.to_device(d)
    dims = hx.dims_of(d, scale)
    ws = tpla.alloc_workspace(dims)
    out = torch.empty(3, 128, 128, dtype=torch.float32, device="cuda")
    old = [tpla.get_option(o) for o in (tpla.OPT_ATTENTION_KERNEL, tpla.OPT_WAIT_LIMIT, tpla.OPT_DEBUG_STALL)]
    try:
        tpla.set_option(tpla.OPT_ATTENTION_KERNEL, 2)
        tpla.set_option(tpla.OPT_WAIT_LIMIT, 20000)         # 20 ms
        tpla.set_option(tpla.OPT_DEBUG_STALL, 1)
        tpla.attention(dims, -1, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], dev["block_table"],
                       dev["seq_lens"], ws)
        assert tpla.check_device_status() == tpla.TPLA_ERR_TIMEOUT
        tpla.set_option(tpla.OPT_DEBUG_STALL, 0)
        tpla.set_option(tpla.OPT_WAIT_LIMIT, 0)
        # the same context still computes correctly
        got = hx.run_gpu(d, scale, dev=dev, kernel="sm100")
        hx.assert_close(got, hx.run_oracle(d, scale), "after time-out")
    finally:
        for o, v in zip((tpla.OPT_ATTENTION_KERNEL, tpla.OPT_WAIT_LIMIT, tpla.OPT_DEBUG_STALL), old):
            tpla.set_option(o, v)
