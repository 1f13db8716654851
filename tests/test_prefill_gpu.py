"""MLA-form prefill on the GPU against the oracle, and the hand-off to TPLA decode.

edgentiq blog, "Prefill-Decode Separation for Optimal Performance": prefill keeps MLA (every head over the
whole latent), decode uses TPLA.  The prompt's outputs are compared with the oracle's causal MLA
attention over the g = 1 append of the same raw latents; then a decode step over the g-shard cache the
prefill wrote is compared with the oracle's decode over a cache the oracle's append filled.
"""

import math

import numpy as np
import pytest
import torch

import gpu_harness as hx
from oracle import tpla_ref as ref
from latent_attention_decode_tpla_b200 import inputs as gen
from latent_attention_decode_tpla_b200 import prefill, tpla

pytestmark = pytest.mark.gpu


def _bf16(x):
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("T,g,transform,chunk", [
    (300, 2, ref.TRANSFORM_HADAMARD, 64),
    (129, 4, ref.TRANSFORM_DENSE, 50),
    (64, 2, ref.TRANSFORM_BLOCK_HADAMARD, 64),
    (1, 2, ref.TRANSFORM_HADAMARD, 64),
])
def test_mla_prefill_and_decode_hand_off(T, g, transform, chunk):
    H, L, R, dv = 128, 512, 64, 128
    gcpu = torch.Generator().manual_seed(1000 + T + g)
    x = _bf16(torch.randn(T, L, generator=gcpu))
    kpe = _bf16(torch.randn(T, R, generator=gcpu))
    q = _bf16(torch.randn(T, H, L, generator=gcpu))
    q_pe = _bf16(torch.randn(T, H, R, generator=gcpu))
    w_uv = _bf16(torch.randn(H, L, dv, generator=gcpu) / math.sqrt(L))
    R_dense = gen.random_orthogonal(L, 7) if transform == ref.TRANSFORM_DENSE else None
    scale = 1 / math.sqrt(192)
    maxp = (T + 63) // 64 + 1                      # one page more than the prompt needs
    P = maxp + 3
    row = torch.randperm(P, generator=gcpu)[:maxp].to(torch.int32)
    dims = tpla.make_dims(B=1, H=H, L=L, R=R, dv=dv, g=g, max_pages_per_seq=maxp, num_pages=P, softmax_scale=scale)
    ckv = torch.zeros((P, g, 64, L // g), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((P, 64, R), dtype=torch.bfloat16, device="cuda")
    out = torch.full((T, H, dv), float("nan"), dtype=torch.float32, device="cuda")
    prefill.mla_prefill(dims, x.cuda(), kpe.cuda(), q.cuda(), q_pe.cuda(), w_uv.cuda(), transform,
                        None if R_dense is None else R_dense.cuda(), None, 1e-6, row.cuda(), ckv, kc, out, chunk=chunk)
    torch.cuda.synchronize()
    assert tpla.check_device_status() == tpla.TPLA_OK
    f = lambda t: t.to(torch.float64).numpy()
    want = ref.mla_prefill(f(x), f(kpe), f(q), f(q_pe), scale, transform=transform,
                           R_dense=None if R_dense is None else f(R_dense), w_uv=f(w_uv))
    hx.assert_close(out.cpu().to(torch.float64).numpy(), want, "prefill T=%d g=%d" % (T, g))

    # hand-off: one decode step of a new query over the prompt, on the cache the prefill wrote
    ckv_o = np.zeros((P, g, 64, L // g))
    kc_o = np.zeros((P, 64, R))
    bt = row.numpy()[None, :]
    ref.append_kv(f(x), f(kpe), np.arange(T), np.repeat(bt, T, axis=0), ckv_o, kc_o, g=g, max_pages_per_seq=maxp,
                  transform=transform, R_dense=None if R_dense is None else f(R_dense))
    qd = _bf16(torch.randn(1, H, L, generator=gcpu))
    qd_pe = _bf16(torch.randn(1, H, R, generator=gcpu))
    o = torch.empty((1, H, dv), dtype=torch.float32, device="cuda")
    tpla.decode(dims, qd.cuda(), qd_pe.cuda(), ckv, kc, row.cuda().reshape(1, -1).contiguous(),
                torch.tensor([T], dtype=torch.int32, device="cuda"), w_uv.cuda(), o, tpla.alloc_workspace(dims))
    torch.cuda.synchronize()
    assert tpla.check_device_status() == tpla.TPLA_OK
    want_d = ref.decode(f(qd), f(qd_pe), ckv_o, kc_o, bt, np.array([T]), scale, max_pages_per_seq=maxp, w_uv=f(w_uv))
    hx.assert_close(o.cpu().to(torch.float64).numpy(), want_d, "decode after prefill")
