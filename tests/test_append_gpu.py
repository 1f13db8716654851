"""GPU parity of tpla_append_kv: orthogonal transform + sliced RMSNorm + paged store.

Layout and index math are bit-exact (R = I and +-1 inputs make every stored
value exact); with a real transform the stored bf16 values are within one
bf16 ulp of the oracle's float64 values rounded to nearest even (the GPU
rounds an fp32 value, so a value within fp32 error of a rounding boundary may
land on the other side), and almost all are identical.
"""

import numpy as np
import pytest
import torch

import gpu_harness as hx
from oracle import tpla_ref as ref
from latent_attention_decode_tpla_b200 import inputs as gen
from latent_attention_decode_tpla_b200 import tpla

pytestmark = pytest.mark.gpu

SENTINEL = torch.tensor(-12345.0).to(torch.bfloat16)


def _setup(B, L, R, g, maxp, seed, shuffle=True):
    num_pages = B * maxp + 3
    bt = gen.block_table(B, maxp, num_pages, seed, shuffle)
    dims = tpla.make_dims(B=B, H=1, L=L, R=R, dv=8, g=g, max_pages_per_seq=maxp, num_pages=num_pages,
                          softmax_scale=1.0)
    ckv = torch.full((num_pages, g, 64, L // g), float(SENTINEL), dtype=torch.bfloat16)
    kpe = torch.full((num_pages, 64, R), float(SENTINEL), dtype=torch.bfloat16)
    return dims, bt, ckv, kpe


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("g", [1, 2, 4, 8])
def test_layout_bit_exact(g):
    B, L, R, maxp = 6, 512, 64, 4
    dims, bt, ckv, kpe = _setup(B, L, R, g, maxp, seed=g)
    rng = np.random.default_rng(g)
    x = torch.from_numpy(rng.choice([-1.0, 1.0], size=(B, L)).astype(np.float32)).to(torch.bfloat16)
    kn = gen.randn((B, R), g, 9)
    pos = torch.tensor([0, 63, 64, 100, 255, 130], dtype=torch.int32)
    ckv_d, kpe_d = ckv.cuda(), kpe.cuda()
    tpla.append_kv(dims, x.cuda(), kn.cuda(), tpla.TRANSFORM_NONE, None, None, 0.0, pos.cuda(), bt.cuda(),
                   ckv_d, kpe_d)
    torch.cuda.synchronize()
    assert tpla.check_device_status() == tpla.TPLA_OK
    ck = hx.to64(ckv)
    kp = hx.to64(kpe)
    ref.append_kv(hx.to64(x), hx.to64(kn), pos.numpy(), bt.numpy(), ck, kp, g=g, max_pages_per_seq=maxp,
                  transform=ref.TRANSFORM_NONE, eps=0.0)
    np.testing.assert_array_equal(_bits(ckv_d), _bits(torch.from_numpy(ck).to(torch.bfloat16)))
    np.testing.assert_array_equal(_bits(kpe_d), _bits(torch.from_numpy(kp).to(torch.bfloat16)))


@pytest.mark.parametrize("transform,g,L,weight", [
    (ref.TRANSFORM_HADAMARD, 2, 512, False), (ref.TRANSFORM_HADAMARD, 4, 512, True),
    (ref.TRANSFORM_DENSE, 4, 512, False), (ref.TRANSFORM_DENSE, 2, 256, True),
    (ref.TRANSFORM_HADAMARD, 2, 64, False), (ref.TRANSFORM_NONE, 1, 512, False),
    (ref.TRANSFORM_HADAMARD, 8, 1024, False),
    (ref.TRANSFORM_BLOCK_HADAMARD, 2, 512, False), (ref.TRANSFORM_BLOCK_HADAMARD, 4, 512, True),
    (ref.TRANSFORM_BLOCK_HADAMARD, 8, 1024, False), (ref.TRANSFORM_BLOCK_HADAMARD, 1, 512, False),
    (ref.TRANSFORM_BLOCK_HADAMARD, 2, 64, False),
])
def test_values_within_one_ulp(transform, g, L, weight):
    B, R, maxp = 64, 64, 2
    dims, bt, ckv, kpe = _setup(B, L, R, g, maxp, seed=L + g)
    x = gen.randn((B, L), 7, 2, 3.0)
    kn = gen.randn((B, R), 7, 3)
    Rd = gen.random_orthogonal(L, 7) if transform == ref.TRANSFORM_DENSE else None
    w = (torch.rand(L, generator=torch.Generator().manual_seed(3)) + 0.5) if weight else None
    pos = torch.randint(0, maxp * 64, (B,), generator=torch.Generator().manual_seed(4), dtype=torch.int32)
    ckv_d, kpe_d = ckv.cuda(), kpe.cuda()
    tpla.append_kv(dims, x.cuda(), kn.cuda(), transform, None if Rd is None else Rd.cuda(),
                   None if w is None else w.cuda(), 1e-6, pos.cuda(), bt.cuda(), ckv_d, kpe_d)
    torch.cuda.synchronize()
    assert tpla.check_device_status() == tpla.TPLA_OK
    ck = hx.to64(ckv)
    kp = hx.to64(kpe)
    ref.append_kv(hx.to64(x), hx.to64(kn), pos.numpy(), bt.numpy(), ck, kp, g=g, max_pages_per_seq=maxp,
                  transform=transform, R_dense=None if Rd is None else Rd.numpy().astype(np.float64),
                  norm_weight=None if w is None else w.numpy().astype(np.float64), eps=1e-6)
    got = hx.to64(ckv_d)
    # compare as bf16 bit patterns: |difference| <= 1 ulp means adjacent patterns of the same sign
    gb = _bits(ckv_d).astype(np.int64)
    ob = _bits(torch.from_numpy(ck).to(torch.bfloat16)).astype(np.int64)
    same_sign = np.sign(got) == np.sign(ck)
    assert np.all((gb == ob) | (same_sign & (np.abs(gb - ob) <= 1))), "more than one ulp"
    assert np.mean(gb == ob) >= 0.999
    np.testing.assert_array_equal(_bits(kpe_d), _bits(torch.from_numpy(kp).to(torch.bfloat16)))


def test_bad_positions_are_skipped_and_reported():
    B, L, R, g, maxp = 3, 512, 64, 2, 2
    dims, bt, ckv, kpe = _setup(B, L, R, g, maxp, seed=1)
    x = gen.randn((B, L), 1, 2)
    kn = gen.randn((B, R), 1, 3)
    pos = torch.tensor([5, maxp * 64, -1], dtype=torch.int32)     # only the first is inside
    ckv_d, kpe_d = ckv.cuda(), kpe.cuda()
    tpla.append_kv(dims, x.cuda(), kn.cuda(), tpla.TRANSFORM_HADAMARD, None, None, 1e-6, pos.cuda(), bt.cuda(),
                   ckv_d, kpe_d)
    assert tpla.check_device_status() == tpla.TPLA_ERR_INDEX
    assert tpla.check_device_status() == tpla.TPLA_OK          # the status word was cleared
    changed = (_bits(ckv_d) != _bits(ckv)).reshape(ckv.shape[0], g, 64, -1).any(axis=(1, 3))
    page = int(bt[0, 0])
    assert changed[page, 5] and changed.sum() == 1
    # a page table entry outside the cache is skipped as well
    bt_bad = bt.clone()
    bt_bad[0, 0] = dims.num_pages + 7
    tpla.append_kv(dims, x.cuda(), kn.cuda(), tpla.TRANSFORM_HADAMARD, None, None, 1e-6,
                   torch.tensor([5, 6, 7], dtype=torch.int32).cuda(), bt_bad.cuda(), ckv_d, kpe_d)
    assert tpla.check_device_status() == tpla.TPLA_ERR_INDEX
