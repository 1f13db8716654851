"""Pins of the float64 oracle against things other than itself.

Each test ties one oracle function to a closed form, an invariant the TPLA
pages imply, a textbook/library routine, or brute-force loops on tiny inputs,
so that a dropped term, a wrong sign, index or shard, or a transposed operand
fails at least one of them.  CPU only.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.linalg
import torch

from oracle import tpla_ref as ref
from latent_attention_decode_tpla_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
P = ref.PAGE_SIZE


def _np(t):
    return t.to(torch.float64).numpy() if isinstance(t, torch.Tensor) else np.asarray(t, dtype=np.float64)


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_round_matches_torch_cast():
    # library routine: torch's float32 -> bfloat16 cast is round-to-nearest-even
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-30, 30, 20000),
                        rng.standard_normal(1000) * 1e-39]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = ref.bf16_round(x.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_bf16_round_ties_and_overflow():
    # ties go to the even significand
    assert ref.bf16_round(1.0 + 2.0 ** -8) == 1.0
    assert ref.bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert ref.bf16_round(-(1.0 + 2.0 ** -8)) == -1.0
    # just above a tie rounds up
    assert ref.bf16_round(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7
    # largest finite bfloat16, and overflow past its rounding boundary
    bmax = (2 - 2.0 ** -7) * 2.0 ** 127
    assert ref.bf16_round(bmax) == bmax
    assert np.isinf(ref.bf16_round(2.0 ** 128 - 2.0 ** 119))
    # subnormal quantum 2**-133
    assert ref.bf16_round(3 * 2.0 ** -134) == 2 * 2.0 ** -133
    assert ref.bf16_round(0.0) == 0.0


# ---------------------------------------------------------------- Hadamard

def test_hadamard_golden_h8():
    rows = [list(map(float, ln.split())) for ln in open(os.path.join(GOLDEN, "hadamard8.txt"))
            if ln.strip() and not ln.startswith("#")]
    np.testing.assert_array_equal(ref.sylvester_hadamard(8), np.array(rows))


@pytest.mark.parametrize("n", [1, 2, 16, 64, 512])
def test_hadamard_library_walsh_and_orthogonal(n):
    h = ref.sylvester_hadamard(n)
    np.testing.assert_array_equal(h, scipy.linalg.hadamard(n).astype(np.float64))
    i, j = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    walsh = np.vectorize(lambda a: (-1.0) ** bin(a).count("1"))(i & j)
    np.testing.assert_array_equal(h, walsh)
    np.testing.assert_array_equal(h @ h.T, n * np.eye(n))
    t = ref.transform_matrix(ref.TRANSFORM_HADAMARD, n)
    np.testing.assert_allclose(t @ t.T, np.eye(n), atol=1e-13)


def test_dense_transform_is_caller_matrix_and_orthogonal():
    Rd = gen.random_orthogonal(64, seed=0).numpy().astype(np.float64)
    t = ref.transform_matrix(ref.TRANSFORM_DENSE, 64, Rd)
    np.testing.assert_array_equal(t, Rd)
    np.testing.assert_allclose(t @ t.T, np.eye(64), atol=1e-6)


@pytest.mark.parametrize("L,g", [(4, 2), (64, 4), (512, 2), (512, 8)])
def test_block_hadamard_is_per_shard_sylvester(L, g):
    # library routine: scipy's Sylvester Hadamard of order L/g on every diagonal block, zero elsewhere
    Ls = L // g
    t = ref.transform_matrix(ref.TRANSFORM_BLOCK_HADAMARD, L, None, g)
    want = scipy.linalg.block_diag(*([scipy.linalg.hadamard(Ls) / math.sqrt(Ls)] * g))
    np.testing.assert_allclose(t, want, rtol=0, atol=1e-15)
    np.testing.assert_allclose(t @ t.T, np.eye(L), atol=1e-13)
    # one block is the full transform
    np.testing.assert_array_equal(ref.transform_matrix(ref.TRANSFORM_BLOCK_HADAMARD, L, None, 1),
                                  ref.transform_matrix(ref.TRANSFORM_HADAMARD, L))


def test_block_hadamard_append_hand_worked_and_shard_local():
    # L = 4, g = 2: each shard's pair (a, b) becomes ((a + b), (a - b)) / sqrt(2), then its own RMSNorm.
    # x = [3, 1, 2, -2]: shard 0 -> [4, 2] / sqrt 2, mean square 5, so c_0 = [4, 2] / sqrt(2 (5 + eps));
    # shard 1 -> [0, 4] / sqrt 2, mean square 4, so c_1 = [0, 4] / sqrt(2 (4 + eps)).
    eps = 1e-6
    c = ref.append_values(np.array([[3.0, 1.0, 2.0, -2.0]]), 2, ref.TRANSFORM_BLOCK_HADAMARD, None, None, eps)
    np.testing.assert_allclose(c[0, 0], np.array([4.0, 2.0]) / math.sqrt(2 * (5 + eps)), rtol=1e-15)
    np.testing.assert_allclose(c[0, 1], np.array([0.0, 4.0]) / math.sqrt(2 * (4 + eps)), rtol=1e-15)
    # the full transform mixes the shards: the same input gives other values
    full = ref.append_values(np.array([[3.0, 1.0, 2.0, -2.0]]), 2, ref.TRANSFORM_HADAMARD, None, None, eps)
    assert np.max(np.abs(full - c)) > 0.1
    # a one-hot input in shard 2 of 4 leaves every other shard zero (no mixing across shards)
    L, g = 64, 4
    x = np.zeros((1, L)); x[0, 2 * 16 + 5] = 1.0
    cb = ref.append_values(x, g, ref.TRANSFORM_BLOCK_HADAMARD, None, None, eps)
    for s in range(g):
        assert np.all(cb[0, s] == 0.0) == (s != 2)
    np.testing.assert_allclose(cb[0, 2], scipy.linalg.hadamard(16)[:, 5] / math.sqrt(1 + 16 * eps), rtol=1e-14)


# ---------------------------------------------------------------- append (transform + sliced RMSNorm)

def test_append_g1_equals_transform_of_rmsnorm():
    # RMS is invariant under an orthogonal R, so with one shard
    # "transform, then RMSNorm" equals R applied to RMSNorm(x).
    rng = np.random.default_rng(2)
    x = rng.standard_normal((5, 64))
    eps = 1e-6
    q64 = np.linalg.qr(rng.standard_normal((64, 64)))[0]      # orthogonal to float64 precision
    for tr, Rd in [(ref.TRANSFORM_HADAMARD, None), (ref.TRANSFORM_DENSE, q64)]:
        Rm = scipy.linalg.hadamard(64) / 8.0 if Rd is None else Rd
        want = (x / np.sqrt(np.mean(x * x, axis=1, keepdims=True) + eps)) @ Rm.T
        got = ref.append_values(x, 1, tr, Rd, None, eps)[:, 0, :]
        np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_append_sliced_rmsnorm_closed_form():
    # L=4, g=2, x = e0 + e2: H_4 x / 2 = [1, 1, 0, 0], so shard 0 normalises to
    # [1, 1] / sqrt(1 + eps) and shard 1 (all zero) stays 0.  Normalising the
    # whole vector first would give sqrt(2) instead: this pins the order.
    eps = 1e-6
    c = ref.append_values(np.array([[1.0, 0.0, 1.0, 0.0]]), 2, ref.TRANSFORM_HADAMARD, None, None, eps)
    np.testing.assert_allclose(c[0, 0], [1 / math.sqrt(1 + eps)] * 2, rtol=1e-15)
    np.testing.assert_array_equal(c[0, 1], [0.0, 0.0])
    # one-hot input: every Hadamard entry is +-1/sqrt(L); signs are column j of H
    L, g, j = 64, 4, 37
    x = np.zeros((1, L)); x[0, j] = 1.0
    c = ref.append_values(x, g, ref.TRANSFORM_HADAMARD, None, None, eps).reshape(L)
    np.testing.assert_allclose(c, scipy.linalg.hadamard(L)[:, j] / math.sqrt(1 + L * eps), rtol=1e-14)
    # norm weight multiplies after normalisation, in the transformed basis
    w = np.arange(1, L + 1, dtype=np.float64)
    cw = ref.append_values(x, g, ref.TRANSFORM_HADAMARD, None, w, eps).reshape(L)
    np.testing.assert_allclose(cw, c * w, rtol=1e-14)


def test_append_each_shard_row_has_unit_rms():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((7, 512)) * 3.0
    c = ref.append_values(x, 4, ref.TRANSFORM_HADAMARD, None, None, 0.0)
    np.testing.assert_allclose(np.mean(c * c, axis=2), 1.0, rtol=1e-13)


def test_append_kv_layout_exact_under_shuffled_pages():
    # R = I and +-1 inputs with eps = 0 give exactly representable values, so the
    # cache must hold exactly x at the flat address ((page*g + s)*64 + slot)*Ls + j.
    B, L, R, g, maxp = 3, 64, 16, 2, 3
    Ls = L // g
    num_pages = B * maxp + 2
    bt = gen.block_table(B, maxp, num_pages, seed=5).numpy()
    rng = np.random.default_rng(5)
    x = rng.choice([-1.0, 1.0], size=(B, L))
    kp = ref.bf16_round(rng.standard_normal((B, R)))
    pos = np.array([0, 64 + 5, 3 * 64 - 1])
    sentinel = 7.0
    ckv = np.full((num_pages, g, P, Ls), sentinel)
    kpe = np.full((num_pages, P, R), sentinel)
    ref.append_kv(x, kp, pos, bt, ckv, kpe, g=g, max_pages_per_seq=maxp,
                  transform=ref.TRANSFORM_NONE, eps=0.0)
    flat = ckv.reshape(-1)
    flat_k = kpe.reshape(-1)
    touched = np.zeros(flat.size, bool)
    touched_k = np.zeros(flat_k.size, bool)
    for b in range(B):
        page = bt[b][pos[b] // 64]
        slot = pos[b] % 64
        for s in range(g):
            for jj in range(Ls):
                a = ((page * g + s) * 64 + slot) * Ls + jj
                assert flat[a] == x[b, s * Ls + jj]
                touched[a] = True
        for r in range(R):
            a = (page * 64 + slot) * R + r
            assert flat_k[a] == kp[b, r]
            touched_k[a] = True
    assert np.all(flat[~touched] == sentinel)
    assert np.all(flat_k[~touched_k] == sentinel)


# ---------------------------------------------------------------- decode

def _small_case(B, H, L, R, dv, g, lens, seed, shuffle=True, dn=None):
    d = gen.make_workload(B=B, H=H, L=L, R=R, dv=dv, g=g, seq_lens=lens, seed=seed,
                          extra_pages=3, shuffle=shuffle, dn=dn)
    return dict(q=_np(d["q"]), q_pe=_np(d["q_pe"]), ckv=_np(d["ckv"]), kpe=_np(d["kpe"]),
                bt=d["block_table"].numpy(), lens=d["seq_lens"].numpy(), w_uv=_np(d["w_uv"]),
                maxp=d["max_pages_per_seq"], raw=d)


def _brute_force(c, scale, shard_only=None, latent=False, probs=None):
    """Scalar loops over b, h, s, t with an explicit page walk (no numpy algebra).

    If ``probs`` is a dict, the softmax weights of every (b, s) with T_b > 0 are
    stored in it as probs[(b, s)][h][t]."""
    q, q_pe, ckv, kpe, bt, lens, w = c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], c["w_uv"]
    B, H, L = q.shape
    g = ckv.shape[1]
    Ls = L // g
    R = q_pe.shape[2]
    dv = w.shape[2]
    shards = range(g) if shard_only is None else [shard_only]
    out = np.zeros((B, H, (len(shards) * Ls) if latent else dv))
    for b in range(B):
        T = int(lens[b])
        for h in range(H):
            for si, s in enumerate(shards):
                if T == 0:
                    continue
                zs = []
                for t in range(T):
                    page, slot = bt[b][t // 64], t % 64
                    acc = 0.0
                    for j in range(Ls):
                        acc += q[b, h, s * Ls + j] * ckv[page, s, slot, j]
                    for r in range(R):
                        acc += q_pe[b, h, r] * kpe[page, slot, r]
                    zs.append(scale * acc)
                m = max(zs)
                es = [math.exp(z - m) for z in zs]
                den = sum(es)
                if probs is not None:
                    probs.setdefault((b, s), [None] * H)[h] = [e / den for e in es]
                o = [0.0] * Ls
                for t in range(T):
                    page, slot = bt[b][t // 64], t % 64
                    for j in range(Ls):
                        o[j] += es[t] / den * ckv[page, s, slot, j]
                if latent:
                    for j in range(Ls):
                        out[b, h, si * Ls + j] = o[j]
                else:
                    for dd in range(dv):
                        acc = 0.0
                        for j in range(Ls):
                            acc += o[j] * w[h, s * Ls + j, dd]
                        out[b, h, dd] += acc
    return out


@pytest.mark.parametrize("g", [1, 2, 4])
def test_decode_matches_brute_force(g):
    c = _small_case(B=4, H=3, L=16, R=4, dv=5, g=g, lens=[0, 1, 65, 130], seed=11)
    scale = 0.37
    got = ref.decode(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], scale,
                     max_pages_per_seq=c["maxp"], w_uv=c["w_uv"])
    np.testing.assert_allclose(got, _brute_force(c, scale), rtol=0, atol=1e-12)
    lat = ref.decode(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], scale,
                     max_pages_per_seq=c["maxp"])
    np.testing.assert_allclose(lat, _brute_force(c, scale, latent=True), rtol=0, atol=1e-12)
    for s in range(g):
        sh = ref.decode_shard(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], scale, s,
                              max_pages_per_seq=c["maxp"], w_uv=c["w_uv"])
        np.testing.assert_allclose(sh, _brute_force(c, scale, shard_only=s), rtol=0, atol=1e-12)


def test_decode_hand_worked_example():
    f = json.load(open(os.path.join(GOLDEN, "hand_tiny.json")))
    L, g, R, dv = f["L"], f["g"], f["R"], f["dv"]
    ckv = np.zeros((1, g, P, L // g))
    kpe = np.zeros((1, P, R))
    for t, (lat, kp) in enumerate(zip(f["tokens_latent"], f["tokens_kpe"])):
        ckv[0, :, t, :] = np.array(lat).reshape(g, L // g)
        kpe[0, t] = kp
    q = np.array(f["q"]).reshape(1, 1, L)
    q_pe = np.array(f["q_pe"]).reshape(1, 1, R)
    w = np.array(f["w_uv_rows"]).reshape(1, L, dv)
    lens = [len(f["tokens_latent"])]
    e = f["expected"]
    kw = dict(max_pages_per_seq=1)
    np.testing.assert_allclose(ref.decode(q, q_pe, ckv, kpe, None, lens, f["scale"], **kw)[0, 0],
                               e["o_shard"], rtol=1e-15)
    np.testing.assert_allclose(ref.decode(q, q_pe, ckv, kpe, None, lens, f["scale"], w_uv=w, **kw)[0, 0],
                               e["out"], rtol=1e-15)
    for s in range(g):
        np.testing.assert_allclose(
            ref.decode_shard(q, q_pe, ckv, kpe, None, lens, f["scale"], s, w_uv=w, **kw)[0, 0],
            e["shard_terms"][s], rtol=1e-15)
    ckv1 = ckv.transpose(0, 2, 1, 3).reshape(1, P, 1, L).transpose(0, 2, 1, 3)
    np.testing.assert_allclose(ref.decode(q, q_pe, ckv1, kpe, None, lens, f["scale"], **kw)[0, 0],
                               e["mla_g1_latent"], rtol=1e-15)
    np.testing.assert_allclose(ref.decode(q, q_pe, ckv1, kpe, None, lens, f["scale"], w_uv=w, **kw)[0, 0],
                               e["mla_g1_out"], rtol=1e-15)


def test_g1_equals_nonabsorbed_mla():
    # absorption is associativity: (W_UK q)^T c = q^T (W_UK^T c), and p (c W_UV) = (p c) W_UV
    B, H, L, R, dn, dv = 2, 4, 32, 8, 12, 10
    c = _small_case(B=B, H=H, L=L, R=R, dv=dv, g=1, lens=[70, 129], seed=21, dn=dn)
    w_uk = _np(c["raw"]["w_uk"])
    q_nope = _np(c["raw"]["q_nope"])
    scale = 1 / math.sqrt(dn + R)
    q_abs = ref.absorb_query(q_nope, w_uk)
    got = ref.decode(q_abs, c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], scale,
                     max_pages_per_seq=c["maxp"], w_uv=c["w_uv"])
    T = int(max(c["lens"]))
    latent = np.zeros((B, T, L))
    kp = np.zeros((B, T, R))
    for b in range(B):
        for t in range(int(c["lens"][b])):
            page, slot = c["bt"][b][t // 64], t % 64
            latent[b, t] = c["ckv"][page, 0, slot]
            kp[b, t] = c["kpe"][page, slot]
    want = ref.mla_nonabsorbed(q_nope, c["q_pe"], latent, kp, w_uk, c["w_uv"], scale, c["lens"])
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kind", ["hadamard", "dense"])
def test_g1_orthogonal_invariance(kind):
    # transforming query, latent and W_UV rows by the same orthogonal R leaves g=1 unchanged
    L = 64
    c = _small_case(B=2, H=3, L=L, R=8, dv=6, g=1, lens=[50, 140], seed=31)
    Rm = (scipy.linalg.hadamard(L) / 8.0) if kind == "hadamard" else \
        np.linalg.qr(np.random.default_rng(9).standard_normal((L, L)))[0]
    q2 = np.einsum("ij,bhj->bhi", Rm, c["q"])
    ckv2 = np.einsum("ij,psj->psi", Rm, c["ckv"][:, 0]).reshape(c["ckv"].shape)
    w2 = np.einsum("ij,hjd->hid", Rm, c["w_uv"])
    kw = dict(max_pages_per_seq=c["maxp"])
    a = ref.decode(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], 0.3, w_uv=c["w_uv"], **kw)
    b = ref.decode(q2, c["q_pe"], ckv2, c["kpe"], c["bt"], c["lens"], 0.3, w_uv=w2, **kw)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_shard_softmax_rows_sum_to_one():
    c = _small_case(B=2, H=5, L=64, R=16, dv=8, g=4, lens=[1, 200], seed=41)
    for b in range(2):
        for s in range(4):
            p = ref.shard_probabilities(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], 0.5,
                                        b, s, max_pages_per_seq=c["maxp"])
            assert p.shape == (5, int(c["lens"][b]))
            assert np.all(p >= 0)
            np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def test_shard_probabilities_match_brute_force():
    # every (sequence, shard) of a g = 4 case on a shuffled page table, including a one-token
    # sequence and tails that end inside a page: the weights must be the brute-force loop's
    # exp(z - max) / sum, head by head and token by token
    c = _small_case(B=3, H=3, L=32, R=4, dv=2, g=4, lens=[1, 70, 129], seed=43)
    scale = 0.45
    probs = {}
    _brute_force(c, scale, probs=probs)
    for b in range(3):
        for s in range(4):
            p = ref.shard_probabilities(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], scale,
                                        b, s, max_pages_per_seq=c["maxp"])
            np.testing.assert_allclose(p, np.array(probs[(b, s)]), rtol=0, atol=1e-14)
    # and the weights of different shards differ (each shard has its own softmax)
    p0 = ref.shard_probabilities(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], scale, 2, 0,
                                 max_pages_per_seq=c["maxp"])
    p3 = ref.shard_probabilities(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], scale, 2, 3,
                                 max_pages_per_seq=c["maxp"])
    assert np.max(np.abs(p0 - p3)) > 1e-3


@pytest.mark.parametrize("g", [1, 2, 4])
def test_gla_decode_matches_brute_force_by_head_group(g):
    # brute force: each head of group s is the scalar loop of shard s alone (no sum over shards)
    c = _small_case(B=3, H=4, L=16, R=4, dv=5, g=g, lens=[0, 65, 130], seed=19)
    scale = 0.33
    kw = dict(max_pages_per_seq=c["maxp"])
    got = ref.gla_decode(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], scale, w_uv=c["w_uv"], **kw)
    lat = ref.gla_decode(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], scale, **kw)
    Hg = 4 // g
    for s in range(g):
        heads = slice(s * Hg, (s + 1) * Hg)
        np.testing.assert_allclose(got[:, heads], _brute_force(c, scale, shard_only=s)[:, heads], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lat[:, heads], _brute_force(c, scale, shard_only=s, latent=True)[:, heads],
                                   rtol=0, atol=1e-12)
    if g == 1:   # one group: MLA
        np.testing.assert_allclose(got, ref.decode(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], scale,
                                                   w_uv=c["w_uv"], **kw), rtol=0, atol=1e-13)
    if g > 1:   # heads must split evenly into the groups
        with pytest.raises(ValueError):
            ref.gla_decode(c["q"][:, :3], c["q_pe"][:, :3], c["ckv"], c["kpe"], c["bt"], c["lens"], scale, **kw)


def _to_g1(ckv):
    n, g, _, Ls = ckv.shape
    return ckv.transpose(0, 2, 1, 3).reshape(n, P, g * Ls)[:, None]


@pytest.mark.parametrize("g", [2, 4])
def test_special_cases(g):
    c = _small_case(B=3, H=4, L=32, R=8, dv=6, g=g, lens=[1, 77, 150], seed=51)
    kw = dict(max_pages_per_seq=c["maxp"])
    w = c["w_uv"]
    out = ref.decode(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], 0.4, w_uv=w, **kw)
    # seq_len 1: every softmax is [1], so out = W_UV^T c_0 for every g
    page = c["bt"][0][0]
    c0 = c["ckv"][page, :, 0, :].reshape(-1)
    np.testing.assert_allclose(out[0], np.einsum("l,hld->hd", c0, w), rtol=0, atol=1e-13)
    # q~ = 0: all shards share the RoPE-only softmax, so TPLA(g) equals MLA (g = 1) exactly
    qz = np.zeros_like(c["q"])
    a = ref.decode(qz, c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], 0.4, w_uv=w, **kw)
    b = ref.decode(qz, c["q_pe"], _to_g1(c["ckv"]), c["kpe"], c["bt"], c["lens"], 0.4, w_uv=w, **kw)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)
    # scale = 0: uniform weights, out = W_UV^T mean_t c_t
    u = ref.decode(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], 0.0, w_uv=w, **kw)
    for bb in range(3):
        T = int(c["lens"][bb])
        rows = [c["ckv"][c["bt"][bb][t // 64], :, t % 64, :].reshape(-1) for t in range(T)]
        np.testing.assert_allclose(u[bb], np.einsum("l,hld->hd", np.mean(rows, axis=0), w),
                                   rtol=0, atol=1e-13)
    # the per-shard terms sum to the full result (the all-reduce is a sum)
    tot = sum(ref.decode_shard(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], 0.4, s,
                               w_uv=w, **kw) for s in range(g))
    np.testing.assert_allclose(tot, out, rtol=0, atol=1e-13)


def test_identity_page_table_and_empty_sequences():
    c = _small_case(B=3, H=2, L=16, R=4, dv=3, g=2, lens=[0, 64, 100], seed=61, shuffle=False)
    kw = dict(max_pages_per_seq=c["maxp"])
    a = ref.decode(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], 0.7, w_uv=c["w_uv"], **kw)
    b = ref.decode(c["q"], c["q_pe"], c["ckv"], c["kpe"], None, c["lens"], 0.7, w_uv=c["w_uv"], **kw)
    np.testing.assert_array_equal(a, b)
    assert np.all(a[0] == 0.0)


def test_tokens_past_seq_len_are_ignored():
    c = _small_case(B=1, H=2, L=16, R=4, dv=3, g=2, lens=[70], seed=71)
    kw = dict(max_pages_per_seq=c["maxp"])
    a = ref.decode(c["q"], c["q_pe"], c["ckv"], c["kpe"], c["bt"], c["lens"], 0.7, w_uv=c["w_uv"], **kw)
    ckv = c["ckv"].copy()
    page = c["bt"][0][1]
    ckv[page, :, 6:, :] = 1e6      # slots 70.. of the tail page
    b = ref.decode(c["q"], c["q_pe"], ckv, c["kpe"], c["bt"], c["lens"], 0.7, w_uv=c["w_uv"], **kw)
    np.testing.assert_array_equal(a, b)


# ---------------------------------------------------------------- MLA-form prefill

def test_mla_prefill_matches_brute_force():
    # independent statement: Sylvester H_8 from scipy, one RMSNorm over the whole row, bf16 by torch's
    # cast, then scalar loops for the causal softmax and the W_UV projection
    rng = np.random.default_rng(17)
    T, H, L, R, dv = 5, 2, 8, 4, 3
    x = rng.standard_normal((T, L))
    kpe = np.asarray(torch.from_numpy(rng.standard_normal((T, R))).to(torch.bfloat16).to(torch.float64))
    q = rng.standard_normal((T, H, L))
    q_pe = rng.standard_normal((T, H, R))
    w = rng.standard_normal((H, L, dv))
    scale, eps = 0.37, 1e-6
    Hm = scipy.linalg.hadamard(L) / math.sqrt(L)
    c = []
    for t in range(T):
        y = Hm @ x[t]
        y = y / math.sqrt(sum(v * v for v in y) / L + eps)
        c.append(torch.tensor(y).to(torch.bfloat16).to(torch.float64).numpy())
    want = np.zeros((T, H, dv))
    for t in range(T):
        for h in range(H):
            zs = [scale * (sum(q[t, h, j] * c[i][j] for j in range(L)) + sum(q_pe[t, h, r] * kpe[i, r] for r in range(R)))
                  for i in range(t + 1)]
            m = max(zs)
            es = [math.exp(z - m) for z in zs]
            den = sum(es)
            for d in range(dv):
                want[t, h, d] = sum(es[i] / den * sum(c[i][j] * w[h, j, d] for j in range(L)) for i in range(t + 1))
    got = ref.mla_prefill(x, kpe, q, q_pe, scale, transform=ref.TRANSFORM_HADAMARD, eps=eps, w_uv=w)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    # the first token sees only itself: out_0 = W_UV^T c_0 for every head
    np.testing.assert_allclose(got[0], np.einsum('l,hld->hd', c[0], w), rtol=1e-12, atol=1e-12)
    # without W_UV the rows are convex combinations of the latent rows seen so far
    lat = ref.mla_prefill(x, kpe, q, q_pe, scale, transform=ref.TRANSFORM_HADAMARD, eps=eps)
    np.testing.assert_allclose(lat[0], np.broadcast_to(c[0], (H, L)), rtol=1e-12)
    C = np.stack(c)
    for t in range(T):
        assert np.all(lat[t] <= C[:t + 1].max(axis=0) + 1e-12) and np.all(lat[t] >= C[:t + 1].min(axis=0) - 1e-12)


def test_mla_prefill_last_token_is_the_g1_decode_over_the_prompt():
    # the last prompt token's output is a g = 1 decode of a sequence whose cache holds the prompt
    rng = np.random.default_rng(5)
    T, H, L, R, dv = 70, 3, 16, 4, 5
    x = rng.standard_normal((T, L))
    kpe = np.asarray(torch.from_numpy(rng.standard_normal((T, R))).to(torch.bfloat16).to(torch.float64))
    q = rng.standard_normal((T, H, L))
    q_pe = rng.standard_normal((T, H, R))
    w = rng.standard_normal((H, L, dv))
    out = ref.mla_prefill(x, kpe, q, q_pe, 0.2, transform=ref.TRANSFORM_HADAMARD, w_uv=w)
    ckv = np.zeros((2, 1, 64, L)); kc = np.zeros((2, 64, R))
    c = ref.bf16_round(ref.append_values(x, 1, ref.TRANSFORM_HADAMARD))[:, 0, :]
    for t in range(T):
        ckv[t // 64, 0, t % 64] = c[t]
        kc[t // 64, t % 64] = kpe[t]
    for t in (0, 63, 64, T - 1):
        dec = ref.decode(q[t][None], q_pe[t][None], ckv, kc, np.array([[0, 1]]), np.array([t + 1]), 0.2,
                         max_pages_per_seq=2, w_uv=w)
        np.testing.assert_allclose(out[t], dec[0], rtol=1e-12, atol=1e-12)
