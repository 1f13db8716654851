"""Seeded synthetic inputs for TPLA decode (shared by tests, bench and smoke).

This module only draws random numbers and builds index tables; it holds none
of the method's arithmetic, so the GPU path and the CPU oracle can both be fed
from it without sharing any computation.  Every tensor has its own sub-seed
so that changing one shape does not perturb the others:

    q~ (absorbed query) 0, q_pe 1, raw latent x 2, k_pe 3, W_UV 4,
    dense orthogonal transform 5, sequence lengths 6, page permutation 7,
    new-token latent 8, new-token k_pe 9, W_UK 10, q_nope 11.

Value recipe: q~, q_pe, k_pe and the raw latent ~ N(0, 1) (times ``value_scale``
per tensor when a workload asks for N(0,1)/sqrt(dim)); W_UV ~ N(0,1)/sqrt(L).
The dense transform is the Q factor of the QR decomposition of an N(0,1)
L x L matrix with column signs fixed by sign(diag(R)) -- a seeded random
orthogonal matrix that stands in for a calibrated PCA basis.
"""

import math

import numpy as np
import torch

PAGE_SIZE = 64

SUB_Q, SUB_QPE, SUB_X, SUB_KPE, SUB_WUV, SUB_RDENSE, SUB_LENS, SUB_PERM, \
    SUB_XNEW, SUB_KPENEW, SUB_WUK, SUB_QNOPE = range(12)


def _gen(seed, sub):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1000 + int(sub))
    return g


def randn(shape, seed, sub, std=1.0, dtype=torch.bfloat16, chunk_elems=1 << 26):
    """N(0, std^2) samples drawn in float32 on the CPU, then cast (RN-even) to ``dtype``.

    Large tensors are drawn in slices along dim 0 from one generator, so the
    values do not depend on the slice size beyond the fixed ``chunk_elems``.
    """
    shape = tuple(int(s) for s in shape)
    gen = _gen(seed, sub)
    n = 1
    for s in shape:
        n *= s
    if n <= chunk_elems or len(shape) == 1:
        x = torch.randn(*shape, generator=gen, dtype=torch.float32)
        if std != 1.0:
            x = x * std
        return x.to(dtype)
    out = torch.empty(shape, dtype=dtype)
    row = n // shape[0]
    step = max(1, chunk_elems // row)
    for i in range(0, shape[0], step):
        j = min(shape[0], i + step)
        x = torch.randn((j - i,) + shape[1:], generator=gen, dtype=torch.float32)
        if std != 1.0:
            x = x * std
        out[i:j] = x.to(dtype)
    return out


def random_orthogonal(L, seed):
    """Seeded random orthogonal L x L matrix (float32), the PCA stand-in."""
    a = torch.randn(L, L, generator=_gen(seed, SUB_RDENSE), dtype=torch.float64).numpy()
    q, r = np.linalg.qr(a)
    q = q * np.sign(np.diag(r))[None, :]
    return torch.from_numpy(q.astype(np.float32))


def seq_lengths(B, lo, hi, seed):
    """Sequence lengths uniform on the integers [lo, hi]."""
    return torch.randint(lo, hi + 1, (B,), generator=_gen(seed, SUB_LENS), dtype=torch.int32)


def block_table(B, max_pages_per_seq, num_pages, seed, shuffle=True):
    """[B, max_pages_per_seq] int32 page table: a seeded permutation of the physical pages."""
    if num_pages < B * max_pages_per_seq:
        raise ValueError("not enough pages")
    if shuffle:
        perm = torch.randperm(num_pages, generator=_gen(seed, SUB_PERM)).to(torch.int32)
    else:
        perm = torch.arange(num_pages, dtype=torch.int32)
    return perm[: B * max_pages_per_seq].reshape(B, max_pages_per_seq).contiguous()


def pages_for(T):
    return (int(T) + PAGE_SIZE - 1) // PAGE_SIZE


def make_workload(*, B, H, L, R, dv, g, seq_lens, seed=0, extra_pages=0, shuffle=True,
                  q_std=1.0, qpe_std=1.0, x_std=1.0, kpe_std=1.0, wuv_std=None,
                  dn=None, with_new_token=True, cache_values="normal"):
    """All inputs of one decode step, as CPU tensors.

    seq_lens: list/tensor of per-sequence lengths (tokens already cached).
    cache_values: "normal" fills every cache slot with N(0,1) bf16 (unit RMS,
    like the output of sliced RMSNorm); "none" leaves the latent cache zero so
    that the caller can fill it by appending ``x`` (the raw pre-norm latent of
    every cached token, returned as ``x_all`` [B, Tmax, L]).
    """
    seq_lens = torch.as_tensor(seq_lens, dtype=torch.int32).reshape(B)
    tmax = int(seq_lens.max().item()) if B > 0 else 0
    maxp = max(1, pages_for(tmax + (1 if with_new_token else 0)))
    num_pages = B * maxp + extra_pages
    Ls = L // g
    d = dict(B=B, H=H, L=L, R=R, dv=dv, g=g, Ls=Ls, max_pages_per_seq=maxp, num_pages=num_pages)
    d["q"] = randn((B, H, L), seed, SUB_Q, q_std)
    d["q_pe"] = randn((B, H, R), seed, SUB_QPE, qpe_std)
    if cache_values == "normal":
        d["ckv"] = randn((num_pages, g, PAGE_SIZE, Ls), seed, SUB_X, 1.0)
    else:
        d["ckv"] = torch.zeros((num_pages, g, PAGE_SIZE, Ls), dtype=torch.bfloat16)
        d["x_all"] = randn((B, max(tmax, 1), L), seed, SUB_X, x_std)
    d["kpe"] = randn((num_pages, PAGE_SIZE, R), seed, SUB_KPE, kpe_std)
    d["block_table"] = block_table(B, maxp, num_pages, seed, shuffle)
    d["seq_lens"] = seq_lens
    d["w_uv"] = randn((H, L, dv), seed, SUB_WUV, (1.0 / math.sqrt(L)) if wuv_std is None else wuv_std)
    if with_new_token:
        d["x_new"] = randn((B, L), seed, SUB_XNEW, x_std)
        d["kpe_new"] = randn((B, R), seed, SUB_KPENEW, kpe_std)
    if dn is not None:
        d["w_uk"] = randn((H, L, dn), seed, SUB_WUK, 1.0 / math.sqrt(L))
        d["q_nope"] = randn((B, H, dn), seed, SUB_QNOPE, 1.0)
    return d


# Workloads of the benchmark configurations (shapes of DeepSeek-V3 and Kimi-K2 attention).
# scale = 1/sqrt(qk_nope_head_dim + rope_dim).
WORKLOADS = {
    "tiny_g2": dict(B=1, H=8, L=64, R=16, dv=32, g=2, T=128, qk_nope=32, transform=1,
                    stds=dict(q_std=1 / math.sqrt(64), qpe_std=1 / math.sqrt(16),
                              x_std=1 / math.sqrt(64), kpe_std=1 / math.sqrt(16))),
    "mla_g1_dsv3_b1_4k": dict(B=1, H=128, L=512, R=64, dv=128, g=1, T=4096, qk_nope=128, transform=1),
    "mla_g1_dsv3_b8_32k": dict(B=8, H=128, L=512, R=64, dv=128, g=1, T=32768, qk_nope=128, transform=1),
    "tpla_g2_dsv3_b1_32k": dict(B=1, H=128, L=512, R=64, dv=128, g=2, T=32768, qk_nope=128, transform=1),
    "tpla_g2_dsv3_b16_32k": dict(B=16, H=128, L=512, R=64, dv=128, g=2, T=32768, qk_nope=128, transform=1),
    "tpla_g4_kimi_b8_32k": dict(B=8, H=64, L=512, R=64, dv=128, g=4, T=32768, qk_nope=128, transform=2),
    "tpla_g2_dsv3_b64_mixed": dict(B=64, H=128, L=512, R=64, dv=128, g=2, T=(1024, 65536),
                                   qk_nope=128, transform=1),
}


def workload_seq_lens(spec, seed=0):
    T = spec["T"]
    if isinstance(T, tuple):
        return seq_lengths(spec["B"], T[0], T[1], seed)
    return torch.full((spec["B"],), int(T), dtype=torch.int32)


def softmax_scale(spec):
    return 1.0 / math.sqrt(spec["qk_nope"] + spec["R"])
