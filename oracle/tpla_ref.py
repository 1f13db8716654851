"""Float64 CPU oracle for TPLA decode (Tensor-Parallel Latent Attention).

TEST INFRASTRUCTURE ONLY. This module is the slow, obviously-correct statement
of what the GPU path computes. Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it; the product path
(``latent_attention_decode_tpla_b200``) never does, and this module imports
nothing from it.  Plain numpy in float64; ``numpy.matmul``/``einsum`` are the
only library primitives used as steps.

Sources (the paper "TPLA: Tensor Parallel Latent Attention for Efficient
Disaggregated Prefill & Decode Inference", arXiv 2508.15881):
  [ABS]   the paper's abstract (chatpaper.ai, fugumt.com and searcharxiv.org
          pages): MLA caches one low-rank latent per token; TPLA splits the
          latent and every head's input dimension into shards, runs attention
          independently on each shard and sums the shard results (all-reduce);
          orthogonal transforms (Hadamard, PCA) are applied before slicing.
  [BLOG]  edgentiq blog "Enhancing LLM Efficiency: A New Approach to
          Tensor-Parallel Latent Attention", sections "Introducing TPLA",
          "How TPLA Works: Smart Slicing and Reparameterization" (RMSNorm
          slicing and softmax slicing after an orthogonal transform) and
          "Prefill-Decode Separation" (decode is memory-bound and uses TPLA).
  [PBOT]  paperbot summary page, extended abstract: the cache is named cKV;
          RMSNorm and softmax get orthogonal reparameterisations.

Readings where the pages are silent:
  * the decoupled RoPE key is replicated: every shard adds the full
    q_pe . k_pe term to its scores;
  * the softmax scale is the caller's ``scale`` for every shard (no
    per-shard compensation);
  * shard results are summed (the all-reduce is a sum);
  * transform first, then per-shard RMSNorm: y = R x, c_s = y_s / sqrt(mean(y_s^2) + eps),
    optionally times a weight in the transformed basis;
  * Hadamard = Sylvester construction in natural order, scaled by 1/sqrt(L);
    the block variant applies H_{L/g} / sqrt(L/g) to each shard's slice alone;
  * stored cache values are rounded to bfloat16, round-to-nearest-even;
  * tokens at positions >= seq_len are ignored; an empty sequence gives 0.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
closed forms, invariants, textbook/library routines or brute force.
"""

import numpy as np

PAGE_SIZE = 64          # tokens per cache page (layout of the paged latent cache)

TRANSFORM_NONE = 0
TRANSFORM_HADAMARD = 1
TRANSFORM_DENSE = 2
TRANSFORM_BLOCK_HADAMARD = 3


# --------------------------------------------------------------------------
# number format
# --------------------------------------------------------------------------

def bf16_round(x):
    """Round float64 values to the nearest bfloat16 value (ties to even).

    bfloat16 keeps 8 significant bits and the float32 exponent range, so a
    normal number with 2**(e-1) <= |x| < 2**e has quantum 2**(e-8); below the
    smallest normal 2**-126 the quantum is fixed at 2**-133. Results that
    reach 2**128 overflow to infinity. Returned as float64.
    """
    x = np.asarray(x, dtype=np.float64)
    finite = np.isfinite(x)
    xf = np.where(finite, x, 0.0)
    _, e = np.frexp(xf)
    e = np.maximum(e, -125)
    q = np.ldexp(np.rint(np.ldexp(xf, 8 - e)), e - 8)   # np.rint rounds half to even
    q = np.where(np.abs(q) >= 2.0 ** 128, np.copysign(np.inf, xf), q)
    return np.where(finite, q, x)


# --------------------------------------------------------------------------
# orthogonal reparameterisation  [ABS], [BLOG "How TPLA Works"], [PBOT]
# --------------------------------------------------------------------------

def sylvester_hadamard(n):
    """Unnormalised Sylvester Hadamard matrix of order n (a power of two).

    H_1 = [1];  H_2k = [[H_k, H_k], [H_k, -H_k]]  (natural order).
    """
    if n < 1 or (n & (n - 1)) != 0:
        raise ValueError("Hadamard order must be a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def transform_matrix(transform, L, R_dense=None, g=1):
    """The L x L orthogonal matrix R applied to each new latent before slicing.

    transform 0: identity; 1: Sylvester Hadamard / sqrt(L); 2: the caller's dense
    matrix (the PCA stand-in; a seeded random orthogonal matrix in the tests);
    3: block-diagonal, one Sylvester Hadamard / sqrt(L/g) per shard slice of
    L/g columns, so that each shard's values come from its own slice of the raw
    latent only (a "Hadamard-like" transform cheaper than the full one, the
    pages' named direction for future transforms; the full transform is the
    g = 1 case).
    """
    if transform == TRANSFORM_NONE:
        return np.eye(L)
    if transform == TRANSFORM_HADAMARD:
        return sylvester_hadamard(L) / np.sqrt(L)
    if transform == TRANSFORM_BLOCK_HADAMARD:
        if L % g:
            raise ValueError("L must be divisible by g")
        Ls = L // g
        m = np.zeros((L, L))
        for s in range(g):
            m[s * Ls:(s + 1) * Ls, s * Ls:(s + 1) * Ls] = sylvester_hadamard(Ls) / np.sqrt(Ls)
        return m
    if transform == TRANSFORM_DENSE:
        if R_dense is None:
            raise ValueError("dense transform needs R_dense")
        return np.asarray(R_dense, dtype=np.float64).reshape(L, L)
    raise ValueError("unknown transform %r" % (transform,))


def append_values(latent_raw, g, transform=TRANSFORM_HADAMARD, R_dense=None,
                  norm_weight=None, eps=1e-6):
    """Unrounded cache values of new tokens: transform, then sliced RMSNorm.

    latent_raw: [B, L] pre-norm latent of the new tokens.
    Returns float64 [B, g, L/g]:  y = R x;  c_s = y_s / sqrt(mean(y_s**2) + eps)
    (times norm_weight[s-slice] if given), one RMSNorm per shard s
    ([BLOG "How TPLA Works": RMSNorm slicing after an orthogonal transform]).
    """
    x = np.asarray(latent_raw, dtype=np.float64)
    B, L = x.shape
    if L % g:
        raise ValueError("L must be divisible by g")
    Ls = L // g
    Rm = transform_matrix(transform, L, R_dense, g)
    y = x @ Rm.T                                    # y_b = R x_b
    ys = y.reshape(B, g, Ls)
    ms = np.mean(ys * ys, axis=2, keepdims=True)
    c = ys / np.sqrt(ms + eps)
    if norm_weight is not None:
        c = c * np.asarray(norm_weight, dtype=np.float64).reshape(1, g, Ls)
    return c


def page_of(block_table, b, logical_page, max_pages_per_seq):
    """Physical page holding logical page ``logical_page`` of sequence b.

    block_table None means the identity layout: page = b * max_pages_per_seq + logical_page.
    """
    if block_table is None:
        return b * max_pages_per_seq + logical_page
    return int(np.asarray(block_table)[b, logical_page])


def append_kv(latent_raw, kpe_new, positions, block_table, ckv_cache, kpe_cache, *,
              g, max_pages_per_seq, transform=TRANSFORM_HADAMARD, R_dense=None,
              norm_weight=None, eps=1e-6):
    """Write one new token per sequence into the paged, shard-contiguous cache.

    ckv_cache: [num_pages, g, 64, L/g]; kpe_cache: [num_pages, 64, R] (modified
    in place).  Token b goes to page block_table[b][pos // 64], slot pos % 64,
    for every shard s; k_pe is copied unchanged (it arrives after RoPE).
    """
    c = bf16_round(append_values(latent_raw, g, transform, R_dense, norm_weight, eps))
    kp = np.asarray(kpe_new, dtype=np.float64)
    for b in range(c.shape[0]):
        pos = int(positions[b])
        page = page_of(block_table, b, pos // PAGE_SIZE, max_pages_per_seq)
        slot = pos % PAGE_SIZE
        ckv_cache[page, :, slot, :] = c[b]
        kpe_cache[page, slot, :] = kp[b]
    return ckv_cache, kpe_cache


# --------------------------------------------------------------------------
# decode  [ABS]: per-shard attention, per-shard softmax, sum of shard results
# --------------------------------------------------------------------------

def gather_sequence(ckv_cache, kpe_cache, block_table, b, T, max_pages_per_seq):
    """The first T tokens of sequence b: latent [T, g, Ls] and RoPE key [T, R]."""
    t = np.arange(T)
    pages = np.array([page_of(block_table, b, int(p), max_pages_per_seq)
                      for p in t // PAGE_SIZE], dtype=np.int64).reshape(T)
    slots = t % PAGE_SIZE
    C = np.asarray(ckv_cache, dtype=np.float64)[pages, :, slots, :]
    K = np.asarray(kpe_cache, dtype=np.float64)[pages, slots, :]
    return C, K


def shard_attention(q_s, q_pe, C_s, K_pe, scale):
    """One shard's attention for all heads of one sequence.

    q_s [H, Ls] (the absorbed query slice), q_pe [H, R], C_s [T, Ls], K_pe [T, R].
    Scores z = scale * (q_s C_s^T + q_pe K_pe^T)  (replicated RoPE term);
    p = softmax over tokens (this shard's own softmax); o_s = p C_s.
    Returns (p [H, T], o_s [H, Ls]).
    """
    z = scale * (q_s @ C_s.T + q_pe @ K_pe.T)
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    p = e / e.sum(axis=1, keepdims=True)
    return p, p @ C_s


def decode_latent(q, q_pe, ckv_cache, kpe_cache, block_table, seq_lens, scale, *,
                  max_pages_per_seq, shards=None):
    """Per-shard attention outputs o[b, s] = p_{b,s} C_{b,s}  ->  [B, len(shards), H, Ls].

    q [B, H, L] absorbed queries (already in the transformed basis), q_pe [B, H, R].
    Sequences with seq_len 0 give zeros.
    """
    q = np.asarray(q, dtype=np.float64)
    q_pe = np.asarray(q_pe, dtype=np.float64)
    B, H, L = q.shape
    g = ckv_cache.shape[1]
    Ls = L // g
    shards = list(range(g)) if shards is None else list(shards)
    o = np.zeros((B, len(shards), H, Ls))
    for b in range(B):
        T = int(seq_lens[b])
        if T == 0:
            continue
        C, K = gather_sequence(ckv_cache, kpe_cache, block_table, b, T, max_pages_per_seq)
        for i, s in enumerate(shards):
            _, o[b, i] = shard_attention(q[b, :, s * Ls:(s + 1) * Ls], q_pe[b], C[:, s, :], K, scale)
    return o


def project_shards(o, w_uv, shards):
    """sum_s  W_UV_h[s-rows]^T o_{b,h,s}  ->  [B, H, dv]  (the all-reduce as a sum)."""
    w = np.asarray(w_uv, dtype=np.float64)
    Ls = o.shape[-1]
    out = np.zeros((o.shape[0], o.shape[2], w.shape[2]))
    for i, s in enumerate(shards):
        out += np.einsum('bhl,hld->bhd', o[:, i], w[:, s * Ls:(s + 1) * Ls, :])
    return out


def decode(q, q_pe, ckv_cache, kpe_cache, block_table, seq_lens, scale, *,
           max_pages_per_seq, w_uv=None):
    """TPLA decode over all g shards.

    With w_uv [H, L, dv]: out [B, H, dv] = sum over shards of the shard's
    up-projected output.  Without: the latent outputs concatenated over
    shards, [B, H, L].  With g = 1 this is MLA decode in absorbed form.
    """
    g = ckv_cache.shape[1]
    o = decode_latent(q, q_pe, ckv_cache, kpe_cache, block_table, seq_lens, scale,
                      max_pages_per_seq=max_pages_per_seq)
    if w_uv is None:
        return np.concatenate([o[:, s] for s in range(g)], axis=2)
    return project_shards(o, w_uv, list(range(g)))


def decode_shard(q, q_pe, ckv_cache, kpe_cache, block_table, seq_lens, scale, shard, *,
                 max_pages_per_seq, w_uv=None):
    """The work of one tensor-parallel rank: shard ``shard`` only.

    With w_uv: that shard's term W_UV[s-rows]^T o_s, [B, H, dv] (the input of
    the all-reduce).  Without: o_s, [B, H, L/g].
    """
    o = decode_latent(q, q_pe, ckv_cache, kpe_cache, block_table, seq_lens, scale,
                      max_pages_per_seq=max_pages_per_seq, shards=[shard])
    if w_uv is None:
        return o[:, 0]
    return project_shards(o, w_uv, [shard])


def gla_decode(q, q_pe, ckv_cache, kpe_cache, block_table, seq_lens, scale, *, max_pages_per_seq, w_uv=None):
    """GLA-style decode, the contrast the edgentiq blog draws in "Introducing TPLA": heads are split
    into g groups as well as the latent, and head group s (heads s*H/g .. (s+1)*H/g - 1) attends to
    latent shard s only, with no sum over shards.  Per head h of group s:
    z_t = scale * (q~_h[s-slice] . c_{t,s} + q_pe_h . k_pe_t), o = softmax(z) C_s, and
    out_h = W_UV_h[s-rows]^T o (or o itself without w_uv: [B, H, L/g]).  H must be a multiple of g.
    """
    q = np.asarray(q, dtype=np.float64)
    q_pe = np.asarray(q_pe, dtype=np.float64)
    B, H, L = q.shape
    g = ckv_cache.shape[1]
    if H % g:
        raise ValueError("H must be a multiple of g")
    Ls, Hg = L // g, H // g
    w = None if w_uv is None else np.asarray(w_uv, dtype=np.float64)
    out = np.zeros((B, H, Ls if w is None else w.shape[2]))
    for b in range(B):
        T = int(seq_lens[b])
        if T == 0:
            continue
        C, K = gather_sequence(ckv_cache, kpe_cache, block_table, b, T, max_pages_per_seq)
        for s in range(g):
            heads = slice(s * Hg, (s + 1) * Hg)
            _, o = shard_attention(q[b, heads, s * Ls:(s + 1) * Ls], q_pe[b, heads], C[:, s, :], K, scale)
            out[b, heads] = o if w is None else np.einsum('hl,hld->hd', o, w[heads, s * Ls:(s + 1) * Ls, :])
    return out


def mla_prefill(latent_raw, kpe_new, q, q_pe, scale, *, transform=TRANSFORM_HADAMARD, R_dense=None,
                norm_weight=None, eps=1e-6, w_uv=None):
    """Prefill of one prompt in MLA form ([BLOG] "Prefill-Decode Separation": prefill keeps MLA, decode uses
    TPLA): every head attends over the whole latent, normalised by one RMSNorm over all L columns.

    latent_raw [T, L] pre-norm latents and kpe_new [T, R] RoPE keys of the prompt's tokens; q [T, H, L]
    absorbed queries and q_pe [T, H, R], all in the transformed basis.  The latent rows are the g = 1
    append rounded like the cache, c_i = bf16(R x_i / sqrt(mean((R x_i)^2) + eps)); token t attends
    causally: z_i = scale * (q~_t . c_i + q_pe_t . k_pe_i) for i <= t, o_t = softmax(z) C, and
    out_t = W_UV^T o_t (o_t itself without w_uv).  Returns [T, H, dv] or [T, H, L].
    """
    c = bf16_round(append_values(latent_raw, 1, transform, R_dense, norm_weight, eps))[:, 0, :]   # [T, L]
    K = np.asarray(kpe_new, dtype=np.float64)
    q = np.asarray(q, dtype=np.float64)
    q_pe = np.asarray(q_pe, dtype=np.float64)
    T, H, L = q.shape
    w = None if w_uv is None else np.asarray(w_uv, dtype=np.float64)
    out = np.zeros((T, H, L if w is None else w.shape[2]))
    for t in range(T):
        _, o = shard_attention(q[t], q_pe[t], c[:t + 1], K[:t + 1], scale)
        out[t] = o if w is None else np.einsum('hl,hld->hd', o, w)
    return out


def shard_probabilities(q, q_pe, ckv_cache, kpe_cache, block_table, seq_lens, scale, b, s, *,
                        max_pages_per_seq):
    """Softmax weights p [H, T_b] of sequence b on shard s (for invariant checks)."""
    q = np.asarray(q, dtype=np.float64)
    g = ckv_cache.shape[1]
    Ls = q.shape[2] // g
    T = int(seq_lens[b])
    C, K = gather_sequence(ckv_cache, kpe_cache, block_table, b, T, max_pages_per_seq)
    p, _ = shard_attention(q[b, :, s * Ls:(s + 1) * Ls], np.asarray(q_pe, dtype=np.float64)[b],
                           C[:, s, :], K, scale)
    return p


# --------------------------------------------------------------------------
# explicit (non-absorbed) MLA, the g = 1 reference  [ABS]: TPLA is drop-in for MLA
# --------------------------------------------------------------------------

def mla_nonabsorbed(q_nope, q_pe, latent, kpe, w_uk, w_uv, scale, seq_lens):
    """Ordinary multi-head attention with per-head keys and values rebuilt from the latent.

    q_nope [B, H, dn], q_pe [B, H, R], latent [B, T, L], kpe [B, T, R],
    w_uk [H, L, dn], w_uv [H, L, dv].  For head h and token t:
    k_t = [w_uk_h^T c_t ; kpe_t], v_t = w_uv_h^T c_t, q = [q_nope_h ; q_pe_h].
    Returns [B, H, dv].
    """
    q_nope = np.asarray(q_nope, dtype=np.float64)
    q_pe = np.asarray(q_pe, dtype=np.float64)
    latent = np.asarray(latent, dtype=np.float64)
    kpe = np.asarray(kpe, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    w_uv = np.asarray(w_uv, dtype=np.float64)
    B, H, _ = q_nope.shape
    out = np.zeros((B, H, w_uv.shape[2]))
    for b in range(B):
        T = int(seq_lens[b])
        if T == 0:
            continue
        c = latent[b, :T]
        for h in range(H):
            k_nope = c @ w_uk[h]                  # [T, dn]
            v = c @ w_uv[h]                       # [T, dv]
            z = scale * (k_nope @ q_nope[b, h] + kpe[b, :T] @ q_pe[b, h])
            z = z - z.max()
            p = np.exp(z)
            p = p / p.sum()
            out[b, h] = p @ v
    return out


def absorb_query(q_nope, w_uk):
    """q~_{b,h} = w_uk_h q_nope_{b,h}  ([B, H, L]): the query in latent space."""
    return np.einsum('hld,bhd->bhl', np.asarray(w_uk, dtype=np.float64),
                     np.asarray(q_nope, dtype=np.float64))
