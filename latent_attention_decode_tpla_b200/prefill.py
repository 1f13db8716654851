"""MLA-form prefill of one prompt, handing the cache off to TPLA decode.

edgentiq blog, "Prefill-Decode Separation for Optimal Performance": prefill keeps the MLA form (every head
attends over the whole latent, normalised by one RMSNorm over all of it), while decode uses TPLA over the
sliced cache.  ``mla_prefill`` runs, on the library's kernels:

1. ``tpla_append_kv`` with one shard into a scratch cache: the prompt's latent rows R x / rms(R x);
2. ``mla_decode`` over that cache for every prompt token t, as a batch of sequences of lengths t + 1
   sharing the prompt's pages (causal attention), in chunks of ``chunk`` tokens that bound the split-KV
   workspace;
3. ``tpla_append_kv`` with the model's g shards into the caller's paged cache at positions 0 .. T-1
   (transform, per-shard RMSNorm), from which decode continues.

Step 2 computes MLA attention in its absorbed form on tensor cores (the one-shard kernel); it reads each
prompt page once per later query token, mostly from L2, and does the absorbed form's FLOPs, so it is a
correct prefill, not a compute-optimal one (that is a flash-attention kernel over the decompressed keys and
values).  This module only creates index tensors and calls the library.
"""

import torch

from . import tpla


def mla_prefill(dims, latent_raw, kpe_new, q, q_pe, w_uv, transform, R_dense, norm_weight, eps, block_table_row,
                ckv_cache, kpe_cache, out, chunk=64, stream=None):
    """Prefill one prompt of T tokens.

    dims: the model's dims (H, L, R, dv, g, softmax_scale, and the paged cache's max_pages_per_seq and
    num_pages; B is not used).  latent_raw [T, L] and kpe_new [T, R] bf16: the prompt's pre-norm latents
    and RoPE keys; q [T, H, L] and q_pe [T, H, R] bf16: its absorbed queries in the transformed basis;
    w_uv [H, L, dv] bf16 or None; transform, R_dense, norm_weight, eps as for tpla_append_kv;
    block_table_row [max_pages_per_seq] int32: the sequence's pages in ``ckv_cache`` [num_pages, g, 64, L/g]
    and ``kpe_cache`` [num_pages, 64, R], which receive the prompt; out [T, H, dv] fp32 (or [T, H, L]
    without w_uv).  Returns ``out``.
    """
    T = latent_raw.shape[0]
    if T == 0:
        return out
    if chunk < 1:
        raise ValueError("chunk must be positive")
    if T > dims.max_pages_per_seq * tpla.PAGE_SIZE:
        raise ValueError("the prompt does not fit the sequence's pages")
    dev = latent_raw.device
    npg = (T + tpla.PAGE_SIZE - 1) // tpla.PAGE_SIZE
    common = dict(H=dims.H, L=dims.L, R=dims.R, dv=dims.dv, softmax_scale=dims.softmax_scale)
    pos = torch.arange(T, dtype=torch.int32, device=dev)

    # 1. the prompt's unsliced latent rows in a scratch one-shard cache (pages 0 .. npg-1)
    c1 = torch.empty((npg, 1, tpla.PAGE_SIZE, dims.L), dtype=torch.bfloat16, device=dev)
    k1 = torch.empty((npg, tpla.PAGE_SIZE, dims.R), dtype=torch.bfloat16, device=dev)
    rows1 = torch.arange(npg, dtype=torch.int32, device=dev).expand(T, npg).contiguous()
    tpla.append_kv(tpla.make_dims(B=T, g=1, max_pages_per_seq=npg, num_pages=npg, **common), latent_raw, kpe_new,
                   transform, R_dense, norm_weight, eps, pos, rows1, c1, k1, stream)

    # 2. causal MLA attention: token t is a sequence of length t + 1 over those pages
    cmax = min(chunk, T)
    ws = tpla.alloc_workspace(tpla.make_dims(B=cmax, g=1, max_pages_per_seq=npg, num_pages=npg, **common), dev)
    for t0 in range(0, T, cmax):
        c = min(cmax, T - t0)
        lens = torch.arange(t0 + 1, t0 + c + 1, dtype=torch.int32, device=dev)
        tpla.mla_decode(tpla.make_dims(B=c, g=1, max_pages_per_seq=npg, num_pages=npg, **common),
                        q[t0:t0 + c], q_pe[t0:t0 + c], c1, k1, rows1[:c], lens, w_uv, out[t0:t0 + c], ws, stream)

    # 3. the g-shard cache that decode reads
    rows = block_table_row.reshape(1, -1).expand(T, -1).contiguous()
    tpla.append_kv(tpla.make_dims(B=T, g=dims.g, max_pages_per_seq=dims.max_pages_per_seq, num_pages=dims.num_pages,
                                  **common),
                   latent_raw, kpe_new, transform, R_dense, norm_weight, eps, pos, rows, ckv_cache, kpe_cache, stream)
    return out
