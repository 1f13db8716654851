"""GLA-style decode on the library's kernels, the contrast the TPLA pages draw.

edgentiq blog, "Introducing TPLA": GLA splits the heads into g groups along with the latent, so a
head of group s sees latent shard s only, while TPLA lets every head see every shard (one softmax
per shard, shard results summed).  For head h of group s, GLA's output is TPLA's shard-s term for
that head, without the other shards' terms.  Both read the same cache bytes per shard; GLA computes
H/g heads per shard instead of H.

gla_decode runs, for each group s, the library's tpla_decode_shard on that group's heads alone
(their query rows, RoPE query rows and W_UV rows as dense tensors) and places the result in the
group's rows of ``out``.  This module only slices and copies tensors; the attention, its softmax and
the W_UV projection run in the library's kernels.
"""

import torch

from . import tpla


def group_dims(dims):
    """Dims of one head group: H/g heads, the same g-shard cache."""
    if dims.H % dims.g:
        raise ValueError("H must be a multiple of g for GLA-style head groups")
    return tpla.make_dims(B=dims.B, H=dims.H // dims.g, L=dims.L, R=dims.R, dv=dims.dv, g=dims.g,
                          max_pages_per_seq=dims.max_pages_per_seq, num_pages=dims.num_pages,
                          softmax_scale=dims.softmax_scale, page_size=dims.page_size)


def gla_decode(dims, q, q_pe, ckv, kpe, block_table, seq_lens, w_uv, out, workspace=None, stream=None):
    """GLA-style decode into ``out``: [B, H, dv] fp32 with w_uv, else [B, H, L/g] (each head's latent
    output over its group's shard).  Arguments as tpla.decode; H a multiple of g."""
    gd = group_dims(dims)
    hg = gd.H
    ws = workspace if workspace is not None else tpla.alloc_workspace(gd)
    cols = out.shape[-1]
    part = torch.empty((dims.B, hg, cols), dtype=torch.float32, device=out.device)
    for s in range(dims.g):
        heads = slice(s * hg, (s + 1) * hg)
        tpla.decode_shard(gd, s, q[:, heads].contiguous(), q_pe[:, heads].contiguous(), ckv, kpe, block_table,
                          seq_lens, None if w_uv is None else w_uv[heads], part, ws, stream)
        out[:, heads] = part
    return out
