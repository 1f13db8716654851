"""Tensor-parallel TPLA decode: one process per GPU, latent shard s on rank s.

What the pages describe (TPLA paper, Abstract; edgentiq blog "Introducing TPLA"): the latent cKV
and each head's absorbed query are cut into g shards; device s keeps shard s of the latent cache
(and the RoPE key), runs attention over its shard with its own softmax, up-projects with its rows
of W_UV, and the devices add their outputs with an all-reduce.

Each rank's work is the library's own kernels on its slice: ``tpla_append_kv_shard`` writes the
rank's slice of every new token into its one-shard cache, and ``tpla_decode`` on dims with latent
width L/g and one shard (the rank's query slice and W_UV rows) gives the rank's term; the sum of
the terms is ``tpla_decode``'s result on the g-shard cache.  ``torch.distributed.all_reduce``
(NCCL between GPUs) adds the terms.  This module only marshals arguments and calls the collective.
"""

import torch
import torch.distributed as dist

from . import tpla


def rank_dims(dims):
    """Dims of one rank's decode: latent width L/g, one shard (the rest as ``dims``)."""
    if dims.L % dims.g:
        raise ValueError("L must be divisible by g")
    return tpla.make_dims(B=dims.B, H=dims.H, L=dims.L // dims.g, R=dims.R, dv=dims.dv, g=1,
                          max_pages_per_seq=dims.max_pages_per_seq, num_pages=dims.num_pages,
                          softmax_scale=dims.softmax_scale, page_size=dims.page_size)


def query_slice(q, g, shard):
    """Rank ``shard``'s columns of the absorbed query [B, H, L] as a dense [B, H, L/g] tensor."""
    ls = q.shape[-1] // g
    return q[..., shard * ls:(shard + 1) * ls].contiguous()


def w_uv_rows(w_uv, g, shard):
    """Rank ``shard``'s rows of W_UV [H, L, dv] as a dense [H, L/g, dv] tensor."""
    ls = w_uv.shape[1] // g
    return w_uv[:, shard * ls:(shard + 1) * ls, :].contiguous()


def cache_slice(ckv, shard):
    """Rank ``shard``'s slice of a g-shard cache [P, g, 64, L/g] as a one-shard cache [P, 64, L/g]."""
    return ckv[:, shard].contiguous()


class TensorParallelDecode:
    """One rank of TPLA decode at TP degree g = the process group's size (shard = rank).

    dims: the model's dims (L the full latent width, g the TP degree).  Per rank the caller holds
    a one-shard latent cache [num_pages, 64, L/g], the RoPE cache [num_pages, 64, R], its query
    slice [B, H, L/g] (``query_slice``) and its W_UV rows [H, L/g, dv] (``w_uv_rows``).
    """

    def __init__(self, dims, group=None):
        self.group = group
        initialized = dist.is_available() and dist.is_initialized()
        self.rank = dist.get_rank(group) if initialized else 0
        self.world = dist.get_world_size(group) if initialized else 1
        if dims.g != self.world:
            raise ValueError("the TP degree g (%d) must equal the process group's size (%d)" % (dims.g, self.world))
        self.dims = dims
        self.shard = self.rank
        self.local = rank_dims(dims)

    def workspace(self, device=None):
        return tpla.alloc_workspace(self.local, device)

    def append(self, latent_raw, kpe_new, transform, R_dense, norm_weight, eps, positions, block_table,
               ckv_local, kpe, stream=None):
        """This rank's slice of one new token per sequence (the whole raw latent goes in: the
        transform mixes all of it) into its one-shard cache."""
        tpla.append_kv_shard(self.dims, self.shard, latent_raw, kpe_new, transform, R_dense, norm_weight, eps,
                             positions, block_table, ckv_local, kpe, stream)

    def decode(self, q_local, q_pe, ckv_local, kpe, block_table, seq_lens, w_uv_local, out, workspace,
               stream=None, reduce=True):
        """This rank's term W_UV[shard rows]^T o_shard into ``out`` [B, H, dv] fp32, then (reduce=True)
        the all-reduce that leaves the sum over all ranks (the whole TPLA output) in every rank."""
        tpla.decode(self.local, q_local, q_pe, ckv_local, kpe, block_table, seq_lens, w_uv_local, out, workspace,
                    stream)
        if reduce and self.world > 1:
            all_reduce_terms(out, self.group, stream)
        return out


def all_reduce_terms(out, group=None, stream=None):
    """Sum the ranks' output terms in place (the all-reduce of the TPLA pages), on ``stream``."""
    if stream is not None and out.is_cuda:
        with torch.cuda.stream(stream):
            dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    else:
        dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)
    return out
