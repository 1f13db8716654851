"""Tensor-parallel decode on CPU: two ranks over gloo, the oracle standing in for each rank's kernels.

Rank s holds shard s of the latent cache as a one-shard cache, its columns of the absorbed query and
its rows of W_UV; its term is attention over that slice alone, and the all-reduce of the terms is
TPLA's output (TPLA paper, Abstract: shard results are combined by an all-reduce).  This checks the
slicing helpers and the reduction of latent_attention_decode_tpla_b200.tp against the oracle's whole
decode; the kernels of each rank are checked on the GPU (test_tp_gpu.py).
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from oracle import tpla_ref as ref
    from latent_attention_decode_tpla_b200 import inputs as gen
    from latent_attention_decode_tpla_b200 import tp, tpla
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = world
        d = gen.make_workload(B=3, H=4, L=32, R=8, dv=6, g=g, seq_lens=[1, 70, 130], seed=13)
        f64 = lambda t: t.to(torch.float64)
        scale = 0.41
        # this rank's slices (the helpers of the TP module)
        q_local = tp.query_slice(f64(d["q"]), g, rank)
        w_local = tp.w_uv_rows(f64(d["w_uv"]), g, rank)
        c_local = tp.cache_slice(f64(d["ckv"]), rank)            # [P, 64, L/g]
        dims = tpla.make_dims(B=3, H=4, L=32, R=8, dv=6, g=g, max_pages_per_seq=d["max_pages_per_seq"],
                              num_pages=d["num_pages"], softmax_scale=scale)
        local = tp.rank_dims(dims)
        assert (local.L, local.g, local.H, local.num_pages) == (32 // g, 1, 4, d["num_pages"])
        # the rank's term: attention over its slice alone (the oracle in place of the rank's kernels)
        kw = dict(max_pages_per_seq=d["max_pages_per_seq"])
        term = ref.decode(q_local.numpy(), f64(d["q_pe"]).numpy(), c_local[:, None].numpy(), f64(d["kpe"]).numpy(),
                          d["block_table"].numpy(), d["seq_lens"].numpy(), scale, w_uv=w_local.numpy(), **kw)
        shard_term = ref.decode_shard(f64(d["q"]).numpy(), f64(d["q_pe"]).numpy(), f64(d["ckv"]).numpy(),
                                      f64(d["kpe"]).numpy(), d["block_table"].numpy(), d["seq_lens"].numpy(), scale,
                                      rank, w_uv=f64(d["w_uv"]).numpy(), **kw)
        np.testing.assert_allclose(term, shard_term, rtol=0, atol=1e-13)
        out = torch.from_numpy(term.copy())
        tp.all_reduce_terms(out)
        full = ref.decode(f64(d["q"]).numpy(), f64(d["q_pe"]).numpy(), f64(d["ckv"]).numpy(), f64(d["kpe"]).numpy(),
                          d["block_table"].numpy(), d["seq_lens"].numpy(), scale, w_uv=f64(d["w_uv"]).numpy(), **kw)
        err = float(np.max(np.abs(out.numpy() - full)))
        # the module refuses a TP degree other than the group's size
        bad = tpla.make_dims(B=3, H=4, L=32, R=8, dv=6, g=2 * g, max_pages_per_seq=2, num_pages=8,
                             softmax_scale=scale)
        try:
            tp.TensorParallelDecode(bad)
            refused = False
        except ValueError:
            refused = True
        r = tp.TensorParallelDecode(dims)
        item = (rank, err, refused, r.shard, r.world)
    finally:
        dist.destroy_process_group()
    results.put(item)


@pytest.mark.parametrize("world", [2, 4])
def test_tp_terms_sum_to_tpla_over_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, refused, shard, w in res:
        assert err < 1e-12, (rank, err)
        assert refused and shard == rank and w == world
