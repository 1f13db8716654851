"""Tensor-parallel decode on the GPU: each rank's kernels, and the whole rank module over gloo.

Rank s appends its slice of every token into a one-shard cache (tpla_append_kv_shard) and decodes it
with tpla_decode at latent width L/g; the sum of the ranks' terms is TPLA's output (TPLA paper,
Abstract: shard results are combined by an all-reduce).  The first test runs the ranks one after the
other in one process (one GPU is all a test gets here) and checks the one-shard caches bit for bit
against the g-shard append, each term against the oracle's per-shard decode and their sum against
the oracle's decode.  The second runs two ranks as two processes on the same GPU through
latent_attention_decode_tpla_b200.tp, with gloo carrying the all-reduce (the kernels of one rank never
wait on another's).
"""

import math
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import gpu_harness as hx
from oracle import tpla_ref as ref
from latent_attention_decode_tpla_b200 import inputs as gen
from latent_attention_decode_tpla_b200 import tp, tpla

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _virtual_batch(d):
    """Every cached token of every sequence as one append call: token i of sequence b is entry
    (b, i) of a batch whose page-table rows repeat sequence b's row."""
    lens = [int(t) for t in d["seq_lens"]]
    bt = d["block_table"]
    rows, pos, x, kp = [], [], [], []
    for b, T in enumerate(lens):
        for i in range(T):
            rows.append(bt[b])
            pos.append(i)
            x.append(d["x_all"][b, i])
            kp.append(d["kpe"][bt[b, i // 64], i % 64])
    return (torch.stack(rows).contiguous(), torch.tensor(pos, dtype=torch.int32), torch.stack(x).contiguous(),
            torch.stack(kp).contiguous())


def _fill(d, g, transform, R_dense):
    """g-shard cache and the g one-shard caches, all written on the GPU from the same raw latents."""
    bt_v, pos_v, x_v, kp_v = (t.cuda() for t in _virtual_batch(d))
    dims_v = tpla.make_dims(B=len(pos_v), H=d["H"], L=d["L"], R=d["R"], dv=d["dv"], g=g,
                            max_pages_per_seq=d["max_pages_per_seq"], num_pages=d["num_pages"], softmax_scale=1.0)
    P, Ls = d["num_pages"], d["L"] // g
    ckv = torch.zeros((P, g, 64, Ls), dtype=torch.bfloat16, device="cuda")
    kpe = torch.zeros((P, 64, d["R"]), dtype=torch.bfloat16, device="cuda")
    tpla.append_kv(dims_v, x_v, kp_v, transform, R_dense, None, 1e-6, pos_v, bt_v, ckv, kpe)
    ranks = []
    for s in range(g):
        c = torch.full((P, 64, Ls), -7.0, dtype=torch.bfloat16, device="cuda")     # unwritten slots keep -7
        k = torch.zeros_like(kpe)
        tpla.append_kv_shard(dims_v, s, x_v, kp_v, transform, R_dense, None, 1e-6, pos_v, bt_v, c, k)
        ranks.append((c, k))
    torch.cuda.synchronize()
    assert tpla.check_device_status() == tpla.TPLA_OK
    return ckv, kpe, ranks


@pytest.mark.parametrize("g,H,transform", [
    (2, 128, ref.TRANSFORM_HADAMARD), (4, 64, ref.TRANSFORM_DENSE), (2, 128, ref.TRANSFORM_BLOCK_HADAMARD),
])
def test_rank_kernels_sum_to_tpla(g, H, transform):
    lens = [300, 70, 129]
    d = gen.make_workload(B=3, H=H, L=512, R=64, dv=128, g=g, seq_lens=lens, seed=41 + g, extra_pages=2,
                          cache_values="none")
    R_dense = gen.random_orthogonal(512, 41).cuda() if transform == ref.TRANSFORM_DENSE else None
    ckv, kpe, ranks = _fill(d, g, transform, R_dense)
    used = torch.zeros(d["num_pages"], 64, dtype=torch.bool)
    for b, T in enumerate(lens):
        for i in range(T):
            used[d["block_table"][b, i // 64], i % 64] = True
    for s, (c, k) in enumerate(ranks):
        # the rank's cache holds exactly shard s of the g-shard append in the written slots
        got, want = c.cpu(), ckv[:, s].cpu()
        assert torch.equal(got[used].view(torch.int16), want[used].view(torch.int16))
        assert torch.all(got[~used] == -7.0)
        assert torch.equal(k.cpu()[used].view(torch.int16), kpe.cpu()[used].view(torch.int16))
    scale = 1 / math.sqrt(192)
    dims = hx.dims_of(d, scale)
    local = tp.rank_dims(dims)
    q, q_pe, w = d["q"].cuda(), d["q_pe"].cuda(), d["w_uv"].cuda()
    bt, sl = d["block_table"].cuda(), d["seq_lens"].cuda()
    d_or = dict(d, ckv=ckv.cpu(), kpe=kpe.cpu())
    total = torch.zeros(3, H, 128, dtype=torch.float32, device="cuda")
    for s, (c, k) in enumerate(ranks):
        out = torch.full((3, H, 128), float("nan"), dtype=torch.float32, device="cuda")
        tpla.decode(local, tp.query_slice(q, g, s), q_pe, c, k, bt, sl, tp.w_uv_rows(w, g, s), out,
                    tpla.alloc_workspace(local))
        torch.cuda.synchronize()
        assert tpla.check_device_status() == tpla.TPLA_OK
        hx.assert_close(hx.to64(out), hx.run_oracle(d_or, scale, mode="shard", shard=s), "rank %d term" % s)
        total += out
    hx.assert_close(hx.to64(total), hx.run_oracle(d_or, scale), "sum of the rank terms")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_process(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    import gpu_harness as h
    from latent_attention_decode_tpla_b200 import inputs as gen
    from latent_attention_decode_tpla_b200 import tp, tpla
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lens = [200, 65, 1]
        d = gen.make_workload(B=3, H=128, L=512, R=64, dv=128, g=world, seq_lens=lens, seed=5, extra_pages=1,
                              cache_values="none")
        scale = 1 / math.sqrt(192)
        dims = h.dims_of(d, scale)
        r = tp.TensorParallelDecode(dims)
        bt_v, pos_v, x_v, kp_v = (t.cuda() for t in _virtual_batch(d))
        dims_v = tpla.make_dims(B=len(pos_v), H=128, L=512, R=64, dv=128, g=world,
                                max_pages_per_seq=d["max_pages_per_seq"], num_pages=d["num_pages"], softmax_scale=1.0)
        c = torch.zeros((d["num_pages"], 64, 512 // world), dtype=torch.bfloat16, device="cuda")
        k = torch.zeros((d["num_pages"], 64, 64), dtype=torch.bfloat16, device="cuda")
        tp.TensorParallelDecode(dims_v).append(x_v, kp_v, tpla.TRANSFORM_HADAMARD, None, None, 1e-6, pos_v, bt_v, c, k)
        out = torch.empty(3, 128, 128, dtype=torch.float32, device="cuda")
        r.decode(tp.query_slice(d["q"].cuda(), world, rank), d["q_pe"].cuda(), c, k, d["block_table"].cuda(),
                 d["seq_lens"].cuda(), tp.w_uv_rows(d["w_uv"].cuda(), world, rank), out, r.workspace())
        torch.cuda.synchronize()
        ok = tpla.check_device_status() == tpla.TPLA_OK
        # the oracle's whole decode on the g-shard cache built from the same raw latents
        h.oracle_fill_cache(d, tpla.TRANSFORM_HADAMARD)
        ma, rr = h.errors(h.to64(out), h.run_oracle(d, scale))
        results.put((rank, ok, ma, rr))
    finally:
        dist.destroy_process_group()


def test_two_ranks_over_gloo_on_one_gpu():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_process, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, ok, ma, rr in res:
        assert ok, rank
        assert ma <= hx.MAX_ABS and rr <= hx.REL_RMS, (rank, ma, rr)
