"""Helpers for the GPU parity tests: run the C ABI on seeded inputs and the
float64 oracle on the same bf16 values, and compare them."""

import numpy as np
import torch

from oracle import tpla_ref as ref
from latent_attention_decode_tpla_b200 import inputs as gen
from latent_attention_decode_tpla_b200 import tpla

# Tolerances on fp32 outputs (bf16 inputs, fp32 accumulation).
MAX_ABS = 2e-2
REL_RMS = 1e-3

KERNELS = {"simt": 1, "sm100": 2}
# kernels reported by TPLA_OPT_LAST_ATTENTION_KERNEL for each forced choice: the tcgen05 choice runs
# the 128-token-tile kernel (2) for L/g <= 256 and the CTA-pair kernel (3) for L/g = 512
RAN = {"simt": (1,), "sm100": (2, 3)}


class tile_tokens:
    """Context manager: tokens per tile of the tcgen05 kernel for L/g <= 256 (64, 128; 0 = default)."""

    def __init__(self, tokens):
        self.tokens = tokens

    def __enter__(self):
        self.old = tpla.get_option(tpla.OPT_TILE_TOKENS)
        tpla.set_option(tpla.OPT_TILE_TOKENS, self.tokens)
        return self

    def __exit__(self, *exc):
        tpla.set_option(tpla.OPT_TILE_TOKENS, self.old)
        return False


def to64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


def oracle_fill_cache(d, transform, R_dense=None, eps=1e-6):
    """Fill d['ckv'] (CPU) by the oracle's append of every cached token's raw latent d['x_all']."""
    B, g, Ls = d["B"], d["g"], d["Ls"]
    ckv = to64(d["ckv"])
    bt = d["block_table"].numpy()
    Rd = None if R_dense is None else R_dense.numpy().astype(np.float64)
    for b in range(B):
        T = int(d["seq_lens"][b])
        if T == 0:
            continue
        x = to64(d["x_all"][b, :T])
        c = ref.bf16_round(ref.append_values(x, g, transform, Rd, None, eps))   # [T, g, Ls]
        t = np.arange(T)
        ckv[bt[b, t // 64], :, t % 64, :] = c
    d["ckv"] = torch.from_numpy(ckv).to(torch.bfloat16)
    return d


def dims_of(d, scale, B=None):
    return tpla.make_dims(B=d["B"] if B is None else B, H=d["H"], L=d["L"], R=d["R"], dv=d["dv"], g=d["g"],
                          max_pages_per_seq=d["max_pages_per_seq"], num_pages=d["num_pages"],
                          softmax_scale=scale)


def to_device(d):
    keys = ("q", "q_pe", "ckv", "kpe", "block_table", "seq_lens", "w_uv", "x_new", "kpe_new")
    return {k: d[k].cuda() for k in keys if k in d}


def run_gpu(d, scale, mode="full", shard=0, with_wuv=True, dev=None, block_table=True, kernel=None):
    """Decode through the C ABI; returns the fp32 output as float64 numpy.

    mode: "full" (tpla_decode), "shard" (tpla_decode_shard), "mla" (mla_decode).
    """
    dev = dev or to_device(d)
    dims = dims_of(d, scale)
    B, H, L, dv, g = d["B"], d["H"], d["L"], d["dv"], d["g"]
    cols = dv if with_wuv else (L if mode != "shard" else L // g)
    out = torch.full((B, H, cols), float("nan"), dtype=torch.float32, device="cuda")
    ws = tpla.alloc_workspace(dims)
    w = dev["w_uv"] if with_wuv else None
    bt = dev["block_table"] if block_table else None
    old = tpla.get_option(tpla.OPT_ATTENTION_KERNEL)
    if kernel is not None:
        tpla.set_option(tpla.OPT_ATTENTION_KERNEL, KERNELS[kernel])
    try:
        if mode == "full":
            tpla.decode(dims, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], bt, dev["seq_lens"], w, out, ws)
        elif mode == "shard":
            tpla.decode_shard(dims, shard, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], bt, dev["seq_lens"],
                              w, out, ws)
        elif mode == "mla":
            tpla.mla_decode(dims, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], bt, dev["seq_lens"], w, out, ws)
        else:
            raise ValueError(mode)
        used = tpla.get_option(tpla.OPT_LAST_ATTENTION_KERNEL)
    finally:
        tpla.set_option(tpla.OPT_ATTENTION_KERNEL, old)
    torch.cuda.synchronize()
    assert tpla.check_device_status() == tpla.TPLA_OK
    if kernel is not None:
        assert used in RAN[kernel], "asked for %s, ran kernel %d" % (kernel, used)
    return to64(out)


def run_oracle(d, scale, mode="full", shard=0, with_wuv=True, batch=None):
    """Oracle output for all sequences, or for the sequences in ``batch`` (rows in that order)."""
    idx = list(range(d["B"])) if batch is None else list(batch)
    sub_lens = [int(d["seq_lens"][b]) for b in idx]
    q = to64(d["q"][idx])
    q_pe = to64(d["q_pe"][idx])
    bt = d["block_table"].numpy()[idx]
    ckv = d["ckv"]
    kpe = d["kpe"]
    # gather only the pages these sequences use, so huge caches are not converted whole
    used = np.unique(np.concatenate([bt[i, :gen.pages_for(n)] for i, n in enumerate(sub_lens)] + [[0]]))
    remap = np.zeros(d["num_pages"], dtype=np.int64)
    remap[used] = np.arange(len(used))
    ckv_s = ckv[torch.from_numpy(used)].to(torch.float64).numpy()
    kpe_s = kpe[torch.from_numpy(used)].to(torch.float64).numpy()
    bt_s = remap[bt]
    w = to64(d["w_uv"]) if with_wuv else None
    kw = dict(max_pages_per_seq=d["max_pages_per_seq"], w_uv=w)
    if mode == "shard":
        return ref.decode_shard(q, q_pe, ckv_s, kpe_s, bt_s, sub_lens, scale, shard, **kw)
    return ref.decode(q, q_pe, ckv_s, kpe_s, bt_s, sub_lens, scale, **kw)


def errors(got, want):
    diff = got - want
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.sqrt(np.sum(want * want)))
    rel = float(np.sqrt(np.sum(diff * diff)) / den) if den > 0 else float(np.sqrt(np.sum(diff * diff)))
    return max_abs, rel


def assert_close(got, want, what="", max_abs=MAX_ABS, rel_rms=REL_RMS):
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), what + ": non-finite output"
    ma, rr = errors(got, want)
    assert ma <= max_abs and rr <= rel_rms, "%s: max-abs %.3g (<= %.3g), rel-RMS %.3g (<= %.3g)" % (
        what, ma, max_abs, rr, rel_rms)
    return ma, rr


def sm100_available(d):
    """True if the tcgen05 kernel serves this shape (forced-kernel calls return UNSUPPORTED otherwise)."""
    dims = dims_of(d, 0.1)
    old = tpla.get_option(tpla.OPT_ATTENTION_KERNEL)
    tpla.set_option(tpla.OPT_ATTENTION_KERNEL, 2)
    try:
        dev = {k: torch.zeros(16, dtype=torch.bfloat16, device="cuda") for k in ("q", "q_pe", "ckv", "kpe")}
        lens = torch.zeros(d["B"], dtype=torch.int32, device="cuda")    # all empty: no work launched
        ws = tpla.alloc_workspace(dims)
        try:
            tpla.attention(dims, -1, dev["q"], dev["q_pe"], dev["ckv"], dev["kpe"], None, lens, ws)
        except tpla.TplaError as e:
            if e.status == tpla.TPLA_ERR_UNSUPPORTED:
                return False
            raise
        torch.cuda.synchronize()
        return True
    finally:
        tpla.set_option(tpla.OPT_ATTENTION_KERNEL, old)
