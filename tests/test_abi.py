"""The C ABI without a GPU: the library loads, exports what include/tpla.h
declares, sizes workspaces on the host, and rejects bad arguments before any
CUDA call (so these calls never touch a device, with or without a GPU)."""

import ctypes
import os
import re

import pytest

from latent_attention_decode_tpla_b200 import tpla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tpla.h")

# fake, 16-byte aligned addresses: only ever passed to calls that fail validation
FAKE = [ctypes.c_void_p(0x10000 * (i + 1)) for i in range(12)]


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


def dims(**kw):
    base = dict(B=2, H=128, L=512, R=64, dv=128, g=2, max_pages_per_seq=8, num_pages=16,
                softmax_scale=192 ** -0.5)
    base.update(kw)
    return tpla.make_dims(**base)


def test_library_loads_and_exports_every_header_symbol():
    L = tpla.lib()
    names = header_functions()
    assert set(tpla.EXPORTED) == set(names), names
    for n in names:
        assert hasattr(L, n), n
    assert "sm_100a" in tpla.version()


def test_status_strings():
    for code in range(8):
        s = tpla.status_string(code)
        assert s.startswith("TPLA_") or code == 0
    assert tpla.status_string(0) == "TPLA_OK"
    assert "unknown" in tpla.status_string(99)


def test_workspace_size_host_only():
    ws = tpla.workspace_size(dims())
    # (160 workers + B*g) slots of H*(L/g) fp32 partials plus log-sum-exps
    slots = 160 + 2 * 2
    assert ws >= slots * 128 * 256 * 4 + slots * 128 * 4
    assert tpla.workspace_size(dims(B=16)) > ws
    assert tpla.workspace_size(dims(g=3)) == 0
    assert tpla.workspace_size(dims(page_size=32)) == 0
    assert tpla.workspace_size(dims(H=129)) == 0


def _decode(L, d, ws_bytes=1 << 40, q=FAKE[0], out=FAKE[7]):
    return L.tpla_decode(ctypes.byref(d) if d is not None else None, q, FAKE[1], FAKE[2], FAKE[3], None,
                         FAKE[5], None, out, FAKE[8], ws_bytes, None)


def test_validation_returns_before_any_cuda_call():
    L = tpla.lib()
    assert _decode(L, None) == tpla.TPLA_ERR_INVALID_ARG
    assert _decode(L, dims(g=3)) == tpla.TPLA_ERR_UNSUPPORTED
    assert _decode(L, dims(L=500)) == tpla.TPLA_ERR_UNSUPPORTED
    assert _decode(L, dims(R=48)) == tpla.TPLA_ERR_UNSUPPORTED
    assert _decode(L, dims(dv=12)) == tpla.TPLA_ERR_UNSUPPORTED
    assert _decode(L, dims(H=0)) == tpla.TPLA_ERR_INVALID_ARG
    assert _decode(L, dims(B=-1)) == tpla.TPLA_ERR_INVALID_ARG
    assert _decode(L, dims(softmax_scale=float("nan"))) == tpla.TPLA_ERR_INVALID_ARG
    assert _decode(L, dims(), q=None) == tpla.TPLA_ERR_INVALID_ARG
    assert _decode(L, dims(), q=ctypes.c_void_p(0x10008)) == tpla.TPLA_ERR_INVALID_ARG   # misaligned
    assert _decode(L, dims(), out=None) == tpla.TPLA_ERR_INVALID_ARG
    assert _decode(L, dims(), ws_bytes=1024) == tpla.TPLA_ERR_WORKSPACE
    # identity page table needs B * max_pages_per_seq pages
    assert _decode(L, dims(num_pages=15)) == tpla.TPLA_ERR_INVALID_ARG
    # mla_decode needs a g = 1 cache layout
    d = dims()
    assert L.mla_decode(ctypes.byref(d), *FAKE[:4], None, FAKE[5], None, FAKE[7], FAKE[8], 1 << 40,
                        None) == tpla.TPLA_ERR_LAYOUT
    # shard index range
    for s in (-1, 2):
        assert L.tpla_decode_shard(ctypes.byref(d), s, *FAKE[:4], None, FAKE[5], None, FAKE[7], FAKE[8],
                                   1 << 40, None) == tpla.TPLA_ERR_INVALID_ARG
    assert L.tpla_attention(ctypes.byref(d), 5, *FAKE[:4], None, FAKE[5], FAKE[8], 1 << 40,
                            None) == tpla.TPLA_ERR_INVALID_ARG
    assert L.tpla_combine(ctypes.byref(d), 0, FAKE[5], None, FAKE[7], FAKE[8], 16, None) == \
        tpla.TPLA_ERR_WORKSPACE


def test_empty_batch_is_a_noop_without_cuda():
    L = tpla.lib()
    d = dims(B=0)
    assert _decode(L, d) == tpla.TPLA_OK
    assert L.tpla_append_kv(ctypes.byref(d), None, None, 1, None, None, 1e-6, None, None, None, None,
                            None) == tpla.TPLA_OK


def test_append_validation():
    L = tpla.lib()
    d = dims()
    args = [FAKE[0], FAKE[1]]
    rest = [FAKE[4], None, FAKE[6], FAKE[7], None]
    assert L.tpla_append_kv(ctypes.byref(d), *args, 7, None, None, 1e-6, *rest) == tpla.TPLA_ERR_INVALID_ARG
    assert L.tpla_append_kv(ctypes.byref(d), *args, 4, None, None, 1e-6, *rest) == tpla.TPLA_ERR_INVALID_ARG
    assert L.tpla_append_kv(ctypes.byref(d), *args, -1, None, None, 1e-6, *rest) == tpla.TPLA_ERR_INVALID_ARG
    assert L.tpla_append_kv(ctypes.byref(d), *args, 2, None, None, 1e-6, *rest) == tpla.TPLA_ERR_INVALID_ARG
    assert L.tpla_append_kv(ctypes.byref(d), *args, 1, None, None, -1.0, *rest) == tpla.TPLA_ERR_INVALID_ARG
    assert L.tpla_append_kv(ctypes.byref(d), None, FAKE[1], 1, None, None, 1e-6, *rest) == \
        tpla.TPLA_ERR_INVALID_ARG
    assert L.tpla_append_kv(ctypes.byref(dims(g=3)), *args, 1, None, None, 1e-6, *rest) == \
        tpla.TPLA_ERR_UNSUPPORTED
    # one tensor-parallel rank's append: the shard must be one of the g shards
    for shard in (-1, d.g, d.g + 5):
        assert L.tpla_append_kv_shard(ctypes.byref(d), shard, *args, 1, None, None, 1e-6, *rest) == \
            tpla.TPLA_ERR_INVALID_ARG
    assert L.tpla_append_kv_shard(ctypes.byref(d), 0, *args, 7, None, None, 1e-6, *rest) == tpla.TPLA_ERR_INVALID_ARG


def test_options_roundtrip():
    old = tpla.get_option(tpla.OPT_ATTENTION_KERNEL)
    try:
        for v in (1, 2, 0):
            tpla.set_option(tpla.OPT_ATTENTION_KERNEL, v)
            assert tpla.get_option(tpla.OPT_ATTENTION_KERNEL) == v
        with pytest.raises(tpla.TplaError):
            tpla.set_option(tpla.OPT_ATTENTION_KERNEL, 5)
        with pytest.raises(tpla.TplaError):
            tpla.set_option(99, 0)
        assert tpla.get_option(99) == -1
    finally:
        tpla.set_option(tpla.OPT_ATTENTION_KERNEL, old)


def test_binding_rejects_cpu_tensors():
    import torch
    d = dims(B=1)
    t = torch.zeros(4, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        tpla.decode(d, t, t, t, t, None, t, None, t, torch.zeros(16, dtype=torch.uint8))
