"""ctypes binding of libtpla.so (C ABI in include/tpla.h).

Argument marshalling only: every function passes device pointers, sizes and
the current CUDA stream to the library entry point of the same name and
raises TplaError on a non-zero status.  No computation happens here and there
is no fallback: if the library is missing, every call raises.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtpla.so")

TPLA_OK = 0
TPLA_ERR_INVALID_ARG = 1
TPLA_ERR_UNSUPPORTED = 2
TPLA_ERR_LAYOUT = 3
TPLA_ERR_WORKSPACE = 4
TPLA_ERR_CUDA = 5
TPLA_ERR_TIMEOUT = 6
TPLA_ERR_INDEX = 7

TRANSFORM_NONE = 0
TRANSFORM_HADAMARD = 1
TRANSFORM_DENSE = 2
TRANSFORM_BLOCK_HADAMARD = 3

OPT_ATTENTION_KERNEL = 1
OPT_MAX_WORKERS = 2
OPT_WAIT_LIMIT = 3
OPT_DEBUG_STALL = 4
OPT_LAST_ATTENTION_KERNEL = 5
OPT_TILE_TOKENS = 6

PAGE_SIZE = 64

EXPORTED = ("tpla_status_string", "tpla_decode_workspace_size", "tpla_decode", "tpla_decode_shard",
            "mla_decode", "tpla_attention", "tpla_combine", "tpla_append_kv",
            "tpla_check_device_status", "tpla_set_option", "tpla_get_option", "tpla_version",
            "tpla_decode_static", "tpla_append_kv_shard")


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int), ("R", ctypes.c_int),
                ("dv", ctypes.c_int), ("g", ctypes.c_int), ("page_size", ctypes.c_int),
                ("max_pages_per_seq", ctypes.c_int), ("num_pages", ctypes.c_int),
                ("softmax_scale", ctypes.c_float)]


def make_dims(*, B, H, L, R, dv, g, max_pages_per_seq, num_pages, softmax_scale, page_size=PAGE_SIZE):
    return Dims(int(B), int(H), int(L), int(R), int(dv), int(g), int(page_size),
                int(max_pages_per_seq), int(num_pages), float(softmax_scale))


class TplaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, status_string(status), status))


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_F = ctypes.c_float
_DIMS = ctypes.POINTER(Dims)


def lib():
    """The loaded libtpla.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libtpla.so is not built (python -m latent_attention_decode_tpla_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        dec = [_DIMS, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
        sigs = {
            "tpla_status_string": ([_I], ctypes.c_char_p),
            "tpla_decode_workspace_size": ([_DIMS], _SZ),
            "tpla_decode": (dec, _I),
            "tpla_decode_shard": ([_DIMS, _I] + dec[1:], _I),
            "mla_decode": (dec, _I),
            "tpla_attention": ([_DIMS, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P], _I),
            "tpla_combine": ([_DIMS, _I, _P, _P, _P, _P, _SZ, _P], _I),
            "tpla_append_kv": ([_DIMS, _P, _P, _I, _P, _P, _F, _P, _P, _P, _P, _P], _I),
            "tpla_append_kv_shard": ([_DIMS, _I, _P, _P, _I, _P, _P, _F, _P, _P, _P, _P, _P], _I),
            "tpla_check_device_status": ([_P], _I),
            "tpla_set_option": ([_I, _I], _I),
            "tpla_get_option": ([_I], _I),
            "tpla_version": ([], ctypes.c_char_p),
            "tpla_decode_static": ([_DIMS, _P, _P, _P, _P, _P, _P, _P, _P, _P], _I),
        }
        for name, (args, res) in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def status_string(status):
    return lib().tpla_status_string(int(status)).decode()


def version():
    return lib().tpla_version().decode()


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _bf16(t):
    if t is not None and t.dtype != torch.bfloat16:
        raise TypeError("expected a bfloat16 tensor, got %s" % t.dtype)
    return _ptr(t)


def _i32(t):
    if t is not None and t.dtype != torch.int32:
        raise TypeError("expected an int32 tensor, got %s" % t.dtype)
    return _ptr(t)


def _f32(t):
    if t is not None and t.dtype != torch.float32:
        raise TypeError("expected a float32 tensor, got %s" % t.dtype)
    return _ptr(t)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status, where):
    if status != TPLA_OK:
        raise TplaError(status, where)


def workspace_size(dims):
    return int(lib().tpla_decode_workspace_size(ctypes.byref(dims)))


def alloc_workspace(dims, device=None):
    n = workspace_size(dims)
    if n == 0:
        raise TplaError(TPLA_ERR_UNSUPPORTED, "tpla_decode_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def decode(dims, q, q_pe, ckv, kpe, block_table, seq_lens, w_uv, out, workspace, stream=None):
    _check(lib().tpla_decode(ctypes.byref(dims), _bf16(q), _bf16(q_pe), _bf16(ckv), _bf16(kpe),
                             _i32(block_table), _i32(seq_lens), _bf16(w_uv), _f32(out), _ptr(workspace),
                             workspace.numel(), _stream(stream)), "tpla_decode")
    return out


def decode_shard(dims, shard, q, q_pe, ckv, kpe, block_table, seq_lens, w_uv, out, workspace, stream=None):
    _check(lib().tpla_decode_shard(ctypes.byref(dims), int(shard), _bf16(q), _bf16(q_pe), _bf16(ckv),
                                   _bf16(kpe), _i32(block_table), _i32(seq_lens), _bf16(w_uv), _f32(out),
                                   _ptr(workspace), workspace.numel(), _stream(stream)), "tpla_decode_shard")
    return out


def mla_decode(dims, q, q_pe, ckv, kpe, block_table, seq_lens, w_uv, out, workspace, stream=None):
    _check(lib().mla_decode(ctypes.byref(dims), _bf16(q), _bf16(q_pe), _bf16(ckv), _bf16(kpe),
                            _i32(block_table), _i32(seq_lens), _bf16(w_uv), _f32(out), _ptr(workspace),
                            workspace.numel(), _stream(stream)), "mla_decode")
    return out


def decode_static(dims, q, q_pe, ckv, kpe, block_table, seq_lens, w_uv, out, stream=None):
    """tpla_decode without a workspace: scratch is the library's fixed 32 MiB device array."""
    _check(lib().tpla_decode_static(ctypes.byref(dims), _bf16(q), _bf16(q_pe), _bf16(ckv), _bf16(kpe),
                                    _i32(block_table), _i32(seq_lens), _bf16(w_uv), _f32(out), _stream(stream)),
           "tpla_decode_static")
    return out


def attention(dims, shard, q, q_pe, ckv, kpe, block_table, seq_lens, workspace, stream=None):
    _check(lib().tpla_attention(ctypes.byref(dims), int(shard), _bf16(q), _bf16(q_pe), _bf16(ckv),
                                _bf16(kpe), _i32(block_table), _i32(seq_lens), _ptr(workspace),
                                workspace.numel(), _stream(stream)), "tpla_attention")


def combine(dims, shard, seq_lens, w_uv, out, workspace, stream=None):
    _check(lib().tpla_combine(ctypes.byref(dims), int(shard), _i32(seq_lens), _bf16(w_uv), _f32(out),
                              _ptr(workspace), workspace.numel(), _stream(stream)), "tpla_combine")
    return out


def append_kv(dims, latent_raw, kpe_new, transform, R_dense, norm_weight, eps, positions, block_table,
              ckv, kpe, stream=None):
    _check(lib().tpla_append_kv(ctypes.byref(dims), _bf16(latent_raw), _bf16(kpe_new), int(transform),
                                _f32(R_dense), _f32(norm_weight), float(eps), _i32(positions),
                                _i32(block_table), _bf16(ckv), _bf16(kpe), _stream(stream)),
           "tpla_append_kv")


def append_kv_shard(dims, shard, latent_raw, kpe_new, transform, R_dense, norm_weight, eps, positions,
                    block_table, ckv_shard, kpe, stream=None):
    _check(lib().tpla_append_kv_shard(ctypes.byref(dims), int(shard), _bf16(latent_raw), _bf16(kpe_new),
                                      int(transform), _f32(R_dense), _f32(norm_weight), float(eps),
                                      _i32(positions), _i32(block_table), _bf16(ckv_shard), _bf16(kpe),
                                      _stream(stream)), "tpla_append_kv_shard")


def check_device_status(stream=None):
    """Synchronise the stream and return (and clear) the device status code."""
    return int(lib().tpla_check_device_status(_stream(stream)))


def set_option(option, value):
    _check(lib().tpla_set_option(int(option), int(value)), "tpla_set_option")


def get_option(option):
    return int(lib().tpla_get_option(int(option)))
