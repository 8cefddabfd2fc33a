"""Thin ctypes binding of libtq.so, with the C ABI's own entry-point names.

Only argument marshalling happens here: every step of quantisation and
attention runs in the library's CUDA kernels.  PyTorch provides device
memory and the current stream.  Importing this module loads libtq.so and
raises ImportError when it is missing (build it with
``python -m bit_kv_cache_tq_b200.build``); there is no fallback path.
"""

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtq.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError("libtq.so is not built (run: python -m bit_kv_cache_tq_b200.build)")
_lib = ctypes.CDLL(_LIB_PATH)

TQ_OK, TQ_ERR_INVALID_ARG, TQ_ERR_UNSUPPORTED, TQ_ERR_CAPACITY = 0, 1, 2, 3
TQ_ERR_CUDA, TQ_ERR_TIMEOUT, TQ_ERR_DEVICE, TQ_ERR_ALIGNMENT = 4, 5, 6, 7
TQ_MODE_TURBO, TQ_MODE_INT8 = 0, 1
TQ_F32, TQ_BF16, TQ_F16 = 0, 1, 2
TQ_DEVERR_POSITION, TQ_DEVERR_SEQLEN, TQ_DEVERR_TIMEOUT, TQ_DEVERR_PAGE = 0x1, 0x2, 0x4, 0x8
TQ_PARAM_PREFETCH_EARLY = 0x1

# every symbol include/tq.h declares
EXPORTED = (
    "tq_status_string", "tq_abi_version", "tq_codebook_init", "tq_rotation_signs", "tq_qjl_matrix",
    "tq_cache_bytes", "tq_decode_workspace_bytes", "tq_quantize_append", "tq_dequantize",
    "tq_decode_attention", "tq_append_decode_attention", "tq_decode_attention_static", "tq_read_device_error",
    "tq_quantize_append_paged", "tq_decode_attention_paged", "tq_append_decode_attention_paged",
    "tq_prefill_attention", "tq_decode_static_fill", "tq_prefill_workspace_bytes",
)

# Bytes of the library's own decode scratch per device (tq_decode_attention_static).
TQ_DECODE_STATIC_SCRATCH_BYTES = 16 << 20


class tq_codebook(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int32), ("bits", ctypes.c_int32),
                ("centroids", ctypes.c_double * 16), ("boundaries", ctypes.c_double * 15),
                ("fp16_scale", ctypes.c_double)]

    @property
    def centroid_array(self):
        return np.array(self.centroids[: 1 << self.bits])

    @property
    def boundary_array(self):
        return np.array(self.boundaries[: (1 << self.bits) - 1])


class tq_params(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("k_mode", ctypes.c_int32), ("v_mode", ctypes.c_int32), ("k_bits", ctypes.c_int32),
                ("v_bits", ctypes.c_int32), ("qjl_dims", ctypes.c_int32), ("seed", ctypes.c_uint64),
                ("sm_scale", ctypes.c_float), ("sparse_v_threshold", ctypes.c_float),
                ("flags", ctypes.c_uint32), ("reserved", ctypes.c_uint32)]


class tq_cache(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("k_codes", ctypes.c_void_p), ("k_norms", ctypes.c_void_p),
                ("k_qjl", ctypes.c_void_p), ("k_gamma", ctypes.c_void_p),
                ("v_codes", ctypes.c_void_p), ("v_norms", ctypes.c_void_p),
                ("qjl_matrix", ctypes.c_void_p)]


class tq_block_table(ctypes.Structure):
    _fields_ = [("d_table", ctypes.c_void_p), ("batch", ctypes.c_int32), ("max_blocks", ctypes.c_int32)]


_P = ctypes.POINTER
_lib.tq_status_string.restype = ctypes.c_char_p
_lib.tq_status_string.argtypes = [ctypes.c_int]
_lib.tq_abi_version.restype = ctypes.c_int32
_lib.tq_abi_version.argtypes = []
_lib.tq_codebook_init.argtypes = [ctypes.c_int32, ctypes.c_int32, _P(tq_codebook)]
_lib.tq_rotation_signs.argtypes = [ctypes.c_uint64, ctypes.c_int32, ctypes.c_void_p]
_lib.tq_qjl_matrix.argtypes = [ctypes.c_uint64, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p]
_lib.tq_cache_bytes.argtypes = [_P(tq_params), ctypes.c_int32, ctypes.c_int32, _P(ctypes.c_size_t * 6)]
_lib.tq_decode_workspace_bytes.argtypes = [_P(tq_params), ctypes.c_int32, ctypes.c_int32, _P(ctypes.c_size_t)]
_lib.tq_quantize_append.argtypes = [_P(tq_params), _P(tq_codebook), _P(tq_codebook), ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_int, ctypes.c_int32, ctypes.c_void_p,
                                    _P(tq_cache), ctypes.c_void_p, ctypes.c_void_p]
_lib.tq_dequantize.argtypes = [_P(tq_params), _P(tq_codebook), _P(tq_codebook), _P(tq_cache), ctypes.c_int32,
                               ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
_lib.tq_decode_attention.argtypes = [_P(tq_params), _P(tq_codebook), _P(tq_codebook), ctypes.c_void_p, ctypes.c_int,
                                     _P(tq_cache), ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p]
_lib.tq_append_decode_attention.argtypes = [_P(tq_params), _P(tq_codebook), _P(tq_codebook), ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                                            _P(tq_cache), ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p,
                                            ctypes.c_void_p]
_lib.tq_decode_static_fill.argtypes = [ctypes.c_uint8, ctypes.c_void_p]
_lib.tq_decode_attention_static.argtypes = [_P(tq_params), _P(tq_codebook), _P(tq_codebook), ctypes.c_void_p,
                                            ctypes.c_int, _P(tq_cache), ctypes.c_void_p, ctypes.c_int32,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
_lib.tq_read_device_error.argtypes = [ctypes.c_void_p, _P(ctypes.c_uint32), ctypes.c_void_p, ctypes.c_int32]
_lib.tq_quantize_append_paged.argtypes = [_P(tq_params), _P(tq_codebook), _P(tq_codebook), ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_int, ctypes.c_int32, ctypes.c_void_p,
                                          _P(tq_cache), _P(tq_block_table), ctypes.c_void_p, ctypes.c_void_p]
_lib.tq_decode_attention_paged.argtypes = [_P(tq_params), _P(tq_codebook), _P(tq_codebook), ctypes.c_void_p,
                                           ctypes.c_int, _P(tq_cache), _P(tq_block_table), ctypes.c_void_p,
                                           ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
_lib.tq_append_decode_attention_paged.argtypes = [_P(tq_params), _P(tq_codebook), _P(tq_codebook), ctypes.c_void_p,
                                                  ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                                                  _P(tq_cache), _P(tq_block_table), ctypes.c_void_p, ctypes.c_int32,
                                                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                                  ctypes.c_void_p, ctypes.c_void_p]
_lib.tq_prefill_attention.argtypes = [_P(tq_params), _P(tq_codebook), _P(tq_codebook), ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int32,
                                      ctypes.c_void_p, _P(tq_cache), ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p]
_lib.tq_prefill_workspace_bytes.argtypes = [_P(tq_params), ctypes.c_int32, ctypes.c_int32, _P(ctypes.c_size_t)]
for _name in EXPORTED:
    if _name not in ("tq_status_string", "tq_abi_version"):
        getattr(_lib, _name).restype = ctypes.c_int


class TqError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s (%d)" % (where, tq_status_string(status), status))


def _check(status, where):
    if status != TQ_OK:
        raise TqError(status, where)


def _dtype_code(t):
    return {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16, torch.float16: TQ_F16}[t.dtype]


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def library():
    """The loaded ctypes library (for symbol checks)."""
    return _lib


def library_path():
    return _LIB_PATH


# ------------------------------------------------------------------ host calls
def tq_status_string(status):
    return _lib.tq_status_string(int(status)).decode()


def tq_abi_version():
    return int(_lib.tq_abi_version())


def tq_codebook_init(head_dim, bits):
    cb = tq_codebook()
    _check(_lib.tq_codebook_init(head_dim, bits, ctypes.byref(cb)), "tq_codebook_init")
    return cb


def tq_rotation_signs(seed, head_dim):
    out = np.empty(head_dim, dtype=np.float32)
    _check(_lib.tq_rotation_signs(seed, head_dim, out.ctypes.data), "tq_rotation_signs")
    return out


def tq_qjl_matrix(seed, m, head_dim):
    out = np.empty((m, head_dim), dtype=np.float32)
    _check(_lib.tq_qjl_matrix(seed, m, head_dim, out.ctypes.data), "tq_qjl_matrix")
    return out


def make_params(head_dim, num_q_heads, num_kv_heads, k_bits=4, v_bits=2, k_mode=TQ_MODE_TURBO,
                v_mode=TQ_MODE_TURBO, qjl_dims=0, seed=0, sm_scale=0.0, sparse_v_threshold=0.0, flags=0):
    return tq_params(head_dim, num_q_heads, num_kv_heads, k_mode, v_mode, k_bits, v_bits, qjl_dims, seed,
                     sm_scale, sparse_v_threshold, flags, 0)


def tq_cache_bytes(params, batch, capacity):
    sizes = (ctypes.c_size_t * 6)()
    _check(_lib.tq_cache_bytes(ctypes.byref(params), batch, capacity, ctypes.byref(sizes)), "tq_cache_bytes")
    return tuple(int(s) for s in sizes)


def tq_decode_workspace_bytes(params, batch, max_seq_len):
    n = ctypes.c_size_t()
    _check(_lib.tq_decode_workspace_bytes(ctypes.byref(params), batch, max_seq_len, ctypes.byref(n)),
           "tq_decode_workspace_bytes")
    return int(n.value)


def block_table(table):
    """tq_block_table over an int32 CUDA tensor [batch, max_blocks] (kept alive by the caller)."""
    assert table.dtype == torch.int32 and table.is_cuda and table.is_contiguous() and table.dim() == 2
    return tq_block_table(_ptr(table), table.shape[0], table.shape[1])


# -------------------------------------------------------------- cache storage
@dataclass
class CacheTensors:
    """Device tensors of one layer's compressed cache (caller-owned memory)."""
    batch: int
    capacity: int
    k_codes: torch.Tensor
    k_norms: torch.Tensor
    k_qjl: torch.Tensor
    k_gamma: torch.Tensor
    v_codes: torch.Tensor
    v_norms: torch.Tensor
    qjl_matrix: torch.Tensor

    def struct(self):
        return tq_cache(self.batch, self.capacity, _ptr(self.k_codes), _ptr(self.k_norms), _ptr(self.k_qjl),
                        _ptr(self.k_gamma), _ptr(self.v_codes), _ptr(self.v_norms), _ptr(self.qjl_matrix))

    def nbytes(self):
        return sum(t.numel() * t.element_size() for t in (self.k_codes, self.k_norms, self.k_qjl, self.k_gamma,
                                                          self.v_codes, self.v_norms) if t is not None)


def alloc_cache(params, batch, capacity, device="cuda"):
    """Allocate a zeroed cache with torch, shaped [batch][Hkv][capacity][...]."""
    sizes = tq_cache_bytes(params, batch, capacity)
    hkv = params.num_kv_heads
    slots = batch * hkv * capacity

    def buf(nbytes, per_slot, dtype=torch.uint8):
        if nbytes == 0:
            return None
        return torch.zeros(batch, hkv, capacity, per_slot, dtype=dtype, device=device)

    k_codes = buf(sizes[0], sizes[0] // slots)
    k_norms = buf(sizes[1], 1, torch.int16).view(batch, hkv, capacity)
    k_qjl = buf(sizes[2], sizes[2] // slots if sizes[2] else 0)
    k_gamma = buf(sizes[3], 1, torch.int16)
    k_gamma = None if k_gamma is None else k_gamma.view(batch, hkv, capacity)
    v_codes = buf(sizes[4], sizes[4] // slots)
    v_norms = buf(sizes[5], 1, torch.int16).view(batch, hkv, capacity)
    qjl_matrix = None
    if params.qjl_dims:
        qjl_matrix = torch.from_numpy(tq_qjl_matrix(params.seed, params.qjl_dims, params.head_dim)).to(device)
    return CacheTensors(batch, capacity, k_codes, k_norms, k_qjl, k_gamma, v_codes, v_norms, qjl_matrix)


# ------------------------------------------------------------- device calls
def tq_quantize_append(params, kcb, vcb, k_new, v_new, positions, cache, error=None, stream=None):
    """k_new, v_new: [batch, n_new, Hkv, d] CUDA tensors; positions: int32 [batch] CUDA tensor."""
    assert k_new.is_contiguous() and v_new.is_contiguous() and k_new.dtype == v_new.dtype
    assert positions.dtype == torch.int32 and positions.is_cuda
    c = cache.struct()
    st = _lib.tq_quantize_append(ctypes.byref(params), kcb and ctypes.byref(kcb), vcb and ctypes.byref(vcb),
                                 _ptr(k_new), _ptr(v_new), _dtype_code(k_new), k_new.shape[1], _ptr(positions),
                                 ctypes.byref(c), _ptr(error), _stream(stream))
    _check(st, "tq_quantize_append")


def tq_dequantize(params, kcb, vcb, cache, b, start, count, k_out=None, v_out=None, stream=None):
    c = cache.struct()
    st = _lib.tq_dequantize(ctypes.byref(params), kcb and ctypes.byref(kcb), vcb and ctypes.byref(vcb),
                            ctypes.byref(c), b, start, count, _ptr(k_out), _ptr(v_out), _stream(stream))
    _check(st, "tq_dequantize")


def tq_decode_attention(params, kcb, vcb, q, cache, seq_lens, max_seq_len, out, workspace, error=None,
                        stream=None, skip_mask=None):
    """q: [batch, Hq, d] CUDA tensor; seq_lens int32 [batch]; out fp32 [batch, Hq, d]; workspace uint8;
    skip_mask: zeroed int32 [batch, Hq, (max_seq_len + 31) // 32] CUDA tensor or None (Sparse V's dropped
    positions, one bit each)."""
    assert q.is_contiguous() and out.is_contiguous() and out.dtype == torch.float32
    assert seq_lens.dtype == torch.int32 and seq_lens.is_cuda
    c = cache.struct()
    st = _lib.tq_decode_attention(ctypes.byref(params), kcb and ctypes.byref(kcb), vcb and ctypes.byref(vcb),
                                  _ptr(q), _dtype_code(q), ctypes.byref(c), _ptr(seq_lens), max_seq_len, _ptr(out),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(skip_mask),
                                  _ptr(error), _stream(stream))
    _check(st, "tq_decode_attention")


def tq_append_decode_attention(params, kcb, vcb, k_new, v_new, q, cache, seq_lens, max_seq_len, out, workspace,
                               error=None, stream=None, skip_mask=None):
    """Append k_new/v_new ([batch, 1, Hkv, d]) at slot seq_lens-1, then decode attention over seq_lens tokens."""
    assert q.is_contiguous() and out.is_contiguous() and out.dtype == torch.float32
    assert k_new.is_contiguous() and v_new.is_contiguous() and k_new.dtype == v_new.dtype
    assert seq_lens.dtype == torch.int32 and seq_lens.is_cuda
    c = cache.struct()
    st = _lib.tq_append_decode_attention(ctypes.byref(params), kcb and ctypes.byref(kcb), vcb and ctypes.byref(vcb),
                                         _ptr(k_new), _ptr(v_new), _dtype_code(k_new), _ptr(q), _dtype_code(q), ctypes.byref(c),
                                         _ptr(seq_lens), max_seq_len, _ptr(out), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _ptr(skip_mask), _ptr(error),
                                         _stream(stream))
    _check(st, "tq_append_decode_attention")


def tq_decode_static_fill(value, stream=None):
    """Fill the static decode array's counter region with the byte `value` (0: reset)."""
    _check(_lib.tq_decode_static_fill(int(value) & 0xFF, _stream(stream)), "tq_decode_static_fill")


def tq_decode_attention_static(params, kcb, vcb, q, cache, seq_lens, max_seq_len, out, error=None, stream=None):
    """tq_decode_attention on the library's own per-device scratch (no workspace argument)."""
    assert q.is_contiguous() and out.is_contiguous() and out.dtype == torch.float32
    assert seq_lens.dtype == torch.int32 and seq_lens.is_cuda
    c = cache.struct()
    st = _lib.tq_decode_attention_static(ctypes.byref(params), kcb and ctypes.byref(kcb), vcb and ctypes.byref(vcb),
                                         _ptr(q), _dtype_code(q), ctypes.byref(c), _ptr(seq_lens), max_seq_len,
                                         _ptr(out), _ptr(error), _stream(stream))
    _check(st, "tq_decode_attention_static")


def tq_prefill_workspace_bytes(params, batch, n_new):
    n = ctypes.c_size_t(0)
    _check(_lib.tq_prefill_workspace_bytes(ctypes.byref(params), batch, n_new, ctypes.byref(n)),
           "tq_prefill_workspace_bytes")
    return n.value


def tq_prefill_attention(params, kcb, vcb, k_new, v_new, q, positions, cache, out, workspace, error=None,
                         stream=None):
    """Append k_new/v_new ([batch, n_new, Hkv, d]) at slots positions[b] .., then causal attention of
    q ([batch, n_new, Hq, d]) over the cache into out ([batch, n_new, Hq, d] fp32); workspace: a uint8
    CUDA tensor of tq_prefill_workspace_bytes(params, batch, n_new) bytes, any contents (None when that is 0)."""
    assert q.is_contiguous() and out.is_contiguous() and out.dtype == torch.float32
    assert k_new.is_contiguous() and v_new.is_contiguous() and k_new.dtype == v_new.dtype
    assert positions.dtype == torch.int32 and positions.is_cuda
    c = cache.struct()
    st = _lib.tq_prefill_attention(ctypes.byref(params), kcb and ctypes.byref(kcb), vcb and ctypes.byref(vcb),
                                   _ptr(k_new), _ptr(v_new), _dtype_code(k_new), _ptr(q), _dtype_code(q),
                                   k_new.shape[1], _ptr(positions), ctypes.byref(c), _ptr(out), _ptr(workspace),
                                   0 if workspace is None else workspace.numel() * workspace.element_size(),
                                   _ptr(error), _stream(stream))
    _check(st, "tq_prefill_attention")


def tq_quantize_append_paged(params, kcb, vcb, k_new, v_new, positions, pool, table, error=None, stream=None):
    """tq_quantize_append on a paged cache: pool from alloc_cache(params, num_blocks, block_size),
    table an int32 CUDA tensor [batch, max_blocks] of block indices."""
    assert k_new.is_contiguous() and v_new.is_contiguous() and k_new.dtype == v_new.dtype
    assert positions.dtype == torch.int32 and positions.is_cuda
    c, bt = pool.struct(), block_table(table)
    st = _lib.tq_quantize_append_paged(ctypes.byref(params), kcb and ctypes.byref(kcb), vcb and ctypes.byref(vcb),
                                       _ptr(k_new), _ptr(v_new), _dtype_code(k_new), k_new.shape[1],
                                       _ptr(positions), ctypes.byref(c), ctypes.byref(bt), _ptr(error),
                                       _stream(stream))
    _check(st, "tq_quantize_append_paged")


def tq_decode_attention_paged(params, kcb, vcb, q, pool, table, seq_lens, max_seq_len, out, workspace, error=None,
                              stream=None, skip_mask=None):
    """tq_decode_attention on a paged cache (see tq_quantize_append_paged)."""
    assert q.is_contiguous() and out.is_contiguous() and out.dtype == torch.float32
    assert seq_lens.dtype == torch.int32 and seq_lens.is_cuda
    c, bt = pool.struct(), block_table(table)
    st = _lib.tq_decode_attention_paged(ctypes.byref(params), kcb and ctypes.byref(kcb), vcb and ctypes.byref(vcb),
                                        _ptr(q), _dtype_code(q), ctypes.byref(c), ctypes.byref(bt), _ptr(seq_lens),
                                        max_seq_len, _ptr(out), _ptr(workspace),
                                        workspace.numel() * workspace.element_size(), _ptr(skip_mask), _ptr(error),
                                        _stream(stream))
    _check(st, "tq_decode_attention_paged")


def tq_append_decode_attention_paged(params, kcb, vcb, k_new, v_new, q, pool, table, seq_lens, max_seq_len, out,
                                     workspace, error=None, stream=None, skip_mask=None):
    """tq_append_decode_attention on a paged cache (see tq_quantize_append_paged)."""
    assert q.is_contiguous() and out.is_contiguous() and out.dtype == torch.float32
    assert k_new.is_contiguous() and v_new.is_contiguous() and k_new.dtype == v_new.dtype
    assert seq_lens.dtype == torch.int32 and seq_lens.is_cuda
    c, bt = pool.struct(), block_table(table)
    st = _lib.tq_append_decode_attention_paged(ctypes.byref(params), kcb and ctypes.byref(kcb),
                                               vcb and ctypes.byref(vcb), _ptr(k_new), _ptr(v_new),
                                               _dtype_code(k_new), _ptr(q), _dtype_code(q), ctypes.byref(c),
                                               ctypes.byref(bt), _ptr(seq_lens), max_seq_len, _ptr(out),
                                               _ptr(workspace), workspace.numel() * workspace.element_size(),
                                               _ptr(skip_mask), _ptr(error), _stream(stream))
    _check(st, "tq_append_decode_attention_paged")


def tq_read_device_error(error, stream=None, timeout_ms=2000):
    """Return (status, word) for a device uint32 error word."""
    word = ctypes.c_uint32()
    st = _lib.tq_read_device_error(_ptr(error), ctypes.byref(word), _stream(stream), timeout_ms)
    return st, int(word.value)
