"""The C-ABI library on the host (no GPU): exports, codebooks, random numbers,
sizes and argument validation.  No test here launches device work."""

import ctypes
import math
import os
import re

import numpy as np
import pytest

from conftest import ROOT, read_golden
from bit_kv_cache_tq_b200 import tq
from oracle import codebook, rng


def _declared_functions():
    with open(os.path.join(ROOT, "include", "tq.h"), encoding="utf-8") as fh:
        text = fh.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    declared = _declared_functions()
    assert len(declared) >= 11
    for name in declared:
        assert hasattr(tq.library(), name), name
    assert set(tq.EXPORTED) <= set(declared)


def _declared_arities():
    """Parameter count of every function declared in include/tq.h."""
    with open(os.path.join(ROOT, "include", "tq.h"), encoding="utf-8") as fh:
        text = fh.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(tq_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text):
        args = m.group(2).strip()
        out[m.group(1)] = 0 if args in ("", "void") else args.count(",") + 1
    return out


def test_binding_declares_every_argument_type():
    """ctypes passes an undeclared integer argument as a 32-bit int: every
    exported call must declare its argument types, one per C parameter (a
    size_t passed as int reads garbage in its upper half)."""
    arity = _declared_arities()
    for name in tq.EXPORTED:
        f = getattr(tq.library(), name)
        assert f.argtypes is not None, name
        assert len(f.argtypes) == arity[name], (name, len(f.argtypes), arity[name])


def test_abi_version_and_status_strings():
    assert tq.tq_abi_version() == 5
    for st in range(8):
        assert tq.tq_status_string(st)
    assert tq.tq_status_string(99) == "unknown status"


@pytest.mark.parametrize("d,bits", [(64, 2), (64, 3), (64, 4), (128, 2), (128, 3), (128, 4),
                                    (256, 2), (256, 3), (256, 4), (3, 3), (4, 1), (16, 4)])
def test_codebook_matches_oracle(d, bits):
    """Library (incomplete-beta continued fraction) vs oracle (Gauss-Legendre)."""
    cb = tq.tq_codebook_init(d, bits)
    c, t = codebook.lloyd_max(d, bits)
    assert cb.head_dim == d and cb.bits == bits
    assert np.max(np.abs(cb.centroid_array - c)) * math.sqrt(d) < 1e-10
    assert np.max(np.abs(cb.boundary_array - t)) * math.sqrt(d) < 1e-10
    assert np.array_equal(cb.centroid_array, -cb.centroid_array[::-1])


@pytest.mark.parametrize("d,bits", [(128, 2), (128, 3), (128, 4), (256, 4), (64, 3)])
def test_codebook_fp16_scale_keeps_rounding_small(d, bits):
    """The scale the tensor-core kernels apply before fp16 rounding leaves every
    centroid within 2e-4 relative of its fp64 value (sqrt(d) would not)."""
    cb = tq.tq_codebook_init(d, bits)
    assert 8.0 <= cb.fp16_scale < 16.0
    c = cb.centroid_array
    scaled = (c * cb.fp16_scale).astype(np.float32)
    err = np.max(np.abs(scaled.astype(np.float16).astype(np.float64) - scaled) / np.abs(scaled))
    assert err < 2e-4, err


def test_codebook_rejects_bad_arguments():
    with pytest.raises(tq.TqError):
        tq.tq_codebook_init(128, 5)
    with pytest.raises(tq.TqError):
        tq.tq_codebook_init(2, 2)


@pytest.mark.parametrize("seed", [0, 1, 12345, 2 ** 63 + 17])
def test_rotation_signs_match_oracle(seed):
    for d in (64, 128, 256):
        assert np.array_equal(tq.tq_rotation_signs(seed, d), rng.rotation_signs(seed, d))


@pytest.mark.parametrize("seed,m,d", [(0, 64, 128), (7, 32, 64), (99, 128, 256)])
def test_qjl_matrix_matches_oracle(seed, m, d):
    a = tq.tq_qjl_matrix(seed, m, d).astype(np.float64)
    b = rng.qjl_matrix(seed, m, d)
    ulp = np.spacing(np.abs(b).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(a - b) <= ulp)


def test_cache_bytes_layout():
    p = tq.make_params(128, 32, 8, k_bits=4, v_bits=2)
    kc, kn, kq, kg, vc, vn = tq.tq_cache_bytes(p, 2, 1000)
    slots = 2 * 8 * 1000
    assert (kc, kn, kq, kg, vc, vn) == (slots * 64, slots * 2, 0, 0, slots * 32, slots * 2)
    p = tq.make_params(128, 64, 8, k_bits=3, v_bits=2, qjl_dims=64)
    kc, kn, kq, kg, vc, vn = tq.tq_cache_bytes(p, 1, 10)
    assert (kc, kq, kg, vc) == (80 * 48, 80 * 8, 80 * 2, 80 * 32)
    p = tq.make_params(256, 8, 8, k_mode=tq.TQ_MODE_INT8, v_mode=tq.TQ_MODE_INT8)
    kc, kn, _, _, vc, vn = tq.tq_cache_bytes(p, 1, 3)
    assert (kc, kn, vc, vn) == (8 * 3 * 256, 8 * 3 * 2, 8 * 3 * 256, 8 * 3 * 2)


def test_compression_ratios_against_page_table():
    """Bytes per vector against 16-bit storage, d = 128 (golden: page table)."""
    gold = read_golden("compression_formats.txt")
    for name, (bits, lo, hi, pinned) in gold.items():
        bits, lo, hi = int(bits), float(lo), float(hi)
        p = tq.make_params(128, 1, 1, k_bits=bits, v_bits=bits)
        kc, kn, _, _, _, _ = tq.tq_cache_bytes(p, 1, 1)
        ratio = 128 * 2 / (kc + kn)
        if pinned == "yes":
            assert lo - 0.05 <= ratio <= hi + 0.05, (name, ratio)
        else:
            assert ratio > lo, (name, ratio)


def test_bit_presets_against_page():
    gold = read_golden("bit_presets.txt")
    for name, (kb, vb, avg, saving) in gold.items():
        p = tq.make_params(128, 1, 1, k_bits=int(kb), v_bits=int(vb))
        kc, _, _, _, vc, _ = tq.tq_cache_bytes(p, 1, 1)
        avg_bits = (kc + vc) * 8 / (2 * 128)
        assert avg_bits == float(avg), name
        if saving != "-":
            assert 100 * (1 - avg_bits / 16) >= float(saving) - 0.5, name


def test_workspace_bound_grows_with_length_and_batch():
    p = tq.make_params(128, 32, 8)
    a = tq.tq_decode_workspace_bytes(p, 1, 1024)
    b = tq.tq_decode_workspace_bytes(p, 1, 32769)
    c = tq.tq_decode_workspace_bytes(p, 4, 32769)
    assert 0 < a <= b <= c
    assert b >= 32 * 128 * 4  # at least one fp32 partial per query head


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 100, tq.TQ_ERR_INVALID_ARG), ("head_dim", 512, tq.TQ_ERR_UNSUPPORTED),
    ("num_q_heads", 30, tq.TQ_ERR_INVALID_ARG), ("num_q_heads", 8 * 32, tq.TQ_ERR_UNSUPPORTED),
    ("k_bits", 5, tq.TQ_ERR_INVALID_ARG), ("v_bits", 1, tq.TQ_ERR_INVALID_ARG),
    ("qjl_dims", 48, tq.TQ_ERR_INVALID_ARG), ("qjl_dims", 512, tq.TQ_ERR_INVALID_ARG),
    ("k_mode", 3, tq.TQ_ERR_INVALID_ARG), ("sm_scale", -1.0, tq.TQ_ERR_INVALID_ARG),
    ("sparse_v_threshold", 1.5, tq.TQ_ERR_INVALID_ARG), ("flags", 0x2, tq.TQ_ERR_INVALID_ARG),
    ("reserved", 1, tq.TQ_ERR_INVALID_ARG),
])
def test_params_validation(field, value, status):
    p = tq.make_params(128, 32, 8)
    setattr(p, field, value)
    sizes = (ctypes.c_size_t * 6)()
    assert tq.library().tq_cache_bytes(ctypes.byref(p), 1, 16, ctypes.byref(sizes)) == status


def test_qjl_requires_turbo_keys():
    p = tq.make_params(128, 8, 8, k_mode=tq.TQ_MODE_INT8, qjl_dims=64)
    sizes = (ctypes.c_size_t * 6)()
    assert tq.library().tq_cache_bytes(ctypes.byref(p), 1, 16, ctypes.byref(sizes)) == tq.TQ_ERR_INVALID_ARG


def test_entry_points_reject_bad_arguments_before_launch():
    """Host validation runs before any CUDA call, so these need no GPU."""
    lib = tq.library()
    p = tq.make_params(128, 32, 8)
    kcb, vcb = tq.tq_codebook_init(128, 4), tq.tq_codebook_init(128, 2)
    fake = 1 << 20  # never dereferenced: every call below fails validation first
    cache = tq.tq_cache(1, 64, fake, fake, None, None, fake, fake, None)
    args = (ctypes.byref(p), ctypes.byref(kcb), ctypes.byref(vcb))
    # null inputs
    assert lib.tq_quantize_append(*args, None, fake, tq.TQ_BF16, 1, fake, ctypes.byref(cache), None, None) == \
        tq.TQ_ERR_INVALID_ARG
    # misaligned input
    assert lib.tq_quantize_append(*args, fake + 2, fake, tq.TQ_BF16, 1, fake, ctypes.byref(cache), None, None) == \
        tq.TQ_ERR_ALIGNMENT
    # more new tokens than the cache holds
    assert lib.tq_quantize_append(*args, fake, fake, tq.TQ_BF16, 65, fake, ctypes.byref(cache), None, None) == \
        tq.TQ_ERR_CAPACITY
    # codebook of the wrong width
    assert lib.tq_quantize_append(ctypes.byref(p), ctypes.byref(vcb), ctypes.byref(vcb), fake, fake, tq.TQ_BF16, 1,
                                  fake, ctypes.byref(cache), None, None) == tq.TQ_ERR_INVALID_ARG
    # misaligned cache array
    bad = tq.tq_cache(1, 64, fake + 4, fake, None, None, fake, fake, None)
    assert lib.tq_quantize_append(*args, fake, fake, tq.TQ_BF16, 1, fake, ctypes.byref(bad), None, None) == \
        tq.TQ_ERR_ALIGNMENT
    # QJL on without its arrays
    pq = tq.make_params(128, 32, 8, k_bits=3, qjl_dims=64)
    k3 = tq.tq_codebook_init(128, 3)
    assert lib.tq_quantize_append(ctypes.byref(pq), ctypes.byref(k3), ctypes.byref(vcb), fake, fake, tq.TQ_BF16, 1,
                                  fake, ctypes.byref(cache), None, None) == tq.TQ_ERR_INVALID_ARG
    # dequantize range outside the cache
    assert lib.tq_dequantize(*args, ctypes.byref(cache), 0, 60, 8, fake, fake, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_dequantize(*args, ctypes.byref(cache), 1, 0, 8, fake, fake, None) == tq.TQ_ERR_INVALID_ARG
    # decode: null workspace, bad max length, misaligned output
    assert lib.tq_decode_attention(*args, fake, tq.TQ_BF16, ctypes.byref(cache), fake, 64, fake, None, 0, None, None,
                                   None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention(*args, fake, tq.TQ_BF16, ctypes.byref(cache), fake, 0, fake, fake, 1 << 20, None,
                                   None, None) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_decode_attention(*args, fake, tq.TQ_BF16, ctypes.byref(cache), fake, 64, fake + 8, fake, 1 << 20,
                                   None, None, None) == tq.TQ_ERR_ALIGNMENT
    # a skip mask that is not 4-byte aligned
    assert lib.tq_decode_attention(*args, fake, tq.TQ_BF16, ctypes.byref(cache), fake, 64, fake, fake, 1 << 20,
                                   fake + 2, None, None) == tq.TQ_ERR_ALIGNMENT
    # error-word reader
    word = ctypes.c_uint32()
    assert lib.tq_read_device_error(None, ctypes.byref(word), None, 10) == tq.TQ_ERR_INVALID_ARG


def test_append_decode_rejects_bad_arguments_before_launch():
    lib = tq.library()
    p = tq.make_params(128, 32, 8)
    kcb, vcb = tq.tq_codebook_init(128, 4), tq.tq_codebook_init(128, 2)
    fake = 1 << 20
    cache = tq.tq_cache(1, 64, fake, fake, None, None, fake, fake, None)
    args = (ctypes.byref(p), ctypes.byref(kcb), ctypes.byref(vcb))
    tail = (fake, tq.TQ_BF16, ctypes.byref(cache), fake, 64, fake, fake, 1 << 20, None, None, None)
    assert lib.tq_append_decode_attention(*args, None, fake, tq.TQ_BF16, *tail) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_append_decode_attention(*args, fake, None, tq.TQ_BF16, *tail) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_append_decode_attention(*args, fake + 4, fake, tq.TQ_BF16, *tail) == tq.TQ_ERR_ALIGNMENT
    assert lib.tq_append_decode_attention(*args, fake, fake, 7, *tail) == tq.TQ_ERR_INVALID_ARG


def test_paged_entry_points_reject_bad_arguments_before_launch():
    """Block-table checks (block size a multiple of 16, a table, at least one
    sequence and block) and the paged capacity run before any CUDA call."""
    lib = tq.library()
    p = tq.make_params(128, 32, 8)
    kcb, vcb = tq.tq_codebook_init(128, 4), tq.tq_codebook_init(128, 2)
    fake = 1 << 20
    pool = tq.tq_cache(8, 64, fake, fake, None, None, fake, fake, None)  # 8 blocks of 64 tokens
    table = tq.tq_block_table(fake, 2, 4)                                  # 2 sequences x 4 blocks
    args = (ctypes.byref(p), ctypes.byref(kcb), ctypes.byref(vcb))

    def append(pool_, table_, n_new=1):
        return lib.tq_quantize_append_paged(*args, fake, fake, tq.TQ_BF16, n_new, fake, ctypes.byref(pool_),
                                            table_ and ctypes.byref(table_), None, None)

    def decode(pool_, table_):
        return lib.tq_decode_attention_paged(*args, fake, tq.TQ_BF16, ctypes.byref(pool_),
                                             table_ and ctypes.byref(table_), fake, 64, fake, None, 0, None, None, None)

    assert append(pool, None) == tq.TQ_ERR_INVALID_ARG
    assert append(pool, tq.tq_block_table(None, 2, 4)) == tq.TQ_ERR_INVALID_ARG
    assert append(pool, tq.tq_block_table(fake, 0, 4)) == tq.TQ_ERR_INVALID_ARG
    assert append(pool, tq.tq_block_table(fake, 2, 0)) == tq.TQ_ERR_INVALID_ARG
    assert append(tq.tq_cache(8, 24, fake, fake, None, None, fake, fake, None), table) == tq.TQ_ERR_INVALID_ARG
    # a sequence holds max_blocks * block_size = 256 tokens
    assert append(pool, table, n_new=257) == tq.TQ_ERR_CAPACITY
    assert decode(pool, None) == tq.TQ_ERR_INVALID_ARG
    assert decode(tq.tq_cache(8, 8, fake, fake, None, None, fake, fake, None), table) == tq.TQ_ERR_INVALID_ARG
    # null workspace
    assert decode(pool, table) == tq.TQ_ERR_INVALID_ARG
    assert lib.tq_append_decode_attention_paged(*args, None, fake, tq.TQ_BF16, fake, tq.TQ_BF16,
                                                ctypes.byref(pool), ctypes.byref(table), fake, 64, fake, fake,
                                                1 << 20, None, None, None) == tq.TQ_ERR_INVALID_ARG


def test_binding_constants_match_the_header():
    """Status codes, modes, dtypes, device-error bits and flags: the binding's
    numbers are the header's."""
    with open(os.path.join(ROOT, "include", "tq.h"), encoding="utf-8") as fh:
        text = fh.read()
    defines = {m.group(1): int(m.group(2), 16) for m in re.finditer(r"#define (TQ_[A-Z_]+) (0x[0-9a-fA-F]+)u", text)}
    enums = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(TQ_[A-Z0-9_]+) = (\d+)", text)}
    for name in ("TQ_DEVERR_POSITION", "TQ_DEVERR_SEQLEN", "TQ_DEVERR_TIMEOUT", "TQ_DEVERR_PAGE",
                 "TQ_PARAM_PREFETCH_EARLY"):
        assert getattr(tq, name) == defines[name], name
    for name in ("TQ_OK", "TQ_ERR_INVALID_ARG", "TQ_ERR_UNSUPPORTED", "TQ_ERR_CAPACITY", "TQ_ERR_CUDA",
                 "TQ_ERR_TIMEOUT", "TQ_ERR_DEVICE", "TQ_ERR_ALIGNMENT", "TQ_MODE_TURBO", "TQ_MODE_INT8",
                 "TQ_F32", "TQ_BF16", "TQ_F16"):
        assert getattr(tq, name) == enums[name], name
