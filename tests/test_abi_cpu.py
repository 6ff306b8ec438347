"""CPU checks of the C ABI: the library loads, exports every symbol that
include/rcx.h declares, and rejects bad arguments before launching anything."""

import ctypes
import os
import re

import numpy as np
import pytest

from rope_context_extension_scaled_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "rcx.h")


def declared_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(rcx_\w+)\s*\(", txt, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("rcx_rope_freqs", "rcx_rope_apply", "rcx_attn_blockwise_fwd", "rcx_merge_partials"):
        assert n in names
    assert set(names) == set(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
        assert ctypes.cast(getattr(lib, n), ctypes.c_void_p).value


def test_release_staging_without_pools_is_a_no_op(lib):
    # no host-buffer call has run in this process: nothing to trim, no CUDA call
    assert lib.rcx_release_staging() == 0


def test_version_and_status_strings(lib):
    assert lib.rcx_abi_version() == 100
    assert _lib.status_string(0) == "ok"
    assert "misaligned" in _lib.status_string(-3)


def test_argument_errors_return_before_launch(lib):
    null = _lib.RcxTensor()
    one = (ctypes.c_double * 64)(*([1.0] * 64))
    # no inv_freq
    assert lib.rcx_rope_apply(null, null, null, null, None, 0, None, None) == _lib.RCX_ERR_INVALID_ARG
    # null tensors
    assert lib.rcx_attn_blockwise_fwd(null, null, null, null, null, 0, 0, 0, 1.0, 0, 0, None, 0, one, 0,
                                      None) == _lib.RCX_ERR_INVALID_ARG
    assert lib.rcx_merge_partials(null, null, null, null, null, null, None) == _lib.RCX_ERR_INVALID_ARG
    assert lib.rcx_ring_attn_fwd(null, null, null, null, null, 0, 0, 0, 1.0, None, 0, None, 0, None, 0,
                                 None) == _lib.RCX_ERR_INVALID_ARG
    st = ctypes.c_int(0)
    assert lib.rcx_device_status(None, None) == _lib.RCX_ERR_INVALID_ARG
    assert lib.rcx_debug_inject_wait_timeout(-1) == _lib.RCX_ERR_INVALID_ARG


def _host_tensor(ptr, dtype, shape, stride):
    t = _lib.RcxTensor()
    t.ptr, t.dtype = ptr, dtype
    for i in range(4):
        t.shape[i], t.stride[i] = shape[i], stride[i]
    return t


def test_attention_shape_and_flag_checks(lib):
    buf = (ctypes.c_uint8 * 4096)()
    p = ctypes.addressof(buf)
    q = _host_tensor(p, _lib.RCX_BF16, (1, 4, 3, 128), (1536, 384, 128, 1))   # Hq = 3
    k = _host_tensor(p, _lib.RCX_BF16, (1, 4, 2, 128), (1024, 256, 128, 1))   # Hkv = 2 does not divide
    lse = _lib.RcxTensor()
    f = (ctypes.c_double * 64)()
    assert lib.rcx_attn_blockwise_fwd(q, k, k, q, lse, 0, 0, 0, 1.0, 0, 0, None, 0, f, 0, None) == \
        _lib.RCX_ERR_INVALID_ARG
    bad = _host_tensor(p, _lib.RCX_BF16, (1, 4, 2, 128), (1024, 256, 128, 2))   # d not unit stride
    assert lib.rcx_attn_blockwise_fwd(bad, bad, bad, bad, lse, 0, 0, 0, 1.0, 0, 0, None, 0, f, 0, None) == \
        _lib.RCX_ERR_INVALID_ARG
    q2 = _host_tensor(p, _lib.RCX_BF16, (1, 4, 2, 128), (1024, 256, 128, 1))
    # temperature must be positive; unknown rope flag bits rejected
    assert lib.rcx_attn_blockwise_fwd(q2, q2, q2, q2, lse, 0, 0, 0, 0.0, 0, 0, None, 0, f, 0, None) == \
        _lib.RCX_ERR_INVALID_ARG
    assert lib.rcx_attn_blockwise_fwd(q2, q2, q2, q2, lse, 0, 0, 0, 1.0, 0, 0, None, 0, f, 8, None) == \
        _lib.RCX_ERR_INVALID_ARG
    # rope requested without frequencies
    assert lib.rcx_attn_blockwise_fwd(q2, q2, q2, q2, lse, 0, 0, 0, 1.0, 0, 0, None, 0, None, 1, None) == \
        _lib.RCX_ERR_INVALID_ARG


def test_ring_workspace_size_is_deterministic(lib):
    buf = (ctypes.c_uint8 * 16)()
    p = ctypes.addressof(buf)
    N, Hq, Hkv, D = 1 << 20, 64, 8, 128
    q = _host_tensor(p, _lib.RCX_BF16, (1, N, Hq, D), (N * Hq * D, Hq * D, D, 1))
    k = _host_tensor(p, _lib.RCX_BF16, (1, N, Hkv, D), (N * Hkv * D, Hkv * D, D, 1))
    n0 = lib.rcx_ring_workspace_size(q, k, 65536, 0)
    n1 = lib.rcx_ring_workspace_size(q, k, 65536, _lib.ROTATE_K)
    # fp32 accumulator + its LSE (+ rotated K); later blocks merge into the
    # accumulator in the attention epilogue, so there is no partial buffer
    assert n0 == N * Hq * D * 4 + Hq * N * 4
    assert n1 == n0 + N * Hkv * D * 2


def test_int8_cache_argument_checks(lib):
    """The int8 KV-cache entry points reject wrong dtypes and shapes before any launch."""
    fake = 1 << 20   # never dereferenced: every case fails validation first
    x = _host_tensor(fake, _lib.RCX_BF16, (1, 16, 2, 128), (4096, 256, 128, 1))
    c8 = _host_tensor(fake, _lib.RCX_I8, (1, 16, 2, 128), (4096, 256, 128, 1))
    c_bf = _host_tensor(fake, _lib.RCX_BF16, (1, 16, 2, 128), (4096, 256, 128, 1))
    c_bad = _host_tensor(fake, _lib.RCX_I8, (1, 15, 2, 128), (4096, 256, 128, 1))
    x32 = _host_tensor(fake, _lib.RCX_F32, (1, 16, 2, 128), (4096, 256, 128, 1))
    x64 = _host_tensor(fake, _lib.RCX_BF16, (1, 16, 2, 64), (2048, 128, 64, 1))
    sc = ctypes.c_void_p(fake)
    assert lib.rcx_kv_quantize_int8(x, c_bf, sc, None) == _lib.RCX_ERR_INVALID_ARG    # codes not int8
    assert lib.rcx_kv_quantize_int8(x, c_bad, sc, None) == _lib.RCX_ERR_INVALID_ARG   # shape mismatch
    assert lib.rcx_kv_quantize_int8(x32, c8, sc, None) == _lib.RCX_ERR_UNSUPPORTED    # fp32 cache
    assert lib.rcx_kv_quantize_int8(x64, c8, sc, None) == _lib.RCX_ERR_UNSUPPORTED    # d != 128
    assert lib.rcx_kv_quantize_int8(x, c8, None, None) == _lib.RCX_ERR_INVALID_ARG    # no scale buffer
    q = _host_tensor(fake, _lib.RCX_BF16, (1, 1, 8, 128), (1024, 1024, 128, 1))
    null = _lib.RcxTensor()
    assert lib.rcx_attn_decode_int8_workspace_size(q, c_bf) == -1                     # bf16 k
    # bf16 cache passed to the int8 entry point, and int8 cache to the bf16 one
    assert lib.rcx_attn_decode_int8_fwd(q, c_bf, sc, c_bf, sc, q, null, 0, 0, 1.0, 15, None, 0, None, 0, None, 0,
                                        None) == _lib.RCX_ERR_INVALID_ARG
    assert lib.rcx_attn_decode_fwd(q, c8, c8, q, null, 0, 0, 1.0, 15, None, 0, None, 0, None, 0,
                                   None) == _lib.RCX_ERR_INVALID_ARG
    # missing scales
    assert lib.rcx_attn_decode_int8_fwd(q, c8, None, c8, sc, q, null, 0, 0, 1.0, 15, None, 0, None, 0, None, 0,
                                        None) == _lib.RCX_ERR_INVALID_ARG
