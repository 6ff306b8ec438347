"""ctypes binding of librcx.so (include/rcx.h): argument marshalling only.

Every step of the computation runs in the library's CUDA kernels; this module
turns torch tensors into rcx_tensor views (data pointer, dtype, shape,
strides), passes the current CUDA stream, and maps status codes to
exceptions.  PyTorch provides device memory and streams.  If the library is
missing, load() raises: there is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librcx.so")

RCX_OK, RCX_ERR_INVALID_ARG, RCX_ERR_UNSUPPORTED, RCX_ERR_ALIGNMENT, RCX_ERR_CUDA, RCX_ERR_DEVICE_TIMEOUT = \
    0, -1, -2, -3, -4, -5
RCX_F32, RCX_BF16, RCX_I8 = 0, 1, 2
PLAIN, PI, NTK, DYN_NTK, NTK_PARTS, YARN = range(6)
ROTATE_Q, ROTATE_K = 1, 2

# every symbol include/rcx.h declares
EXPORTS = (
    "rcx_abi_version", "rcx_status_string", "rcx_rope_freqs", "rcx_rope_apply",
    "rcx_attn_blockwise_fwd", "rcx_merge_partials", "rcx_ring_workspace_size",
    "rcx_ring_attn_fwd", "rcx_ring_attn_fwd_host", "rcx_device_status",
    "rcx_debug_inject_wait_timeout", "rcx_stats_enable_timing", "rcx_stats_reset", "rcx_stats_read",
    "rcx_ring_attn_fwd_noalloc", "rcx_rope_freqs_per_pair", "rcx_attn_decode_workspace_size",
    "rcx_attn_decode_fwd", "rcx_kv_quantize_int8", "rcx_attn_decode_int8_workspace_size",
    "rcx_attn_decode_int8_fwd", "rcx_attn_blockwise_merge_fwd", "rcx_release_staging",
)
NOALLOC_SCRATCH_BYTES = 32 << 20   # RCX_NOALLOC_SCRATCH_BYTES in include/rcx.h
KERNEL_KINDS = {"rope_apply": 0, "attn_tc": 1, "attn_simt": 2, "merge": 3, "decode": 4}


class RcxError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


class RcxTensor(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("dtype", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


_lib = None


def load():
    """Load librcx.so (built in-tree); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is not built: run `python -m rope_context_extension_scaled_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    T = RcxTensor
    i64, f64, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
    pd = ctypes.POINTER(ctypes.c_double)
    lib.rcx_abi_version.restype = ctypes.c_int
    lib.rcx_status_string.restype = ctypes.c_char_p
    lib.rcx_status_string.argtypes = [ctypes.c_int]
    lib.rcx_rope_freqs.argtypes = [ctypes.c_int, f64, ctypes.c_int, i64, i64, f64, f64, pd, pd]
    lib.rcx_rope_apply.argtypes = [T, T, T, T, vp, i64, pd, vp]
    lib.rcx_rope_freqs_per_pair.argtypes = [f64, ctypes.c_int, pd, pd]
    lib.rcx_rope_freqs_per_pair.restype = ctypes.c_int
    lib.rcx_attn_decode_workspace_size.argtypes = [T, T]
    lib.rcx_attn_decode_workspace_size.restype = i64
    lib.rcx_attn_decode_fwd.argtypes = [T, T, T, T, T, i64, i64, f64, i64, vp, i64, pd, ctypes.c_int, vp, i64, vp]
    lib.rcx_attn_decode_fwd.restype = ctypes.c_int
    lib.rcx_kv_quantize_int8.argtypes = [T, T, vp, vp]
    lib.rcx_attn_decode_int8_workspace_size.argtypes = [T, T]
    lib.rcx_attn_decode_int8_workspace_size.restype = i64
    lib.rcx_attn_decode_int8_fwd.argtypes = [T, T, vp, T, vp, T, T, i64, i64, f64, i64, vp, i64, pd, ctypes.c_int,
                                             vp, i64, vp]
    lib.rcx_attn_decode_int8_fwd.restype = ctypes.c_int
    lib.rcx_attn_blockwise_fwd.argtypes = [T, T, T, T, T, i64, i64, i64, f64, i64, i64, vp, i64, pd,
                                           ctypes.c_int, vp]
    lib.rcx_attn_blockwise_merge_fwd.argtypes = [T, T, T, T, T, T, T, i64, i64, i64, f64, i64, i64, vp, i64, pd,
                                                 ctypes.c_int, vp]
    lib.rcx_attn_blockwise_merge_fwd.restype = ctypes.c_int
    lib.rcx_release_staging.argtypes = []
    lib.rcx_release_staging.restype = ctypes.c_int
    lib.rcx_merge_partials.argtypes = [T, T, T, T, T, T, vp]
    lib.rcx_ring_workspace_size.argtypes = [T, T, i64, ctypes.c_int]
    lib.rcx_ring_workspace_size.restype = i64
    lib.rcx_ring_attn_fwd.argtypes = [T, T, T, T, T, i64, i64, i64, f64, vp, i64, pd, ctypes.c_int, vp, i64, vp]
    lib.rcx_ring_attn_fwd_host.argtypes = [T, T, T, T, T, i64, i64, i64, f64, vp, i64, pd, ctypes.c_int, vp]
    lib.rcx_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_int)]
    lib.rcx_ring_attn_fwd_noalloc.argtypes = [T, T, T, T, T, i64, i64, i64, f64, vp, i64, pd, ctypes.c_int, vp]
    lib.rcx_ring_attn_fwd_noalloc.restype = ctypes.c_int
    lib.rcx_debug_inject_wait_timeout.argtypes = [i64]
    lib.rcx_stats_enable_timing.argtypes = [ctypes.c_int]
    lib.rcx_stats_read.argtypes = [ctypes.c_int, ctypes.POINTER(i64), ctypes.POINTER(f64)]
    for name in ("rcx_rope_freqs", "rcx_rope_apply", "rcx_attn_blockwise_fwd", "rcx_merge_partials",
                 "rcx_ring_attn_fwd", "rcx_ring_attn_fwd_host", "rcx_device_status",
                 "rcx_debug_inject_wait_timeout", "rcx_stats_enable_timing", "rcx_stats_reset",
                 "rcx_stats_read"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(st):
    return load().rcx_status_string(int(st)).decode()


def _check(st, what):
    if st != RCX_OK:
        raise RcxError(st, what)


def _dtype_code(t: torch.Tensor):
    if t.dtype == torch.float32:
        return RCX_F32
    if t.dtype == torch.bfloat16:
        return RCX_BF16
    if t.dtype == torch.int8:
        return RCX_I8
    raise TypeError(f"unsupported dtype {t.dtype}")


def view(t):
    """rcx_tensor of a [B, N, H, d] torch tensor (None -> null view)."""
    r = RcxTensor()
    if t is None:
        return r
    if t.dim() != 4:
        raise ValueError("expected a 4-D [B, N, H, d] tensor")
    r.ptr = t.data_ptr()
    r.dtype = _dtype_code(t)
    for i in range(4):
        r.shape[i] = t.shape[i]
        r.stride[i] = t.stride(i)
    return r


def lse_view(t):
    """rcx_tensor of a [B, H, N] fp32 LSE tensor (None -> null view)."""
    r = RcxTensor()
    if t is None:
        return r
    if t.dim() != 3 or t.dtype != torch.float32:
        raise ValueError("expected a 3-D [B, H, N] float32 tensor")
    r.ptr = t.data_ptr()
    r.dtype = RCX_F32
    for i in range(3):
        r.shape[i] = t.shape[i]
        r.stride[i] = t.stride(i)
    r.shape[3] = 1
    r.stride[3] = 1
    return r


def _freq_ptr(inv_freq):
    if inv_freq is None:
        return None, None
    arr = np.ascontiguousarray(np.asarray(inv_freq, dtype=np.float64))
    return arr, arr.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _pos(positions):
    if positions is None:
        return None, 0
    if positions.dtype != torch.int64:
        raise TypeError("positions must be int64")
    return ctypes.c_void_p(positions.data_ptr()), positions.numel()


# ----------------------------------------------------------------- entry points

def rope_freqs(scheme, base, d, L_train, L_target, alpha=1.0, beta=32.0):
    out = np.zeros(d // 2, dtype=np.float64)
    t = ctypes.c_double(0.0)
    st = load().rcx_rope_freqs(int(scheme), float(base), int(d), int(L_train), int(L_target), float(alpha),
                               float(beta), out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), ctypes.byref(t))
    _check(st, "rcx_rope_freqs")
    return out, t.value


def rope_freqs_per_pair(base, d, factors):
    """theta_i / factors[i] (per-plane rescaling); returns float64 [d/2]."""
    f = np.ascontiguousarray(np.asarray(factors, dtype=np.float64))
    if f.shape != (d // 2,):
        raise ValueError("need d/2 factors")
    out = np.zeros(d // 2, dtype=np.float64)
    st = load().rcx_rope_freqs_per_pair(float(base), int(d), f.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                        out.ctypes.data_as(ctypes.POINTER(ctypes.c_double)))
    _check(st, "rcx_rope_freqs_per_pair")
    return out


def rope_apply(q, k, inv_freq, positions=None, q_out=None, k_out=None):
    """Rotate q and/or k (either may be None).  Default: in place."""
    q_out = q if (q_out is None) else q_out
    k_out = k if (k_out is None) else k_out
    arr, fp = _freq_ptr(inv_freq)
    pp, npos = _pos(positions)
    dev = (q if q is not None else k).device
    st = load().rcx_rope_apply(view(q), view(k), view(q_out if q is not None else None),
                               view(k_out if k is not None else None), pp, npos, fp, _stream(dev))
    _check(st, "rcx_rope_apply")
    return q_out, k_out


def attn_blockwise_fwd(q, k, v, o=None, lse=None, kv_block=0, window=0, n_sink=0, temperature=1.0,
                       q_start=0, k_start=0, positions=None, inv_freq=None, rope_flags=0, want_lse=True,
                       out_dtype=None):
    B, N, H, D = q.shape
    if o is None:
        o = torch.empty(B, N, H, D, dtype=out_dtype or q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    arr, fp = _freq_ptr(inv_freq)
    pp, npos = _pos(positions)
    st = load().rcx_attn_blockwise_fwd(view(q), view(k), view(v), view(o), lse_view(lse), int(kv_block),
                                       int(window), int(n_sink), float(temperature), int(q_start), int(k_start),
                                       pp, npos, fp, int(rope_flags), _stream(q.device))
    _check(st, "rcx_attn_blockwise_fwd")
    return o, lse


def attn_blockwise_merge_fwd(q, k, v, o, lse, acc, acc_lse, kv_block=0, window=0, n_sink=0, temperature=1.0,
                             q_start=0, k_start=0, positions=None, inv_freq=None, rope_flags=0):
    """Attention over this call's keys merged into the partial (acc, acc_lse)
    in the kernel's epilogue; o / lse may be acc / acc_lse (in place)."""
    arr, fp = _freq_ptr(inv_freq)
    pp, npos = _pos(positions)
    st = load().rcx_attn_blockwise_merge_fwd(view(q), view(k), view(v), view(o), lse_view(lse), view(acc),
                                             lse_view(acc_lse), int(kv_block), int(window), int(n_sink),
                                             float(temperature), int(q_start), int(k_start), pp, npos, fp,
                                             int(rope_flags), _stream(q.device))
    _check(st, "rcx_attn_blockwise_merge_fwd")
    return o, lse


def merge_partials(o_a, lse_a, o_b, lse_b, o_out=None, lse_out=None):
    st = load().rcx_merge_partials(view(o_a), lse_view(lse_a), view(o_b), lse_view(lse_b), view(o_out),
                                   lse_view(lse_out), _stream(o_a.device))
    _check(st, "rcx_merge_partials")
    return (o_a, lse_a) if o_out is None else (o_out, lse_out)


def ring_workspace_size(q, k, kv_block, rope_flags):
    n = load().rcx_ring_workspace_size(view(q), view(k), int(kv_block), int(rope_flags))
    if n < 0:
        raise RcxError(RCX_ERR_INVALID_ARG, "rcx_ring_workspace_size")
    return int(n)


def ring_attn_fwd(q, k, v, o=None, lse=None, kv_block=0, window=0, n_sink=0, temperature=1.0, positions=None,
                  inv_freq=None, rope_flags=0, workspace=None, want_lse=True):
    B, N, H, D = q.shape
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, N, dtype=torch.float32, device=q.device)
    need = ring_workspace_size(q, k, kv_block, rope_flags)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    arr, fp = _freq_ptr(inv_freq)
    pp, npos = _pos(positions)
    st = load().rcx_ring_attn_fwd(view(q), view(k), view(v), view(o), lse_view(lse), int(kv_block), int(window),
                                  int(n_sink), float(temperature), pp, npos, fp, int(rope_flags),
                                  ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(q.device))
    _check(st, "rcx_ring_attn_fwd")
    return o, lse


def ring_attn_fwd_host(q, k, v, o, lse=None, kv_block=0, window=0, n_sink=0, temperature=1.0, positions=None,
                       inv_freq=None, rope_flags=0, stream=None):
    """Same as ring_attn_fwd on HOST tensors (pinned for full copy speed); synchronous."""
    arr, fp = _freq_ptr(inv_freq)
    pp, npos = (None, 0) if positions is None else (ctypes.c_void_p(positions.data_ptr()), positions.numel())
    s = ctypes.c_void_p(stream.cuda_stream if stream is not None else torch.cuda.current_stream().cuda_stream)
    st = load().rcx_ring_attn_fwd_host(view(q), view(k), view(v), view(o), lse_view(lse), int(kv_block),
                                       int(window), int(n_sink), float(temperature), pp, npos, fp, int(rope_flags), s)
    _check(st, "rcx_ring_attn_fwd_host")
    return o, lse


def release_staging():
    """Return the staging memory rcx_ring_attn_fwd_host keeps between calls."""
    _check(load().rcx_release_staging(), "rcx_release_staging")


def device_status(device=None):
    v = ctypes.c_int(0)
    _check(load().rcx_device_status(_stream(device), ctypes.byref(v)), "rcx_device_status")
    return v.value


def debug_inject_wait_timeout(spins):
    _check(load().rcx_debug_inject_wait_timeout(int(spins)), "rcx_debug_inject_wait_timeout")


def stats_enable_timing(on=True):
    _check(load().rcx_stats_enable_timing(1 if on else 0), "rcx_stats_enable_timing")


def stats_reset():
    _check(load().rcx_stats_reset(), "rcx_stats_reset")


def stats_read():
    """{kind: (launches, elapsed_ms)} for every kernel kind."""
    out = {}
    for name, k in KERNEL_KINDS.items():
        n = ctypes.c_int64(0)
        ms = ctypes.c_double(0.0)
        _check(load().rcx_stats_read(k, ctypes.byref(n), ctypes.byref(ms)), "rcx_stats_read")
        out[name] = (n.value, ms.value)
    return out


def ring_attn_fwd_noalloc(q, k, v, o, lse=None, kv_block=0, window=0, n_sink=0, temperature=1.0, positions=None,
                          inv_freq=None, rope_flags=0):
    """rcx_ring_attn_fwd_noalloc: the ring forward with the library's static
    scratch instead of a caller workspace, for callers that cannot allocate
    device memory.  o (and lse) are caller-provided; nothing is allocated."""
    arr, fp = _freq_ptr(inv_freq)
    pp, npos = _pos(positions)
    st = load().rcx_ring_attn_fwd_noalloc(view(q), view(k), view(v), view(o), lse_view(lse), int(kv_block),
                                          int(window), int(n_sink), float(temperature), pp, npos, fp,
                                          int(rope_flags), _stream(q.device))
    _check(st, "rcx_ring_attn_fwd_noalloc")
    return o, lse


def kv_quantize_int8(x, codes=None, scale=None):
    """Int8 codes [B, N, H, 128] and fp32 scales [B, H, N] (head-major) of a bf16 cache x."""
    B, N, H, _ = x.shape
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    if scale is None:
        scale = torch.empty(B, H, N, dtype=torch.float32, device=x.device)
    if not scale.is_contiguous() or scale.dtype != torch.float32 or tuple(scale.shape) != (B, H, N):
        raise ValueError("scale must be a contiguous float32 [B, H, N] tensor")
    st = load().rcx_kv_quantize_int8(view(x), view(codes), ctypes.c_void_p(scale.data_ptr()), _stream(x.device))
    _check(st, "rcx_kv_quantize_int8")
    return codes, scale


def attn_decode_int8_fwd(q, k, k_scale, v, v_scale, o=None, lse=None, window=0, n_sink=0, temperature=1.0,
                         q_index=None, positions=None, inv_freq=None, rope_flags=0, workspace=None, want_lse=True):
    """attn_decode_fwd over an int8 cache (codes k, v [B, Nk, Hkv, 128], scales [B, Hkv, Nk])."""
    B, _, H, D = q.shape
    if q_index is None:
        q_index = k.shape[1] - 1
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, 1, dtype=torch.float32, device=q.device)
    Bk, Nk, Hkv = k.shape[:3]
    for sc in (k_scale, v_scale):
        if not sc.is_contiguous() or sc.dtype != torch.float32 or tuple(sc.shape) != (Bk, Hkv, Nk):
            raise ValueError("scales must be contiguous float32 [B, Hkv, Nk] tensors")
    need = load().rcx_attn_decode_int8_workspace_size(view(q), view(k))
    if need < 0:
        raise RcxError(RCX_ERR_INVALID_ARG, "rcx_attn_decode_int8_workspace_size")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    arr, fp = _freq_ptr(inv_freq)
    pp, npos = _pos(positions)
    st = load().rcx_attn_decode_int8_fwd(view(q), view(k), ctypes.c_void_p(k_scale.data_ptr()), view(v),
                                         ctypes.c_void_p(v_scale.data_ptr()), view(o), lse_view(lse), int(window),
                                         int(n_sink), float(temperature), int(q_index), pp, npos, fp,
                                         int(rope_flags), ctypes.c_void_p(workspace.data_ptr()), workspace.numel(),
                                         _stream(q.device))
    _check(st, "rcx_attn_decode_int8_fwd")
    return o, lse


def attn_decode_fwd(q, k, v, o=None, lse=None, window=0, n_sink=0, temperature=1.0, q_index=None, positions=None,
                    inv_freq=None, rope_flags=0, workspace=None, want_lse=True):
    """One query token per (batch, head) against a KV cache k, v [B, Nk, Hkv, 128].

    q: [B, 1, Hq, 128]; q_index defaults to Nk - 1 (the newest cached token)."""
    B, _, H, D = q.shape
    if q_index is None:
        q_index = k.shape[1] - 1
    if o is None:
        o = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(B, H, 1, dtype=torch.float32, device=q.device)
    need = load().rcx_attn_decode_workspace_size(view(q), view(k))
    if need < 0:
        raise RcxError(RCX_ERR_INVALID_ARG, "rcx_attn_decode_workspace_size")
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    arr, fp = _freq_ptr(inv_freq)
    pp, npos = _pos(positions)
    st = load().rcx_attn_decode_fwd(view(q), view(k), view(v), view(o), lse_view(lse), int(window), int(n_sink),
                                    float(temperature), int(q_index), pp, npos, fp, int(rope_flags),
                                    ctypes.c_void_p(workspace.data_ptr()), workspace.numel(), _stream(q.device))
    _check(st, "rcx_attn_decode_fwd")
    return o, lse
