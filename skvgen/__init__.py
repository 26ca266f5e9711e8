"""Seeded synthetic inputs for streaming sparse decode attention.

Serves both sides of every parity check: ``host_*`` functions return numpy
arrays in logical (token-major, per KV group) layout for the CPU oracle, and
``device_*`` functions fill torch CUDA tensors (the paged K/V pool) with the
same bits.  The module holds no attention arithmetic: only the random numbers
and the workload recipe (see ``core.h``).

bf16 tensors travel as raw uint16 bit patterns on the host side.
"""
import ctypes
import os

import numpy as np

from . import _build

_HOST = None
_DEV = None

S_Q, S_K, S_V, S_CENTER, S_ASSIGN, S_PERM, S_HEAVY, S_ROUTE, S_ROUTER_W = 1, 2, 3, 4, 5, 6, 7, 8, 9
S_FORECAST_W = 12  # Forecast projection weights (lookahead block selection)

_u64, _u32, _i32, _i64, _p = ctypes.c_uint64, ctypes.c_uint32, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data)


def host_lib():
    global _HOST
    if _HOST is None:
        if not os.path.exists(_build.HOST_SO):
            _build.build(device=False)
        lib = ctypes.CDLL(_build.HOST_SO)
        lib.skvg_host_normal_bf16.argtypes = [_u64, _u32, _u32, _u64, _u64, _p]
        lib.skvg_host_qhat.argtypes = [_p, ctypes.c_int, ctypes.c_int, _p]
        lib.skvg_host_kv_group.argtypes = [_u64, _u32, _u64, _u64, _u64, _u64, ctypes.c_int, _p, _p, _p]
        lib.skvg_host_mixture_offsets.argtypes = [_u64, _u32, _u64, _u64, _u64, _u32, _p]
        lib.skvg_host_mixture_group.argtypes = [_u64, _u32, _u64, _u64, _u64, ctypes.c_int, _u32, _p, _p, _p]
        lib.skvg_host_perm.argtypes = [_u64, _u32, _u32, _i32, _p]
        lib.skvg_host_route_bit.argtypes = [_u64, _u32]
        lib.skvg_host_route_bit.restype = ctypes.c_int
        lib.skvg_host_is_heavy.argtypes = [_u64, _u32, _u64, _u64, _u64]
        lib.skvg_host_is_heavy.restype = ctypes.c_int
        lib.skvg_host_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.skvg_host_f64_to_bf16.restype = ctypes.c_uint16
        lib.skvg_host_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.skvg_host_f32_to_bf16.restype = ctypes.c_uint16
        lib.skvg_host_block_means.argtypes = [_p, _u64, ctypes.c_int, ctypes.c_int, _p]
        lib.skvg_host_key.argtypes = [_u64, _u32, _u32]
        lib.skvg_host_key.restype = _u64
        _HOST = lib
    return _HOST


def dev_lib():
    global _DEV
    if _DEV is None:
        if not os.path.exists(_build.DEV_SO):
            raise RuntimeError("device generator library missing: run __graft_entry__.build()")
        lib = ctypes.CDLL(_build.DEV_SO)
        lib.skvg_dev_normal_bf16.argtypes = [_u64, _u32, _u32, _u64, _u64, _p, _p]
        lib.skvg_dev_qhat.argtypes = [_p] + [ctypes.c_int] * 5 + [_p, _p]
        lib.skvg_dev_kv_paged.argtypes = [_u64, _u32, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u64,
                                          _p, _p, ctypes.c_int, ctypes.c_int, _p, _p, _p, _p]
        lib.skvg_dev_mixture.argtypes = [_u64, _u32, ctypes.c_int, ctypes.c_int, ctypes.c_int, _u64, _u64,
                                         _u32, _p, ctypes.c_int, ctypes.c_int, _p, _p, _p, _p]
        lib.skvg_dev_block_means.argtypes = [_p, _p, _p] + [ctypes.c_int] * 5 + [_p, _p]
        for f in (lib.skvg_dev_normal_bf16, lib.skvg_dev_qhat, lib.skvg_dev_kv_paged, lib.skvg_dev_mixture,
                  lib.skvg_dev_block_means):
            f.restype = ctypes.c_int
        _DEV = lib
    return _DEV


# --------------------------------------------------------------------------- host side

def host_normal_bf16(seed, stream, n, base=0, layer=0):
    out = np.empty(int(n), dtype=np.uint16)
    host_lib().skvg_host_normal_bf16(seed, stream, layer, base, int(n), _ptr(out))
    return out


def host_q(wl, layer=0):
    """q of the whole workload, bf16 bits [B][Tq][Hq][d]."""
    n = wl.B * wl.Tq * wl.Hq * wl.d
    return host_normal_bf16(wl.seed, S_Q, n, layer=layer).reshape(wl.B, wl.Tq, wl.Hq, wl.d)


def host_qhat(q_group):
    """Unit vector (fp64) of the sum of a KV group's query heads, q_group [G][d]."""
    qg = np.ascontiguousarray(q_group, dtype=np.uint16)
    G, d = qg.shape
    out = np.empty(d, dtype=np.float64)
    host_lib().skvg_host_qhat(_ptr(qg), G, d, _ptr(out))
    return out


def host_kv_group(wl, b, kvh, layer=0, t0=0, n=None, q=None):
    """Logical K, V [n][d] (bf16 bits) of KV group (b, kvh), tokens [t0, t0+n)."""
    L = wl.seq_len(b)
    if n is None:
        n = L - t0
    g = b * wl.Hkv + kvh
    K = np.empty((n, wl.d), dtype=np.uint16)
    V = np.empty((n, wl.d), dtype=np.uint16)
    qhat = None
    if wl.structured:
        if q is None:
            q = host_q(wl, layer)
        G = wl.Hq // wl.Hkv
        qhat = host_qhat(q[b, 0, kvh * G:(kvh + 1) * G])
    host_lib().skvg_host_kv_group(wl.seed, layer, g, wl.Lmax, t0, n, wl.d,
                                  _ptr(qhat) if qhat is not None else None, _ptr(K), _ptr(V))
    return K, V


def host_mixture_group(wl, b, kvh, layer=0, want_keys=True):
    """Mixture keys [L][d] (cluster-contiguous), cluster offsets [C+1], centroids [C][d]."""
    g = b * wl.Hkv + kvh
    L = wl.seq_len(b)
    C = 1 << wl.c_log2
    off = np.empty(C + 1, dtype=np.int32)
    host_lib().skvg_host_mixture_offsets(wl.seed, layer, g, wl.Lmax, L, wl.c_log2, _ptr(off))
    K = np.empty((L, wl.d), dtype=np.uint16) if want_keys else None
    cent = np.empty((C, wl.d), dtype=np.uint16)
    host_lib().skvg_host_mixture_group(wl.seed, layer, g, wl.Lmax, L, wl.d, wl.c_log2, _ptr(off),
                                       _ptr(K) if K is not None else None, _ptr(cent))
    return K, off, cent


def host_block_means(K, bs=64):
    """Block summaries of one KV group's keys K [L][d] (bf16 bits): [nb][d],
    bf16 of the fp64 mean of each block's keys (the last block may be short)."""
    K = np.ascontiguousarray(K, dtype=np.uint16)
    L, d = K.shape
    out = np.empty(((L + bs - 1) // bs, d), dtype=np.uint16)
    host_lib().skvg_host_block_means(_ptr(K), L, d, bs, _ptr(out))
    return out


def host_forecast_weights(wl, layer=0):
    """Forecast projection weights of a layer, bf16 bits [Hkv][d][d]: seeded
    normals times 2^-4 (exact in bf16), untrained."""
    w = host_normal_bf16(wl.seed, S_FORECAST_W, wl.Hkv * wl.d * wl.d, layer=layer)
    v = bf16_to_f64(w) * 0.0625
    return (v.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16).reshape(wl.Hkv, wl.d, wl.d)


def host_perm(seed, n, stream=S_PERM, layer=0):
    out = np.empty(int(n), dtype=np.int32)
    host_lib().skvg_host_perm(seed, stream, layer, int(n), _ptr(out))
    return out


def route_bit(seed, layer):
    return host_lib().skvg_host_route_bit(seed, layer)


def is_heavy(wl, b, kvh, t, layer=0):
    return host_lib().skvg_host_is_heavy(wl.seed, layer, b * wl.Hkv + kvh, wl.Lmax, t)


def f64_to_bf16(x):
    return host_lib().skvg_host_f64_to_bf16(float(x))


def f32_to_bf16(x):
    return host_lib().skvg_host_f32_to_bf16(float(x))


def bf16_to_f64(bits):
    """bf16 bit patterns (uint16 array) -> float64 values."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------- device side

def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with CUDA error {rc}")


def _stream_ptr(torch):
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def device_normal_bf16(out, seed, stream, layer=0, base=0):
    import torch
    _check(dev_lib().skvg_dev_normal_bf16(seed, stream, layer, base, out.numel(),
                                          ctypes.c_void_p(out.data_ptr()), _stream_ptr(torch)),
           "skvg_dev_normal_bf16")


def device_q(wl, layer=0, device="cuda"):
    import torch
    q = torch.empty((wl.B, wl.Tq, wl.Hq, wl.d), dtype=torch.bfloat16, device=device)
    device_normal_bf16(q, wl.seed, S_Q, layer)
    return q


def device_kv_paged(wl, q, k_pool, v_pool, block_table, seq_lens, layer=0, keys=True, values=True):
    """Fill the paged pool [num_pages][Hkv][bs][d] through the block table."""
    import torch
    qhat = None
    if wl.structured and keys:
        qhat = torch.empty((wl.B * wl.Hkv, wl.d), dtype=torch.float64, device=q.device)
        _check(dev_lib().skvg_dev_qhat(ctypes.c_void_p(q.data_ptr()), wl.B, wl.Tq, wl.Hq, wl.Hkv, wl.d,
                                       ctypes.c_void_p(qhat.data_ptr()), _stream_ptr(torch)),
               "skvg_dev_qhat")
    _check(dev_lib().skvg_dev_kv_paged(
        wl.seed, layer, wl.B, wl.Hkv, wl.d, wl.Lmax, ctypes.c_void_p(seq_lens.data_ptr()),
        ctypes.c_void_p(block_table.data_ptr()), block_table.shape[1], wl.bs,
        ctypes.c_void_p(qhat.data_ptr()) if qhat is not None else None,
        ctypes.c_void_p(k_pool.data_ptr()) if keys else None,
        ctypes.c_void_p(v_pool.data_ptr()) if values else None, _stream_ptr(torch)), "skvg_dev_kv_paged")


def device_mixture(wl, k_pool, block_table, layer=0):
    """Mixture keys into the pool; returns (cluster_off [B][Hkv][C+1] int32, centroids bf16 [B][Hkv][C][d])."""
    import torch
    C = 1 << wl.c_log2
    off = torch.empty((wl.B, wl.Hkv, C + 1), dtype=torch.int32, device=k_pool.device)
    cent = torch.empty((wl.B, wl.Hkv, C, wl.d), dtype=torch.bfloat16, device=k_pool.device)
    _check(dev_lib().skvg_dev_mixture(wl.seed, layer, wl.B, wl.Hkv, wl.d, wl.Lmax, wl.L, wl.c_log2,
                                      ctypes.c_void_p(block_table.data_ptr()), block_table.shape[1], wl.bs,
                                      ctypes.c_void_p(k_pool.data_ptr()), ctypes.c_void_p(off.data_ptr()),
                                      ctypes.c_void_p(cent.data_ptr()), _stream_ptr(torch)),
           "skvg_dev_mixture")
    return off, cent


def device_block_means(wl, k_pool, block_table, seq_lens):
    """Block summaries of every (sequence, KV head) of a paged cache:
    bf16 [B][Hkv][max_blocks][d] (0 past a sequence's end)."""
    import torch
    mb = block_table.shape[1]
    out = torch.empty((wl.B, wl.Hkv, mb, wl.d), dtype=torch.bfloat16, device=k_pool.device)
    _check(dev_lib().skvg_dev_block_means(ctypes.c_void_p(k_pool.data_ptr()),
                                          ctypes.c_void_p(block_table.data_ptr()),
                                          ctypes.c_void_p(seq_lens.data_ptr()), wl.B, wl.Hkv, wl.d, mb,
                                          wl.bs, ctypes.c_void_p(out.data_ptr()), _stream_ptr(torch)),
           "skvg_dev_block_means")
    return out


def device_forecast_weights(wl, layer=0):
    """The same weights as host_forecast_weights, on the device."""
    import torch
    w = torch.empty((wl.Hkv, wl.d, wl.d), dtype=torch.bfloat16, device="cuda")
    device_normal_bf16(w, wl.seed, S_FORECAST_W, layer)
    return w * 0.0625  # a power of two: exact in bf16


def device_shared_context(wl):
    """Inputs of a shared-context workload: one context (that of request 0 of
    `wl`, a mixture) in a pool of its own pages, a block table whose B rows all
    map to those pages, and every request's own query.  Returns q [B][1][Hq][d],
    k_pool, v_pool, block_table [B][max_blocks], seq_lens [B], cluster_off
    [Hkv][C+1] and centroids [Hkv][C][d]."""
    import torch
    one = wl.with_(B=1, shared_context=False)
    bt1, num_pages = block_table_host(one)
    q = device_q(wl)
    q1 = device_q(one)
    shape = (max(num_pages, 1), wl.Hkv, wl.bs, wl.d)
    k_pool = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    v_pool = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    bt = torch.tensor(bt1, dtype=torch.int32, device="cuda")
    sl1 = torch.tensor([one.seq_len(0)], dtype=torch.int32, device="cuda")
    off, cent = device_mixture(one, k_pool, bt)
    device_kv_paged(one, q1, k_pool, v_pool, bt, sl1, keys=False)
    block_table = bt.expand(wl.B, bt.shape[1]).contiguous()
    seq_lens = sl1.expand(wl.B).contiguous()
    return q, k_pool, v_pool, block_table, seq_lens, off[0].contiguous(), cent[0].contiguous()


def host_shared_context(wl, kvh):
    """Logical keys [L][d], values [L][d], cluster offsets [C+1] and centroids
    [C][d] of KV head kvh of a shared-context workload's one context."""
    one = wl.with_(B=1, shared_context=False)
    K, off, cent = host_mixture_group(one, 0, kvh)
    _, V = host_kv_group(one.with_(mixture=False, structured=False), 0, kvh)
    return K, V, off, cent


from .workloads import Workload, WORKLOADS, block_table_host  # noqa: E402,F401
