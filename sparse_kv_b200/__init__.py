"""sparse_kv_b200 -- Python binding of libsparsekv.so (streaming sparse decode
attention for B200 / sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/sparsekv.h.  Tensors are torch
CUDA tensors (PyTorch provides device memory and streams); there is no CPU
fallback, and importing this module raises if the compiled library is
missing.
"""
import ctypes
import math
import os

from . import _build

__all__ = ["attn_decode", "attn_decode_static_ws", "attn_select_centroids",
           "attn_select_centroids_shared", "attn_merge_lse", "attn_forecast", "attn_prefetch_blocks",
           "host_device_pointer",
           "attn_route_layers", "attn_select_centroids2",
           "decode_workspace_size", "decode_launches", "decode_plan",
           "strerror", "status_of_word", "SkvError", "lib", "DEV_BITS"]

SKV_OK, SKV_EINVAL, SKV_EUNSUPPORTED, SKV_ECUDA, SKV_ETIMEOUT, SKV_EWORKSPACE = range(6)
DEV_BITS = {"timeout": 0x1, "bad_page": 0x2, "bad_seqlen": 0x4, "bad_order": 0x8, "bad_segment": 0x10}

_p = ctypes.c_void_p
_i = ctypes.c_int


class _Art(ctypes.Structure):
    _fields_ = [("enable", _i), ("tau", ctypes.c_float), ("phi", ctypes.c_float), ("patience", _i)]


class _Window(ctypes.Structure):
    _fields_ = [("sink_tokens", _i), ("recent_tokens", _i)]


class DecodeArgs(ctypes.Structure):
    """Mirror of skv_decode_args (include/sparsekv.h)."""
    _fields_ = [
        ("q", _p), ("k_pool", _p), ("v_pool", _p), ("block_table", _p), ("seq_lens", _p),
        ("order", _p), ("order_len", _i), ("seg_start", _p), ("seg_end", _p), ("n_seg", _i),
        ("batch", _i), ("q_tokens", _i), ("q_heads", _i), ("kv_heads", _i), ("head_dim", _i),
        ("block_size", _i), ("max_blocks", _i), ("num_pages", _i), ("max_seq_len", _i),
        ("kv_begin", _i), ("kv_end", _i), ("scale", ctypes.c_float), ("art", _Art),
        ("window", _Window), ("causal", _i), ("kv_shards", _i), ("out", _p), ("lse", _p),
        ("blocks_consumed", _p),
        ("status_word", _p), ("workspace", _p), ("workspace_bytes", ctypes.c_size_t),
    ]


class SkvError(RuntimeError):
    def __init__(self, status, where):
        super().__init__(f"{where}: {strerror(status)} (status {status})")
        self.status = status


_LIB = None


def lib():
    """The loaded libsparsekv.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(_build.SO):
            raise RuntimeError(f"libsparsekv.so not found at {_build.SO}; build it with "
                               "`python -c 'import __graft_entry__ as g; g.build()'`")
        L = ctypes.CDLL(_build.SO)
        L.skv_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeArgs)]
        L.skv_decode_workspace_size.restype = ctypes.c_size_t
        L.skv_decode_launches.argtypes = [ctypes.POINTER(DecodeArgs)]
        L.skv_decode_launches.restype = ctypes.c_int
        L.skv_decode_plan_info.argtypes = [ctypes.POINTER(DecodeArgs), ctypes.POINTER(DecodePlan)]
        L.skv_decode_plan_info.restype = _i
        L.attn_decode.argtypes = [ctypes.POINTER(DecodeArgs), _p]
        L.attn_decode.restype = _i
        L.attn_decode_static_ws.argtypes = [ctypes.POINTER(DecodeArgs), _p]
        L.attn_decode_static_ws.restype = _i
        L.attn_select_centroids.argtypes = [_p, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p]
        L.attn_select_centroids.restype = _i
        L.attn_select_centroids_shared.argtypes = [_p, _p, _p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p]
        L.attn_select_centroids_shared.restype = _i
        L.attn_merge_lse.argtypes = [_p, _p, _i, _i, _i, _p, _p, _p]
        L.attn_merge_lse.restype = _i
        L.attn_route_layers.argtypes = [_p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _p, _p]
        L.attn_route_layers.restype = _i
        L.attn_select_centroids2.argtypes = [_p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p]
        L.attn_select_centroids2.restype = _i
        L.attn_forecast.argtypes = [_p, _p, _i, _i, _i, _p, _p]
        L.attn_forecast.restype = _i
        L.skv_host_device_pointer.argtypes = [_p, ctypes.POINTER(_p)]
        L.skv_host_device_pointer.restype = _i
        L.attn_prefetch_blocks.argtypes = [_p, _p, _p, _p, _p] + [_i] * 7 + [_p, _p, _p, _p, _p, _i, _p]
        L.attn_prefetch_blocks.restype = _i
        L.skv_status_of_word.argtypes = [ctypes.c_uint32]
        L.skv_status_of_word.restype = _i
        L.skv_test_withhold_tile.argtypes = [_i, _i]
        L.skv_test_withhold_tile.restype = _i
        L.skv_strerror.argtypes = [_i]
        L.skv_strerror.restype = ctypes.c_char_p
        _LIB = L
    return _LIB


def strerror(status):
    return lib().skv_strerror(int(status)).decode()


def attn_forecast(x, w, f, stream=None):
    """Forecast projection: x bf16 [B, Hkv, d], w bf16 [Hkv, d, d] (input dim
    major) -> f bf16 [B, Hkv, d] (see attn_forecast in include/sparsekv.h)."""
    B, Hkv, d = x.shape
    st = lib().attn_forecast(_ptr(x), _ptr(w), B, Hkv, d, _ptr(f), _stream(stream))
    if st != SKV_OK:
        raise SkvError(st, "attn_forecast")


def host_device_pointer(t):
    """Device-accessible address of a page-locked (pinned) host tensor."""
    p = ctypes.c_void_p()
    st = lib().skv_host_device_pointer(ctypes.c_void_p(t.data_ptr()), ctypes.byref(p))
    if st != SKV_OK:
        raise SkvError(st, "skv_host_device_pointer")
    return p


def attn_prefetch_blocks(k_host, v_host, block_table, seq_lens, block_ids, k_cache, v_cache, seg_start,
                         seg_end, *, max_seq_len, status=None, n_ctas=16, stream=None, host_ptrs=None):
    """Copy the chosen blocks from pinned host pools [P, Hkv, 64, 128] into the
    device caches [B * k, Hkv, 64, 128]; block_ids int32 [B, Hkv, k]; writes the
    cache token ranges seg_start / seg_end [B, Hkv, k] (see attn_prefetch_blocks
    in include/sparsekv.h).  host_ptrs: (k, v) from host_device_pointer, to skip
    the look-up."""
    B, Hkv, k = block_ids.shape
    P, _, _, d = k_host.shape
    kp, vp = host_ptrs if host_ptrs is not None else (host_device_pointer(k_host), host_device_pointer(v_host))
    st = lib().attn_prefetch_blocks(kp, vp, _ptr(block_table), _ptr(seq_lens), _ptr(block_ids), B, Hkv, d, k,
                                    block_table.shape[1], P, int(max_seq_len), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(seg_start), _ptr(seg_end), _ptr(status), int(n_ctas), _stream(stream))
    if st != SKV_OK:
        raise SkvError(st, "attn_prefetch_blocks")


def status_of_word(word):
    """The skv_status a device status word stands for (see skv_status_of_word)."""
    return lib().skv_status_of_word(int(word) & 0xFFFFFFFF)


def test_withhold_tile(cta, entry):
    """Test hook: the next plain decode launch's CTA `cta` withholds ring entry
    `entry`, so its bounded wait expires (see skv_test_withhold_tile)."""
    st = lib().skv_test_withhold_tile(int(cta), int(entry))
    if st != SKV_OK:
        raise SkvError(st, "skv_test_withhold_tile")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def make_decode_args(q, k_pool, v_pool, block_table, seq_lens, out, lse, *, max_seq_len,
                     scale=None, order=None, segments=None, window=None, kv_range=None, art=None,
                     causal=False, kv_shards=0, blocks_consumed=None, status=None, workspace=None):
    """Fill a DecodeArgs from tensors.

    q [B, Tq, Hq, 128] bf16; k_pool/v_pool [P, Hkv, 64, 128] bf16; block_table [B, MB]
    int32; seq_lens [B] int32; out [B, Tq, Hq, 128] fp32; lse [B, Tq, Hq] fp32.
    order: int32 [B, Hkv, n]; segments: (start, end) int32 [B, Hkv, n] each;
    window: (sink, recent); kv_range: (begin, end); art: (tau, phi, patience);
    causal / kv_shards: query chunks (q_tokens > 1), see include/sparsekv.h."""
    B, Tq, Hq, d = q.shape
    P, Hkv, bs, d2 = k_pool.shape
    a = DecodeArgs()
    a.q, a.k_pool, a.v_pool = _ptr(q), _ptr(k_pool), _ptr(v_pool)
    a.block_table, a.seq_lens = _ptr(block_table), _ptr(seq_lens)
    a.batch, a.q_tokens, a.q_heads, a.kv_heads, a.head_dim, a.block_size = B, Tq, Hq, Hkv, d, bs
    a.max_blocks = block_table.shape[1]
    a.num_pages = P
    a.max_seq_len = int(max_seq_len)
    a.scale = float(scale) if scale is not None else 1.0 / math.sqrt(d)
    if order is not None:
        a.order, a.order_len = _ptr(order), order.shape[-1]
    if segments is not None:
        a.seg_start, a.seg_end, a.n_seg = _ptr(segments[0]), _ptr(segments[1]), segments[0].shape[-1]
    if window is not None:
        a.window = _Window(int(window[0]), int(window[1]))
    if kv_range is not None:
        a.kv_begin, a.kv_end = int(kv_range[0]), int(kv_range[1])
    if art is not None:
        a.art = _Art(1, float(art[0]), float(art[1]), int(art[2]))
    a.causal = 1 if causal else 0
    a.kv_shards = int(kv_shards)
    a.out, a.lse = _ptr(out), _ptr(lse)
    a.blocks_consumed = _ptr(blocks_consumed)
    a.status_word = _ptr(status)
    if workspace is not None:
        a.workspace = _ptr(workspace)
        a.workspace_bytes = workspace.numel() * workspace.element_size()
    return a


def decode_workspace_size(*args, **kw):
    """Bytes of workspace attn_decode needs (same arguments as attn_decode)."""
    return lib().skv_decode_workspace_size(ctypes.byref(make_decode_args(*args, **kw)))


class DecodePlan(ctypes.Structure):
    """Mirror of skv_decode_plan (include/sparsekv.h)."""
    _fields_ = [("schedule", _i), ("ctas", _i), ("splits", _i), ("art_chunk_blocks", _i),
                ("art_chunks", _i), ("launches", _i), ("workspace_bytes", ctypes.c_size_t)]


SCHEDULES = {0: "persistent", 1: "cluster", 2: "art", 3: "chunk"}


def decode_plan(*args, **kw):
    """The launch plan attn_decode would follow (see skv_decode_plan_info in
    include/sparsekv.h) as a dict; raises SkvError for invalid arguments."""
    p = DecodePlan()
    st = lib().skv_decode_plan_info(ctypes.byref(make_decode_args(*args, **kw)), ctypes.byref(p))
    if st != SKV_OK:
        raise SkvError(st, "skv_decode_plan_info")
    d = {f: getattr(p, f) for f, _ in DecodePlan._fields_}
    d["schedule"] = SCHEDULES[d["schedule"]]
    return d


def decode_launches(*args, **kw):
    """Kernels one attn_decode call launches for these arguments (see
    skv_decode_launches in include/sparsekv.h)."""
    return lib().skv_decode_launches(ctypes.byref(make_decode_args(*args, **kw)))


def attn_decode(*args, stream=None, **kw):
    """Decode attention over the paged cache (see make_decode_args); raises SkvError."""
    a = make_decode_args(*args, **kw)
    st = lib().attn_decode(ctypes.byref(a), _stream(stream))
    if st != SKV_OK:
        raise SkvError(st, "attn_decode")


def attn_decode_static_ws(*args, stream=None, **kw):
    """attn_decode for callers that cannot allocate device memory: same
    arguments (any workspace is ignored), scratch taken from a fixed array in
    the library (SKV_STATIC_WORKSPACE_BYTES).  Calls share that array, so they
    must not overlap on the GPU.  Raises SkvError."""
    kw.pop("workspace", None)
    a = make_decode_args(*args, **kw)
    st = lib().attn_decode_static_ws(ctypes.byref(a), _stream(stream))
    if st != SKV_OK:
        raise SkvError(st, "attn_decode_static_ws")


def attn_decode_args(a, stream=None):
    """Launch with a prepared DecodeArgs (lowest-overhead path); returns the status."""
    return lib().attn_decode(ctypes.byref(a), _stream(stream))


def attn_select_centroids(q, centroids, cluster_off, topk, sel_ids, seg_start, seg_end, stream=None):
    """q [B, Hq, 128] bf16 (or [B, 1, Hq, 128]); centroids [B, Hkv, C, 128] bf16;
    cluster_off [B, Hkv, C+1] int32; outputs int32 [B, Hkv, topk]."""
    B, Hkv, C, d = centroids.shape
    Hq = q.shape[-2]
    st = lib().attn_select_centroids(_ptr(q), _ptr(centroids), _ptr(cluster_off), B, Hq, Hkv, d, C,
                                     int(topk), _ptr(sel_ids), _ptr(seg_start), _ptr(seg_end),
                                     _stream(stream))
    if st != SKV_OK:
        raise SkvError(st, "attn_select_centroids")


def attn_select_centroids_shared(q, centroids, cluster_off, topk, sel_ids, seg_start, seg_end,
                                 stream=None):
    """q [B, Hq, 128] bf16 (or [B, 1, Hq, 128]), one query per request; centroids
    [Hkv, C, 128] bf16 and cluster_off [Hkv, C+1] int32 shared by every request;
    outputs int32 [B, Hkv, topk]."""
    Hkv, C, d = centroids.shape
    B, Hq = q.shape[0], q.shape[-2]
    st = lib().attn_select_centroids_shared(_ptr(q), _ptr(centroids), _ptr(cluster_off), B, Hq, Hkv, d,
                                            C, int(topk), _ptr(sel_ids), _ptr(seg_start), _ptr(seg_end),
                                            _stream(stream))
    if st != SKV_OK:
        raise SkvError(st, "attn_select_centroids_shared")


def attn_merge_lse(o_parts, lse_parts, out, lse, stream=None):
    """o_parts [S, N, d] fp32, lse_parts [S, N] fp32 -> out [N, d], lse [N]."""
    S, N, d = o_parts.shape
    st = lib().attn_merge_lse(_ptr(o_parts), _ptr(lse_parts), S, N, d, _ptr(out), _ptr(lse),
                              _stream(stream))
    if st != SKV_OK:
        raise SkvError(st, "attn_merge_lse")


def attn_route_layers(q, w, bias, n_prefix, n_suffix, route, logits=None, stream=None):
    """q bf16 [L, B, T, Hq, d]; w fp32 [L, 2 * Hq * d]; bias fp32 [L] or None ->
    route uint8 [L, B] (1: full attention), logits fp32 [L, B] (optional)."""
    L, B, T, Hq, d = q.shape
    st = lib().attn_route_layers(_ptr(q), _ptr(w), _ptr(bias), L, B, T, Hq, d, int(n_prefix),
                                 int(n_suffix), _ptr(logits), _ptr(route), _stream(stream))
    if st != SKV_OK:
        raise SkvError(st, "attn_route_layers")


def attn_select_centroids2(q, coarse, coarse_off, fine, cluster_off, k1, k2, ids, seg_start, seg_end,
                           stream=None):
    """q bf16 [B, Hq, d] (or [B, 1, Hq, d]); coarse bf16 [B, Hkv, C1, d]; coarse_off int32
    [B, Hkv, C1 + 1]; fine bf16 [B, Hkv, C, d]; cluster_off int32 [B, Hkv, C + 1] ->
    ids, seg_start, seg_end int32 [B, Hkv, k2] (unused slots: id -1, empty range)."""
    B, Hkv, C1, d = coarse.shape
    C = fine.shape[2]
    Hq = q.shape[-2]
    st = lib().attn_select_centroids2(_ptr(q), _ptr(coarse), _ptr(coarse_off), _ptr(fine), _ptr(cluster_off),
                                      B, Hq, Hkv, d, C1, C, int(k1), int(k2), _ptr(ids), _ptr(seg_start),
                                      _ptr(seg_end), _stream(stream))
    if st != SKV_OK:
        raise SkvError(st, "attn_select_centroids2")
