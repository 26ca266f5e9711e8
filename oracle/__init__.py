"""CPU fp64 oracle for streaming sparse decode attention -- TEST INFRASTRUCTURE.

Only tests/, the smoke check in __graft_entry__ and the CPU-baseline leg of
bench.py may import this package.  The library never does: it has no CPU
fallback.  The numeric work lives in oracle.c (plain C, fp64, OpenMP over
independent units); this module marshals numpy arrays and builds the key sets
each option attends, following the pages:

* full traversal           -- every token of the sequence
* ART traversal            -- block 0 first, then the caller's order
                              ("ART" 2.4: attention sinks, orthogonal order)
* sink + recent window     -- tokens [0, sink) U [L - recent, L)
                              ("Flux Attention" 2: sparse layers keep minimal KV;
                              "Pulsar Attention" Phase 1: 64-token sink prefix)
* selected clusters        -- the union of the chosen clusters' key ranges
                              ("Squeezed Attention" Q2, steps 2-3)
* causal query chunk       -- chunk token t sees the context and chunk keys 0..t
* shard merge              -- "Pulsar Attention" Phase 2
* layer routing            -- "Flux Attention" 2 (Layer Router: prefix and
                              suffix pooling of the query tensor, hard routing)
* shared-context selection -- "Squeezed Attention" Q1 (one fixed context,
                              clustered once, shared by every request)
* lookahead block choice   -- "SparDA" 2 (Forecast projection, then the top-k
                              blocks by the projection's dot product with each
                              block's summary)
* two-level selection      -- "Squeezed Attention" Q2 step 4 (hierarchical
                              clustering: coarse clusters first, then the fine
                              clusters inside the chosen coarse ones)

Parity pins for every function are in tests/test_oracle_pins.py.
"""
import ctypes
import os

import numpy as np

from . import _build

_LIB = None
_p = ctypes.c_void_p


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(_build.SO) or os.path.getmtime(_build.SO) < os.path.getmtime(
                os.path.join(_build.HERE, "oracle.c")):
            _build.build()
        L = ctypes.CDLL(_build.SO)
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.orc_attend.argtypes = [i64, i32, i32, _p, _p, _p, i64, _p, _p, i64, dbl, _p, _p]
        L.orc_art_metrics.argtypes = [_p, _p, i32, _p, _p]
        L.orc_art_stop.argtypes = [_p, i32, i32, dbl, dbl, i32, _p]
        L.orc_art_stop.restype = i32
        L.orc_art.argtypes = [i64, i32, i32, _p, _p, _p, i64, _p, i32, _p, _p, i64, dbl, dbl, dbl,
                              i32, i32, _p, _p, _p, _p, _p]
        L.orc_select.argtypes = [i64, i32, i32, _p, _p, i32, i32, _p, _p]
        L.orc_max_threads.restype = i32
        L.orc_set_threads.argtypes = [i32]
        L.orc_merge.argtypes = [i32, i64, i32, _p, _p, _p, _p]
        L.orc_forecast.argtypes = [i64, i32, _p, _p, _p]
        _LIB = L
    return _LIB


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


# --------------------------------------------------------------------------- key sets

def keys_full(L):
    return np.arange(L, dtype=np.int64)


def keys_window(L, sink, recent):
    """Tokens [0, sink) U [L - recent, L), as one sorted set (overlap counted once)."""
    s = set(range(min(sink, L)))
    s.update(range(max(0, L - recent), L))
    return np.array(sorted(s), dtype=np.int64)


def keys_segments(starts, ends):
    """Union of token ranges [starts[i], ends[i])."""
    s = set()
    for a, b in zip(starts, ends):
        s.update(range(int(a), int(b)))
    return np.array(sorted(s), dtype=np.int64)


def keys_chunk(L_ctx, t):
    """Chunk token t (0-based) sees context keys [0, L_ctx) and chunk keys 0..t."""
    return np.arange(L_ctx + t + 1, dtype=np.int64)


def art_traversal(nb, order=None):
    """ART traversal: block 0 first ("ART" 2.4), then `order` without block 0.

    order=None means recency-first: nb-1, nb-2, ..., 1."""
    if order is None:
        order = list(range(nb - 1, -1, -1))
    return np.array([0] + [int(j) for j in order if int(j) != 0], dtype=np.int32)


# --------------------------------------------------------------------------- numeric entry points

def attend(q, K, V, idx, scale):
    """Plain softmax attention.  q [U][nq][d] bf16 bits; K, V [U][Lk][d];
    idx: list (per unit) of lists (per query row) of key index arrays.
    Returns O [U][nq][d], lse [U][nq] (fp64)."""
    q, K, V = _u16(q), _u16(K), _u16(V)
    U, nq, d = q.shape
    Lk = K.shape[1]
    stride = max(1, max(len(r) for u in idx for r in u))
    I = np.zeros((U, nq, stride), dtype=np.int64)
    M = np.zeros((U, nq), dtype=np.int64)
    for u in range(U):
        for r in range(nq):
            n = len(idx[u][r])
            I[u, r, :n] = idx[u][r]
            M[u, r] = n
    O = np.empty((U, nq, d), dtype=np.float64)
    lse = np.empty((U, nq), dtype=np.float64)
    lib().orc_attend(U, nq, d, _ptr(q), _ptr(K), _ptr(V), Lk, _ptr(I), _ptr(M), stride, scale,
                     _ptr(O), _ptr(lse))
    return O, lse


def art_metrics(x_prev, x):
    a = np.ascontiguousarray(x_prev, dtype=np.float64)
    b = np.ascontiguousarray(x, dtype=np.float64)
    ds, dc = ctypes.c_double(), ctypes.c_double()
    lib().orc_art_metrics(_ptr(a), _ptr(b), a.size, ctypes.byref(ds), ctypes.byref(dc))
    return ds.value, dc.value


def art_stop(x, tau, phi, patience):
    """Stopping rule on a probe trajectory x [T][n] -> (blocks consumed, min margin)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    mg = ctypes.c_double()
    c = lib().orc_art_stop(_ptr(x), x.shape[0], x.shape[1], tau, phi, patience, ctypes.byref(mg))
    return c, mg.value


def art(q, K, V, Ls, bs, blocks, scale, tau, phi, patience, n_probe=8, forced=None):
    """Sequential ART per query head.  q [U][G][d]; K, V [U][Lk][d]; Ls [U];
    blocks: list (per unit) of traversal arrays.  forced: None or int [U][G].
    Returns O [U][G][d], lse [U][G], consumed [U][G], margin [U][G]."""
    q, K, V = _u16(q), _u16(K), _u16(V)
    U, G, d = q.shape
    Lk = K.shape[1]
    stride = max(1, max(len(b) for b in blocks))
    Bl = np.zeros((U, stride), dtype=np.int32)
    nb = np.zeros(U, dtype=np.int32)
    for u in range(U):
        Bl[u, :len(blocks[u])] = blocks[u]
        nb[u] = len(blocks[u])
    Ls = np.ascontiguousarray(Ls, dtype=np.int64)
    fo = None if forced is None else np.ascontiguousarray(forced, dtype=np.int32)
    O = np.empty((U, G, d))
    lse = np.empty((U, G))
    cons = np.empty((U, G), dtype=np.int32)
    mg = np.empty((U, G))
    lib().orc_art(U, G, d, _ptr(q), _ptr(K), _ptr(V), Lk, _ptr(Ls), bs, _ptr(Bl), _ptr(nb), stride,
                  scale, tau, phi, patience, n_probe, _ptr(fo), _ptr(O), _ptr(lse), _ptr(cons), _ptr(mg))
    return O, lse, cons, mg


def select(q, cent, k):
    """Centroid top-k per unit.  q [U][G][d]; cent [U][C][d].  Returns ids [U][k]
    (ascending) and all scores [U][C] (fp64)."""
    q, cent = _u16(q), _u16(cent)
    U, G, d = q.shape
    C = cent.shape[1]
    ids = np.empty((U, k), dtype=np.int32)
    sc = np.empty((U, C))
    lib().orc_select(U, G, d, _ptr(q), _ptr(cent), C, k, _ptr(ids), _ptr(sc))
    return ids, sc


def select_shared(q, cent, k):
    """Centroid top-k for a batch of requests over ONE shared fixed context
    ("Squeezed Attention" Q1: the fixed context is clustered offline once and
    reused by every request; Q2 step 2 per request): request u's selection is
    the per-sequence selection of select() with its own query against the
    shared centroids.  q [U][G][d]; cent [C][d] (bf16 bits).  Returns ids
    [U][k] (ascending) and scores [U][C] (fp64)."""
    q = _u16(q)
    cent = _u16(cent)
    U = q.shape[0]
    return select(q, np.broadcast_to(cent, (U,) + cent.shape), k)


def forecast(x, w):
    """Forecast projection ("SparDA" 2: one Forecast head per GQA group maps
    layer l's activation to the query that ranks layer l+1's KV blocks):
    f[u][j] = bf16(sum_i w[u][i][j] x[u][i]) with the sum in fp32, one fused
    multiply-add per term in ascending i, rounded to nearest even.
    x [U][d], w [U][d][d] (input dim major), bf16 bits.  Returns f [U][d] bits."""
    x, w = _u16(x), _u16(w)
    U, d = x.shape
    f = np.empty((U, d), dtype=np.uint16)
    lib().orc_forecast(U, d, _ptr(x), _ptr(w), _ptr(f))
    return f


def keys_blocks(ids, L, bs=64):
    """Token set of logical blocks `ids` of a sequence of L tokens (the keys a
    layer attends once its chosen blocks are fetched)."""
    s = set()
    for j in ids:
        if int(j) >= 0:
            s.update(range(int(j) * bs, min((int(j) + 1) * bs, L)))
    return np.array(sorted(s), dtype=np.int64)


def select2(q, coarse, coarse_off, fine, k1, k2):
    """Two-level centroid selection ("Squeezed Attention" Q2 step 4,
    hierarchical clustering).  Per unit: pick the k1 best coarse clusters by
    select(); their fine clusters (coarse cluster i owns the fine clusters
    coarse_off[i] .. coarse_off[i+1] - 1) are the candidates; pick the
    min(k2, #candidates) best candidates by select() over the candidates'
    centroids.  Ties go to the lower index at both levels.
      q [U][G][d], coarse [U][C1][d], fine [U][C][d] (bf16 bits);
      coarse_off [U][C1 + 1] (int).
    Returns fine ids [U][k2], ascending, then -1 for unused slots."""
    q, coarse, fine = _u16(q), _u16(coarse), _u16(fine)
    U = q.shape[0]
    out = np.full((U, k2), -1, dtype=np.int32)
    for u in range(U):
        ids1, _ = select(q[u:u + 1], coarse[u:u + 1], k1)
        cand = np.concatenate([np.arange(coarse_off[u][i], coarse_off[u][i + 1]) for i in ids1[0]]
                              + [np.zeros(0, dtype=np.int64)]).astype(np.int64)
        if cand.size == 0:
            continue
        kk = min(k2, cand.size)
        local, _ = select(q[u:u + 1], fine[u:u + 1, cand], kk)
        out[u, :kk] = cand[local[0]]
    return out


def merge(o_parts, lse_parts):
    """Exact LSE merge.  o_parts [S][N][d], lse_parts [S][N] -> O [N][d], lse [N]."""
    o = np.ascontiguousarray(o_parts, dtype=np.float64)
    l = np.ascontiguousarray(lse_parts, dtype=np.float64)
    S, N, d = o.shape
    out = np.empty((N, d))
    lse = np.empty(N)
    lib().orc_merge(S, N, d, _ptr(o), _ptr(l), _ptr(out), _ptr(lse))
    return out, lse


def topk_boundary_gap(scores, k):
    """Relative gap between the k-th and (k+1)-th best score of each unit
    (ranking by score desc, index asc); +inf when k >= C."""
    out = []
    for s in np.atleast_2d(scores):
        C = s.shape[0]
        if k >= C:
            out.append(np.inf)
            continue
        order = sorted(range(C), key=lambda i: (-s[i], i))
        a, b = s[order[k - 1]], s[order[k]]
        out.append(abs(a - b) / max(abs(a), 1e-300))
    return np.array(out)


def _bf16_values(bits):
    """bf16 bit patterns -> float64 values (the upper half of an fp32)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def route(q, w, bias, n_prefix, n_suffix):
    """Flux-style layer routing ("Flux Attention" 2, Layer Router): the start
    and end tokens of each layer's query tensor are pooled (mean over the
    first n_prefix and the last n_suffix tokens), a linear map of the two
    pooled vectors gives the layer's logit, and inference routes hard: full
    attention where the logit is above zero.
      q     bf16 bits [L][B][T][F] (F = q_heads * head_dim, a query row)
      w     [L][2F] weights (prefix features first), bias [L]
    Returns the logits z [L][B] (fp64) and the route bits [L][B] (1 = full)."""
    x = _bf16_values(q)
    T = x.shape[2]
    prefix = x[:, :, :n_prefix, :].mean(axis=2)
    suffix = x[:, :, T - n_suffix:, :].mean(axis=2)
    f = np.concatenate([prefix, suffix], axis=-1)  # [L][B][2F]
    z = np.einsum("lbf,lf->lb", f, np.asarray(w, dtype=np.float64)) + np.asarray(bias, dtype=np.float64)[:, None]
    return z, (z > 0).astype(np.uint8)


def threads():
    """OpenMP threads the oracle's loops use."""
    return int(lib().orc_max_threads())


def set_threads(n):
    """Use n threads from now on (for timing the oracle on one core)."""
    lib().orc_set_threads(int(n))
