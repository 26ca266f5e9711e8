"""Shared helpers for the GPU parity tests: device inputs from the seeded
generator, oracle inputs for sampled KV groups, and the tolerance checks.

Tolerances (fp32 GPU path vs fp64 oracle on bf16 inputs):
  O     max |O_gpu - O_ref| <= 2e-3            (values ~N(0,1))
  LSE   |lse_gpu - lse_ref| <= 1e-4 * max(1, |lse_ref|)
Integer outputs (selected ids, blocks consumed) must match exactly, except
decisions the oracle marks as near-threshold (ART margin <= 1e-3, top-k
boundary gap <= 1e-5), which are counted and re-checked against the oracle
forced to the GPU's decision.
"""
import numpy as np

import oracle
import skvgen

ATOL_O = 2e-3
RTOL_LSE = 1e-4
ART_FLAG_MARGIN = 1e-3
TOPK_FLAG_GAP = 1e-5


def device_workload(wl, layer=0, nan_fill=True, keys=True, values=True):
    """q, paged pools, block table and seq_lens on cuda for workload `wl`."""
    import torch
    bt_host, num_pages = skvgen.block_table_host(wl, layer)
    dev = "cuda"
    q = skvgen.device_q(wl, layer)
    shape = (max(num_pages, 1), wl.Hkv, wl.bs, wl.d)
    k_pool = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    v_pool = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    if nan_fill:  # rows never written stay NaN: reading them would poison the output
        k_pool.fill_(float("nan"))
        v_pool.fill_(float("nan"))
    block_table = torch.tensor(bt_host, dtype=torch.int32, device=dev)
    seq_lens = torch.tensor([wl.seq_len(b) for b in range(wl.B)], dtype=torch.int32, device=dev)
    extra = {}
    if wl.mixture:
        off, cent = skvgen.device_mixture(wl, k_pool, block_table, layer)
        skvgen.device_kv_paged(wl, q, k_pool, v_pool, block_table, seq_lens, layer, keys=False)
        extra = dict(cluster_off=off, centroids=cent)
    else:
        skvgen.device_kv_paged(wl, q, k_pool, v_pool, block_table, seq_lens, layer)
    return dict(q=q, k_pool=k_pool, v_pool=v_pool, block_table=block_table, seq_lens=seq_lens,
                bt_host=bt_host, num_pages=num_pages, **extra)


def outputs(wl, device="cuda"):
    """Output buffers filled with NaN: a row the kernels never write cannot pass
    as a stale copy of an earlier call's result."""
    import torch
    out = torch.full((wl.B, wl.Tq, wl.Hq, wl.d), float("nan"), dtype=torch.float32, device=device)
    lse = torch.full((wl.B, wl.Tq, wl.Hq), float("nan"), dtype=torch.float32, device=device)
    return out, lse


def run_decode(wl, dev, **opts):
    """Call attn_decode; returns (out [B,Hq,d], lse [B,Hq], consumed [B,Hq], status) on host."""
    import torch
    import sparse_kv_b200 as skv
    out, lse = outputs(wl)
    consumed = torch.full((wl.B, wl.Hq), -1, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = (dev["q"], dev["k_pool"], dev["v_pool"], dev["block_table"], dev["seq_lens"], out, lse)
    kw = dict(max_seq_len=opts.pop("max_seq_len", wl.Lmax), blocks_consumed=consumed, status=status,
              scale=wl.scale)
    kw.update(opts)
    n = skv.decode_workspace_size(*args, **kw)
    ws = torch.empty(max(n, 16) // 4 + 4, dtype=torch.float32, device="cuda") if n else None
    skv.attn_decode(*args, workspace=ws, **kw)
    torch.cuda.synchronize()
    return (out[:, 0].cpu().numpy().astype(np.float64), lse[:, 0].cpu().numpy().astype(np.float64),
            consumed.cpu().numpy(), int(status.item()) & 0xFFFFFFFF)


def group_inputs(wl, b, kvh, layer=0, q=None):
    """Oracle inputs of KV group (b, kvh): q [G][d], K, V [L][d] (bf16 bits)."""
    if q is None:
        q = skvgen.host_q(wl, layer)
    G = wl.G
    qg = q[b, 0, kvh * G:(kvh + 1) * G]
    if wl.mixture:
        K, _, _ = skvgen.host_mixture_group(wl, b, kvh, layer)
        _, V = skvgen.host_kv_group(wl.with_(structured=False), b, kvh, layer)
    else:
        K, V = skvgen.host_kv_group(wl, b, kvh, layer, q=q)
    return qg, K, V


def check_close(O_gpu, lse_gpu, O_ref, lse_ref, what=""):
    O_gpu, O_ref = np.asarray(O_gpu), np.asarray(O_ref)
    lse_gpu, lse_ref = np.asarray(lse_gpu), np.asarray(lse_ref)
    both_empty = np.isneginf(lse_ref) & np.isneginf(lse_gpu)
    assert np.all(np.isfinite(O_gpu)), f"{what}: non-finite output"
    err = np.abs(O_gpu - O_ref).max() if O_ref.size else 0.0
    assert err <= ATOL_O, f"{what}: max |dO| = {err:.3e}"
    with np.errstate(invalid="ignore"):
        ok = both_empty | (np.abs(lse_gpu - lse_ref) <= RTOL_LSE * np.maximum(1.0, np.abs(lse_ref)))
    assert np.all(ok), f"{what}: LSE mismatch {lse_gpu[~ok][:4]} vs {lse_ref[~ok][:4]}"
    return err


def oracle_keys_attend(wl, b, kvh, keys, layer=0, q=None):
    qg, K, V = group_inputs(wl, b, kvh, layer, q)
    return oracle.attend(qg[None], K[None], V[None], [[keys] * wl.G], wl.scale)


def check_art(wl, dev_res, b, kvh, order=None, layer=0, q=None, tau=None, phi=None, patience=None):
    """Compare one group's ART result with the oracle; returns number of flagged heads."""
    O_g, lse_g, cons_g, _ = dev_res
    tau = wl.tau if tau is None else tau
    phi = wl.phi if phi is None else phi
    patience = wl.patience if patience is None else patience
    qg, K, V = group_inputs(wl, b, kvh, layer, q)
    L = wl.seq_len(b)
    trav = oracle.art_traversal(wl.nb(b), order)
    O, lse, cons, mg = oracle.art(qg[None], K[None], V[None], [L], wl.bs, [trav], wl.scale, tau, phi,
                                  patience)
    G = wl.G
    hs = slice(kvh * G, (kvh + 1) * G)
    flagged = 0
    cg = cons_g[b, hs]
    if not np.array_equal(cg, cons[0]):
        bad = np.nonzero(cg != cons[0])[0]
        for h in bad:
            assert mg[0, h] <= ART_FLAG_MARGIN, (
                f"ART stop differs for (b={b}, h={kvh * G + h}): gpu {cg[h]} vs oracle {cons[0, h]}, "
                f"margin {mg[0, h]:.3e}")
        flagged = len(bad)
        O, lse, _, _ = oracle.art(qg[None], K[None], V[None], [L], wl.bs, [trav], wl.scale, tau, phi,
                                  patience, forced=cg[None])
    check_close(O_g[b, hs], lse_g[b, hs], O[0], lse[0], f"ART group ({b},{kvh})")
    return flagged, cons[0], mg[0]


def check_topk_valid(ids_gpu, scores, k, what=""):
    """ids_gpu (k ids) is a valid top-k of `scores` (fp64, ranked by score desc,
    index asc) up to near ties at the boundary: k distinct ids in ascending
    order; every id whose score lies clearly above the k-th best score is kept;
    every kept id scores at least the k-th best score, both within the flag
    gap TOPK_FLAG_GAP (relative to the k-th score)."""
    s = np.asarray(scores, dtype=np.float64)
    ids = np.asarray(ids_gpu, dtype=np.int64)
    assert ids.shape == (k,), f"{what}: {ids.shape} ids, expected {k}"
    assert np.all(np.diff(ids) > 0), f"{what}: ids not strictly ascending"
    assert ids.min() >= 0 and ids.max() < s.shape[0], f"{what}: id out of range"
    order = sorted(range(s.shape[0]), key=lambda i: (-s[i], i))
    kth = s[order[k - 1]]
    band = TOPK_FLAG_GAP * max(abs(kth), 1e-300)
    must = {i for i in range(s.shape[0]) if s[i] > kth + band}
    kept = set(int(i) for i in ids)
    assert must <= kept, f"{what}: ids {sorted(must - kept)[:4]} score above the boundary but were dropped"
    low = [i for i in kept if s[i] < kth - band]
    assert not low, f"{what}: ids {low[:4]} score below the k-th best but were kept"


def check_selection(wl, ids_gpu, groups, q=None):
    """ids must equal the oracle's except at flagged near-tie boundaries, where
    the GPU's choice must still be a valid top-k (check_topk_valid)."""
    q = skvgen.host_q(wl) if q is None else q
    flagged = 0
    for (b, kvh) in groups:
        _, off, cent = skvgen.host_mixture_group(wl, b, kvh, want_keys=False)
        qg = q[b, 0, kvh * wl.G:(kvh + 1) * wl.G]
        ids, sc = oracle.select(qg[None], cent[None], wl.topk)
        if not np.array_equal(ids[0], ids_gpu[b, kvh]):
            gap = oracle.topk_boundary_gap(sc, wl.topk)[0]
            assert gap <= TOPK_FLAG_GAP, f"selection differs for ({b},{kvh}), gap {gap:.2e}"
            check_topk_valid(ids_gpu[b, kvh], sc[0], wl.topk, f"selection ({b},{kvh})")
            flagged += 1
    return flagged
