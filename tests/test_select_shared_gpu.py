"""Centroid selection over one shared fixed context ("Squeezed Attention" Q1:
the fixed context is clustered once and reused by every request), then
attention over each request's chosen clusters in that one context.

Checks: the ids equal the oracle's (shared centroids, each request's own
summed query) except at flagged near ties, where they must still be a valid
top-k; they equal what the per-sequence selection returns when given the same
centroids for every request (same arithmetic, so bit-identical keys); and the
attention over the chosen ranges, read through a block table whose rows all
map to the one context, matches the oracle."""
import numpy as np
import pytest

import oracle
import skvgen
from helpers import TOPK_FLAG_GAP, check_close, check_topk_valid, run_decode

pytestmark = pytest.mark.gpu


def _shared(B, L, c_log2, topk, seed):
    return skvgen.Workload("shr", B=B, Hq=16, Hkv=4, L=L, mixture=True, c_log2=c_log2, topk=topk,
                           shared_context=True, seed=seed)


@pytest.mark.parametrize("B,L,c_log2,topk", [(5, 9000, 7, 13), (12, 20000, 9, 51), (1, 4096, 6, 64)])
def test_shared_selection_and_attention(B, L, c_log2, topk):
    import torch
    import sparse_kv_b200 as skv
    wl = _shared(B, L, c_log2, topk, seed=700 + B)
    q, k_pool, v_pool, bt, sl, off, cent = skvgen.device_shared_context(wl)
    C = 1 << c_log2
    shape = (B, wl.Hkv, topk)
    ids = torch.full(shape, -7, dtype=torch.int32, device="cuda")
    ss, se = torch.full_like(ids, -7), torch.full_like(ids, -7)
    skv.attn_select_centroids_shared(q, cent, off, topk, ids, ss, se)
    # the per-sequence call with the centroids repeated for every request
    ids2, ss2, se2 = torch.empty_like(ids), torch.empty_like(ids), torch.empty_like(ids)
    cent_b = cent.unsqueeze(0).expand(B, *cent.shape).contiguous()
    off_b = off.unsqueeze(0).expand(B, *off.shape).contiguous()
    skv.attn_select_centroids(q, cent_b, off_b, topk, ids2, ss2, se2)
    torch.cuda.synchronize()
    ids_h, ss_h, se_h = ids.cpu().numpy(), ss.cpu().numpy(), se.cpu().numpy()
    np.testing.assert_array_equal(ids_h, ids2.cpu().numpy())
    np.testing.assert_array_equal(ss_h, ss2.cpu().numpy())
    np.testing.assert_array_equal(se_h, se2.cpu().numpy())
    qh = skvgen.host_q(wl)
    flagged = 0
    ctx = {kvh: skvgen.host_shared_context(wl, kvh) for kvh in range(wl.Hkv)}
    for kvh in range(wl.Hkv):
        K, V, off_h, cent_h = ctx[kvh]
        np.testing.assert_array_equal(off_h, off[kvh].cpu().numpy())
        ref_ids, sc = oracle.select_shared(qh[:, 0, kvh * wl.G:(kvh + 1) * wl.G], cent_h, topk)
        for b in range(B):
            if not np.array_equal(ref_ids[b], ids_h[b, kvh]):
                gap = oracle.topk_boundary_gap(sc[b:b + 1], topk)[0]
                assert gap <= TOPK_FLAG_GAP, f"request {b} head {kvh}: gap {gap:.2e}"
                check_topk_valid(ids_h[b, kvh], sc[b], topk, f"request {b} head {kvh}")
                flagged += 1
            np.testing.assert_array_equal(ss_h[b, kvh], off_h[ids_h[b, kvh]])
            np.testing.assert_array_equal(se_h[b, kvh], off_h[ids_h[b, kvh] + 1])
    assert flagged <= 1
    # attention over each request's chosen ranges of the one shared context
    dev = dict(q=q, k_pool=k_pool, v_pool=v_pool, block_table=bt, seq_lens=sl)
    O_g, lse_g, _, status = run_decode(wl, dev, segments=(ss, se))
    assert status == 0
    for b in sorted({0, B - 1}):
        for kvh in (0, wl.Hkv - 1):
            K, V, off_h, _ = ctx[kvh]
            keys = oracle.keys_segments(ss_h[b, kvh], se_h[b, kvh])
            qg = qh[b, 0, kvh * wl.G:(kvh + 1) * wl.G]
            O, lse = oracle.attend(qg[None], K[None], V[None], [[keys] * wl.G], wl.scale)
            hs = slice(kvh * wl.G, (kvh + 1) * wl.G)
            check_close(O_g[b, hs], lse_g[b, hs], O[0], lse[0], f"request {b} head {kvh}")


def test_per_sequence_selection_cluster_split_matches_oracle():
    """The per-sequence call (one CTA per KV group) over 1 to 320 groups and
    256 to 4096 clusters, with top-k from 7 to 300."""
    import torch
    import sparse_kv_b200 as skv
    for B, Hkv, c_log2, topk in [(1, 1, 12, 300), (2, 8, 10, 102), (40, 8, 8, 7)]:
        wl = skvgen.Workload("psel", B=B, Hq=Hkv * 4, Hkv=Hkv, L=max(4096, 1 << c_log2), mixture=True,
                             c_log2=c_log2, topk=topk, seed=740 + B)
        from helpers import device_workload, check_selection
        dev = device_workload(wl)
        shape = (B, Hkv, topk)
        ids = torch.full(shape, -7, dtype=torch.int32, device="cuda")
        ss, se = torch.empty_like(ids), torch.empty_like(ids)
        skv.attn_select_centroids(dev["q"], dev["centroids"], dev["cluster_off"], topk, ids, ss, se)
        torch.cuda.synchronize()
        groups = sorted({(0, 0), (B - 1, Hkv - 1), (B // 2, Hkv // 2)})
        assert check_selection(wl, ids.cpu().numpy(), groups) <= 1
