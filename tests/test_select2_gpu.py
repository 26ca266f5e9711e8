"""GPU parity of attn_select_centroids2 (two-level centroid selection,
"Squeezed Attention" Q2 step 4) against the CPU fp64 oracle, and attention over
the chosen clusters' keys through attn_decode's segment traversal."""
import numpy as np
import pytest

import oracle
import skvgen
from helpers import TOPK_FLAG_GAP, check_close, device_workload, oracle_keys_attend, outputs

pytestmark = pytest.mark.gpu


def _bf16(x):
    import torch
    return torch.tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _data(B, Hkv, G, d, sizes, seed, toks_per_fine=5):
    """Fine centroids (generator normals), coarse clusters of the given sizes
    (in fine clusters, possibly 0) with centroids = fp64 means rounded to bf16,
    and key ranges of toks_per_fine tokens per fine cluster."""
    C1, C = len(sizes), int(sum(sizes))
    q = skvgen.host_normal_bf16(seed, skvgen.S_Q, B * G * Hkv * d).reshape(B, G * Hkv, d)
    fine = skvgen.host_normal_bf16(seed, skvgen.S_CENTER, B * Hkv * C * d).reshape(B, Hkv, C, d)
    off1 = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    fv = skvgen.bf16_to_f64(fine)
    coarse = np.zeros((B, Hkv, C1, d), dtype=np.uint16)
    for i in range(C1):
        if sizes[i]:
            coarse[:, :, i] = _bf16(fv[:, :, off1[i]:off1[i + 1]].mean(axis=2))
        else:
            coarse[:, :, i] = _bf16(np.full((B, Hkv, d), -4.0))  # an empty cluster scores low
    coarse_off = np.broadcast_to(off1, (B, Hkv, C1 + 1)).copy()
    cluster_off = np.broadcast_to(np.arange(C + 1, dtype=np.int32) * toks_per_fine, (B, Hkv, C + 1)).copy()
    return q, coarse, coarse_off, fine, cluster_off


def _run(q, coarse, coarse_off, fine, cluster_off, k1, k2):
    import torch
    import sparse_kv_b200 as skv
    B, Hkv = coarse.shape[:2]
    dev = lambda a, dt: torch.tensor(a.astype(np.int32) if dt == torch.int32 else a.view(np.int16), dtype=dt, device="cuda")
    t = dict(q=dev(q, torch.int16).view(torch.bfloat16), coarse=dev(coarse, torch.int16).view(torch.bfloat16),
             co=dev(coarse_off, torch.int32), fine=dev(fine, torch.int16).view(torch.bfloat16),
             clo=dev(cluster_off, torch.int32))
    ids = torch.full((B, Hkv, k2), 777, dtype=torch.int32, device="cuda")
    ss, se = torch.empty_like(ids), torch.empty_like(ids)
    skv.attn_select_centroids2(t["q"], t["coarse"], t["co"], t["fine"], t["clo"], k1, k2, ids, ss, se)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), ss.cpu().numpy(), se.cpu().numpy(), t, (ids, ss, se)


def _check(q, coarse, coarse_off, fine, cluster_off, k1, k2):
    ids, ss, se, _, _ = _run(q, coarse, coarse_off, fine, cluster_off, k1, k2)
    B, Hkv, C1, d = coarse.shape
    G = q.shape[1] // Hkv
    flagged = 0
    for b in range(B):
        for h in range(Hkv):
            qg = q[b, h * G:(h + 1) * G][None]
            want = oracle.select2(qg, coarse[b, h][None], coarse_off[b, h][None], fine[b, h][None], k1, k2)[0]
            if not np.array_equal(ids[b, h], want):
                # a near tie at either level may be decided either way in fp32
                _, s1 = oracle.select(qg, coarse[b, h][None], k1)
                g1 = oracle.topk_boundary_gap(s1, k1)[0]
                _, s2 = oracle.select(qg, fine[b, h][None], fine.shape[2])
                assert min(g1, _cand_gap(s2[0], coarse_off[b, h], want, ids[b, h], k2)) <= TOPK_FLAG_GAP, \
                    f"({b},{h}): {ids[b, h]} vs {want}"
                flagged += 1
            n = int((want >= 0).sum())
            np.testing.assert_array_equal(ss[b, h, :n], cluster_off[b, h][want[:n]])
            np.testing.assert_array_equal(se[b, h, :n], cluster_off[b, h][want[:n] + 1])
            assert np.all(ids[b, h, n:] == -1) and np.all(ss[b, h, n:] == 0) and np.all(se[b, h, n:] == 0)
    return flagged


def _cand_gap(scores, off, want, got, k2):
    """Relative score gap at the second level's boundary among the candidates
    the oracle used (the union of both answers' coarse parents)."""
    parents = set(np.searchsorted(off, [f for f in list(want) + list(got) if f >= 0], side="right") - 1)
    cand = [f for p in sorted(parents) for f in range(off[p], off[p + 1])]
    return oracle.topk_boundary_gap(scores[cand][None], min(k2, len(cand)))[0]


def test_select2_matches_oracle_uniform():
    # 32 coarse clusters of 32 fine ones (1024 fine clusters), keep 4 then 102
    flagged = _check(*_data(2, 2, 4, 128, [32] * 32, seed=0xA1), k1=4, k2=102)
    assert flagged <= 1


def test_select2_matches_oracle_ragged_and_empty():
    rng = np.random.default_rng(5)
    sizes = list(rng.integers(0, 9, 40))
    sizes[3] = 0
    flagged = _check(*_data(3, 2, 2, 128, sizes, seed=0xA2), k1=7, k2=20)
    assert flagged <= 1


def test_select2_fewer_candidates_than_k2():
    # 2 kept coarse clusters of 3 fine ones: 6 candidates for 9 slots
    _check(*_data(1, 2, 4, 128, [3] * 8, seed=0xA3), k1=2, k2=9)


def test_select2_keep_all_coarse_is_the_flat_selection():
    import torch
    import sparse_kv_b200 as skv
    q, coarse, coarse_off, fine, cluster_off = _data(2, 2, 4, 128, [16] * 16, seed=0xA4)
    ids2, _, _, t, _ = _run(q, coarse, coarse_off, fine, cluster_off, 16, 50)
    ids1 = torch.empty((2, 2, 50), dtype=torch.int32, device="cuda")
    s1, e1 = torch.empty_like(ids1), torch.empty_like(ids1)
    skv.attn_select_centroids(t["q"], t["fine"], t["clo"], 50, ids1, s1, e1)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ids2, ids1.cpu().numpy())


def test_select2_then_attend_the_chosen_keys():
    # the chosen fine clusters' key ranges (with unused slots as empty ranges)
    # feed attn_decode's segment traversal; compare with the oracle's attention
    import torch
    import sparse_kv_b200 as skv
    wl = skvgen.Workload("s2", B=1, Hq=8, Hkv=2, L=64 * 40, paging="perm", seed=0xA5)
    dev = device_workload(wl)
    q = skvgen.host_q(wl)[:, 0]  # [B][Hq][d]
    sizes = [4] * 10  # 40 fine clusters of 64 tokens: the whole cache
    _, coarse, coarse_off, fine, cluster_off = _data(1, 2, 4, 128, sizes, seed=0xA6, toks_per_fine=64)
    ids, ss, se, _, (ids_d, ss_d, se_d) = _run(q, coarse, coarse_off, fine, cluster_off, 2, 12)
    out, lse = outputs(wl)
    args = (dev["q"], dev["k_pool"], dev["v_pool"], dev["block_table"], dev["seq_lens"], out, lse)
    kw = dict(max_seq_len=wl.Lmax, scale=wl.scale, segments=(ss_d, se_d))
    skv.attn_decode(*args, **kw)
    torch.cuda.synchronize()
    O, L = out[:, 0].cpu().numpy().astype(np.float64), lse[:, 0].cpu().numpy().astype(np.float64)
    qh = skvgen.host_q(wl)
    for kvh in range(2):
        keys = np.concatenate([np.arange(a, b) for a, b in zip(ss[0, kvh], se[0, kvh])])
        Oo, Lo = oracle_keys_attend(wl, 0, kvh, keys, 0, qh)
        hs = slice(kvh * 4, kvh * 4 + 4)
        check_close(O[0, hs], L[0, hs], Oo[0], Lo[0], f"group (0,{kvh})")
