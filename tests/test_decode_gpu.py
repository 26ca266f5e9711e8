"""GPU parity: the CUDA path (through the C ABI) against the CPU fp64 oracle
on the same seeded inputs."""
import numpy as np
import pytest

import oracle
import skvgen
from helpers import (TOPK_FLAG_GAP, check_art, check_close, check_selection, check_topk_valid,
                     device_workload, group_inputs, oracle_keys_attend, outputs, run_decode)

pytestmark = pytest.mark.gpu


def _torch():
    import torch
    return torch


# ----------------------------------------------------------------------------- generator

def test_device_generator_matches_host_bits():
    torch = _torch()
    wl = skvgen.Workload("g", B=3, Hq=8, Hkv=2, L=300, lens=[300, 65, 1], structured=True,
                         paging="perm", seed=77)
    dev = device_workload(wl)
    qh = skvgen.host_q(wl)
    qd = dev["q"].view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(qd, qh)
    kp = dev["k_pool"].view(torch.int16).cpu().numpy().view(np.uint16)
    vp = dev["v_pool"].view(torch.int16).cpu().numpy().view(np.uint16)
    for b in range(wl.B):
        for kvh in range(wl.Hkv):
            K, V = skvgen.host_kv_group(wl, b, kvh, q=qh)
            for t in range(wl.seq_len(b)):
                pg = dev["bt_host"][b, t // 64]
                np.testing.assert_array_equal(kp[pg, kvh, t % 64], K[t])
                np.testing.assert_array_equal(vp[pg, kvh, t % 64], V[t])


def test_device_mixture_matches_host_bits():
    torch = _torch()
    wl = skvgen.Workload("m", B=2, Hq=8, Hkv=2, L=1500, mixture=True, c_log2=5, topk=4, seed=78)
    dev = device_workload(wl)
    kp = dev["k_pool"].view(torch.int16).cpu().numpy().view(np.uint16)
    cent = dev["centroids"].view(torch.int16).cpu().numpy().view(np.uint16)
    off = dev["cluster_off"].cpu().numpy()
    for b in range(2):
        for kvh in range(2):
            K, o, c = skvgen.host_mixture_group(wl, b, kvh)
            np.testing.assert_array_equal(off[b, kvh], o)
            np.testing.assert_array_equal(cent[b, kvh], c)
            for t in range(0, 1500, 7):
                pg = dev["bt_host"][b, t // 64]
                np.testing.assert_array_equal(kp[pg, kvh, t % 64], K[t])


# ----------------------------------------------------------------------------- full traversal

def _check_all_groups(wl, res, keys_fn, layer=0):
    O_g, lse_g = res[0], res[1]
    q = skvgen.host_q(wl, layer)
    worst = 0.0
    for b in range(wl.B):
        for kvh in range(wl.Hkv):
            O, lse = oracle_keys_attend(wl, b, kvh, keys_fn(b), layer, q)
            hs = slice(kvh * wl.G, (kvh + 1) * wl.G)
            worst = max(worst, check_close(O_g[b, hs], lse_g[b, hs], O[0], lse[0], f"group ({b},{kvh})"))
    return worst


def test_cfg1_full_traversal():
    wl = skvgen.WORKLOADS["cfg1_b1_h8_l4k"]
    dev = device_workload(wl)
    res = run_decode(wl, dev)
    assert res[3] == 0
    _check_all_groups(wl, res, lambda b: oracle.keys_full(wl.seq_len(b)))
    assert np.all(res[2] == 64)


@pytest.mark.parametrize("G,Hkv,L", [(8, 1, 4096), (4, 1, 4096), (1, 2, 64 * 40 + 9), (2, 3, 64 * 5)])
def test_split_cluster_sizes(G, Hkv, L):
    # one KV group walked by clusters of up to 16 CTAs (G = 8 runs one CTA per
    # SM, so 16 pieces need 16 SMs; a size that cannot be resident is halved)
    import sparse_kv_b200 as skv
    wl = skvgen.Workload("cs", B=1, Hq=G * Hkv, Hkv=Hkv, L=L, paging="perm", seed=80 + G)
    dev = device_workload(wl)
    out, lse = outputs(wl)
    args = (dev["q"], dev["k_pool"], dev["v_pool"], dev["block_table"], dev["seq_lens"], out, lse)
    assert skv.decode_launches(*args, max_seq_len=wl.Lmax) == 1
    res = run_decode(wl, dev)
    assert res[3] == 0
    _check_all_groups(wl, res, lambda b: oracle.keys_full(wl.seq_len(b)))
    np.testing.assert_array_equal(res[2], wl.nb(0))


def test_split_merge_repeats():
    # The split schedule (small walks) merges inside the kernel: the pieces of a
    # group form one cluster, and rank 0 combines them from the cluster's
    # shared memory.  Three calls must give the oracle's result, bit-identical.
    import sparse_kv_b200 as skv
    torch = _torch()
    lens = [4096, 64 * 7 + 3, 0]
    wl = skvgen.Workload("w", B=3, Hq=8, Hkv=2, L=max(lens), lens=lens, paging="perm", seed=71)
    dev = device_workload(wl)
    out = torch.empty((wl.B, 1, wl.Hq, wl.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((wl.B, 1, wl.Hq), dtype=torch.float32, device="cuda")
    consumed = torch.full((wl.B, wl.Hq), -1, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    args = (dev["q"], dev["k_pool"], dev["v_pool"], dev["block_table"], dev["seq_lens"], out, lse)
    kw = dict(max_seq_len=wl.Lmax, blocks_consumed=consumed, status=status, scale=wl.scale)
    assert skv.decode_launches(*args, **kw) == 1
    assert skv.decode_workspace_size(*args, **kw) == 0
    first = None
    for it in range(3):
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        skv.attn_decode(*args, **kw)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        res = (out[:, 0].cpu().numpy().astype(np.float64), lse[:, 0].cpu().numpy().astype(np.float64),
               consumed.cpu().numpy(), 0)
        if first is None:
            _check_all_groups(wl, res, lambda b: oracle.keys_full(wl.seq_len(b)))
            first = res
        else:
            np.testing.assert_array_equal(res[0], first[0])
            np.testing.assert_array_equal(res[1], first[1])
        nb = np.array([wl.nb(b) for b in range(wl.B)])
        np.testing.assert_array_equal(res[2], np.repeat(nb[:, None], wl.Hq, axis=1))


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_ragged_paged_full_traversal(G):
    lens = [1, 63, 64, 65, 200, 1000, 0, 4097]
    wl = skvgen.Workload("r", B=len(lens), Hq=2 * G, Hkv=2, L=max(lens), lens=lens, paging="perm",
                         seed=100 + G)
    dev = device_workload(wl)
    res = run_decode(wl, dev)
    assert res[3] == 0
    _check_all_groups(wl, res, lambda b: oracle.keys_full(wl.seq_len(b)))
    nb = np.array([wl.nb(b) for b in range(wl.B)])
    np.testing.assert_array_equal(res[2], np.repeat(nb[:, None], wl.Hq, axis=1))


def test_caller_order_full_traversal_is_permutation_invariant():
    torch = _torch()
    lens = [64 * 37 + 5, 64 * 20]
    wl = skvgen.Workload("o", B=2, Hq=8, Hkv=2, L=max(lens), lens=lens, paging="perm", seed=5)
    dev = device_workload(wl)
    rng = np.random.default_rng(0)
    n = max(wl.nb(b) for b in range(2))
    order = np.zeros((2, 2, n), dtype=np.int32)
    for b in range(2):
        for h in range(2):
            nb = wl.nb(b)
            order[b, h, :nb] = rng.permutation(nb)
            order[b, h, nb:] = rng.integers(0, nb, n - nb)  # duplicates: attended twice
    res = run_decode(wl, dev, order=torch.tensor(order, device="cuda"))
    assert res[3] == 0
    q = skvgen.host_q(wl)
    for b in range(2):
        for kvh in range(2):
            keys = np.concatenate([np.arange(64 * j, min(64 * j + 64, wl.seq_len(b))) for j in order[b, kvh]])
            O, lse = oracle_keys_attend(wl, b, kvh, keys, q=q)
            hs = slice(kvh * 4, kvh * 4 + 4)
            check_close(res[0][b, hs], res[1][b, hs], O[0], lse[0])
    # order covering exactly the blocks once equals natural full traversal
    o2 = np.stack([np.stack([rng.permutation(wl.nb(0))] * 2)] * 1)
    wl1 = wl.with_(B=1, lens=[lens[0]], L=lens[0])
    dev1 = device_workload(wl1)
    a = run_decode(wl1, dev1, order=torch.tensor(o2.astype(np.int32), device="cuda"))
    bfull = run_decode(wl1, dev1)
    np.testing.assert_allclose(a[0], bfull[0], atol=2e-5)
    np.testing.assert_allclose(a[1], bfull[1], rtol=1e-6)


@pytest.mark.parametrize("sink,recent", [(64, 4096), (64, 256), (10, 100), (0, 130), (200, 0), (64, 10 ** 6)])
def test_sink_recent_window(sink, recent):
    lens = [5000, 300, 64, 129, 1]
    wl = skvgen.Workload("w", B=len(lens), Hq=8, Hkv=2, L=max(lens), lens=lens, paging="perm", seed=9)
    dev = device_workload(wl)
    res = run_decode(wl, dev, window=(sink, recent))
    assert res[3] == 0
    _check_all_groups(wl, res, lambda b: oracle.keys_window(wl.seq_len(b), sink, recent))


@pytest.mark.parametrize("rng_", [(0, 64), (100, 1000), (1, 4096), (4000, 4100), (3000, 3000)])
def test_kv_token_range(rng_):
    lens = [4100, 3500]
    wl = skvgen.Workload("k", B=2, Hq=8, Hkv=2, L=max(lens), lens=lens, paging="perm", seed=19)
    dev = device_workload(wl)
    res = run_decode(wl, dev, kv_range=rng_)
    assert res[3] == 0
    a, e = rng_
    _check_all_groups(wl, res, lambda b: np.arange(a, min(e, wl.seq_len(b))))


def test_token_segments_unaligned():
    torch = _torch()
    lens = [3000, 2000]
    wl = skvgen.Workload("s", B=2, Hq=8, Hkv=2, L=max(lens), lens=lens, paging="perm", seed=29)
    dev = device_workload(wl)
    rng = np.random.default_rng(3)
    n_seg = 9
    ss = np.zeros((2, 2, n_seg), dtype=np.int32)
    se = np.zeros((2, 2, n_seg), dtype=np.int32)
    for b in range(2):
        for h in range(2):
            cuts = np.sort(rng.choice(np.arange(1, lens[b]), 2 * n_seg, replace=False))
            ss[b, h], se[b, h] = cuts[0::2], cuts[1::2]
            se[b, h, -1] = lens[b] + 50  # clipped to seq_len
            ss[b, h, 0] = se[b, h, 0]    # an empty segment
    res = run_decode(wl, dev, segments=(torch.tensor(ss, device="cuda"), torch.tensor(se, device="cuda")))
    assert res[3] == 0
    q = skvgen.host_q(wl)
    for b in range(2):
        for kvh in range(2):
            keys = oracle.keys_segments(ss[b, kvh], np.minimum(se[b, kvh], lens[b]))
            O, lse = oracle_keys_attend(wl, b, kvh, keys, q=q)
            hs = slice(kvh * 4, kvh * 4 + 4)
            check_close(res[0][b, hs], res[1][b, hs], O[0], lse[0])


def test_token_segments_many():
    # long segment lists (420 per group: the producer warp resolves them in
    # batches of 32), segments of 1 to 300 tokens (some over more than two
    # pages), empty ones, and ones past seq_len
    torch = _torch()
    lens = [20000, 13001, 700]
    wl = skvgen.Workload("sp", B=3, Hq=8, Hkv=2, L=max(lens), lens=lens, paging="perm", seed=41)
    dev = device_workload(wl)
    n_seg = 420
    rng = np.random.default_rng(5)
    ss = np.zeros((3, 2, n_seg), dtype=np.int32)
    se = np.zeros((3, 2, n_seg), dtype=np.int32)
    for b in range(3):
        for h in range(2):
            pos = 0
            for i in range(n_seg):
                gap = int(rng.integers(0, 40))
                ln = int(rng.choice([0, 1, 5, 63, 64, 65, 130, 300]))
                ss[b, h, i] = pos + gap
                se[b, h, i] = pos + gap + ln
                pos = se[b, h, i]
    res = run_decode(wl, dev, segments=(torch.tensor(ss, device="cuda"), torch.tensor(se, device="cuda")))
    assert res[3] == 0
    q = skvgen.host_q(wl)
    for b in range(3):
        for kvh in range(2):
            keys = oracle.keys_segments(np.minimum(ss[b, kvh], lens[b]), np.minimum(se[b, kvh], lens[b]))
            assert len(keys) > 0
            O, lse_o = oracle_keys_attend(wl, b, kvh, keys, q=q)
            hs = slice(kvh * 4, kvh * 4 + 4)
            check_close(res[0][b, hs], res[1][b, hs], O[0], lse_o[0], f"group ({b},{kvh})")


# ----------------------------------------------------------------------------- ART

def test_art_zero_thresholds_is_full_attention():
    lens = [64 * 30 + 7, 64 * 5]
    wl = skvgen.Workload("a0", B=2, Hq=8, Hkv=2, L=max(lens), lens=lens, paging="perm", seed=31)
    dev = device_workload(wl)
    res = run_decode(wl, dev, art=(0.0, 0.0, 4))
    assert res[3] == 0
    _check_all_groups(wl, res, lambda b: oracle.keys_full(wl.seq_len(b)))
    nb = np.array([wl.nb(b) for b in range(2)])
    np.testing.assert_array_equal(res[2], np.repeat(nb[:, None], 8, axis=1))


@pytest.mark.parametrize("tau,phi,p", [(1e-3, 1e-4, 4), (3e-2, 3e-3, 2), (1e-2, 1e-3, 1)])
def test_art_structured_small(tau, phi, p):
    # sink + heavy structure (token 0 key + 6 qhat, 1% heavy + 4 qhat), recency-first
    lens = [64 * 60, 64 * 33 + 20, 64 * 8]
    wl = skvgen.Workload("as", B=3, Hq=8, Hkv=2, L=max(lens), lens=lens, structured=True,
                         paging="perm", seed=41)
    dev = device_workload(wl)
    res = run_decode(wl, dev, art=(tau, phi, p))
    assert res[3] == 0
    q = skvgen.host_q(wl)
    flagged = 0
    for b in range(3):
        for kvh in range(2):
            f, _, _ = check_art(wl, res, b, kvh, q=q, tau=tau, phi=phi, patience=p)
            flagged += f
    assert flagged <= 2


@pytest.mark.parametrize("p", [1, 2, 3, 4])
def test_art_always_passing_stops_after_one_plus_p_blocks(p):
    # thresholds no probe change can reach (d_scale < 10, 1 - cos < 2.5): every
    # test passes, so each head stops after block 0 and p more blocks
    lens = [64 * 40, 64 * 3 + 1]
    wl = skvgen.Workload("ap", B=2, Hq=8, Hkv=2, L=max(lens), lens=lens, structured=True,
                         paging="perm", seed=43, softmax_scale=0.3)
    dev = device_workload(wl)
    res = run_decode(wl, dev, art=(10.0, 2.5, p))
    assert res[3] == 0
    assert np.all(res[2][0] == 1 + p)
    assert np.all(res[2][1] == min(1 + p, 4))
    q = skvgen.host_q(wl)
    for b in range(2):
        for kvh in range(2):
            check_art(wl, res, b, kvh, q=q, tau=10.0, phi=2.5, patience=p)


@pytest.mark.parametrize("G", [1, 2, 8])
def test_art_other_group_sizes(G):
    lens = [64 * 21 + 9, 64 * 6]
    wl = skvgen.Workload("ag", B=2, Hq=2 * G, Hkv=2, L=max(lens), lens=lens, structured=True,
                         paging="perm", seed=44 + G, softmax_scale=0.3)
    dev = device_workload(wl)
    q = skvgen.host_q(wl)
    for tau, phi, p in [(10.0, 2.5, 2), (0.0, 0.0, 1), (3e-2, 3e-3, 2)]:
        res = run_decode(wl, dev, art=(tau, phi, p))
        assert res[3] == 0
        for b in range(2):
            for kvh in range(2):
                check_art(wl, res, b, kvh, q=q, tau=tau, phi=phi, patience=p)


@pytest.mark.parametrize("tau,phi,p", [(2e-2, 2e-3, 2), (1e-2, 5e-4, 3)])
def test_art_stops_across_many_chunks(tau, phi, p):
    # 130..256 blocks per sequence (5..8 chunks of 32 blocks): heads of one group
    # stop in different chunks (blocks ~38..214), some never; later chunks of a
    # group keep running for the heads still live and pass stopped heads on
    lens = [64 * 256, 64 * 200 + 17, 64 * 130]
    wl = skvgen.Workload("am", B=3, Hq=8, Hkv=2, L=max(lens), lens=lens, structured=True,
                         paging="perm", seed=61)
    dev = device_workload(wl)
    res = run_decode(wl, dev, art=(tau, phi, p))
    assert res[3] == 0
    q = skvgen.host_q(wl)
    flagged = 0
    for b in range(3):
        for kvh in range(2):
            f, _, _ = check_art(wl, res, b, kvh, q=q, tau=tau, phi=phi, patience=p)
            flagged += f
    assert flagged <= 2


def test_art_early_stop_skips_later_chunks():
    # every test passes: each head stops after 1 + p blocks, inside the first
    # chunk of sequences of up to 400 blocks; the chunks taken later issue no
    # loads (or, if already in flight, pass the stopped state on)
    p = 3
    lens = [64 * 400, 64 * 333 + 5, 64 * 40, 64 * 2 + 1] * 2
    wl = skvgen.Workload("ae", B=8, Hq=8, Hkv=2, L=max(lens), lens=lens, structured=True,
                         paging="perm", seed=62, softmax_scale=0.3)
    dev = device_workload(wl)
    res = run_decode(wl, dev, art=(10.0, 2.5, p))
    assert res[3] == 0
    for b in range(wl.B):
        assert np.all(res[2][b] == min(1 + p, wl.nb(b)))
    q = skvgen.host_q(wl)
    for b in (0, 1, 3):
        for kvh in range(2):
            check_art(wl, res, b, kvh, q=q, tau=10.0, phi=2.5, patience=p)


def test_art_caller_order_across_chunks():
    # a caller order over 150 blocks (5 chunks) that also lists block 0 again
    torch = _torch()
    wl = skvgen.Workload("ac", B=1, Hq=8, Hkv=2, L=64 * 150, structured=True, seed=63)
    dev = device_workload(wl)
    rng = np.random.default_rng(2)
    order = np.stack([rng.permutation(150) for _ in range(2)])[None].astype(np.int32)
    tau, phi, p = 2e-2, 2e-3, 2
    res = run_decode(wl, dev, art=(tau, phi, p), order=torch.tensor(order, device="cuda"))
    assert res[3] == 0
    q = skvgen.host_q(wl)
    for kvh in range(2):
        check_art(wl, res, 0, kvh, order=list(order[0, kvh]), q=q, tau=tau, phi=phi, patience=p)


def test_art_with_caller_order_skips_block0_in_list():
    torch = _torch()
    wl = skvgen.Workload("ao", B=1, Hq=8, Hkv=2, L=64 * 50, structured=True, seed=47)
    dev = device_workload(wl)
    rng = np.random.default_rng(1)
    order = np.stack([rng.permutation(50) for _ in range(2)])[None].astype(np.int32)
    res = run_decode(wl, dev, art=(3e-2, 3e-3, 2), order=torch.tensor(order, device="cuda"))
    q = skvgen.host_q(wl)
    for kvh in range(2):
        check_art(wl, res, 0, kvh, order=list(order[0, kvh]), q=q, tau=3e-2, phi=3e-3, patience=2)


# ----------------------------------------------------------------------------- device-side errors

def test_bad_page_and_seqlen_are_reported():
    torch = _torch()
    wl = skvgen.Workload("e", B=2, Hq=8, Hkv=2, L=640, paging="perm", seed=53)
    dev = device_workload(wl)
    bt = dev["block_table"].clone()
    bt[0, 3] = 10 ** 6
    dev2 = dict(dev, block_table=bt)
    res = run_decode(wl, dev2)
    assert res[3] & 0x2
    keys = np.concatenate([np.arange(0, 192), np.arange(256, 640)])
    O, lse = oracle_keys_attend(wl, 0, 1, keys)
    check_close(res[0][0, 4:8], res[1][0, 4:8], O[0], lse[0])
    sl = dev["seq_lens"].clone()
    sl[1] = 10 ** 6
    res = run_decode(wl, dict(dev, seq_lens=sl))
    assert res[3] & 0x4
    assert np.all(np.isneginf(res[1][1])) and np.all(res[0][1] == 0)


# ----------------------------------------------------------------------------- merge

def test_merge_lse_matches_oracle():
    torch = _torch()
    import sparse_kv_b200 as skv
    rng = np.random.default_rng(7)
    S, N, d = 9, 333, 128
    o = rng.standard_normal((S, N, d)).astype(np.float32)
    l = (rng.standard_normal((S, N)) * 5).astype(np.float32)
    l[2, :50] = -np.inf
    l[:, 7] = -np.inf  # all partials empty
    out = torch.empty((N, d), device="cuda")
    lse = torch.empty(N, device="cuda")
    skv.attn_merge_lse(torch.tensor(o, device="cuda"), torch.tensor(l, device="cuda"), out, lse)
    Om, lm = oracle.merge(o.astype(np.float64), l.astype(np.float64))
    got_o, got_l = out.cpu().numpy(), lse.cpu().numpy()
    assert np.isneginf(got_l[7]) and np.all(got_o[7] == 0)
    check_close(got_o, got_l, Om, lm)


def test_sharded_partials_merge_to_unsharded():
    torch = _torch()
    import sparse_kv_b200 as skv
    wl = skvgen.Workload("sh", B=2, Hq=8, Hkv=2, L=5000, paging="perm", seed=59)
    dev = device_workload(wl)
    bounds = [0, 700, 2048, 2049, 4100, 5000]
    outs, lses = [], []
    for a, e in zip(bounds[:-1], bounds[1:]):
        r = run_decode(wl, dev, kv_range=(a, e))
        outs.append(r[0].reshape(-1, 128))
        lses.append(r[1].reshape(-1))
    out = torch.empty((16, 128), device="cuda")
    lse = torch.empty(16, device="cuda")
    skv.attn_merge_lse(torch.tensor(np.array(outs), dtype=torch.float32, device="cuda"),
                       torch.tensor(np.array(lses), dtype=torch.float32, device="cuda"), out, lse)
    full = run_decode(wl, dev)
    check_close(out.cpu().numpy(), lse.cpu().numpy(), full[0].reshape(-1, 128), full[1].reshape(-1))
    _check_all_groups(wl, (out.cpu().numpy().reshape(2, 8, 128), lse.cpu().numpy().reshape(2, 8)),
                      lambda b: oracle.keys_full(5000))


# ----------------------------------------------------------------------------- centroid selection

def _select(wl, dev):
    torch = _torch()
    import sparse_kv_b200 as skv
    shape = (wl.B, wl.Hkv, wl.topk)
    ids = torch.empty(shape, dtype=torch.int32, device="cuda")
    ss = torch.empty(shape, dtype=torch.int32, device="cuda")
    se = torch.empty(shape, dtype=torch.int32, device="cuda")
    skv.attn_select_centroids(dev["q"], dev["centroids"], dev["cluster_off"], wl.topk, ids, ss, se)
    torch.cuda.synchronize()
    return ids, ss, se


def test_select_and_attend_small_mixture():
    wl = skvgen.Workload("m", B=2, Hq=8, Hkv=2, L=3000, mixture=True, c_log2=6, topk=7, seed=61)
    dev = device_workload(wl)
    ids, ss, se = _select(wl, dev)
    ids_h = ids.cpu().numpy()
    groups = [(b, h) for b in range(2) for h in range(2)]
    assert check_selection(wl, ids_h, groups) == 0
    off = dev["cluster_off"].cpu().numpy()
    np.testing.assert_array_equal(ss.cpu().numpy(), np.take_along_axis(off, ids_h, axis=2))
    np.testing.assert_array_equal(se.cpu().numpy(), np.take_along_axis(off, ids_h + 1, axis=2))
    res = run_decode(wl, dev, segments=(ss, se))
    assert res[3] == 0
    q = skvgen.host_q(wl)
    for b, kvh in groups:
        keys = oracle.keys_segments(off[b, kvh, ids_h[b, kvh]], off[b, kvh, ids_h[b, kvh] + 1])
        O, lse = oracle_keys_attend(wl, b, kvh, keys, q=q)
        hs = slice(kvh * 4, kvh * 4 + 4)
        check_close(res[0][b, hs], res[1][b, hs], O[0], lse[0])


@pytest.mark.parametrize("C", [1, 255, 256, 257, 768, 1000, 4096])
def test_select_pair_halves_every_chunk_count(C):
    """The per-sequence selection splits a group's centroid rows, in chunks of
    256, between the two CTAs of a pair: one chunk (the second CTA scores
    nothing), a ragged last chunk, odd and even chunk counts, and the largest C.
    Random bf16 queries and centroids; ids against the oracle's top-k."""
    torch = _torch()
    import sparse_kv_b200 as skv
    B, Hq, Hkv, d = 2, 8, 2, 128
    G, k = Hq // Hkv, min(C, 37)
    qb = skvgen.host_normal_bf16(900 + C, skvgen.S_Q, B * Hq * d).reshape(B, Hq, d)
    cb = skvgen.host_normal_bf16(900 + C, skvgen.S_CENTER, B * Hkv * C * d).reshape(B, Hkv, C, d)
    off = np.ascontiguousarray(np.broadcast_to(np.arange(C + 1, dtype=np.int32) * 5, (B, Hkv, C + 1)))

    def as_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)

    ids = torch.empty((B, Hkv, k), dtype=torch.int32, device="cuda")
    ss, se = torch.empty_like(ids), torch.empty_like(ids)
    skv.attn_select_centroids(as_bf16(qb), as_bf16(cb), torch.from_numpy(off).cuda(), k, ids, ss, se)
    torch.cuda.synchronize()
    ids_h = ids.cpu().numpy()
    for b in range(B):
        for h in range(Hkv):
            want, sc = oracle.select(qb[b, h * G:(h + 1) * G][None], cb[b, h][None], k)
            if not np.array_equal(want[0], ids_h[b, h]):
                assert oracle.topk_boundary_gap(sc, k)[0] <= TOPK_FLAG_GAP, f"C={C} ({b},{h})"
                check_topk_valid(ids_h[b, h], sc[0], k, f"C={C} ({b},{h})")
    np.testing.assert_array_equal(ss.cpu().numpy(), np.take_along_axis(off, ids_h, axis=2))
    np.testing.assert_array_equal(se.cpu().numpy(), np.take_along_axis(off, ids_h + 1, axis=2))


def test_select_ties_go_to_lower_index():
    torch = _torch()
    import sparse_kv_b200 as skv
    C, k = 300, 17
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    q[0, :, 0] = 1.0
    vals = np.random.default_rng(2).integers(0, 6, C).astype(np.float32)  # many exact ties
    cent = torch.zeros((1, 1, C, 128), dtype=torch.bfloat16, device="cuda")
    cent[0, 0, :, 0] = torch.tensor(vals, device="cuda")
    off = torch.arange(C + 1, dtype=torch.int32, device="cuda").view(1, 1, C + 1)
    ids = torch.empty((1, 1, k), dtype=torch.int32, device="cuda")
    ss, se = torch.empty_like(ids), torch.empty_like(ids)
    skv.attn_select_centroids(q, cent, off, k, ids, ss, se)
    want = sorted(sorted(range(C), key=lambda c: (-vals[c], c))[:k])
    assert ids.cpu().numpy()[0, 0].tolist() == want
