"""Parity at the full workload sizes the benchmark times, on sampled KV groups
(the oracle recomputes each sampled group from the seeded generator)."""
import numpy as np
import pytest

import oracle
import skvgen
from helpers import (check_art, check_close, check_selection, device_workload, oracle_keys_attend,
                     run_decode)

pytestmark = pytest.mark.gpu

SAMPLE = [(0, 0), (5, 3), (10, 6), (15, 7)]


@pytest.fixture(scope="module")
def cfg2():
    wl = skvgen.WORKLOADS["cfg2_b16_h32_l32k"]
    return wl, device_workload(wl, nan_fill=False), skvgen.host_q(wl)


def test_cfg2_full_traversal_sampled(cfg2):
    wl, dev, q = cfg2
    res = run_decode(wl, dev)
    assert res[3] == 0
    for b, kvh in SAMPLE:
        O, lse = oracle_keys_attend(wl, b, kvh, oracle.keys_full(wl.L), q=q)
        hs = slice(kvh * 4, kvh * 4 + 4)
        check_close(res[0][b, hs], res[1][b, hs], O[0], lse[0], f"cfg2 group ({b},{kvh})")
    assert np.all(res[2] == wl.nb(0))
    # every row is finite and normalised-looking (|O| bounded by max |v| = 6)
    assert np.all(np.isfinite(res[0])) and np.abs(res[0]).max() <= 6.0


def test_cfg2_art_sampled(cfg2):
    wl, dev, q = cfg2
    res = run_decode(wl, dev, art=(wl.tau, wl.phi, wl.patience))
    assert res[3] == 0
    flagged = 0
    for b, kvh in SAMPLE:
        f, cons, mg = check_art(wl, res, b, kvh, q=q)
        flagged += f
    assert flagged <= 2


@pytest.fixture(scope="module")
def cfg3():
    wl = skvgen.WORKLOADS["cfg3_b8_h32_l64k_c1024_k102"]
    return wl, device_workload(wl, nan_fill=False), skvgen.host_q(wl)


def test_cfg3_selection_and_attention_sampled(cfg3):
    import torch
    import sparse_kv_b200 as skv
    wl, dev, q = cfg3
    shape = (wl.B, wl.Hkv, wl.topk)
    ids = torch.empty(shape, dtype=torch.int32, device="cuda")
    ss, se = torch.empty_like(ids), torch.empty_like(ids)
    skv.attn_select_centroids(dev["q"], dev["centroids"], dev["cluster_off"], wl.topk, ids, ss, se)
    torch.cuda.synchronize()
    ids_h = ids.cpu().numpy()
    sample = [(0, 0), (3, 5), (7, 7)]
    assert check_selection(wl, ids_h, sample, q=q) <= 1
    res = run_decode(wl, dev, segments=(ss, se))
    assert res[3] == 0
    off = dev["cluster_off"].cpu().numpy()
    for b, kvh in sample:
        sel = ids_h[b, kvh]
        keys = oracle.keys_segments(off[b, kvh, sel], off[b, kvh, sel + 1])
        O, lse = oracle_keys_attend(wl, b, kvh, keys, q=q)
        hs = slice(kvh * 4, kvh * 4 + 4)
        check_close(res[0][b, hs], res[1][b, hs], O[0], lse[0], f"cfg3 group ({b},{kvh})")


def _cfg5_layer(fa_wanted):
    wl = skvgen.WORKLOADS["cfg5_b8_h32_l128k_32layers"]
    for l in range(wl.n_layers):
        if (skvgen.route_bit(wl.seed, l) == 1) == fa_wanted:
            return wl, l
    pytest.skip("no layer with that route")


def test_cfg5_sparse_layer_window_sampled():
    wl, l = _cfg5_layer(False)
    lw = wl.with_(paging="window")
    dev = device_workload(lw, layer=l, nan_fill=True)  # only the window's pages exist
    res = run_decode(lw, dev, window=(wl.sink, wl.recent))
    assert res[3] == 0
    q = skvgen.host_q(lw, l)
    keys = oracle.keys_window(wl.L, wl.sink, wl.recent)
    for b, kvh in [(0, 0), (7, 7)]:
        O, lse = oracle_keys_attend(lw, b, kvh, keys, layer=l, q=q)
        hs = slice(kvh * 4, kvh * 4 + 4)
        check_close(res[0][b, hs], res[1][b, hs], O[0], lse[0], f"cfg5 SA layer {l} ({b},{kvh})")


def test_cfg5_full_layer_art_sampled():
    wl, l = _cfg5_layer(True)
    dev = device_workload(wl, layer=l, nan_fill=False)
    res = run_decode(wl, dev, art=(wl.tau, wl.phi, wl.patience))
    assert res[3] == 0
    q = skvgen.host_q(wl, l)
    flagged = 0
    for b, kvh in [(0, 0), (6, 5)]:
        f, _, _ = check_art(wl, res, b, kvh, layer=l, q=q)
        flagged += f
    assert flagged <= 2
