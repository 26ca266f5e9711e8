"""Lookahead block selection and prefetch from host memory ("SparDA",
technical summary section 2).  Layer l's Forecast projection of its activation
ranks layer l+1's blocks by their summaries; the top-k blocks are copied from a
page-locked host pool into a device cache by the gather kernel (reading host
memory through its device-mapped address); layer l+1 then attends the cache.

Checks, against the oracle on the same seeded inputs: the Forecast output bit
for bit (fp32 fused multiply-adds in input order, one bf16 rounding, the
precision that decides the block ids on both sides); the block ids (exact up
to flagged near ties, then a valid top-k); every cached row bit for bit
against the host pool; the attention over the cache against exact attention
over the chosen blocks' tokens."""
import numpy as np
import pytest

import oracle
import skvgen
from helpers import TOPK_FLAG_GAP, check_close, check_topk_valid, device_workload, group_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("lens,topk", [([5000, 5000], 9), ([5000, 3001, 1280], 12), ([200], 3)])
def test_forecast_select_prefetch_attend(lens, topk):
    import torch
    import sparse_kv_b200 as skv
    B, Hkv, G = len(lens), 2, 4
    wl = skvgen.Workload("pf", B=B, Hq=Hkv * G, Hkv=Hkv, L=max(lens), lens=lens, paging="perm",
                         seed=800 + topk)
    d, mb = wl.d, wl.max_blocks
    # layer 1's cache lives in host memory; layer 0 supplies the Forecast input
    dev1 = device_workload(wl, layer=1, nan_fill=False)
    k_host = dev1["k_pool"].cpu().pin_memory()
    v_host = dev1["v_pool"].cpu().pin_memory()
    summ = skvgen.device_block_means(wl, dev1["k_pool"], dev1["block_table"], dev1["seq_lens"])
    q0 = skvgen.device_q(wl, layer=0)
    x = q0[:, 0, ::G].contiguous()                       # head 0 of every GQA group
    w = skvgen.device_forecast_weights(wl, layer=0)
    f = torch.empty_like(x)
    skv.attn_forecast(x, w, f)
    off = torch.tensor([[[min(j * 64, L) for j in range(mb + 1)]] * Hkv for L in lens],
                       dtype=torch.int32, device="cuda")
    shape = (B, Hkv, topk)
    ids = torch.empty(shape, dtype=torch.int32, device="cuda")
    ss0, se0 = torch.empty_like(ids), torch.empty_like(ids)
    skv.attn_select_centroids(f, summ, off, topk, ids, ss0, se0)
    k_cache = torch.full((B * topk, Hkv, 64, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    v_cache = torch.full_like(k_cache, float("nan"))
    ss, se = torch.full_like(ids, -7), torch.full_like(ids, -7)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    skv.attn_prefetch_blocks(k_host, v_host, dev1["block_table"], dev1["seq_lens"], ids, k_cache, v_cache,
                             ss, se, max_seq_len=wl.Lmax, status=status, n_ctas=5)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # --- Forecast, bit for bit
    x_h = skvgen.host_q(wl, 0)[:, 0, ::G]
    w_h = skvgen.host_forecast_weights(wl, 0)
    f_ref = oracle.forecast(x_h.reshape(B * Hkv, d), np.tile(w_h, (B, 1, 1)))
    np.testing.assert_array_equal(f.view(torch.int16).cpu().numpy().view(np.uint16).reshape(B * Hkv, d), f_ref)
    # --- block ids against the oracle's choice from the same summaries
    ids_h = ids.cpu().numpy()
    kc = k_cache.view(torch.int16).cpu().numpy().view(np.uint16)
    kh = k_host.view(torch.int16).numpy().view(np.uint16)
    bt_h = dev1["bt_host"]
    flagged = 0
    q1 = skvgen.host_q(wl, 1)
    O_g_all = {}
    for b in range(B):
        for kvh in range(Hkv):
            qg, K, V = group_inputs(wl, b, kvh, layer=1, q=q1)
            nbk = wl.nb(b)
            summ_h = np.zeros((mb, d), dtype=np.uint16)
            summ_h[:nbk] = skvgen.host_block_means(K)
            ref, sc = oracle.select(f_ref[b * Hkv + kvh][None, None], summ_h[None], topk)
            if not np.array_equal(ref[0], ids_h[b, kvh]):
                assert oracle.topk_boundary_gap(sc, topk)[0] <= TOPK_FLAG_GAP
                check_topk_valid(ids_h[b, kvh], sc[0], topk, f"({b},{kvh})")
                flagged += 1
            # --- the cache holds exactly the chosen blocks' rows
            for i, j in enumerate(ids_h[b, kvh]):
                n = max(0, min(64, wl.seq_len(b) - j * 64)) if j < nbk else 0
                assert ss.cpu().numpy()[b, kvh, i] == i * 64 and se.cpu().numpy()[b, kvh, i] == i * 64 + n
                if n:
                    np.testing.assert_array_equal(kc[b * topk + i, kvh, :n], kh[bt_h[b, j], kvh, :n])
    assert flagged <= 1
    # --- layer 1 attends the cache
    bt_c = torch.arange(B * topk, dtype=torch.int32, device="cuda").view(B, topk)
    sl_c = torch.full((B,), topk * 64, dtype=torch.int32, device="cuda")
    q1_d = skvgen.device_q(wl, layer=1)
    out = torch.empty((B, 1, wl.Hq, d), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, 1, wl.Hq), dtype=torch.float32, device="cuda")
    skv.attn_decode(q1_d, k_cache, v_cache, bt_c, sl_c, out, lse, max_seq_len=topk * 64, scale=wl.scale,
                    segments=(ss, se), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for b in range(B):
        for kvh in range(Hkv):
            qg, K, V = group_inputs(wl, b, kvh, layer=1, q=q1)
            keys = oracle.keys_blocks(ids_h[b, kvh], wl.seq_len(b))
            O, l = oracle.attend(qg[None], K[None], V[None], [[keys] * G], wl.scale)
            hs = slice(kvh * G, (kvh + 1) * G)
            check_close(out[b, 0, hs].cpu().numpy(), lse[b, 0, hs].cpu().numpy(), O[0], l[0], f"({b},{kvh})")
