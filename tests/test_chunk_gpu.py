"""Query-chunk attention on the tensor cores (q_tokens > 1) against the oracle.

Every partial (one shard, or the chunk's own keys under the causal mask) and
every merged result is held to the same tolerances as decode: max |dO| <= 2e-3
and |dlse| <= 1e-4 * max(1, |lse|).  The kernel carries P into the P.V product
as two bf16 terms (hi + lo), so the weights keep about 16 significant bits; a
single bf16 term would miss 2e-3 on partials dominated by a few keys (the first
tokens of the causal chunk, peaky logits).
"""
import numpy as np
import pytest

import oracle
import skvgen
from helpers import check_close, device_workload

pytestmark = pytest.mark.gpu


def chunk_call(wl, dev, n_parts, kv_range=None, causal=False, shards=0, out=None, lse=None):
    import torch
    import sparse_kv_b200 as skv
    if out is None:
        out = torch.full((max(shards, 1), wl.B, wl.Tq, wl.Hq, wl.d), float("nan"), device="cuda")
        lse = torch.full((max(shards, 1), wl.B, wl.Tq, wl.Hq), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    skv.attn_decode(dev["q"], dev["k_pool"], dev["v_pool"], dev["block_table"], dev["seq_lens"],
                    out, lse, max_seq_len=wl.Lmax, scale=wl.scale, kv_range=kv_range, causal=causal,
                    kv_shards=shards, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, lse


def oracle_rows(wl, b, key_fn, q=None):
    """Oracle O, lse for every (t, h) of sequence b; key_fn(t) -> key indices."""
    q = skvgen.host_q(wl) if q is None else q
    O = np.zeros((wl.Tq, wl.Hq, wl.d))
    lse = np.zeros((wl.Tq, wl.Hq))
    for kvh in range(wl.Hkv):
        K, V = skvgen.host_kv_group(wl, b, kvh, q=q)
        qg = q[b, :, kvh * wl.G:(kvh + 1) * wl.G]                   # [Tq][G][d]
        qq = qg.reshape(1, wl.Tq * wl.G, wl.d)
        idx = [[key_fn(r // wl.G) for r in range(wl.Tq * wl.G)]]
        o, l = oracle.attend(qq, K[None], V[None], idx, wl.scale)
        O[:, kvh * wl.G:(kvh + 1) * wl.G] = o[0].reshape(wl.Tq, wl.G, wl.d)
        lse[:, kvh * wl.G:(kvh + 1) * wl.G] = l[0].reshape(wl.Tq, wl.G)
    return O, lse


def check_partial(got_o, got_l, O, lse, what):
    """A partial against exact attention over its key set (decode tolerances)."""
    return check_close(got_o, got_l, O, lse, what)


@pytest.mark.parametrize("G,Tq", [(4, 32), (4, 40), (2, 64), (8, 16)])
def test_chunk_whole_sequence(G, Tq):
    lens = [700, 64 * 3]
    wl = skvgen.Workload("c1", B=2, Hq=2 * G, Hkv=2, L=max(lens), lens=lens, Tq=Tq, paging="perm",
                         seed=300 + G + Tq)
    dev = device_workload(wl)
    out, lse = chunk_call(wl, dev, 1)
    q = skvgen.host_q(wl)
    for b in range(2):
        O, l = oracle_rows(wl, b, lambda t: oracle.keys_full(wl.seq_len(b)), q)
        check_partial(out[0, b].cpu().numpy(), lse[0, b].cpu().numpy(), O, l, f"seq {b}")


def test_chunk_causal_tail_and_shards_merge_exactly():
    import torch
    import sparse_kv_b200 as skv
    Tq, ctx = 32, 1000
    wl = skvgen.Workload("c2", B=2, Hq=8, Hkv=2, L=ctx + Tq, Tq=Tq, paging="perm", seed=331)
    dev = device_workload(wl)
    q = skvgen.host_q(wl)
    S = 3
    parts_o = torch.full((S + 1, wl.B, Tq, wl.Hq, wl.d), float("nan"), device="cuda")
    parts_l = torch.full((S + 1, wl.B, Tq, wl.Hq), float("nan"), device="cuda")
    chunk_call(wl, dev, S, kv_range=(0, ctx), shards=S, out=parts_o[:S], lse=parts_l[:S])
    chunk_call(wl, dev, 1, kv_range=(ctx, ctx + Tq), causal=True, out=parts_o[S:], lse=parts_l[S:])
    # each partial against the oracle on its own key set
    for s in range(S):
        a, e = s * ctx // S, (s + 1) * ctx // S
        for b in range(2):
            O, l = oracle_rows(wl, b, lambda t: np.arange(a, e), q)
            check_partial(parts_o[s, b].cpu().numpy(), parts_l[s, b].cpu().numpy(), O, l,
                          f"shard {s} seq {b}")
    for b in range(2):
        O, l = oracle_rows(wl, b, lambda t: np.arange(ctx, ctx + t + 1), q)
        check_partial(parts_o[S, b].cpu().numpy(), parts_l[S, b].cpu().numpy(), O, l,
                      f"causal chunk seq {b}")
    # merged = unsharded causal attention over context + chunk ("Pulsar Attention" Phase 2)
    N = wl.B * Tq * wl.Hq
    mo = torch.empty((N, wl.d), device="cuda")
    ml = torch.empty(N, device="cuda")
    skv.attn_merge_lse(parts_o.view(S + 1, N, wl.d), parts_l.view(S + 1, N), mo, ml)
    torch.cuda.synchronize()
    mo = mo.view(wl.B, Tq, wl.Hq, wl.d).cpu().numpy()
    ml = ml.view(wl.B, Tq, wl.Hq).cpu().numpy()
    for b in range(2):
        O, l = oracle_rows(wl, b, lambda t: oracle.keys_chunk(ctx, t), q)
        check_close(mo[b], ml[b], O, l, f"merged seq {b}")


def test_chunk_full_size_sampled():
    """8 context shards of 16384 keys + the causal 128-token chunk, batch 4,
    32 q / 8 KV heads, merged and checked on sampled rows."""
    import torch
    import sparse_kv_b200 as skv
    wl = skvgen.WORKLOADS["cfg4_b4_h32_l128k_chunk128"]
    ctx, Tq, S = wl.L - wl.chunk, wl.Tq, wl.shards
    dev = device_workload(wl, nan_fill=False)
    parts_o = torch.empty((S + 1, wl.B, Tq, wl.Hq, wl.d), device="cuda")
    parts_l = torch.empty((S + 1, wl.B, Tq, wl.Hq), device="cuda")
    chunk_call(wl, dev, S, kv_range=(0, ctx), shards=S, out=parts_o[:S], lse=parts_l[:S])
    chunk_call(wl, dev, 1, kv_range=(ctx, ctx + Tq), causal=True, out=parts_o[S:], lse=parts_l[S:])
    N = wl.B * Tq * wl.Hq
    mo = torch.empty((N, wl.d), device="cuda")
    ml = torch.empty(N, device="cuda")
    skv.attn_merge_lse(parts_o.view(S + 1, N, wl.d), parts_l.view(S + 1, N), mo, ml)
    torch.cuda.synchronize()
    mo = mo.view(wl.B, Tq, wl.Hq, wl.d).cpu().numpy()
    ml = ml.view(wl.B, Tq, wl.Hq).cpu().numpy()
    q = skvgen.host_q(wl)
    rng = np.random.default_rng(4)
    for (b, kvh) in [(0, 0), (3, 7)]:
        K, V = skvgen.host_kv_group(wl, b, kvh, q=q)
        for t in list(rng.choice(Tq, 3, replace=False)) + [0, Tq - 1]:
            qg = q[b, t, kvh * wl.G:(kvh + 1) * wl.G][None]
            O, l = oracle.attend(qg, K[None], V[None], [[oracle.keys_chunk(ctx, t)] * wl.G], wl.scale)
            hs = slice(kvh * wl.G, (kvh + 1) * wl.G)
            check_close(mo[b, t, hs], ml[b, t, hs], O[0], l[0], f"cfg4 b{b} t{t} kvh{kvh}")


@pytest.mark.parametrize("scale", [0.35, 1.0])
def test_chunk_peaky_partials(scale):
    """Sink + heavy-token keys and a large softmax scale: a few keys carry most of
    every row's weight, the case where rounding the weights hurts most.  Each
    shard's partial and the causal chunk partial are held to 2e-3."""
    Tq, ctx, S = 48, 1500, 2
    wl = skvgen.Workload("cpk", B=2, Hq=8, Hkv=2, L=ctx + Tq, Tq=Tq, paging="perm", structured=True,
                         softmax_scale=scale, seed=340 + int(scale * 100))
    dev = device_workload(wl)
    q = skvgen.host_q(wl)
    import torch
    parts_o = torch.full((S + 1, wl.B, Tq, wl.Hq, wl.d), float("nan"), device="cuda")
    parts_l = torch.full((S + 1, wl.B, Tq, wl.Hq), float("nan"), device="cuda")
    chunk_call(wl, dev, S, kv_range=(0, ctx), shards=S, out=parts_o[:S], lse=parts_l[:S])
    chunk_call(wl, dev, 1, kv_range=(ctx, ctx + Tq), causal=True, out=parts_o[S:], lse=parts_l[S:])
    worst = 0.0
    for b in range(2):
        for s in range(S):
            a, e = s * ctx // S, (s + 1) * ctx // S
            O, l = oracle_rows(wl, b, lambda t: np.arange(a, e), q)
            worst = max(worst, check_partial(parts_o[s, b].cpu().numpy(), parts_l[s, b].cpu().numpy(),
                                             O, l, f"peaky shard {s} seq {b}"))
        O, l = oracle_rows(wl, b, lambda t: np.arange(ctx, ctx + t + 1), q)
        worst = max(worst, check_partial(parts_o[S, b].cpu().numpy(), parts_l[S, b].cpu().numpy(), O, l,
                                         f"peaky causal chunk seq {b}"))
    print(f"peaky chunk partials (scale {scale}): max |dO| = {worst:.3e}")
