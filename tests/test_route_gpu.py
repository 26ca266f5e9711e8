"""GPU parity of attn_route_layers (per-layer hard routing, "Flux Attention"
section 2) against the CPU fp64 oracle, on seeded inputs."""
import numpy as np
import pytest

import oracle
import skvgen

pytestmark = pytest.mark.gpu


def _inputs(L, B, T, Hq, d, seed):
    import torch
    F = Hq * d
    q = torch.empty((L, B, T, Hq, d), dtype=torch.bfloat16, device="cuda")
    skvgen.device_normal_bf16(q, seed, skvgen.S_Q)
    q_host = skvgen.host_normal_bf16(seed, skvgen.S_Q, q.numel()).reshape(L, B, T, F)
    # weights and biases: generator values scaled by powers of two (exact in fp32)
    w = skvgen.bf16_to_f64(skvgen.host_normal_bf16(seed, skvgen.S_ROUTER_W, L * 2 * F)).reshape(L, 2 * F) / 32
    bias = skvgen.bf16_to_f64(skvgen.host_normal_bf16(seed, skvgen.S_ROUTER_W, L, base=L * 2 * F)) / 8
    return q, q_host, w, bias


def _check(L, B, T, Hq, d, n_p, n_s, seed, with_bias=True):
    import torch
    import sparse_kv_b200 as skv
    q, q_host, w, bias = _inputs(L, B, T, Hq, d, seed)
    if not with_bias:
        bias = np.zeros(L)
    w_d = torch.tensor(w, dtype=torch.float32, device="cuda")
    b_d = torch.tensor(bias, dtype=torch.float32, device="cuda") if with_bias else None
    route = torch.full((L, B), 7, dtype=torch.uint8, device="cuda")
    logits = torch.full((L, B), float("nan"), dtype=torch.float32, device="cuda")
    skv.attn_route_layers(q, w_d, b_d, n_p, n_s, route, logits)
    torch.cuda.synchronize()
    z_ref, r_ref = oracle.route(q_host, w, bias, n_p, n_s)
    z, r = logits.cpu().numpy().astype(np.float64), route.cpu().numpy()
    # Error bound of the kernel's fp32 arithmetic (eps = 2^-24): each pooled
    # feature is a sequential sum of n rows (error <= n eps sum|x|), and the
    # dot product sums 16 terms per 8-feature chunk, a thread's chunks in
    # turn, then a tree over the block and the bias (error <= (2F/256 + 16)
    # eps sum|w f| covers any block size up to 2^16); a factor 4 of margin.
    eps = 2.0 ** -24
    x = skvgen.bf16_to_f64(q_host)
    pre, suf = x[:, :, :n_p], x[:, :, T - n_s:]
    m = np.concatenate([np.abs(pre).mean(axis=2), np.abs(suf).mean(axis=2)], axis=-1)
    f = np.concatenate([pre.mean(axis=2), suf.mean(axis=2)], axis=-1)
    F2 = 2 * Hq * d
    tol = 4 * eps * (max(n_p, n_s) * np.einsum("lbf,lf->lb", m, np.abs(w))
                     + (F2 / 256 + 16) * (np.einsum("lbf,lf->lb", np.abs(f), np.abs(w)) + np.abs(bias)[:, None])) + 1e-7
    assert np.all(np.abs(z - z_ref) <= tol), np.max(np.abs(z - z_ref) / tol)
    decided = np.abs(z_ref) > tol
    np.testing.assert_array_equal(r[decided], r_ref[decided])
    assert set(np.unique(r)) <= {0, 1}
    return int((~decided).sum())


@pytest.mark.parametrize("L,B,T,Hq,d,n_p,n_s", [
    (4, 5, 37, 8, 128, 16, 9),      # ragged row counts (not multiples of 8)
    (3, 2, 1, 4, 128, 1, 1),        # one token: prefix = suffix
    (2, 3, 20, 2, 64, 20, 20),      # prefix and suffix cover everything
    (5, 1, 300, 1, 8, 64, 64),      # F = 8: one chunk per CTA
])
def test_route_matches_oracle(L, B, T, Hq, d, n_p, n_s):
    _check(L, B, T, Hq, d, n_p, n_s, seed=0x707 + T)


def test_route_without_bias():
    _check(3, 4, 50, 8, 128, 32, 16, seed=0x808, with_bias=False)


def test_route_full_size():
    # 32 layers x 8 sequences, 64 prefix + 64 suffix tokens of 32 x 128 query
    # features each (the routed decode stack's shape)
    flagged = _check(32, 8, 128, 32, 128, 64, 64, seed=0x909)
    assert flagged <= 16  # logits within the error bound of zero: either route is correct
