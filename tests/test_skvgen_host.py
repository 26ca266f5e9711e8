"""Host side of the seeded input generator (no GPU)."""
from fractions import Fraction

import numpy as np
import torch

import skvgen


def test_f32_to_bf16_matches_torch_rne():
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(2000).astype(np.float32),
                        # exact halfway cases between bf16 neighbours
                        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 3.0 + 2 ** -7],
                                 dtype=np.float32)])
    want = torch.tensor(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([skvgen.f32_to_bf16(v) for v in x], dtype=np.uint16)
    np.testing.assert_array_equal(got, want)


def _bf16_exact_round(x):
    """Reference: nearest bf16 (ties to even) by exact rational arithmetic."""
    if x == 0:
        return 0
    fx = Fraction(x)
    sign = 0x8000 if fx < 0 else 0
    a = abs(fx)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 7)
    q = a / ulp
    n = int(q)
    r = q - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    val = n * ulp  # in [2^e, 2^(e+1)]
    e2 = e + (1 if n == 256 else 0)
    mant = (int(val / Fraction(2) ** e2 * 128)) - 128
    return sign | ((e2 + 127) << 7) | mant


def test_f64_to_bf16_single_rounding():
    rng = np.random.default_rng(6)
    xs = list(rng.standard_normal(500) * 4)
    # values whose double rounding through fp32 would differ from one rounding:
    # just above a bf16 halfway point by less than an fp32 ulp
    xs += [1 + 2 ** -8 + 2 ** -40, 1 + 2 ** -8 - 2 ** -40, -(3 + 2 ** -7 + 2 ** -35), 1 + 2 ** -8]
    for x in xs:
        assert skvgen.f64_to_bf16(x) == _bf16_exact_round(x), x


def test_normal_samples_moments_and_range():
    x = skvgen.bf16_to_f64(skvgen.host_normal_bf16(42, skvgen.S_K, 200000))
    assert abs(x.mean()) < 0.01
    assert abs(x.var() - 1.0) < 0.01
    assert x.min() >= -6 and x.max() <= 6
    # counter-based: any sub-range regenerates the same values
    y = skvgen.bf16_to_f64(skvgen.host_normal_bf16(42, skvgen.S_K, 100, base=5000))
    np.testing.assert_array_equal(x[5000:5100], y)


def test_perm_is_permutation():
    p = skvgen.host_perm(3, 8192)
    assert sorted(p) == list(range(8192))
    assert not np.array_equal(p, np.arange(8192))


def test_structured_keys_sink_and_heavy():
    wl = skvgen.Workload("t", B=2, Hq=8, Hkv=2, L=5000, structured=True, seed=17)
    q = skvgen.host_q(wl)
    K, V = skvgen.host_kv_group(wl, 1, 1, q=q)
    plain = wl.with_(structured=False)
    K0, V0 = skvgen.host_kv_group(plain, 1, 1)
    np.testing.assert_array_equal(V, V0)
    heavy = [t for t in range(1, 5000) if skvgen.is_heavy(wl, 1, 1, t)]
    assert 20 < len(heavy) < 85  # ~1% of 5000
    qh = skvgen.host_qhat(q[1, 0, 4:8])
    assert abs(np.linalg.norm(qh) - 1) < 1e-15
    diff = skvgen.bf16_to_f64(K) - skvgen.bf16_to_f64(K0)
    changed = sorted(set(np.nonzero(np.abs(diff).sum(axis=1))[0]))
    assert changed == [0] + heavy
    # the shift is coef * qhat, up to one bf16 rounding of the sum
    np.testing.assert_allclose(diff[0], 6 * qh, atol=2 * 2 ** -7 * 8)
    np.testing.assert_allclose(diff[heavy[0]], 4 * qh, atol=2 * 2 ** -7 * 8)


def test_mixture_offsets_and_centroids():
    wl = skvgen.Workload("m", B=1, Hq=4, Hkv=1, L=4096, mixture=True, c_log2=6, seed=21)
    K, off, cent = skvgen.host_mixture_group(wl, 0, 0)
    assert off[0] == 0 and off[-1] == 4096 and np.all(np.diff(off) >= 0)
    sizes = np.diff(off)
    assert sizes.mean() == 64 and sizes.std() < 16
    Kf = skvgen.bf16_to_f64(K)
    Cf = skvgen.bf16_to_f64(cent)
    for c in range(64):
        if sizes[c]:
            m = Kf[off[c]:off[c + 1]].mean(axis=0)
            np.testing.assert_allclose(Cf[c], m, rtol=2 ** -8, atol=1e-30)
    # members sit near their centroid (sigma 0.3 around a N(0,1) center)
    within = np.linalg.norm(Kf[off[3]:off[4]] - Cf[3], axis=1).mean()
    across = np.linalg.norm(Kf[off[3]:off[4]] - Cf[4], axis=1).mean()
    assert within < 0.5 * across


def test_block_tables():
    wl = skvgen.Workload("p", B=3, Hq=4, Hkv=1, L=200, lens=[200, 64, 1], paging="perm", seed=5)
    bt, n = skvgen.block_table_host(wl)
    assert n == 4 + 1 + 1 and bt.shape == (3, 4)
    used = sorted(bt[bt >= 0].tolist())
    assert used == list(range(6))
    assert list(bt[1]) [1:] == [-1, -1, -1] and list(bt[2])[1:] == [-1, -1, -1]
    w = skvgen.Workload("w", B=1, Hq=4, Hkv=1, L=64 * 100, paging="window", sink=64, recent=64 * 3)
    bt, n = skvgen.block_table_host(w)
    assert n == 4 and list(np.nonzero(bt[0] >= 0)[0]) == [0, 97, 98, 99]
