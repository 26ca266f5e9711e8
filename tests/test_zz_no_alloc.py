"""attn_decode_static_ws: decode for callers that cannot allocate device memory.

Such a caller passes inputs and outputs only; the scratch comes from a fixed
array inside the library.  The call must give what attn_decode gives (with a
caller-allocated workspace) on the same inputs, on consecutive calls that
reuse the array, and must refuse work that needs more scratch than the array
holds.  Kept in its own file, collected last.
"""
import os
import re

import numpy as np
import pytest

import skvgen
from helpers import ATOL_O, RTOL_LSE, device_workload, outputs

pytestmark = pytest.mark.gpu

_HDR = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                         "sparsekv.h")).read()
STATIC_BYTES = int(re.search(r"#define SKV_STATIC_WORKSPACE_BYTES \((\d+)u \* 1024u \* 1024u\)",
                             _HDR).group(1)) * 1024 * 1024


def _decode_pair(wl, dev, **kw):
    import torch
    import sparse_kv_b200 as skv
    args = (dev["q"], dev["k_pool"], dev["v_pool"], dev["block_table"], dev["seq_lens"])
    ref_o, ref_l = outputs(wl)
    n = skv.decode_workspace_size(*args, ref_o, ref_l, max_seq_len=wl.Lmax, **kw)
    assert n <= STATIC_BYTES
    ws = torch.empty(n // 4 + 4, dtype=torch.float32, device="cuda") if n else None
    ref_c = torch.full((wl.B, wl.Hq), -1, dtype=torch.int32, device="cuda")
    skv.attn_decode(*args, ref_o, ref_l, max_seq_len=wl.Lmax, workspace=ws, blocks_consumed=ref_c, **kw)
    got_o, got_l = outputs(wl)
    got_c = torch.full((wl.B, wl.Hq), -1, dtype=torch.int32, device="cuda")
    skv.attn_decode_static_ws(*args, got_o, got_l, max_seq_len=wl.Lmax, blocks_consumed=got_c, **kw)
    torch.cuda.synchronize()
    return (ref_o.cpu().numpy(), ref_l.cpu().numpy(), got_o.cpu().numpy(), got_l.cpu().numpy(),
            ref_c.cpu().numpy(), got_c.cpu().numpy())


def _close(a_o, a_l, b_o, b_l, a_c=None, b_c=None):
    assert np.all(np.isfinite(b_o))
    if a_c is not None:
        np.testing.assert_array_equal(a_c, b_c)
    assert np.abs(a_o - b_o).max() <= ATOL_O
    both_inf = np.isneginf(a_l) & np.isneginf(b_l)
    with np.errstate(invalid="ignore"):
        ok = both_inf | (np.abs(a_l - b_l) <= RTOL_LSE * np.maximum(1.0, np.abs(a_l)))
    assert np.all(ok)


def test_static_workspace_matches_caller_workspace_on_consecutive_calls():
    # first call: a batch split over many CTAs (scratch holds per-warp partials)
    wl1 = skvgen.Workload("na1", B=4, Hq=32, Hkv=8, L=8192, paging="perm", structured=True, seed=901)
    r1 = _decode_pair(wl1, device_workload(wl1))
    _close(*r1)
    # second call reuses the array with different shapes and a sink + recent window
    # (a walk long enough to need scratch too)
    lens = [30000, 64, 1, 25000, 0]
    wl2 = skvgen.Workload("na2", B=5, Hq=16, Hkv=4, L=max(lens), lens=lens, paging="perm", seed=902)
    r2 = _decode_pair(wl2, device_workload(wl2), window=(64, 20000))
    _close(*r2)
    # and the first workload again, now with stale contents from the second
    r3 = _decode_pair(wl1, device_workload(wl1))
    _close(*r3)
    np.testing.assert_array_equal(r1[2], r3[2])


def test_static_workspace_art_around_other_calls():
    """ART keeps control words (an item counter, ready flags, stop chunks) and
    look-back records in its scratch; they must be reset by every call even
    when the array holds another call's data.  ART at the Llama shape, then a
    persistent walk, then ART again, then a small walk that needs no scratch:
    outputs and blocks consumed equal the caller-workspace call's exactly."""
    wl = skvgen.Workload("na4", B=4, Hq=32, Hkv=8, L=12000, paging="perm", structured=True, seed=904)
    dev = device_workload(wl)
    # thresholds at which heads do stop (so stop chunks and re-folds are exercised)
    art = dict(art=(5e-2, 5e-3, 2))
    r1 = _decode_pair(wl, dev, **art)
    _close(*r1)
    np.testing.assert_array_equal(r1[0], r1[2])
    assert (r1[4] < wl.nb(0)).any()  # some head stopped early
    wl2 = skvgen.Workload("na5", B=3, Hq=16, Hkv=4, L=30000, paging="perm", seed=905)
    _close(*_decode_pair(wl2, device_workload(wl2)))
    r2 = _decode_pair(wl, dev, **art)
    _close(*r2)
    np.testing.assert_array_equal(r1[2], r2[2])
    np.testing.assert_array_equal(r1[5], r2[5])
    wl3 = skvgen.Workload("na6", B=1, Hq=8, Hkv=2, L=3000, paging="perm", seed=906)
    _close(*_decode_pair(wl3, device_workload(wl3)))


def test_static_workspace_refuses_oversized_work():
    import torch
    import sparse_kv_b200 as skv
    # 8192 KV groups of 8 query heads need about 280 MB of partial records: more than the array
    wl = skvgen.Workload("na3", B=1024, Hq=64, Hkv=8, L=64, seed=903)
    q = torch.zeros((wl.B, 1, wl.Hq, 128), dtype=torch.bfloat16, device="cuda")
    pool = torch.zeros((wl.B, wl.Hkv, 64, 128), dtype=torch.bfloat16, device="cuda")
    bt = torch.arange(wl.B, dtype=torch.int32, device="cuda").view(wl.B, 1)
    sl = torch.full((wl.B,), 64, dtype=torch.int32, device="cuda")
    o, l = outputs(wl)
    need = skv.decode_workspace_size(q, pool, pool, bt, sl, o, l, max_seq_len=64)
    assert need > STATIC_BYTES
    with pytest.raises(skv.SkvError) as e:
        skv.attn_decode_static_ws(q, pool, pool, bt, sl, o, l, max_seq_len=64)
    assert e.value.status == skv.SKV_EWORKSPACE
