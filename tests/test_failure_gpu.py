"""Failure detection on the GPU without a fault: a bounded wait made to expire.

The test hook skv_test_withhold_tile makes one CTA's producer warp stop before
a given ring entry, so that CTA's consumer warps wait for a tile that never
arrives.  Their wait is bounded (1 s of %globaltimer); when it expires they set
SKV_DEV_TIMEOUT in the status word, the producer drains the copies it issued,
and the kernel returns.  The call must come back within seconds with the
timeout bit set, and the context must stay usable: the next call, without the
hook, is exact again.  Nothing here faults, traps or hangs a GPU.
"""
import time

import numpy as np
import pytest

import oracle
import skvgen
from helpers import check_close, device_workload, oracle_keys_attend, run_decode

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,cta,entry", [
    # 8 KV groups x 320 tiles: the persistent schedule (296 CTAs, then the record merge)
    (dict(B=1, Hq=32, Hkv=8, L=320 * 64), 5, 2),
    # a small walk: one cluster of CTAs per KV group, merged in distributed shared memory
    (dict(B=1, Hq=8, Hkv=2, L=4096), 1, 1),
])
def test_withheld_tile_times_out_and_the_next_call_is_exact(shape, cta, entry):
    import sparse_kv_b200 as skv
    wl = skvgen.Workload("fail", paging="perm", seed=950 + cta, **shape)
    dev = device_workload(wl)
    skv.test_withhold_tile(cta, entry)
    t0 = time.monotonic()
    _, _, _, status = run_decode(wl, dev)
    elapsed = time.monotonic() - t0
    assert status & skv.DEV_BITS["timeout"], f"status {status:#x}"
    assert skv.status_of_word(status) == skv.SKV_ETIMEOUT
    assert elapsed < 30.0, elapsed  # bounded: 1 s per wait, a few waits in a row at most
    # the hook was one-shot and the context is fine: the same call is exact again
    O_g, lse_g, cons, status = run_decode(wl, dev)
    assert status == 0
    q = skvgen.host_q(wl)
    for kvh in (0, wl.Hkv - 1):
        O, lse = oracle_keys_attend(wl, 0, kvh, oracle.keys_full(wl.L), q=q)
        hs = slice(kvh * wl.G, (kvh + 1) * wl.G)
        check_close(O_g[0, hs], lse_g[0, hs], O[0], lse[0], f"after timeout, group {kvh}")
    assert np.all(cons == wl.nb(0))
