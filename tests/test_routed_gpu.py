"""The routed layer stack as a whole ("Flux Attention" 2: per-layer hard routing
between full attention and a sink + recent window).  Four consecutive layers
of the cfg5 shape (batch 8, 32 q / 8 KV heads, context 131072) go through the
benchmark's own dispatch, one attn_decode per layer on one stream, mixing both
routes; each layer's sampled KV groups are checked against the oracle for that
layer's route bit: ART over the whole cache (block 0 first, recency-first) for
a full layer, exact attention over tokens [0, 64) U [L - 4096, L) for a sparse
one."""
import numpy as np
import pytest

import oracle
import skvgen
from helpers import check_art, check_close, oracle_keys_attend

pytestmark = pytest.mark.gpu

LAYERS = range(2, 6)  # route bits 0, 1, 0, 1 for the cfg5 seed
SAMPLE = [(0, 0), (7, 7)]


def test_routed_stack_layers_match_their_routes():
    import torch
    import bench
    import sparse_kv_b200 as skv
    wl = skvgen.WORKLOADS["cfg5_b8_h32_l128k_32layers"]
    bits = [skvgen.route_bit(wl.seed, l) for l in LAYERS]
    assert 0 in bits and 1 in bits, bits
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    step = bench.build_routed(torch, skv, skvgen, wl, status, layer_ids=LAYERS)
    # clear the outputs, then run the whole dispatch once more (the builder ran it once)
    for ly in step.tensors["layers"]:
        ly["out"].fill_(float("nan"))
        ly["lse"].fill_(float("nan"))
        ly["consumed"].fill_(-1)
    step.run()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    keys_sa = oracle.keys_window(wl.L, wl.sink, wl.recent)
    flagged = 0
    for ly in step.tensors["layers"]:
        l = ly["layer"]
        assert ly["fa"] == (skvgen.route_bit(wl.seed, l) == 1)
        out = ly["out"][:, 0].cpu().numpy().astype(np.float64)
        lse = ly["lse"][:, 0].cpu().numpy().astype(np.float64)
        cons = ly["consumed"].cpu().numpy()
        q = skvgen.host_q(wl, l)
        for b, kvh in SAMPLE:
            hs = slice(kvh * wl.G, (kvh + 1) * wl.G)
            if ly["fa"]:
                f, _, _ = check_art(wl, (out, lse, cons, 0), b, kvh, layer=l, q=q)
                flagged += f
            else:
                O, l_ref = oracle_keys_attend(wl, b, kvh, keys_sa, layer=l, q=q)
                check_close(out[b, hs], lse[b, hs], O[0], l_ref[0], f"layer {l} SA ({b},{kvh})")
                assert np.all(cons[b, hs] == 65), cons[b, hs]  # block 0 + the last 64 blocks
    assert flagged <= 2
