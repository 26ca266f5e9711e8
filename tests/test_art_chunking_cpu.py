"""The chunked form of the ART stopping rule, as the GPU arbiter evaluates
it, against the sequential rule of the oracle (no GPU).

The probe after block t is the online-softmax combination of blocks 0..t,
which is associative ("ART" 2.1: the partial output is exposed after every
block).  The GPU splits a head's traversal into chunks of CB blocks, forms the
chunk-local prefix after every block, combines it with the previous chunk's
inclusive prefix, and decides all CB blocks of a chunk at once: block t passes
when d_scale < tau and d_dir < phi (and a previous probe exists); the run of
passes at t is the passes after the last failure at or before t inside the
chunk, or the previous chunk's run plus the chunk's passes up to t when
nothing failed; the head stops at the first t whose run reaches the patience.
This file replays that formulation in float64 and checks that it stops where
the oracle's sequential walk stops.
"""
import numpy as np
import pytest

import oracle


def _blocks(rng, T, rows=64, n=8, drift=1.0):
    """Per-block online-softmax pieces (m, l, O[0:n]) of random scores/values;
    later blocks get lower scores so that the probe settles (heads do stop)."""
    out = []
    for t in range(T):
        s = rng.standard_normal(rows) - drift * np.log1p(t)
        v = rng.standard_normal((rows, n))
        m = s.max()
        e = np.exp(s - m)
        out.append((m, e.sum(), e @ v))
    return out


def _combine(a, b):
    if a is None:
        return b
    m = max(a[0], b[0])
    fa, fb = np.exp(a[0] - m), np.exp(b[0] - m)
    return (m, a[1] * fa + b[1] * fb, a[2] * fa + b[2] * fb)


def _sequential_probes(blocks):
    x, acc = [], None
    for blk in blocks:
        acc = _combine(acc, blk)
        x.append(acc[2] / acc[1])
    return np.array(x)


def _chunked_stop(blocks, CB, tau, phi, patience):
    """Blocks consumed under the chunked decision (the arbiter's formulation)."""
    T = len(blocks)
    prev, prev_x, run = None, None, 0  # inclusive prefix, probe and run after the previous chunk
    for c0 in range(0, T, CB):
        chunk = blocks[c0:c0 + CB]
        local, xs = None, []
        for blk in chunk:  # chunk-local prefix after every block, then the global prefix
            local = _combine(local, blk)
            g = _combine(prev, local)
            xs.append(g[2] / g[1])
        passes = []
        for i, x in enumerate(xs):
            xp = xs[i - 1] if i > 0 else prev_x
            if xp is None:
                passes.append(False)  # the first consumed block has nothing to compare with
                continue
            ds, dc = oracle.art_metrics(xp, x)
            passes.append(ds < tau and dc < phi)
        for i in range(len(xs)):
            fails = [j for j in range(i + 1) if not passes[j]]
            r = (sum(passes[fails[-1] + 1:i + 1]) if fails else run + sum(passes[:i + 1]))
            if r >= patience:
                return c0 + i + 1
        fails = [j for j in range(len(xs)) if not passes[j]]
        run = sum(passes[fails[-1] + 1:]) if fails else run + sum(passes)
        prev, prev_x = _combine(prev, local), xs[-1]
    return T


@pytest.mark.parametrize("CB", [1, 3, 16, 32])
def test_chunked_rule_stops_where_the_sequential_rule_stops(CB):
    rng = np.random.default_rng(7 + CB)
    stops = []
    for trial in range(40):
        T = int(rng.integers(1, 120))
        blocks = _blocks(rng, T, drift=rng.uniform(0.5, 3.0))
        tau = 10 ** rng.uniform(-3, -0.5)
        phi = 10 ** rng.uniform(-4, -1)
        p = int(rng.integers(1, 6))
        x = _sequential_probes(blocks)
        want, margin = oracle.art_stop(x, tau, phi, p)
        got = _chunked_stop(blocks, CB, tau, phi, p)
        if margin > 1e-9:  # a decision this close to a threshold may round either way
            assert got == want, (trial, T, CB, tau, phi, p)
        stops.append(want < T)
    assert sum(stops) >= 10  # most trials stop before the end of their walk
