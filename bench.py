#!/usr/bin/env python
"""Benchmark: streaming decode attention over a paged bf16 KV cache on B200.

Default workload: Llama-3.1-8B-shaped decode, batch 16, 32 query / 8 KV heads,
head_dim 128, context 32768 in 64-token pages scattered by a seeded
permutation, sink + 1% heavy-token key structure (synthetic, seeded).  One
step = one attn_decode call over the whole batch (full traversal: plan, tile
fetch, scores, online softmax, P.V, split-KV merge).  The same inputs are then
decoded with ART run-time termination (tau 1e-3, phi 1e-4, patience 4,
recency-first) and reported under "art".

Metric: effective KV GB/s = algorithmic K+V bytes (tokens x kv_heads x 512 B)
/ device time, plus attended tokens/s.  Inputs (2 GiB of KV per step) are far
larger than the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU: independent replicas (the path has no exchange step); value is the
sum over ranks of bytes / max-over-ranks time.
"""
import argparse
import ctypes
import json
import math
import os
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn effective KV GB/s (fraction of B200 HBM peak); attended tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="cfg2_b16_h32_l32k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-art", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="time the headline workload only (skip the other workloads' lines)")
    return ap.parse_args()


def tensor_peak(power_capped):
    """Dense bf16 peak: the burst figure while the clocks held (no power cap
    seen during the timed region), else the sustained one."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if power_capped:
            return d["bf16_tflops_sustained"], "measured sustained bf16 (sw_power_cap seen)"
        return d["bf16_tflops"], "measured burst bf16 (no power cap seen)"
    return (1400.0, "fallback sustained bf16") if power_capped else (1590.0, "fallback burst bf16")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], "measured"
    return 6650.0, "fallback"


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every millisecond
    in a background thread while the timed region runs (read-only queries; a
    short timed region still yields several samples)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, uuid, period_s=0.001):
        self.uuid, self.period = uuid, period_s
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.ok = False

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(self.uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report it, do not guess
            self.err = str(e)
            return self
        self.stop = threading.Event()
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()
        return self

    def _run(self):
        nv = self.nv
        while not self.stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, name in self.REASONS.items():
                    if bits & k:
                        self.reasons.add(name)
            except Exception:
                pass
            self.stop.wait(self.period)

    def __exit__(self, *exc):
        if self.ok:
            self.stop.set()
            self.t.join(timeout=2)

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- CPU baseline (oracle)

def _oracle_sample(wl, n_groups):
    import numpy as np
    import skvgen
    q = skvgen.host_q(wl)
    step = max(1, wl.B * wl.Hkv // n_groups)
    groups = [(g // wl.Hkv, g % wl.Hkv) for g in range(0, wl.B * wl.Hkv, step)][:n_groups]
    Ks, Vs, qs = [], [], []
    for b, kvh in groups:
        K, V = skvgen.host_kv_group(wl, b, kvh, q=q)
        Ks.append(K)
        Vs.append(V)
        qs.append(q[b, 0, kvh * wl.G:(kvh + 1) * wl.G])
    keys = [[np.arange(wl.L)] * wl.G for _ in groups]
    return np.stack(qs), np.stack(Ks), np.stack(Vs), keys, groups


def cpu_baseline(wl, budget_s=20.0, chunk=16):
    """The fp64 oracle, as it stands, on a bounded sample of the workload:
    full-traversal attention of whole KV groups (all G query heads each), in
    chunks of `chunk` groups until every group is done or `budget_s` of oracle
    time is spent."""
    import oracle
    total_groups = wl.B * wl.Hkv
    done, t_oracle = 0, 0.0
    while done < total_groups and t_oracle < budget_s:
        n = min(chunk, total_groups - done)
        qs, Ks, Vs, keys, _ = _oracle_sample_range(wl, done, n)
        t0 = time.perf_counter()
        oracle.attend(qs, Ks, Vs, keys, wl.scale)
        t_oracle += time.perf_counter() - t0
        done += n
    nbytes = done * wl.L * wl.d * 2 * 2
    cores = oracle.threads()
    # the same oracle on one thread, over a few KV groups
    n1 = min(8, total_groups)
    qs, Ks, Vs, keys, _ = _oracle_sample_range(wl, 0, n1)
    oracle.set_threads(1)
    try:
        t0 = time.perf_counter()
        oracle.attend(qs, Ks, Vs, keys, wl.scale)
        t1 = time.perf_counter() - t0
    finally:
        oracle.set_threads(cores)
    return {"value": nbytes / t_oracle / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} of {total_groups} KV groups of {wl.name}, full traversal, fp64 "
                      f"oracle time {t_oracle:.2f} s",
            "one_core": {"value": n1 * wl.L * wl.d * 2 * 2 / t1 / 1e9, "unit": "GB/s",
                         "sample": f"{n1} KV groups, oracle time {t1:.2f} s"}}


def _oracle_sample_range(wl, g0, n):
    import numpy as np
    import skvgen
    q = skvgen.host_q(wl)
    Ks, Vs, qs = [], [], []
    for g in range(g0, g0 + n):
        b, kvh = g // wl.Hkv, g % wl.Hkv
        K, V = skvgen.host_kv_group(wl, b, kvh, q=q)
        Ks.append(K)
        Vs.append(V)
        qs.append(q[b, 0, kvh * wl.G:(kvh + 1) * wl.G])
    keys = [[np.arange(wl.L)] * wl.G for _ in range(n)]
    return np.stack(qs), np.stack(Ks), np.stack(Vs), keys, None


def run_reference(args):
    """--impl reference: the CPU oracle, as it stands, on the host cores (rank
    0 only).  Each step is the oracle's full-traversal attention over a bounded
    sample of the workload (4 of its KV groups), so that the run ends within a
    few minutes."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    import skvgen
    wl = skvgen.WORKLOADS[args.workload]
    n_groups = 4
    qs, Ks, Vs, keys, groups = _oracle_sample(wl, n_groups)
    for _ in range(args.warmup):
        oracle.attend(qs, Ks, Vs, keys, wl.scale)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attend(qs, Ks, Vs, keys, wl.scale)
    dt = (time.perf_counter() - t0) / args.steps
    nbytes = n_groups * wl.L * wl.d * 4
    v = nbytes / dt / 1e9
    cores = oracle.threads()
    sample = f"{n_groups} of {wl.B * wl.Hkv} KV groups of {wl.name} per step, full traversal, fp64"
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": wl.name, "sample_groups": n_groups},
           "cpu_baseline": {"value": v, "unit": "GB/s", "kind": "oracle", "cores": cores,
                            "sample": sample},
           "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# --------------------------------------------------------------------------- our arm

class Step:
    """One benchmark step: `run()` launches it on the current stream; `nbytes`
    are the algorithmic bytes it moves; `launches` our kernels per step."""

    def __init__(self, run, nbytes, launches, extra=None):
        self.run, self.nbytes, self.launches, self.extra = run, nbytes, launches, extra or {}


def _paged_inputs(torch, skvgen, wl, layer=0):
    bt_host, num_pages = skvgen.block_table_host(wl, layer)
    q = skvgen.device_q(wl, layer)
    k_pool = torch.empty((max(num_pages, 1), wl.Hkv, wl.bs, wl.d), dtype=torch.bfloat16, device="cuda")
    v_pool = torch.empty_like(k_pool)
    block_table = torch.tensor(bt_host, device="cuda")
    seq_lens = torch.tensor([wl.seq_len(b) for b in range(wl.B)], dtype=torch.int32, device="cuda")
    return q, k_pool, v_pool, block_table, seq_lens


def build_decode(torch, skv, skvgen, wl, status, art=None, inputs=None, layer=0):
    """Full-traversal (or ART: art = (tau, phi, patience)) decode of one paged
    workload (layer `layer` of its seeded inputs); `inputs` = (q, k_pool,
    v_pool, block_table, seq_lens) of another step to share its cache."""
    if inputs is None:
        q, k_pool, v_pool, bt, sl = _paged_inputs(torch, skvgen, wl, layer=layer)
        skvgen.device_kv_paged(wl, q, k_pool, v_pool, bt, sl, layer=layer)
    else:
        q, k_pool, v_pool, bt, sl = inputs
    out = torch.empty((wl.B, 1, wl.Hq, wl.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((wl.B, 1, wl.Hq), dtype=torch.float32, device="cuda")
    consumed = torch.zeros((wl.B, wl.Hq), dtype=torch.int32, device="cuda")
    common = (q, k_pool, v_pool, bt, sl, out, lse)
    kw = dict(max_seq_len=wl.Lmax, scale=wl.scale, status=status, blocks_consumed=consumed)
    if art is not None:
        kw["art"] = tuple(art)
    n = skv.decode_workspace_size(*common, **kw)
    ws = torch.empty(max(n, 16) // 4 + 4, dtype=torch.float32, device="cuda") if n else None
    a = skv.make_decode_args(*common, workspace=ws, **kw)
    L = skv.lib()

    def run():
        st = L.attn_decode(ctypes.byref(a), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        if st != 0:
            raise skv.SkvError(st, "attn_decode")

    step = Step(run, wl.kv_bytes(), L.skv_decode_launches(ctypes.byref(a)))
    # keep every tensor the raw pointers in `a` refer to alive with the step
    step.tensors = dict(q=q, k_pool=k_pool, v_pool=v_pool, bt=bt, sl=sl, out=out, lse=lse,
                        consumed=consumed, ws=ws, kw=kw, common=common)
    return step


def build_select(torch, skv, skvgen, wl, status):
    """Centroid scoring + top-k, then attention over the chosen clusters' keys."""
    q, k_pool, v_pool, bt, sl = _paged_inputs(torch, skvgen, wl)
    off, cent = skvgen.device_mixture(wl, k_pool, bt)
    skvgen.device_kv_paged(wl, q, k_pool, v_pool, bt, sl, keys=False)
    shape = (wl.B, wl.Hkv, wl.topk)
    ids = torch.empty(shape, dtype=torch.int32, device="cuda")
    ss = torch.empty(shape, dtype=torch.int32, device="cuda")
    se = torch.empty(shape, dtype=torch.int32, device="cuda")
    out = torch.empty((wl.B, 1, wl.Hq, wl.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((wl.B, 1, wl.Hq), dtype=torch.float32, device="cuda")
    kw = dict(max_seq_len=wl.Lmax, scale=wl.scale, status=status, segments=(ss, se))
    n = skv.decode_workspace_size(q, k_pool, v_pool, bt, sl, out, lse, **kw)
    ws = torch.empty(max(n, 16) // 4 + 4, dtype=torch.float32, device="cuda")
    a = skv.make_decode_args(q, k_pool, v_pool, bt, sl, out, lse, workspace=ws, **kw)
    L = skv.lib()
    B, Hq, Hkv, C, k = wl.B, wl.Hq, wl.Hkv, 1 << wl.c_log2, wl.topk
    qp, cp, op = ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(cent.data_ptr()), ctypes.c_void_p(off.data_ptr())
    ip, sp_, ep = (ctypes.c_void_p(t.data_ptr()) for t in (ids, ss, se))

    def run():
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        st = L.attn_select_centroids(qp, cp, op, B, Hq, Hkv, wl.d, C, k, ip, sp_, ep, stream)
        if st != 0:
            raise skv.SkvError(st, "attn_select_centroids")
        st = L.attn_decode(ctypes.byref(a), stream)
        if st != 0:
            raise skv.SkvError(st, "attn_decode")

    run()
    torch.cuda.synchronize()
    sel_tokens = int((se - ss).sum().item())
    nbytes = sel_tokens * wl.d * 4 + cent.numel() * 2 + off.numel() * 4
    step = Step(run, nbytes, 1 + L.skv_decode_launches(ctypes.byref(a)), {"selected_tokens": sel_tokens,
                                 "selected_frac": sel_tokens / (wl.B * wl.Hkv * wl.L),
                                 "centroid_bytes": cent.numel() * 2})
    # keep every tensor the raw pointers above refer to alive with the step
    step.tensors = dict(q=q, k_pool=k_pool, v_pool=v_pool, bt=bt, sl=sl, off=off, cent=cent, ids=ids,
                        ss=ss, se=se, out=out, lse=lse, ws=ws)
    return step


def build_select_shared(torch, skv, skvgen, wl, status):
    """Centroid selection of B requests over one shared fixed context (its
    centroids read once per cluster of up to 8 requests), then each request's
    attention over its chosen clusters' keys in that one context."""
    q, k_pool, v_pool, bt, sl, off, cent = skvgen.device_shared_context(wl)
    shape = (wl.B, wl.Hkv, wl.topk)
    ids = torch.empty(shape, dtype=torch.int32, device="cuda")
    ss = torch.empty(shape, dtype=torch.int32, device="cuda")
    se = torch.empty(shape, dtype=torch.int32, device="cuda")
    out = torch.empty((wl.B, 1, wl.Hq, wl.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((wl.B, 1, wl.Hq), dtype=torch.float32, device="cuda")
    kw = dict(max_seq_len=wl.Lmax, scale=wl.scale, status=status, segments=(ss, se))
    n = skv.decode_workspace_size(q, k_pool, v_pool, bt, sl, out, lse, **kw)
    ws = torch.empty(max(n, 16) // 4 + 4, dtype=torch.float32, device="cuda")
    a = skv.make_decode_args(q, k_pool, v_pool, bt, sl, out, lse, workspace=ws, **kw)
    L = skv.lib()
    C, k = 1 << wl.c_log2, wl.topk
    qp, cp, op = ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(cent.data_ptr()), ctypes.c_void_p(off.data_ptr())
    ip, sp_, ep = (ctypes.c_void_p(t.data_ptr()) for t in (ids, ss, se))

    def run():
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        st = L.attn_select_centroids_shared(qp, cp, op, wl.B, wl.Hq, wl.Hkv, wl.d, C, k, ip, sp_, ep, stream)
        if st != 0:
            raise skv.SkvError(st, "attn_select_centroids_shared")
        st = L.attn_decode(ctypes.byref(a), stream)
        if st != 0:
            raise skv.SkvError(st, "attn_decode")

    run()
    torch.cuda.synchronize()
    sel_tokens = int((se - ss).sum().item())
    nbytes = sel_tokens * wl.d * 4 + cent.numel() * 2 + off.numel() * 4
    step = Step(run, nbytes, 1 + L.skv_decode_launches(ctypes.byref(a)),
                {"selected_tokens": sel_tokens, "selected_frac": sel_tokens / (wl.B * wl.Hkv * wl.L),
                 "centroid_bytes": cent.numel() * 2,
                 "centroid_bytes_per_request_copy": wl.B * cent.numel() * 2,
                 "note": "one shared context: centroid bytes counted once for all requests"})
    step.tensors = dict(q=q, k_pool=k_pool, v_pool=v_pool, bt=bt, sl=sl, off=off, cent=cent, ids=ids,
                        ss=ss, se=se, out=out, lse=lse, ws=ws)
    return step


def build_lookahead(torch, skv, skvgen, wl, status, n_ctas=20):
    """Lookahead prefetch ("SparDA" 2) on a pair of cfg5-shaped layers: layer
    l is a full-attention layer whose cache is on the GPU (ART, as the routed
    stack runs it); layer l+1 keeps its KV in page-locked host memory.  Layer
    l's Forecast picks layer l+1's top-k blocks from their summaries (two small
    kernels), then the gather kernel pulls them into a device cache on a side
    stream while layer l attends on the main stream (the gather's small CTAs
    sit beside the attention kernel's); then layer l+1 attends the cache.
    n_ctas = 20 gather CTAs: alone they take about as long as layer l's
    attention, and each further resident CTA slows that attention more than it
    speeds the copy (the pair measured 0.98 ms at 20 CTAs, 1.16 ms at 64).  Returns (overlapped step, layer-l-alone step,
    prefetch-alone step, layer-(l+1)-alone step)."""
    layers = [l for l in range(wl.n_layers - 1) if skvgen.route_bit(wl.seed, l) == 1]
    l0 = layers[0]
    fa = wl.with_(paging="identity")
    st_fa = build_decode(torch, skv, skvgen, fa, status, art=(wl.tau, wl.phi, wl.patience),
                         inputs=None, layer=l0)
    # layer l0 + 1: generated on the device, moved to page-locked host memory
    q1, k1, v1, bt1, sl1 = _paged_inputs(torch, skvgen, fa, layer=l0 + 1)
    skvgen.device_kv_paged(fa, q1, k1, v1, bt1, sl1, layer=l0 + 1)
    summ = skvgen.device_block_means(fa, k1, bt1, sl1)
    k_host = k1.cpu().pin_memory()
    v_host = v1.cpu().pin_memory()
    del k1, v1
    torch.cuda.empty_cache()
    kp, vp = skv.host_device_pointer(k_host), skv.host_device_pointer(v_host)
    G, k, mb = wl.G, wl.extra["lookahead_blocks"], fa.max_blocks
    q0 = st_fa.tensors["q"]
    x = q0[:, 0, ::G].contiguous()
    w = skvgen.device_forecast_weights(fa, layer=l0)
    f = torch.empty_like(x)
    off = torch.tensor([[[min(j * 64, fa.seq_len(b)) for j in range(mb + 1)]] * wl.Hkv for b in range(wl.B)],
                       dtype=torch.int32, device="cuda")
    ids = torch.empty((wl.B, wl.Hkv, k), dtype=torch.int32, device="cuda")
    ss0, se0, ss, se = (torch.empty_like(ids) for _ in range(4))
    k_cache = torch.empty((wl.B * k, wl.Hkv, 64, wl.d), dtype=torch.bfloat16, device="cuda")
    v_cache = torch.empty_like(k_cache)
    bt_c = torch.arange(wl.B * k, dtype=torch.int32, device="cuda").view(wl.B, k)
    sl_c = torch.full((wl.B,), k * 64, dtype=torch.int32, device="cuda")
    out1 = torch.empty((wl.B, 1, wl.Hq, wl.d), dtype=torch.float32, device="cuda")
    lse1 = torch.empty((wl.B, 1, wl.Hq), dtype=torch.float32, device="cuda")
    a1 = skv.make_decode_args(q1, k_cache, v_cache, bt_c, sl_c, out1, lse1, max_seq_len=k * 64,
                              scale=wl.scale, status=status, segments=(ss, se))
    L = skv.lib()
    side = torch.cuda.Stream()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    cur = lambda: ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def choose(stream_ptr):
        for st in (L.attn_forecast(p(x), p(w), wl.B, wl.Hkv, wl.d, p(f), stream_ptr),
                   L.attn_select_centroids(p(f), p(summ), p(off), wl.B, wl.Hkv, wl.Hkv, wl.d, mb, k, p(ids),
                                           p(ss0), p(se0), stream_ptr)):
            if st != 0:
                raise skv.SkvError(st, "lookahead selection")

    def gather(stream_ptr):
        st = L.attn_prefetch_blocks(kp, vp, p(bt1), p(sl1), p(ids), wl.B, wl.Hkv, wl.d, k, mb, k_host.shape[0],
                                    wl.Lmax, p(k_cache), p(v_cache), p(ss), p(se), p(status), n_ctas, stream_ptr)
        if st != 0:
            raise skv.SkvError(st, "attn_prefetch_blocks")

    def prefetch(stream_ptr):
        choose(stream_ptr)
        gather(stream_ptr)

    def attend_next():
        st = L.attn_decode(ctypes.byref(a1), cur())
        if st != 0:
            raise skv.SkvError(st, "attn_decode")

    def overlapped():
        main = torch.cuda.current_stream()
        choose(cur())                                    # layer l's Forecast picks l+1's blocks
        side.wait_stream(main)
        with torch.cuda.stream(side):
            gather(ctypes.c_void_p(side.cuda_stream))    # the copy from host memory ...
        st_fa.run()                                      # ... while layer l attends
        main.wait_stream(side)
        attend_next()                                    # layer l+1 over the fetched blocks

    copy_bytes = wl.B * wl.Hkv * k * 64 * wl.d * 4       # chosen blocks' K + V (full blocks)
    nb_fa = st_fa.nbytes
    step = Step(overlapped, nb_fa + copy_bytes, st_fa.launches + 4,
                {"layer_full": l0, "layer_offloaded": l0 + 1, "lookahead_blocks": k,
                 "copy_bytes": copy_bytes, "gather_ctas": n_ctas})
    step.tensors = dict(fa=st_fa, q1=q1, bt1=bt1, sl1=sl1, summ=summ, k_host=k_host, v_host=v_host, x=x, w=w,
                        f=f, off=off, ids=ids, ss0=ss0, se0=se0, ss=ss, se=se, k_cache=k_cache,
                        v_cache=v_cache, bt_c=bt_c, sl_c=sl_c, out=out1, lse=lse1, a1=a1, side=side,
                        ptrs=(kp, vp))
    alone_fa = Step(st_fa.run, nb_fa, st_fa.launches)
    alone_pf = Step(lambda: prefetch(cur()), copy_bytes, 3)
    alone_next = Step(attend_next, copy_bytes, L.skv_decode_launches(ctypes.byref(a1)))
    return step, alone_fa, alone_pf, alone_next


def build_routed(torch, skv, skvgen, wl, status, layer_ids=None):
    """Attention layers of a routed stack (all `wl.n_layers`, or `layer_ids`),
    each independent; layer l runs full attention with ART when its seeded
    route bit is 1, else the sink + recent window only, whose cache holds just
    those blocks."""
    layers = []
    for l in (range(wl.n_layers) if layer_ids is None else layer_ids):
        fa = skvgen.route_bit(wl.seed, l) == 1
        lw = wl.with_(paging="identity" if fa else "window")
        q, k_pool, v_pool, bt, sl = _paged_inputs(torch, skvgen, lw, layer=l)
        skvgen.device_kv_paged(lw, q, k_pool, v_pool, bt, sl, layer=l)
        out = torch.empty((wl.B, 1, wl.Hq, wl.d), dtype=torch.float32, device="cuda")
        lse = torch.empty((wl.B, 1, wl.Hq), dtype=torch.float32, device="cuda")
        consumed = torch.zeros((wl.B, wl.Hq), dtype=torch.int32, device="cuda")
        kw = dict(max_seq_len=wl.Lmax, scale=wl.scale, status=status, blocks_consumed=consumed)
        if fa:
            kw["art"] = (wl.tau, wl.phi, wl.patience)
        else:
            kw["window"] = (wl.sink, wl.recent)
        n = skv.decode_workspace_size(q, k_pool, v_pool, bt, sl, out, lse, **kw)
        ws = torch.empty(max(n, 16) // 4 + 4, dtype=torch.float32, device="cuda") if n else None
        a = skv.make_decode_args(q, k_pool, v_pool, bt, sl, out, lse, workspace=ws, **kw)
        layers.append(dict(layer=l, fa=fa, a=a, keep=(q, k_pool, v_pool, bt, sl, out, lse, consumed, ws),
                           out=out, lse=lse, consumed=consumed,
                           launches=skv.lib().skv_decode_launches(ctypes.byref(a))))
    L = skv.lib()

    def run():
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        for ly in layers:
            st = L.attn_decode(ctypes.byref(ly["a"]), stream)
            if st != 0:
                raise skv.SkvError(st, "attn_decode")

    run()
    torch.cuda.synchronize()
    nbytes, fa_n, fa_bytes_full, skipped = 0, 0, 0, []
    win_tokens = len(__import__("oracle").keys_window(wl.L, wl.sink, wl.recent))
    for ly in layers:
        if ly["fa"]:
            fa_n += 1
            grp = ly["consumed"].cpu().numpy().reshape(wl.B, wl.Hkv, wl.G).max(axis=2)
            nbytes += int(grp.sum()) * wl.bs * wl.d * 4
            fa_bytes_full += wl.kv_bytes()
            skipped.append(1.0 - float(grp.sum()) / (wl.B * wl.Hkv * wl.nb(0)))
        else:
            nbytes += wl.B * wl.Hkv * win_tokens * wl.d * 4
    step = Step(run, nbytes, sum(ly["launches"] for ly in layers),
                {"fa_layers": fa_n, "sa_layers": len(layers) - fa_n,
                 "art_blocks_skipped_frac_mean": float(np.mean(skipped)) if skipped else 0.0,
                 "dense_equivalent_bytes": fa_bytes_full + (len(layers) - fa_n) * wl.kv_bytes()})
    step.tensors = dict(layers=layers)
    return step


def build_select_levels(torch, skv, skvgen, wl, sel_step, per=32, k1=8):
    """Centroid selection alone, flat (all C fine centroids) and two-level
    ("Squeezed Attention" Q2 step 4): coarse clusters = runs of `per`
    consecutive fine clusters, centroid = mean of theirs (input preparation,
    as offline clustering would be); keep k1 coarse, then the top-k of their
    fine clusters.  Returns (flat step, two-level step)."""
    T = sel_step.tensors
    q, cent, off = T["q"], T["cent"], T["off"]
    B, Hkv, C, k = wl.B, wl.Hkv, 1 << wl.c_log2, wl.topk
    C1 = C // per
    coarse = cent.view(B, Hkv, C1, per, wl.d).float().mean(dim=3).to(torch.bfloat16).contiguous()
    coarse_off = torch.arange(0, C + 1, per, dtype=torch.int32, device="cuda").expand(B, Hkv, C1 + 1).contiguous()
    outs = [torch.empty((B, Hkv, k), dtype=torch.int32, device="cuda") for _ in range(6)]
    L = skv.lib()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    cur = lambda: ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def flat():
        st = L.attn_select_centroids(p(q), p(cent), p(off), B, wl.Hq, Hkv, wl.d, C, k, p(outs[0]), p(outs[1]),
                                     p(outs[2]), cur())
        if st != 0:
            raise skv.SkvError(st, "attn_select_centroids")

    def two():
        st = L.attn_select_centroids2(p(q), p(coarse), p(coarse_off), p(cent), p(off), B, wl.Hq, Hkv, wl.d,
                                      C1, C, k1, k, p(outs[3]), p(outs[4]), p(outs[5]), cur())
        if st != 0:
            raise skv.SkvError(st, "attn_select_centroids2")

    f = Step(flat, cent.numel() * 2, 1, {"centroids_read": C})
    t = Step(two, coarse.numel() * 2 + B * Hkv * k1 * per * wl.d * 2, 1,
             {"centroids_read": C1 + k1 * per, "coarse": C1, "k1": k1})
    f.tensors = t.tensors = dict(q=q, cent=cent, off=off, coarse=coarse, coarse_off=coarse_off, outs=outs)
    return f, t


def build_router(torch, skv, skvgen, wl, n_prefix=64, n_suffix=64):
    """The routing decision of a routed stack ("Flux Attention" 2, Layer
    Router): pooled prefix and suffix query rows of every layer -> one logit
    and route bit per (layer, sequence).  Synthetic prefill queries (only the
    pooled rows are held) and untrained router weights."""
    L, B, T, F = wl.n_layers, wl.B, n_prefix + n_suffix, wl.Hq * wl.d
    q = torch.empty((L, B, T, wl.Hq, wl.d), dtype=torch.bfloat16, device="cuda")
    skvgen.device_normal_bf16(q, wl.seed, skvgen.S_Q, layer=1 << 20)
    w = torch.empty((L, 2 * F), dtype=torch.bfloat16, device="cuda")
    skvgen.device_normal_bf16(w, wl.seed, skvgen.S_ROUTER_W)
    w = (w.float() / 32).contiguous()
    bias = torch.zeros(L, dtype=torch.float32, device="cuda")
    route = torch.empty((L, B), dtype=torch.uint8, device="cuda")
    logits = torch.empty((L, B), dtype=torch.float32, device="cuda")
    L_ = skv.lib()
    args = (ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(w.data_ptr()), ctypes.c_void_p(bias.data_ptr()),
            L, B, T, wl.Hq, wl.d, n_prefix, n_suffix, ctypes.c_void_p(logits.data_ptr()),
            ctypes.c_void_p(route.data_ptr()))

    def run():
        st = L_.attn_route_layers(*args, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        if st != 0:
            raise skv.SkvError(st, "attn_route_layers")

    step = Step(run, q.numel() * 2 + w.numel() * 4, 1, {"layers": L, "sequences": B,
                                                          "pooled_rows": T, "features": F})
    step.tensors = dict(q=q, w=w, bias=bias, route=route, logits=logits)
    return step


def build_chunk(torch, skv, skvgen, wl, status):
    """Query chunk of Tq tokens: 8 context shards (one launch, one partial per
    shard), the chunk's own keys under a causal mask, and the exact merge."""
    q, k_pool, v_pool, bt, sl = _paged_inputs(torch, skvgen, wl)
    skvgen.device_kv_paged(wl, q, k_pool, v_pool, bt, sl)
    ctx, S = wl.L - wl.chunk, wl.shards
    parts_o = torch.empty((S + 1, wl.B, wl.Tq, wl.Hq, wl.d), dtype=torch.float32, device="cuda")
    parts_l = torch.empty((S + 1, wl.B, wl.Tq, wl.Hq), dtype=torch.float32, device="cuda")
    N = wl.B * wl.Tq * wl.Hq
    out = torch.empty((N, wl.d), dtype=torch.float32, device="cuda")
    lse = torch.empty(N, dtype=torch.float32, device="cuda")
    kw = dict(max_seq_len=wl.Lmax, scale=wl.scale, status=status)
    a_ctx = skv.make_decode_args(q, k_pool, v_pool, bt, sl, parts_o[:S], parts_l[:S],
                                 kv_range=(0, ctx), kv_shards=S, **kw)
    a_tail = skv.make_decode_args(q, k_pool, v_pool, bt, sl, parts_o[S:], parts_l[S:],
                                  kv_range=(ctx, wl.L), causal=True, **kw)
    L = skv.lib()
    po, pl_, op, lp = (ctypes.c_void_p(t.data_ptr()) for t in (parts_o, parts_l, out, lse))

    def run():
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        for a in (a_ctx, a_tail):
            st = L.attn_decode(ctypes.byref(a), stream)
            if st != 0:
                raise skv.SkvError(st, "attn_decode")
        st = L.attn_merge_lse(po, pl_, S + 1, N, wl.d, op, lp, stream)
        if st != 0:
            raise skv.SkvError(st, "attn_merge_lse")

    rows = wl.B * wl.Hq * wl.Tq
    flops = 4.0 * wl.d * rows * ctx + 4.0 * wl.d * wl.B * wl.Hq * (wl.Tq * (wl.Tq + 1) // 2)
    step = Step(run, wl.kv_bytes(), 3, {"flop": flops, "shards": S, "chunk_tokens": wl.Tq})
    step.tensors = dict(q=q, k_pool=k_pool, v_pool=v_pool, bt=bt, sl=sl, parts_o=parts_o,
                        parts_l=parts_l, out=out, lse=lse)
    return step


def max_over_ranks(x, world, dist, device):
    """The largest of every rank's `x` (a device time in ms): the job takes as
    long as its slowest replica.  `x` itself on one rank."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(nbytes_per_rank, world, ms):
    """Whole-job throughput in GB/s: every replica moves `nbytes_per_rank`
    per step, and a step takes `ms` (the max over ranks)."""
    return nbytes_per_rank * world / (ms * 1e-3) / 1e9


class Ctx:
    """What every workload's measurement shares: torch, the process group, the
    peaks and the device status word."""

    def __init__(self, args, torch, dist, world, rank, local):
        import skvgen
        import sparse_kv_b200 as skv
        self.args, self.torch, self.dist = args, torch, dist
        self.world, self.rank, self.local = world, rank, local
        self.skv, self.skvgen = skv, skvgen
        self.hbm_peak, self.peak_kind = peaks()
        self.status = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)

    def timed(self, st, steps, warmup):
        """CUDA-graph replay of `steps` steps, each bracketed by events on the
        launching stream; returns (total ms, max over ranks; per-step ms)."""
        torch = self.torch
        stream = torch.cuda.current_stream()
        for _ in range(warmup):
            st.run()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            st.run()
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        if self.world > 1:
            self.dist.barrier()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(steps)]
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for e0, e1 in evs:
            e0.record(stream)
            g.replay()
            e1.record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        total_ms = t0.elapsed_time(t1)
        per = [e0.elapsed_time(e1) for e0, e1 in evs]
        total_ms = max_over_ranks(total_ms, self.world, self.dist, "cuda")
        del g
        return total_ms, per


def measure_workload(c, name, headline):
    """Build, time and summarise one workload's step; `headline` adds the
    end-to-end leg.  Returns the result dict (the bench line for the
    headline)."""
    torch, skv, skvgen, args = c.torch, c.skv, c.skvgen, c.args
    world, status = c.world, c.status
    wl = skvgen.WORKLOADS[name]
    kind = name.split("_")[0]
    if kind in ("cfg1", "cfg2"):
        step = build_decode(torch, skv, skvgen, wl, status)
    elif kind == "cfg3":
        step = build_select(torch, skv, skvgen, wl, status)
    elif kind == "cfg3s":
        step = build_select_shared(torch, skv, skvgen, wl, status)
    elif kind == "cfg5":
        step = build_routed(torch, skv, skvgen, wl, status)
    elif kind == "cfg5p":
        step, *look_steps = build_lookahead(torch, skv, skvgen, wl, status)
    elif kind == "cfg4":
        step = build_chunk(torch, skv, skvgen, wl, status)
    else:
        raise SystemExit(f"workload {name}: no bench step")
    art_step, sweep_steps, dense_step = None, [], None
    if kind != "cfg5p":
        look_steps = None
    if kind == "cfg2" and not args.no_art:
        T = step.tensors
        shared = (T["q"], T["k_pool"], T["v_pool"], T["bt"], T["sl"])
        art_step = build_decode(torch, skv, skvgen, wl, status, art=(wl.tau, wl.phi, wl.patience),
                                inputs=shared)
        # looser thresholds on the same cache, where heads do stop: savings vs blocks skipped
        for thr in ((5e-2, 5e-3, 2), (2e-2, 2e-3, 2)):
            sweep_steps.append((thr, build_decode(torch, skv, skvgen, wl, status, art=thr, inputs=shared)))
    router_step = build_router(torch, skv, skvgen, wl) if kind == "cfg5" else None
    level_steps = None
    if kind in ("cfg3", "cfg3s"):  # the same cache walked in full, for the savings of the selection
        T = step.tensors
        dense_step = build_decode(torch, skv, skvgen, wl, status,
                                  inputs=(T["q"], T["k_pool"], T["v_pool"], T["bt"], T["sl"]))
    if kind == "cfg3":
        level_steps = build_select_levels(torch, skv, skvgen, wl, step)
    stream = torch.cuda.current_stream()
    n_side = max(10, args.steps // 4)

    with ClockSampler(c.uuid) as clk:
        total_ms, per = c.timed(step, args.steps, args.warmup)
        art_ms = None
        if art_step is not None:
            art_ms, _ = c.timed(art_step, args.steps, args.warmup)
        sweep_ms = [c.timed(st, n_side, args.warmup)[0] / n_side for _, st in sweep_steps]
        dense_ms = (c.timed(dense_step, n_side, args.warmup)[0] / n_side if dense_step is not None else None)
        router_ms = (c.timed(router_step, args.steps, args.warmup)[0] / args.steps
                     if router_step is not None else None)
        level_ms = ([c.timed(st, args.steps, args.warmup)[0] / args.steps for st in level_steps]
                    if level_steps is not None else None)
        look_ms = ([c.timed(st, args.steps, args.warmup)[0] / args.steps for st in look_steps]
                   if look_steps is not None else None)
    clocks = clk.summary()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status word {int(status.item()):#x}")

    ms_step = total_ms / args.steps
    value = job_gbs(step.nbytes, world, ms_step)
    per_launch_ms = statistics.mean(per)
    achieved = step.nbytes / (per_launch_ms * 1e-3) / 1e9

    # ---- end to end through the public API: q (and tables) in from pinned host, O/LSE out
    e2e = None
    if headline and kind in ("cfg1", "cfg2"):
        T = step.tensors
        # one staging buffer each way (q | block table | seq_lens in, O | LSE out, each
        # 256-byte aligned): one host-to-device and one device-to-host copy per step; the
        # call's tensors are views into the device buffers
        ins, outs = (T["q"], T["bt"], T["sl"]), (T["out"], T["lse"])

        def layout(ts):
            offs, n = [], 0
            for t in ts:
                offs.append(n)
                n += (t.numel() * t.element_size() + 255) // 256 * 256
            return offs, n

        def view(buf, off, t):
            return buf[off:off + t.numel() * t.element_size()].view(t.dtype).view(t.shape)

        in_off, in_n = layout(ins)
        out_off, out_n = layout(outs)
        din = torch.zeros(in_n, dtype=torch.uint8, device="cuda")
        dout = torch.zeros(out_n, dtype=torch.uint8, device="cuda")
        hin = torch.zeros(in_n, dtype=torch.uint8).pin_memory()
        hout = torch.zeros(out_n, dtype=torch.uint8).pin_memory()
        for o, t in zip(in_off, ins):
            view(hin, o, t).copy_(t.cpu())
        q_d, bt_d, sl_d = (view(din, o, t) for o, t in zip(in_off, ins))
        out_d, lse_d = (view(dout, o, t) for o, t in zip(out_off, outs))
        common = (q_d, T["k_pool"], T["v_pool"], bt_d, sl_d, out_d, lse_d)

        def e2e_step():
            din.copy_(hin, non_blocking=True)
            skv.attn_decode(*common, workspace=T["ws"], stream=stream, **T["kw"])
            hout.copy_(dout, non_blocking=True)

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            c.dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / args.steps
        e2e_ms = max_over_ranks(e2e_ms, world, c.dist, "cuda")
        # the step's result came back: the host copy of O equals the device-timed run's
        same = bool(torch.equal(view(hout, out_off[0], T["out"]), T["out"].cpu()))
        e2e = {"value": job_gbs(step.nbytes, world, e2e_ms), "unit": "GB/s",
               "h2d_bytes_per_step": in_n, "d2h_bytes_per_step": out_n, "result_matches_device_run": same,
               "note": "KV cache resident in HBM; per step q, block table and seq_lens copied in "
                       "from one page-locked host buffer and O, LSE copied out to another"}

    res = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 in, fp32 accumulate", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.B, "q_heads": wl.Hq, "kv_heads": wl.Hkv,
                   "head_dim": wl.d, "context": wl.L, "page_tokens": wl.bs, "paging": wl.paging,
                   "l2": ("KV cache of 4 MiB fits in L2 (launch-bound case), no flush" if kind == "cfg1"
                          else "inputs larger than L2 (GBs of KV per step), no flush"),
                   "timing": "CUDA-graph replay per step, CUDA events",
                   "parallelism": f"replicas x{world}"},
        "attended_tokens_per_s": step.nbytes / (wl.d * 4) * wl.G * world / (ms_step * 1e-3),
        "kv_tokens_per_s": step.nbytes / (wl.d * 4) * world / (ms_step * 1e-3),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": c.hbm_peak, "unit": "GB/s",
                     "frac": achieved / c.hbm_peak, "peak_kind": c.peak_kind,
                     "frac_of_8000": achieved / 8000.0, "traffic": traffic_for(kind),
                     "kernel": "one step of our kernels (decode + merge; per-kernel shares in profiles/)"},
        "clocks": clocks,
        "step_ms_p10_p50_p90": [float(x) for x in np.percentile(per, [10, 50, 90])],
        "gpu_launches": args.steps * step.launches,
    }
    if step.extra:
        res["step_detail"] = step.extra
    if kind == "cfg4":  # a dense contraction: tensor-core roofline (sustained bf16 peak)
        tf = step.extra["flop"] / (per_launch_ms * 1e-3) / 1e12
        peak_tf, tf_kind = tensor_peak("sw_power_cap" in clocks.get("reasons", []))
        res["metric_tflops"] = step.extra["flop"] * world / (ms_step * 1e-3) / 1e12
        res["roofline"] = {"bound": "tensor", "achieved": tf, "peak": peak_tf, "unit": "TFLOP/s",
                           "frac": tf / peak_tf, "peak_kind": tf_kind, "traffic": traffic_for(kind),
                           "kernel": "one step: chunk kernel x2 + merge"}
    if kind in ("cfg1", "cfg2"):
        res["config"]["traversal"] = "full"
    if art_ms is not None:
        cons = art_step.tensors["consumed"].cpu().numpy()
        grp = cons.reshape(wl.B, wl.Hkv, wl.G).max(axis=2)
        art_bytes = int(grp.sum()) * wl.bs * wl.d * 4
        art_step_ms = art_ms / args.steps
        res["art"] = {"ms_per_step": art_step_ms, "kv_gbs": art_bytes / (art_step_ms * 1e-3) / 1e9,
                      "blocks_consumed_mean": float(cons.mean()), "blocks_total": wl.nb(0),
                      "group_blocks_hist16": np.histogram(grp, bins=16, range=(0, wl.nb(0)))[0].tolist(),
                      "blocks_skipped_frac": 1.0 - float(grp.sum()) / (wl.B * wl.Hkv * wl.nb(0)),
                      "time_vs_full": art_step_ms / ms_step,
                      "attended_tokens_per_s": float(cons.sum()) * wl.bs / (art_step_ms * 1e-3),
                      "tau": wl.tau, "phi": wl.phi, "patience": wl.patience}
        res["gpu_launches"] += args.steps * art_step.launches

        def art_summary(st, ms):
            cons = st.tensors["consumed"].cpu().numpy()
            grp = cons.reshape(wl.B, wl.Hkv, wl.G).max(axis=2)
            skipped = 1.0 - float(grp.sum()) / (wl.B * wl.Hkv * wl.nb(0))
            saved = 1.0 - ms / ms_step
            return {"ms_per_step": ms, "blocks_skipped_frac": skipped, "time_saved_frac": saved,
                    "saved_per_skipped": saved / skipped if skipped > 0 else None,
                    "blocks_consumed_mean": float(cons.mean()),
                    "group_blocks_hist16": np.histogram(grp, bins=16, range=(0, wl.nb(0)))[0].tolist()}
        res["art_sweep"] = [dict(tau=thr[0], phi=thr[1], patience=thr[2], **art_summary(st, ms))
                            for (thr, st), ms in zip(sweep_steps, sweep_ms)]
        res["gpu_launches"] += sum(n_side * st.launches for _, st in sweep_steps)
    if dense_ms is not None:
        res["selection"] = {"dense_ms_per_step": dense_ms, "time_vs_dense": ms_step / dense_ms,
                            "bytes_vs_dense": step.nbytes / wl.kv_bytes(),
                            "note": "same cache walked in full by the plain decode kernel"}
        res["gpu_launches"] += n_side * dense_step.launches
    if level_ms is not None:
        f, t = level_steps
        res["selection_levels"] = {
            "flat": {"ms_per_call": level_ms[0], "centroids_read": f.extra["centroids_read"]},
            "two_level": {"ms_per_call": level_ms[1], **t.extra},
            "note": "selection alone (no attention): flat top-k over all fine centroids vs coarse "
                    "top-k1 then top-k among the kept coarse clusters' fine centroids"}
        res["gpu_launches"] += 2 * args.steps
    if router_ms is not None:
        gbs = router_step.nbytes / (router_ms * 1e-3) / 1e9
        res["router"] = {"ms_per_call": router_ms, "bytes_per_call": router_step.nbytes, "gbs": gbs,
                         "roofline": {"bound": "hbm", "achieved": gbs, "peak": c.hbm_peak, "unit": "GB/s",
                                      "frac": gbs / c.hbm_peak},
                         **router_step.extra,
                         "note": "per-layer route bits from pooled prefix/suffix query rows "
                                 "(untrained weights); outside the timed decode step"}
        res["gpu_launches"] += args.steps * router_step.launches
    if look_ms is not None:
        fa_ms, pf_ms, nx_ms = look_ms
        cb = step.extra["copy_bytes"]
        res["lookahead"] = {
            "ms_overlapped_pair": ms_step, "ms_full_layer_alone": fa_ms, "ms_prefetch_alone": pf_ms,
            "ms_next_layer_alone": nx_ms, "ms_serial_pair": fa_ms + pf_ms + nx_ms,
            "hidden_frac_of_prefetch": (fa_ms + pf_ms + nx_ms - ms_step) / pf_ms if pf_ms > 0 else None,
            "host_to_device_gbs": cb / (pf_ms * 1e-3) / 1e9, "copy_bytes": cb,
            "note": "prefetch = Forecast + block top-k + gather from page-locked host memory (side "
                    "stream, launched first); hidden_frac = (serial - overlapped) / prefetch alone"}
        res["gpu_launches"] += args.steps * sum(st.launches for st in look_steps)
    if e2e is not None:
        res["e2e"] = e2e
    # ---- CPU-baseline leg (rank 0, one GPU): the oracle timed on the host cores, and
    # the same oracle's check of sampled KV groups of what the GPU returned above
    if c.rank == 0 and world == 1 and not args.no_cpu_baseline:
        if headline and kind in ("cfg1", "cfg2"):
            res["cpu_baseline"] = cpu_baseline(wl)
        checks = {}
        if kind in ("cfg1", "cfg2"):
            checks["full"] = oracle_check_full(wl, step)
        if art_step is not None:
            checks["art"] = oracle_check_art(wl, art_step, (wl.tau, wl.phi, wl.patience))
            checks["art_sweep"] = [oracle_check_art(wl, st, thr) for thr, st in sweep_steps]
        if kind == "cfg5p":
            checks["lookahead"] = oracle_check_lookahead(wl, step)
        if kind == "cfg5":
            fa = [ly for ly in step.tensors["layers"] if ly["fa"]]
            if fa:
                checks["art_layer"] = oracle_check_art(wl, fa[0], (wl.tau, wl.phi, wl.patience),
                                                       layer=fa[0]["layer"], n_groups=2)
        if checks:
            res["oracle_check"] = checks
    del step, art_step, sweep_steps, dense_step, router_step, level_steps, look_steps
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return res


def _sample_groups(wl, n):
    """n KV groups spread over the batch and the KV heads."""
    step = max(1, (wl.B * wl.Hkv) // n)
    gs = list(range(0, wl.B * wl.Hkv, step))[:n]
    return [(g // wl.Hkv, (g // wl.Hkv + g) % wl.Hkv) for g in gs]


def oracle_check_full(wl, st, n_groups=4):
    """Full traversal: max |dO| and relative |dlse| of sampled KV groups against
    the oracle (CPU-baseline leg)."""
    import oracle
    import skvgen
    T = st.tensors
    out = T["out"][:, 0].cpu().numpy().astype(np.float64)
    lse = T["lse"][:, 0].cpu().numpy().astype(np.float64)
    q = skvgen.host_q(wl)
    err, lerr = 0.0, 0.0
    groups = _sample_groups(wl, n_groups)
    for b, kvh in groups:
        K, V = skvgen.host_kv_group(wl, b, kvh, q=q)
        qg = q[b, 0, kvh * wl.G:(kvh + 1) * wl.G]
        O, l = oracle.attend(qg[None], K[None], V[None], [[np.arange(wl.seq_len(b))] * wl.G], wl.scale)
        hs = slice(kvh * wl.G, (kvh + 1) * wl.G)
        err = max(err, float(np.abs(out[b, hs] - O[0]).max()))
        lerr = max(lerr, float((np.abs(lse[b, hs] - l[0]) / np.maximum(1.0, np.abs(l[0]))).max()))
    return {"groups": groups, "max_abs_dO": err, "max_rel_dlse": lerr, "tol_O": 2e-3, "tol_lse": 1e-4}


def oracle_check_art(wl, st, thr, layer=0, n_groups=8, flag_margin=1e-3):
    """ART decisions of sampled KV groups against the sequential fp64 oracle
    (CPU-baseline leg).  A head whose blocks consumed differ from the oracle's is
    "flagged" when the oracle's decision margin (relative distance of d_scale
    or d_dir to its threshold) is within flag_margin, else "mismatched"; its
    output is compared with the oracle forced to the GPU's stop."""
    import oracle
    import skvgen
    tau, phi, pat = thr
    T = st.tensors if hasattr(st, "tensors") else st
    out = T["out"][:, 0].cpu().numpy().astype(np.float64)
    lse = T["lse"][:, 0].cpu().numpy().astype(np.float64)
    cons = T["consumed"].cpu().numpy()
    q = skvgen.host_q(wl, layer)
    flagged = mismatched = stop_diff = 0
    err, lerr = 0.0, 0.0
    groups = _sample_groups(wl, n_groups)
    for b, kvh in groups:
        K, V = skvgen.host_kv_group(wl, b, kvh, layer, q=q)
        qg = q[b, 0, kvh * wl.G:(kvh + 1) * wl.G]
        trav = [oracle.art_traversal(wl.nb(b))]
        O, l, c_ref, mg = oracle.art(qg[None], K[None], V[None], [wl.seq_len(b)], wl.bs, trav, wl.scale,
                                     tau, phi, pat)
        hs = slice(kvh * wl.G, (kvh + 1) * wl.G)
        cg = cons[b, hs]
        diff = np.nonzero(cg != c_ref[0])[0]
        for h in diff:
            if mg[0, h] <= flag_margin:
                flagged += 1
            else:
                mismatched += 1
        if len(diff):
            stop_diff = max(stop_diff, int(np.abs(cg - c_ref[0]).max()))
            O, l, _, _ = oracle.art(qg[None], K[None], V[None], [wl.seq_len(b)], wl.bs, trav, wl.scale,
                                    tau, phi, pat, forced=cg[None])
        err = max(err, float(np.abs(out[b, hs] - O[0]).max()))
        lerr = max(lerr, float((np.abs(lse[b, hs] - l[0]) / np.maximum(1.0, np.abs(l[0]))).max()))
    return {"tau": tau, "phi": phi, "patience": pat, "layer": layer, "groups": len(groups),
            "heads": len(groups) * wl.G, "flagged_near_threshold": flagged, "mismatched": mismatched,
            "max_stop_diff_blocks": stop_diff, "max_abs_dO": err, "max_rel_dlse": lerr,
            "flag_margin": flag_margin}


def oracle_check_lookahead(wl, st, n_groups=2):
    """The offloaded layer of the lookahead pair on sampled KV groups (CPU-baseline
    leg): Forecast bits, chosen blocks and attention over them against the oracle."""
    import oracle
    import skvgen
    T = st.tensors
    l0 = st.extra["layer_full"]
    fa = wl.with_(paging="identity")
    k, G, d = st.extra["lookahead_blocks"], wl.G, wl.d
    f = T["f"].view(torch_int16()).cpu().numpy().view(np.uint16)
    ids = T["ids"].cpu().numpy()
    out = T["out"][:, 0].cpu().numpy().astype(np.float64)
    lse = T["lse"][:, 0].cpu().numpy().astype(np.float64)
    q0, q1 = skvgen.host_q(fa, l0), skvgen.host_q(fa, l0 + 1)
    w = skvgen.host_forecast_weights(fa, l0)
    res = {"groups": [], "forecast_bits_equal": True, "ids_equal": 0, "ids_flagged": 0, "max_abs_dO": 0.0,
           "max_rel_dlse": 0.0}
    for b, kvh in _sample_groups(wl, n_groups):
        res["groups"].append((b, kvh))
        fr = oracle.forecast(q0[b, 0, kvh * G][None], w[kvh][None])[0]
        res["forecast_bits_equal"] &= bool(np.array_equal(fr, f[b, kvh]))
        K, V = skvgen.host_kv_group(fa, b, kvh, l0 + 1, q=q1)
        summ = skvgen.host_block_means(K)
        ref, sc = oracle.select(fr[None, None], summ[None], k)
        if np.array_equal(ref[0], ids[b, kvh]):
            res["ids_equal"] += 1
        elif oracle.topk_boundary_gap(sc, k)[0] <= 1e-5:
            res["ids_flagged"] += 1
        keys = oracle.keys_blocks(ids[b, kvh], wl.seq_len(b))
        qg = q1[b, 0, kvh * G:(kvh + 1) * G]
        O, l = oracle.attend(qg[None], K[None], V[None], [[keys] * G], wl.scale)
        hs = slice(kvh * G, (kvh + 1) * G)
        res["max_abs_dO"] = max(res["max_abs_dO"], float(np.abs(out[b, hs] - O[0]).max()))
        res["max_rel_dlse"] = max(res["max_rel_dlse"],
                                  float((np.abs(lse[b, hs] - l[0]) / np.maximum(1.0, np.abs(l[0]))).max()))
    return res


def torch_int16():
    import torch
    return torch.int16


# the other workloads measured in the default run, after the headline
SIDE_WORKLOADS = ["cfg1_b1_h8_l4k", "cfg3_b8_h32_l64k_c1024_k102", "cfg3s_b8_h32_l64k_shared",
                  "cfg4_b4_h32_l128k_chunk128", "cfg5_b8_h32_l128k_32layers",
                  "cfg5p_b8_h32_l128k_lookahead16"]
SIDE_KEYS = ["value", "unit", "ms_per_step", "step_ms_p10_p50_p90", "roofline", "clocks", "config",
             "gpu_launches", "step_detail", "metric_tflops", "selection", "selection_levels", "router",
             "lookahead", "oracle_check", "attended_tokens_per_s"]


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    c = Ctx(args, torch, dist, world, rank, local)
    res = measure_workload(c, args.workload, headline=True)
    if args.workload == "cfg2_b16_h32_l32k" and not args.headline_only:
        res["configs"] = {}
        for name in SIDE_WORKLOADS:
            r = measure_workload(c, name, headline=False)
            res["configs"][name] = {k: r[k] for k in SIDE_KEYS if k in r}
            res["gpu_launches_side"] = res.get("gpu_launches_side", 0) + r["gpu_launches"]
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


# dominant kernel of each workload's step and the sources it is built from
KERNEL_SOURCES = {
    "decode_kernel": ["decode.cu", "tile.cuh", "common.cuh", "decode.cuh"],
    "art_kernel": ["art.cu", "tile.cuh", "common.cuh", "decode.cuh"],
    "chunk_kernel": ["chunk.cu", "common.cuh", "decode.cuh"],
    "select_kernel": ["select.cu", "common.cuh"],
}
DOMINANT = {"cfg1": "decode_kernel", "cfg2": "decode_kernel", "cfg3": "decode_kernel", "cfg3s": "decode_kernel",
            "cfg4": "chunk_kernel", "cfg5": "art_kernel"}


def kernel_sha(kernel):
    """Hash of the sources a kernel is compiled from (first 16 hex digits)."""
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "sparse_kv_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(kind):
    """DRAM bytes (read + write) per launch of the workload's dominant kernel
    from the committed ncu summary (profiles/traffic.json), if it was taken on
    the kernel's current sources; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p) or kind not in DOMINANT:
        return None
    kernel = DOMINANT[kind]
    rec = json.load(open(p)).get(kind)
    if not rec or rec.get("kernel") != kernel or rec.get("sources_sha") != kernel_sha(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


if __name__ == "__main__":
    main()
