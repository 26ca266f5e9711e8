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
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], "measured"
    return 6650.0, "fallback"


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML every few ms in a
    background thread while the timed region runs (read-only queries)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, uuid, period_s=0.005):
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
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": nbytes / t_oracle / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} of {total_groups} KV groups of {wl.name}, full traversal, fp64 "
                      f"oracle time {t_oracle:.2f} s"}


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
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
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

def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import numpy as np
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))

    import skvgen
    import sparse_kv_b200 as skv
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    wl = skvgen.WORKLOADS[args.workload]
    hbm_peak, peak_kind = peaks()

    # ---- inputs resident in HBM
    bt_host, num_pages = skvgen.block_table_host(wl)
    q = skvgen.device_q(wl)
    k_pool = torch.empty((num_pages, wl.Hkv, wl.bs, wl.d), dtype=torch.bfloat16, device="cuda")
    v_pool = torch.empty_like(k_pool)
    block_table = torch.tensor(bt_host, device="cuda")
    seq_lens = torch.full((wl.B,), wl.L, dtype=torch.int32, device="cuda")
    skvgen.device_kv_paged(wl, q, k_pool, v_pool, block_table, seq_lens)
    out = torch.empty((wl.B, 1, wl.Hq, wl.d), dtype=torch.float32, device="cuda")
    lse = torch.empty((wl.B, 1, wl.Hq), dtype=torch.float32, device="cuda")
    consumed = torch.zeros((wl.B, wl.Hq), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    common = (q, k_pool, v_pool, block_table, seq_lens, out, lse)
    kw = dict(max_seq_len=wl.L, scale=wl.scale, status=status)
    ws_n = skv.decode_workspace_size(*common, **kw)
    ws = torch.empty(max(ws_n, 16) // 4 + 4, dtype=torch.float32, device="cuda")
    a_full = skv.make_decode_args(*common, workspace=ws, **kw)
    a_art = skv.make_decode_args(*common, art=(wl.tau, wl.phi, wl.patience), blocks_consumed=consumed,
                                 **kw)
    stream = torch.cuda.current_stream()
    sp = ctypes.c_void_p(stream.cuda_stream)
    L = skv.lib()
    kv_bytes = wl.kv_bytes()
    head_tokens = wl.B * wl.L * wl.Hq

    def launch(a):
        st = L.attn_decode(ctypes.byref(a), sp)
        if st != 0:
            raise skv.SkvError(st, "attn_decode")

    def timed(a, steps, warmup):
        for _ in range(warmup):
            launch(a)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for e0, e1 in evs:
            e0.record(stream)
            launch(a)
            e1.record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
        total_ms = t0.elapsed_time(t1)
        per = [e0.elapsed_time(e1) for e0, e1 in evs]
        if world > 1:
            t = torch.tensor([total_ms], device="cuda")
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            total_ms = float(t.item())
        return total_ms, per

    uuid = "GPU-" + str(torch.cuda.get_device_properties(local).uuid)
    with ClockSampler(uuid) as clk:
        total_ms, per = timed(a_full, args.steps, args.warmup)
        art_ms, art_per = (None, None)
        if not args.no_art:
            art_ms, art_per = timed(a_art, args.steps, args.warmup)
    clocks = clk.summary()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status word {int(status.item()):#x}")

    ms_step = total_ms / args.steps
    value = kv_bytes * world / (ms_step * 1e-3) / 1e9
    per_launch_ms = statistics.mean(per)
    achieved = kv_bytes / (per_launch_ms * 1e-3) / 1e9

    # ---- end to end through the public API: q, tables in from pinned host, O/LSE out
    q_h = q.cpu().pin_memory()
    bt_h = block_table.cpu().pin_memory()
    sl_h = seq_lens.cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()

    def e2e_step():
        q.copy_(q_h, non_blocking=True)
        block_table.copy_(bt_h, non_blocking=True)
        seq_lens.copy_(sl_h, non_blocking=True)
        skv.attn_decode(*common, workspace=ws, stream=stream, **kw)
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / args.steps
    if world > 1:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    h2d = q.numel() * 2 + block_table.numel() * 4 + seq_lens.numel() * 4
    d2h = out.numel() * 4 + lse.numel() * 4

    res = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 in, fp32 accumulate", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.B, "q_heads": wl.Hq, "kv_heads": wl.Hkv,
                   "head_dim": wl.d, "context": wl.L, "page_tokens": wl.bs, "paging": wl.paging,
                   "traversal": "full", "l2": "inputs larger than L2 (2 GiB KV per step), no flush",
                   "parallelism": f"replicas x{world}"},
        "attended_tokens_per_s": head_tokens * world / (ms_step * 1e-3),
        "kv_tokens_per_s": wl.B * wl.L * wl.Hkv * world / (ms_step * 1e-3),
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_kind": peak_kind,
                     "frac_of_8000": achieved / 8000.0, "traffic": None,
                     "kernel": "decode_kernel + split merge (one attn_decode call)"},
        "clocks": clocks,
        "gpu_launches": args.steps * (2 if ws_n > 0 else 1) + (args.steps if not args.no_art else 0),
    }
    if art_ms is not None:
        cons = consumed.cpu().numpy()
        # loads stop per KV group when all of its heads stopped: bytes = max over the group
        grp = cons.reshape(wl.B, wl.Hkv, wl.G).max(axis=2)
        art_bytes = int(grp.sum()) * wl.bs * wl.d * 4
        art_step = art_ms / args.steps
        res["art"] = {"ms_per_step": art_step, "kv_gbs": art_bytes / (art_step * 1e-3) / 1e9,
                      "blocks_consumed_mean": float(cons.mean()), "blocks_total": wl.nb(0),
                      "blocks_skipped_frac": 1.0 - float(grp.sum()) / (wl.B * wl.Hkv * wl.nb(0)),
                      "time_vs_full": art_step / ms_step,
                      "attended_tokens_per_s": float(cons.sum()) * wl.bs / (art_step * 1e-3),
                      "tau": wl.tau, "phi": wl.phi, "patience": wl.patience}
    res["e2e"] = {"value": kv_bytes * world / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                  "note": "KV cache resident in HBM; per step q, block table and seq_lens copied in "
                          "from pinned host memory and O, LSE copied out"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wl)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
