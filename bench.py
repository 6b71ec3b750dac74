"""Benchmark of the HISA indexer on B200: selections/s on the 32K decode workload.

One step = one decode step of a 64-sequence batch at 32K context: append the
new key of every sequence to the cache (hisa_append: trailing block mean
recomputed) and run the two-stage selection for every sequence's new last
position (hisa_select: H_I=64, d_I=128, B=128, m=64, k=2048).  Inputs are
seeded synthetic block-clustered keys (hisa_inputs) resident in HBM; L2 is
flushed (256 MiB write) between timed steps, outside the timed events.

The JSON line also carries: the flat-scan comparison (dsa_flat_select on
the same rows: speedup and mean IoU), the roofline of the dominant kernel
(stage-2 token scoring, HBM-bound), the pool kernel's bandwidth, an
end-to-end figure through the public API with host buffers, SM clocks
sampled during the timed region, and the CPU oracle timed on a bounded
sample of the same workload.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Multi-GPU (torchrun): every rank runs its own 64 sequences (weak scaling, no
data-path collective); time = max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(cfg=1, name="decode-32k-b64")
L2_FLUSH_BYTES = 256 << 20


def iou(a_row, b_row) -> float:
    """|A & B| / |A | B| of two index rows, -1 padding excluded."""
    a = set(int(v) for v in a_row if v >= 0)
    b = set(int(v) for v in b_row if v >= 0)
    if not a and not b:
        return 1.0
    return len(a & b) / len(a | b)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16_tflops=p["bf16_tflops"], source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, source="fallback")


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """SM clock and throttle reasons sampled through NVML from a background
    thread while the timed region runs (about every millisecond)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.samples = []
        self.max_mhz = None
        self.err = None

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = self._handle(pynvml)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report no clocks
            self.err = repr(e)
            self.thread = None
            return self
        self.stop = threading.Event()

        def loop():
            while not self.stop.is_set():
                try:
                    mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((mhz, rs))
                except Exception as e:
                    self.err = repr(e)
                    break
                self.stop.wait(0.001)

        self.thread = threading.Thread(target=loop, daemon=True)
        self.thread.start()
        return self

    def _handle(self, pynvml):
        import torch
        uuid = None
        try:
            uuid = str(torch.cuda.get_device_properties(self.device_index).uuid)
        except Exception:
            pass
        if uuid:
            u = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            try:
                return pynvml.nvmlDeviceGetHandleByUUID(u)
            except Exception:
                pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        idx = int(vis.split(",")[self.device_index]) if vis and vis.split(",")[0].isdigit() \
            else self.device_index
        return pynvml.nvmlDeviceGetHandleByIndex(idx)

    def __exit__(self, *exc):
        if getattr(self, "thread", None) is not None:
            self.stop.set()
            self.thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "samples": 0, "reasons": [],
                    "note": self.err or "no samples"}
        mhz = [m for m, _ in self.samples]
        reasons = set()
        for _, rs in self.samples:
            for bit, name in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        return {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": self.max_mhz,
                "samples": len(mhz), "reasons": sorted(reasons)}


# --------------------------------------------------------------- workload


QUERY_SETS = 32


def make_workload(steps_total: int, seed_shift: int = 0):
    """The 32K decode workload with room for `steps_total` appended keys per
    sequence; decode step s uses query set s % QUERY_SETS."""
    from hisa_inputs import make_config
    spec_cap = 32768 + steps_total
    case = make_config(WORKLOAD["cfg"], cap=spec_cap, append_steps=steps_total,
                       append_query_sets=QUERY_SETS, seed=20260330 + WORKLOAD["cfg"] + seed_shift)
    return case


def algorithmic_bytes(case):
    """Bytes the method must move per query row in each kernel (decode, bf16)."""
    H, d, B, m, k = case.H, case.d, case.B, case.m, case.k
    nb = -(-case.cap // B)
    q = H * d * 2 + H * 4
    token_score = m * B * d * 2 + q + m * 4 + m * B * 4      # keys + Q,w + block ids + score keys
    block_score = nb * 2 * d * 2 + q + nb * 4                 # hi/lo representatives + Q,w + keys
    return dict(token_score=token_score, block_score=block_score,
                step=token_score + block_score + m * B * 4 + k * 4 + nb * 4 + 2 * d + 2 * B * d,
                flat_row=case.cap * d * 2 + q + case.cap * 4)


def traffic_record():
    """ncu DRAM bytes per launch of the token-scoring kernel, if taken on this source."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    src = os.path.join(ROOT, "hierarchical_top_indexer_b200", "csrc", "score.cu")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path))
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    ent = rec.get("token_score")
    if not ent or ent.get("score_cu_sha256_16") != sha:
        return None
    return ent.get("bytes_per_launch")


# --------------------------------------------------------------------- GPU


def capture_steps(fns, dev):
    """One CUDA graph per step: fns[i]() is captured as it would run (the
    library's launches, with their programmatic-launch edges), so replaying it
    puts no host work between a step's kernels.  The library allocates and
    synchronises nothing inside a call, so its calls capture as they are."""
    import torch
    cap = torch.cuda.Stream(dev)
    graphs = []
    for fn in fns:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            fn()
        graphs.append(g)
    torch.cuda.synchronize()
    return graphs


def run_gpu(args, rank, world):
    import torch
    import hierarchical_top_indexer_b200 as hisa

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    K, W = args.steps, args.warmup
    E = args.e2e_steps
    n_flat = args.flat_steps
    n_prof = min(K, 50)
    total_steps = W + K + n_prof + 1 + E
    case = make_workload(total_steps, seed_shift=rank_seed_shift(rank))
    kv = hisa.KVCache.from_case(case, device=dev)
    stream = torch.cuda.current_stream()
    batch, H, d, m, k = case.batch, case.H, case.d, case.m, case.k

    # pool: the index build (also times the pool kernel)
    hisa.hisa_profile_enable(True)
    hisa.hisa_pool_blocks(kv)
    torch.cuda.synchronize()
    hisa.hisa_profile_read(reset=True)
    pool_ms = []
    for _ in range(3):
        hisa.hisa_pool_blocks(kv)
        torch.cuda.synchronize()
        pool_ms.append(hisa.hisa_profile_read(reset=True)["pool"][0])
    hisa.hisa_profile_enable(False)

    # device-resident per-step inputs
    toks = torch.from_numpy(case.append_keys.view(np.int16)).view(torch.bfloat16).to(dev)
    Qs = torch.from_numpy(case.append_Q.view(np.int16)).view(torch.bfloat16).to(dev)
    Ws = torch.from_numpy(case.append_w).to(dev)
    q_seq = torch.arange(batch, dtype=torch.int32, device=dev)
    ws = hisa.workspace(hisa.hisa_decode_step_workspace_bytes(kv, H, m, k), dev)
    idx = torch.empty((2, batch, k), dtype=torch.int32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    nsets = Qs.shape[0]

    def step(s, out):
        # one decode step: every sequence's new key appended, then its new
        # last position selected (hisa_decode_step = hisa_append + hisa_select)
        hisa.hisa_decode_step(kv, toks[s], Qs[s % nsets], Ws[s % nsets], m, k, ws=ws, idx=out)

    for s in range(W):
        step(s, idx[s % 2])
        flush.fill_(7)
    torch.cuda.synchronize()
    graphs = capture_steps([lambda s=W + i: step(s, idx[s % 2]) for i in range(K)], dev)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        wall0 = time.perf_counter()
        for i in range(K):
            ev[i][0].record(stream)
            graphs[i].replay()
            ev[i][1].record(stream)
            flush.fill_(7)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = float(sum(step_ms))
    total_ms = max_over_ranks(total_ms, world, dev)
    # Per-kernel durations: the same steps again, captured as graphs like the
    # timed ones but with an event pair around every launch (separate pass:
    # those events stop the launches from overlapping, so the timed steps
    # above run without them).
    hisa.hisa_profile_enable(True)
    hisa.hisa_profile_read(reset=True)
    pgraphs = capture_steps([lambda s=W + K + i: step(s, idx[s % 2]) for i in range(n_prof)], dev)
    torch.cuda.synchronize()
    for g in pgraphs:
        g.replay()
        flush.fill_(7)
    torch.cuda.synchronize()
    phases = hisa.hisa_profile_read(reset=True)
    hisa.hisa_profile_enable(False)
    del pgraphs
    launches = sum(n for _, n in phases.values()) * K // n_prof

    # select-only comparison: HISA vs the flat scan on the same rows
    s_cmp = W + K + n_prof
    hisa.hisa_append(kv, toks[s_cmp])
    fws = hisa.workspace(hisa.dsa_flat_workspace_bytes(kv, batch, H, k), dev)
    fidx = torch.empty((batch, k), dtype=torch.int32, device=dev)
    hidx = torch.empty((batch, k), dtype=torch.int32, device=dev)

    def time_calls(fn, n):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for _ in range(2):
            fn()
            flush.fill_(7)
        for a, b in evs:
            a.record(stream)
            fn()
            b.record(stream)
            flush.fill_(7)
        torch.cuda.synchronize()
        return float(np.median([a.elapsed_time(b) for a, b in evs]))

    qc, wc = Qs[s_cmp % nsets], Ws[s_cmp % nsets]
    hisa_sel_ms = time_calls(lambda: hisa.hisa_select(kv, qc, wc, q_seq, None, m, k,
                                                      ws=ws, idx=hidx), n_flat)
    flat_ms = time_calls(lambda: hisa.dsa_flat_select(kv, qc, wc, q_seq, None, k,
                                                      ws=fws, idx=fidx), n_flat)
    torch.cuda.synchronize()
    hi, fi = hidx.cpu().numpy(), fidx.cpu().numpy()
    mean_iou = float(np.mean([iou(a, b) for a, b in zip(hi, fi)]))

    # end to end through the public API with host buffers
    e2e = None
    if E > 0:
        e2e = run_e2e(hisa, kv, case, toks, Qs, Ws, q_seq, ws, stream, W + K + n_prof + 1, E)
    assert kv.status_bits() == 0, f"device status {kv.status_bits():#x}"

    peaks = measured_peaks()
    ab = algorithmic_bytes(case)
    tok_ms, tok_n = phases["token_score"]
    tok_launch_s = tok_ms / max(tok_n, 1) / 1e3
    tok_bytes = ab["token_score"] * batch
    achieved = tok_bytes / tok_launch_s / 1e9
    nb = -(-case.cap // case.B)
    pool_bytes = batch * 32768 * d * 2 + batch * nb * (d * 4 + 2 * d * 2)
    pool_gbs = pool_bytes / (float(np.median(pool_ms)) / 1e3) / 1e9
    kernels = {name: {"ms_per_launch": (ms / n if n else None), "launches_profiled": n,
                      "share": ms / max(sum(x for x, _ in phases.values()), 1e-9)}
               for name, (ms, n) in phases.items() if n}
    return dict(
        total_ms=total_ms, step_ms=step_ms, wall=wall, clocks=clk.summary(), launches=launches,
        kernels=kernels, tok_bytes=tok_bytes, achieved=achieved, peaks=peaks,
        pool_gbs=pool_gbs, pool_ms=float(np.median(pool_ms)), hisa_sel_ms=hisa_sel_ms,
        flat_ms=flat_ms, mean_iou=mean_iou, e2e=e2e, case=case)


def run_e2e(hisa, kv, case, toks, Qs, Ws, q_seq, ws, stream, base, E):
    """The decode step end to end through the public calls: every step copies
    its inputs (new keys, Q, w: one packed pinned buffer per step) from host
    to device, runs hisa_decode_step, and copies its 64 x 2048 indices back to
    pinned host memory.  As a serving loop would, each step's three parts are
    captured once as CUDA graphs (the copy in, the call, the copy out) and
    replayed on three streams, with events for every dependency: the copy in
    of step s overlaps the kernels of step s - 1, the copy out of step s those
    of step s + 1; two device slots hold the inputs and outputs in flight.
    One event pair brackets all E steps; the caches (512 MiB of keys) exceed
    L2, so no flush is needed."""
    import torch
    dev = kv.keys.device
    batch, k, m, H, d = case.batch, case.k, case.m, case.H, case.d
    nsets = Qs.shape[0]
    n_tok, n_q, n_w = batch * d * 2, batch * H * d * 2, batch * H * 4     # bytes
    n_in = n_tok + n_q + n_w
    pin_in = torch.empty((E, n_in), dtype=torch.uint8).pin_memory()
    for i in range(E):
        src = base + i
        pin_in[i, :n_tok] = torch.from_numpy(case.append_keys[src].view(np.uint8).reshape(-1))
        pin_in[i, n_tok:n_tok + n_q] = torch.from_numpy(case.append_Q[src % nsets].view(np.uint8).reshape(-1))
        pin_in[i, n_tok + n_q:] = torch.from_numpy(case.append_w[src % nsets].view(np.uint8).reshape(-1))
    pin_out = torch.empty((E, batch, k), dtype=torch.int32).pin_memory()
    dev_in = [torch.empty(n_in, dtype=torch.uint8, device=dev) for _ in range(2)]
    didx = [torch.empty((batch, k), dtype=torch.int32, device=dev) for _ in range(2)]
    views = [(b[:n_tok].view(torch.bfloat16).view(batch, d),
              b[n_tok:n_tok + n_q].view(torch.bfloat16).view(batch, H, d),
              b[n_tok + n_q:].view(torch.float32).view(batch, H)) for b in dev_in]
    s_in, s_out, cap = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    g_in, g_cmp, g_out = [], [], []
    for i in range(E):
        j = i % 2
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s_in):
            dev_in[j].copy_(pin_in[i], non_blocking=True)
        g_in.append(g)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            tok, Q, w = views[j]
            hisa.hisa_decode_step(kv, tok, Q, w, m, k, ws=ws, idx=didx[j])
        g_cmp.append(g)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s_out):
            pin_out[i].copy_(didx[j], non_blocking=True)
        g_out.append(g)
    ev_in = [torch.cuda.Event() for _ in range(E)]
    ev_done = [torch.cuda.Event() for _ in range(E)]
    ev_out = [torch.cuda.Event() for _ in range(E)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    host0 = time.perf_counter()
    t0.record(stream)
    s_in.wait_event(t0)
    s_out.wait_event(t0)
    for i in range(E):                               # (a graph replays on the current stream)
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_done[i - 2])      # step i - 2 no longer reads slot i % 2
            g_in[i].replay()
            ev_in[i].record(s_in)
        stream.wait_event(ev_in[i])
        if i >= 2:
            stream.wait_event(ev_out[i - 2])         # step i - 2's indices have left slot i % 2
        g_cmp[i].replay()
        ev_done[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_done[i])
            g_out[i].replay()
            ev_out[i].record(s_out)
    stream.wait_event(ev_out[E - 1])
    t1.record(stream)
    host_enqueue = time.perf_counter() - host0
    t1.synchronize()
    e2e_ms = t0.elapsed_time(t1)
    del g_in, g_cmp, g_out
    return {"value": batch * E / (e2e_ms / 1e3), "unit": "selections/s",
            "h2d_bytes_per_step": int(n_in), "d2h_bytes_per_step": int(batch * k * 4), "steps": E,
            "ms_per_step": e2e_ms / E, "host_enqueue_ms_per_step": host_enqueue * 1e3 / E,
            "path": "pinned host -> hisa_decode_step (python binding of the C ABI) -> pinned host; "
                    "each step's copy in, call and copy out captured as CUDA graphs and replayed "
                    "on three streams, overlapping the neighbouring steps",
            "l2": "not flushed: the key cache (512 MiB) exceeds L2"}


# ------------------------------------------------------ other workloads


def _median_ms(fn, n, flush, stream, warm=2):
    """Median device time of fn() over n calls, L2 flushed between calls."""
    import torch
    for _ in range(warm):
        fn()
        flush.fill_(7)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for a, b in evs:
        a.record(stream)
        fn()
        b.record(stream)
        flush.fill_(7)
    torch.cuda.synchronize()
    return float(np.median([a.elapsed_time(b) for a, b in evs]))


def _phase_ms(hisa, fn, phase, n):
    """Mean per-launch time of one library phase over n calls (events around every launch)."""
    import torch
    hisa.hisa_profile_enable(True)
    hisa.hisa_profile_read(reset=True)
    for _ in range(n):
        fn()
    torch.cuda.synchronize()
    ph = hisa.hisa_profile_read(reset=True)
    hisa.hisa_profile_enable(False)
    ms, cnt = ph[phase]
    return ms / max(cnt, 1)


def run_workloads(args, dev, peaks):
    """Select-only timings on the other workloads: HISA against the flat scan
    (speedup, mean IoU) at 64K prefill and 128K e4m3 decode, the three-level
    search at 128K, a block size / pooling sweep at 32K, the streaming
    append + select step at 128K, and searches of three and four block
    levels at 128K.  Parity on these sizes is in the GPU tests."""
    import torch
    import hierarchical_top_indexer_b200 as hisa
    from hisa_inputs import make_config

    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    n = args.workload_steps
    out = {}

    def one(cfg):
        case = make_config(cfg)
        kv = hisa.KVCache.from_case(case, device=dev)
        hisa.hisa_pool_blocks(kv)
        Q = torch.from_numpy(case.Q.view(np.int16)).view(torch.bfloat16).to(dev)
        w = torch.from_numpy(case.w).to(dev)
        qs = torch.from_numpy(case.q_seq).to(dev)
        qp = torch.from_numpy(case.q_pos).to(dev)
        n_q, H, m, k = case.n_q, case.H, case.m, case.k
        ws = hisa.workspace(hisa.hisa_select_workspace_bytes(kv, n_q, H, m, k), dev)
        fws = hisa.workspace(hisa.dsa_flat_workspace_bytes(kv, n_q, H, k), dev)
        hidx = torch.empty((n_q, k), dtype=torch.int32, device=dev)
        fidx = torch.empty((n_q, k), dtype=torch.int32, device=dev)
        sel = lambda: hisa.hisa_select(kv, Q, w, qs, qp, m, k, ws=ws, idx=hidx)
        flat = lambda: hisa.dsa_flat_select(kv, Q, w, qs, qp, k, ws=fws, idx=fidx)
        h_ms = _median_ms(sel, n, flush, stream)
        f_ms = _median_ms(flat, max(3, n // 4), flush, stream)
        tok_ms = _phase_ms(hisa, sel, "token_score", 3)
        pool_ms = _phase_ms(hisa, lambda: hisa.hisa_pool_blocks(kv), "pool", 3)
        mi = float(np.mean([iou(a, b) for a, b in zip(hidx.cpu().numpy(), fidx.cpu().numpy())]))
        assert kv.status_bits() == 0, f"device status {kv.status_bits():#x}"
        kbytes = case.d * (1 if case.dtype == "e4m3" else 2) + (4 if case.dtype == "e4m3" else 0)
        mm = min(m, -(-case.cap // case.B))
        tok_bytes = n_q * (mm * case.B * (kbytes + 4) + H * case.d * 2 + H * 4 + mm * 4)
        tok_flops = n_q * mm * case.B * 2 * H * case.d
        pool_bytes = int(case.lens.sum()) * kbytes + case.batch * kv.nblk * case.d * 8
        r = {"rows": n_q, "hisa_ms_per_select": h_ms, "flat_ms_per_select": f_ms,
             "hisa_selections_per_s": n_q / (h_ms / 1e3),
             "flat_selections_per_s": n_q / (f_ms / 1e3), "speedup": f_ms / h_ms,
             "mean_iou_hisa_vs_flat": mi,
             "token_score": {"ms_per_launch": tok_ms,
                             "GB/s": tok_bytes / (tok_ms / 1e3) / 1e9,
                             "hbm_frac": tok_bytes / (tok_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                             "TFLOP/s": tok_flops / (tok_ms / 1e3) / 1e12,
                             "tensor_frac": tok_flops / (tok_ms / 1e3) / 1e12 / peaks["bf16_tflops"]},
             "pool": {"ms": pool_ms, "GB/s": pool_bytes / (pool_ms / 1e3) / 1e9}}
        del kv, ws, fws
        torch.cuda.empty_cache()
        return case, r

    case, r = one(2)
    r["l2"] = "64K x bf16 keys (16 MiB) stay L2-resident across query rows"
    out[case.name] = r
    case, r = one(3)
    r["l2"] = "flushed between calls (cache 528 MiB)"
    out[case.name] = r
    out["tree_" + case.name] = run_tree(case, dev, n, flush, stream, r["hisa_ms_per_select"])
    deep_case, deep_two_ms = case, r["hisa_ms_per_select"]

    # block size / kept-block count / pooling sweep at a fixed candidate
    # budget m * B = 8192 on the 32K decode workload: quality (IoU with the
    # flat scan) against select time
    case = make_config(1)
    Q = torch.from_numpy(case.Q.view(np.int16)).view(torch.bfloat16).to(dev)
    w = torch.from_numpy(case.w).to(dev)
    qs = torch.from_numpy(case.q_seq).to(dev)
    fidx = None
    sweep = []
    for pool in ("mean", "max"):
        for B, m in ((64, 128), (128, 64), (256, 32)):
            kv = hisa.KVCache.from_case(case, device=dev, pool=pool, B=B)
            hisa.hisa_pool_blocks(kv)
            if fidx is None:
                fws = hisa.workspace(hisa.dsa_flat_workspace_bytes(kv, case.n_q, case.H, case.k), dev)
                fidx = hisa.dsa_flat_select(kv, Q, w, qs, None, case.k, ws=fws).cpu().numpy()
                del fws
            ws = hisa.workspace(hisa.hisa_select_workspace_bytes(kv, case.n_q, case.H, m, case.k), dev)
            hidx = torch.empty((case.n_q, case.k), dtype=torch.int32, device=dev)
            ms = _median_ms(lambda: hisa.hisa_select(kv, Q, w, qs, None, m, case.k, ws=ws, idx=hidx),
                            n, flush, stream)
            mi = float(np.mean([iou(a, b) for a, b in zip(hidx.cpu().numpy(), fidx)]))
            assert kv.status_bits() == 0, f"device status {kv.status_bits():#x}"
            sweep.append({"pool": pool, "B": B, "m": m, "hisa_ms_per_select": ms,
                          "selections_per_s": case.n_q / (ms / 1e3), "mean_iou_hisa_vs_flat": mi})
            del kv, ws
            torch.cuda.empty_cache()
    out["pool_sweep_decode-32k-b64"] = sweep
    out["sparse_attention_decode-32k-b64"] = run_attention(dev, n, flush, stream, peaks)

    # streaming append + select for the new last position, one row per step
    case = make_config(4)
    kv = hisa.KVCache.from_case(case, device=dev)
    hisa.hisa_pool_blocks(kv)
    steps = case.append_keys.shape[0]
    toks = torch.from_numpy(case.append_keys.view(np.int16)).view(torch.bfloat16).to(dev)
    AQ = torch.from_numpy(case.append_Q.view(np.int16)).view(torch.bfloat16).to(dev)
    AW = torch.from_numpy(case.append_w).to(dev)
    ws = hisa.workspace(hisa.hisa_decode_step_workspace_bytes(kv, case.H, case.m, case.k), dev)
    idx = torch.empty((1, case.k), dtype=torch.int32, device=dev)
    # one graph per step (the step is a chain of short launches on an
    # L2-resident cache: launch-bound)
    graphs = capture_steps([lambda s=s: hisa.hisa_decode_step(kv, toks[s], AQ[s], AW[s], case.m, case.k,
                                                                ws=ws, idx=idx)
                            for s in range(steps)], dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for s, (a, b) in enumerate(evs):
        a.record(stream)
        graphs[s].replay()
        b.record(stream)
    torch.cuda.synchronize()
    del graphs
    assert kv.status_bits() == 0, f"device status {kv.status_bits():#x}"
    st = [a.elapsed_time(b) for a, b in evs]
    out[case.name] = {"steps": steps, "us_per_step_mean": 1e3 * float(np.mean(st)),
                      "us_per_step_median": 1e3 * float(np.median(st)),
                      "steps_per_s": steps / (sum(st) / 1e3),
                      "l2": "cache (32 MiB) L2-resident; no flush: each step follows the last",
                      "step": "hisa_decode_step (1 key appended, 1 row selected), replayed from a "
                              "CUDA graph per step"}
    # searches of three and four block levels at 128K (last, so that a
    # failure is reported in the line rather than ending the run)
    try:
        out["levels_" + deep_case.name] = run_levels(deep_case, dev, n, flush, stream, deep_two_ms)
    except Exception as e:  # noqa: BLE001
        out["levels_" + deep_case.name] = {"error": f"{type(e).__name__}: {e}"}
    return out


def run_attention(dev, n, flush, stream, peaks):
    """The consumer of the selection on the 32K decode workload: each of the
    64 rows attends with 128 query heads (d = 128, one shared key and value
    head) over the 2048 tokens hisa_select kept.  Key and value caches are
    their own seeded N(0, 1) bf16 tensors [64, 32768, 128], drawn on the
    device.  Reports the attention call's time and roofline next to the
    indexer's select time on the same rows."""
    import torch
    import hierarchical_top_indexer_b200 as hisa
    from hisa_inputs import make_config

    case = make_config(1)
    kv = hisa.KVCache.from_case(case, device=dev)
    hisa.hisa_pool_blocks(kv)
    Q = torch.from_numpy(case.Q.view(np.int16)).view(torch.bfloat16).to(dev)
    w = torch.from_numpy(case.w).to(dev)
    qs = torch.from_numpy(case.q_seq).to(dev)
    n_q, Ha, D, k = case.n_q, 128, 128, case.k
    ws = hisa.workspace(hisa.hisa_select_workspace_bytes(kv, n_q, case.H, case.m, k), dev)
    idx = torch.empty((n_q, k), dtype=torch.int32, device=dev)
    sel = lambda: hisa.hisa_select(kv, Q, w, qs, None, case.m, k, ws=ws, idx=idx)
    sel_ms = _median_ms(sel, n, flush, stream)
    g = torch.Generator(device=dev).manual_seed(20260331)
    Kc = torch.randn((case.batch, case.cap, D), generator=g, device=dev).to(torch.bfloat16)
    Vc = torch.randn((case.batch, case.cap, D), generator=g, device=dev).to(torch.bfloat16)
    Qa = torch.randn((n_q, Ha, D), generator=g, device=dev).to(torch.bfloat16)
    lens = kv.len.clone()
    aws = hisa.workspace(hisa.hisa_sparse_attn_workspace_bytes(n_q, k), dev)
    out = torch.empty((n_q, Ha, D), dtype=torch.float32, device=dev)
    lse = torch.empty((n_q, Ha), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    att = lambda: hisa.hisa_sparse_attn(Qa, Kc, Vc, lens, qs, idx, ws=aws, out=out, lse=lse, status=status)
    att_ms = _median_ms(att, n, flush, stream)
    assert int(status.item()) == 0 and kv.status_bits() == 0
    nbytes = n_q * (k * 2 * D * 2 + Ha * D * 2 + Ha * D * 4 + Ha * 4 + k * 4)
    flops = n_q * 2 * Ha * k * 2 * D
    gbs = nbytes / (att_ms / 1e3) / 1e9
    del Kc, Vc, kv
    torch.cuda.empty_cache()
    return {"rows": n_q, "heads": Ha, "d": D, "k": k,
            "attn_ms_per_call": att_ms, "hisa_select_ms_per_call": sel_ms,
            "indexer_share": sel_ms / (sel_ms + att_ms),
            "attn_roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_call": nbytes,
                              "TFLOP/s": flops / (att_ms / 1e3) / 1e12},
            "l2": "flushed between calls (key and value caches 512 MiB each)"}


def run_tree(case, dev, n, flush, stream, two_level_ms):
    """Three-level search (superblocks of bf blocks, W kept superblocks, then
    the top m blocks under them, then the top k tokens) against the flat scan
    on one workload: select time, work per row and mean IoU."""
    import torch
    import hierarchical_top_indexer_b200 as hisa

    kv = hisa.KVCache.from_case(case, device=dev)
    hisa.hisa_pool_blocks(kv)
    Q = torch.from_numpy(case.Q.view(np.int16)).view(torch.bfloat16).to(dev)
    w = torch.from_numpy(case.w).to(dev)
    qs = torch.from_numpy(case.q_seq).to(dev)
    n_q, H, m, k = case.n_q, case.H, case.m, case.k
    fws = hisa.workspace(hisa.dsa_flat_workspace_bytes(kv, n_q, H, k), dev)
    fidx = hisa.dsa_flat_select(kv, Q, w, qs, None, k, ws=fws).cpu().numpy()
    del fws
    nb = -(-case.cap // case.B)
    rows = []
    for bf, W in ((8, 32), (8, 64), (16, 32)):
        kv2 = hisa.superblock_index(kv, bf)
        hisa.hisa_pool_blocks(kv2)
        ws = hisa.workspace(hisa.hisa_tree_workspace_bytes(kv, kv2, n_q, H, W, m, k), dev)
        idx = torch.empty((n_q, k), dtype=torch.int32, device=dev)
        run = lambda: hisa.hisa_tree_select(kv, kv2, Q, w, qs, None, W, m, k, ws=ws, idx=idx)
        ms = _median_ms(run, n, flush, stream)
        mi = float(np.mean([iou(a, b) for a, b in zip(idx.cpu().numpy(), fidx)]))
        assert kv.status_bits() == 0, f"device status {kv.status_bits():#x}"
        nb2 = kv2.nblk
        rows.append({"bf": bf, "W": W, "m": m, "ms_per_select": ms,
                     "selections_per_s": n_q / (ms / 1e3), "mean_iou_tree_vs_flat": mi,
                     "scores_per_row": {"superblocks": nb2, "blocks": min(W, nb2) * bf,
                                        "tokens": min(m, nb) * case.B}})
        del kv2, ws
        torch.cuda.empty_cache()
    del kv
    torch.cuda.empty_cache()
    return {"two_level_ms_per_select": two_level_ms,
            "two_level_scores_per_row": {"blocks": nb, "tokens": min(m, nb) * case.B},
            "levels": rows, "l2": "flushed between calls"}


def run_levels(case, dev, n, flush, stream, two_level_ms):
    """Searches of three and four block levels (hisa_levels_select; units of
    1024 and 8192 tokens, or 1024, 4096 and 16384, above the workload's
    blocks) against the flat scan on one workload: select time, units and
    token slots scored per row, and mean IoU."""
    import torch
    import hierarchical_top_indexer_b200 as hisa

    kv = hisa.KVCache.from_case(case, device=dev)
    hisa.hisa_pool_blocks(kv)
    Q = torch.from_numpy(case.Q.view(np.int16)).view(torch.bfloat16).to(dev)
    w = torch.from_numpy(case.w).to(dev)
    qs = torch.from_numpy(case.q_seq).to(dev)
    n_q, H, m, k = case.n_q, case.H, case.m, case.k
    fws = hisa.workspace(hisa.dsa_flat_workspace_bytes(kv, n_q, H, k), dev)
    fidx = hisa.dsa_flat_select(kv, Q, w, qs, None, k, ws=fws).cpu().numpy()
    del fws
    rows = []
    for factors, keep in (((8, 64), (m, 32, 8)), ((8, 32, 128), (m, 32, 16, 4))):
        kvs = [kv] + [hisa.superblock_index(kv, f) for f in factors]
        for c in kvs[1:]:
            hisa.hisa_pool_blocks(c)
        ws = hisa.workspace(hisa.hisa_levels_workspace_bytes(kvs, keep, n_q, H, k), dev)
        idx = torch.empty((n_q, k), dtype=torch.int32, device=dev)
        counts = hisa.hisa_levels_select(kvs, Q, w, qs, None, keep, k, inspect=True)["counts"]
        per_row = counts.double().mean(0).cpu().tolist()
        run = lambda: hisa.hisa_levels_select(kvs, Q, w, qs, None, keep, k, ws=ws, idx=idx)
        ms = _median_ms(run, n, flush, stream)
        mi = float(np.mean([iou(a, b) for a, b in zip(idx.cpu().numpy(), fidx)]))
        assert kv.status_bits() == 0, f"device status {kv.status_bits():#x}"
        rows.append({"unit_tokens": [case.B] + [case.B * f for f in factors], "keep": list(keep),
                     "ms_per_select": ms, "selections_per_s": n_q / (ms / 1e3),
                     "mean_iou_vs_flat": mi,
                     "scored_per_row": {"units_per_level": per_row[:-1], "token_slots": per_row[-1]}})
        del kvs, ws
        torch.cuda.empty_cache()
    del kv
    torch.cuda.empty_cache()
    return {"two_level_ms_per_select": two_level_ms, "searches": rows, "l2": "flushed between calls"}


def run_select_only(args):
    """--select-only NAME: hisa_select (or --flat: dsa_flat_select) on one
    workload, `warmup` untimed then `steps` timed calls; for profiling one
    kernel of one workload."""
    import torch
    import hierarchical_top_indexer_b200 as hisa
    from hisa_inputs import CONFIGS, make_config
    cfg = next(i for i, c in CONFIGS.items() if c["name"] == args.select_only)
    dev = torch.device("cuda", 0)
    case = make_config(cfg)
    kv = hisa.KVCache.from_case(case, device=dev)
    hisa.hisa_pool_blocks(kv)
    Q = torch.from_numpy(case.Q.view(np.int16)).view(torch.bfloat16).to(dev)
    w = torch.from_numpy(case.w).to(dev)
    qs = torch.from_numpy(case.q_seq).to(dev)
    qp = torch.from_numpy(case.q_pos).to(dev)
    n_q, H, m, k = case.n_q, case.H, case.m, case.k
    idx = torch.empty((n_q, k), dtype=torch.int32, device=dev)
    if args.flat:
        ws = hisa.workspace(hisa.dsa_flat_workspace_bytes(kv, n_q, H, k), dev)
        fn = lambda: hisa.dsa_flat_select(kv, Q, w, qs, qp, k, ws=ws, idx=idx)
    else:
        ws = hisa.workspace(hisa.hisa_select_workspace_bytes(kv, n_q, H, m, k), dev)
        fn = lambda: hisa.hisa_select(kv, Q, w, qs, qp, m, k, ws=ws, idx=idx)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ms = _median_ms(fn, args.steps, flush, torch.cuda.current_stream(), warm=args.warmup)
    assert kv.status_bits() == 0, f"device status {kv.status_bits():#x}"
    return {"select_only": case.name, "flat": bool(args.flat), "rows": n_q,
            "ms_per_select": ms, "selections_per_s": n_q / (ms / 1e3)}


def run_ncu_case(name: str, reps: int = 3):
    """--ncu-case NAME: a fixed, untimed sequence of library calls on one
    workload, L2 flushed between calls, for ncu captures filtered by kernel
    name (each call kind `reps` times, in this order):
      decode-32k-b64          hisa_pool_blocks, hisa_decode_step, hisa_select,
                              dsa_flat_select (pool, append, block scoring,
                              token scoring, top-k, flat scoring, cluster top-k)
      decode-128k-b32-e4m3    hisa_pool_blocks, hisa_select (e4m3 pool, fp8 scoring)
      prefill-64k-chunk4096   hisa_select (stage 2 on L2-resident keys)
      sparse-attention        hisa_sparse_attn over the decode-32k-b64 selection"""
    import torch
    import hierarchical_top_indexer_b200 as hisa
    from hisa_inputs import CONFIGS, make_config
    dev = torch.device("cuda", 0)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def rep(fn):
        for _ in range(reps):
            fn()
            flush.fill_(7)

    attn = name == "sparse-attention"
    cfg = next(i for i, c in CONFIGS.items() if c["name"] == ("decode-32k-b64" if attn else name))
    steps = reps + 1 if cfg == 1 else 0
    case = make_config(cfg, cap=CONFIGS[cfg]["L"] + steps, append_steps=steps,
                       append_query_sets=1) if steps else make_config(cfg)
    kv = hisa.KVCache.from_case(case, device=dev)
    Q = torch.from_numpy(case.Q.view(np.int16)).view(torch.bfloat16).to(dev)
    w = torch.from_numpy(case.w).to(dev)
    qs = torch.from_numpy(case.q_seq).to(dev)
    qp = torch.from_numpy(case.q_pos).to(dev)
    n_q, H, m, k = case.n_q, case.H, case.m, case.k
    idx = torch.empty((n_q, k), dtype=torch.int32, device=dev)
    ws = hisa.workspace(max(hisa.hisa_select_workspace_bytes(kv, n_q, H, m, k),
                            hisa.dsa_flat_workspace_bytes(kv, n_q, H, k)), dev)
    if not attn:
        rep(lambda: hisa.hisa_pool_blocks(kv))
    else:
        hisa.hisa_pool_blocks(kv)
    if cfg == 1 and not attn:
        toks = torch.from_numpy(case.append_keys.view(np.int16)).view(torch.bfloat16).to(dev)
        AQ = torch.from_numpy(case.append_Q[0].view(np.int16)).view(torch.bfloat16).to(dev)
        AW = torch.from_numpy(case.append_w[0]).to(dev)
        it = iter(range(steps))
        rep(lambda: hisa.hisa_decode_step(kv, toks[next(it)], AQ, AW, m, k, ws=ws, idx=idx))
    rep(lambda: hisa.hisa_select(kv, Q, w, qs, qp, m, k, ws=ws, idx=idx))
    if cfg == 1 and not attn:
        rep(lambda: hisa.dsa_flat_select(kv, Q, w, qs, qp, k, ws=ws, idx=idx))
    if attn:
        g = torch.Generator(device=dev)
        g.manual_seed(20260331)
        Ha, cap = 128, case.cap
        Kc = torch.randn((case.batch, cap, 128), generator=g, device=dev).to(torch.bfloat16)
        Vc = torch.randn((case.batch, cap, 128), generator=g, device=dev).to(torch.bfloat16)
        Qa = torch.randn((n_q, Ha, 128), generator=g, device=dev).to(torch.bfloat16)
        aws = hisa.workspace(hisa.hisa_sparse_attn_workspace_bytes(n_q, k), dev)
        out = torch.empty((n_q, Ha, 128), dtype=torch.float32, device=dev)
        lse = torch.empty((n_q, Ha), dtype=torch.float32, device=dev)
        rep(lambda: hisa.hisa_sparse_attn(Qa, Kc, Vc, kv.len, qs, idx, ws=aws, out=out, lse=lse))
    torch.cuda.synchronize()
    assert kv.status_bits() == 0, f"device status {kv.status_bits():#x}"
    return {"ncu_case": name, "reps": reps}


# ----------------------------------------------------------- CPU baseline


def cpu_oracle_rate(case=None, budget_s: float = 12.0, rows_per_call: int = 16):
    """The oracle as it stands, on all host cores, on a bounded sample of rows."""
    import oracle
    if case is None:
        case = make_workload(1)
    cache = oracle.Cache.of(case)
    threads = host_cores()
    done, t0 = 0, time.perf_counter()
    r0 = 0
    while True:
        rows = np.arange(r0, r0 + rows_per_call) % case.n_q
        oracle.hisa_select(cache, case.Q[rows], case.w[rows], case.q_seq[rows], case.q_pos[rows],
                           case.B, case.m, case.k, threads=threads)
        done += len(rows)
        r0 += rows_per_call
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return dict(value=done / el, unit="selections/s", cores=threads, kind="oracle",
                sample=f"{done} query rows of {WORKLOAD['name']} (HISA oracle, double, pooling "
                       f"from scratch per row), {el:.1f} s wall")


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle on the same workload (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    case = make_workload(1)
    cache = oracle.Cache.of(case)
    threads = host_cores()
    rows_per_step = args.ref_rows
    for s in range(args.warmup):
        rows = (np.arange(rows_per_step) + s * rows_per_step) % case.n_q
        oracle.hisa_select(cache, case.Q[rows], case.w[rows], case.q_seq[rows], case.q_pos[rows],
                           case.B, case.m, case.k, threads=threads)
    t0 = time.perf_counter()
    for s in range(args.steps):
        rows = (np.arange(rows_per_step) + s * rows_per_step) % case.n_q
        oracle.hisa_select(cache, case.Q[rows], case.w[rows], case.q_seq[rows], case.q_pos[rows],
                           case.B, case.m, case.k, threads=threads)
    el = time.perf_counter() - t0
    v = rows_per_step * args.steps / el
    line = {
        "impl": "reference", "metric": "HISA indexer top-k selections/s (decode, 32K context)",
        "value": v, "unit": "selections/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD["name"], "batch": case.batch, "L": 32768, "H_I": case.H,
                   "d_I": case.d, "B": case.B, "m": case.m, "k": case.k,
                   "step": f"{rows_per_step} query rows (bounded sample of the 64-row batch)"},
        "cpu_baseline": {"value": v, "unit": "selections/s", "cores": threads, "kind": "oracle",
                         "sample": f"{rows_per_step} rows per step x {args.steps} steps"},
        "e2e": {"value": v, "unit": "selections/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    return line


# ------------------------------------------------------------------ ranks


def init_ranks(backend: str = "nccl"):
    """(rank, world) from the torchrun environment; joins the process group
    when there is more than one rank.  One process per GPU."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def rank_seed_shift(rank: int) -> int:
    """Every rank draws its own sequences (weak scaling over disjoint batches)."""
    return 1000 * rank


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value: the job's time."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(rows_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job selections/s: the rows every rank finished over the slowest rank's time."""
    return rows_per_rank * steps * world / (max_ms / 1e3)


# -------------------------------------------------------------------- main


def main(argv=None, backend: str = "nccl"):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["hisa", "reference"], default="hisa")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--flat-steps", type=int, default=20)
    ap.add_argument("--ref-rows", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--select-only", default=None,
                    help="time only hisa_select on this workload (a name from hisa_inputs)")
    ap.add_argument("--flat", action="store_true", help="with --select-only: dsa_flat_select")
    ap.add_argument("--ncu-case", default=None,
                    choices=["decode-32k-b64", "decode-128k-b32-e4m3", "prefill-64k-chunk4096",
                             "sparse-attention"],
                    help="run a fixed untimed call sequence on one workload (for ncu captures)")
    ap.add_argument("--attn-only", action="store_true",
                    help="time only the sparse attention over the 32K decode selection")
    ap.add_argument("--workload-steps", type=int, default=20,
                    help="timed selects per extra workload (0: skip them)")
    args = ap.parse_args(argv)
    assert args.warmup >= 3, "at least 3 warm-up steps"

    rank, world = init_ranks(backend)

    try:
        if args.impl == "reference":
            line = run_reference(args, rank, world)
            if line is not None:
                print(json.dumps(line), flush=True)
            return 0

        if args.attn_only:
            if rank == 0:
                import torch
                dev = torch.device("cuda", 0)
                flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
                print(json.dumps(run_attention(dev, args.steps, flush, torch.cuda.current_stream(),
                                               measured_peaks())), flush=True)
            return 0

        if args.select_only:
            if rank == 0:
                print(json.dumps(run_select_only(args)), flush=True)
            return 0

        if args.ncu_case:
            if rank == 0:
                print(json.dumps(run_ncu_case(args.ncu_case)), flush=True)
            return 0

        r = run_gpu(args, rank, world)
        if rank != 0:
            return 0
        case = r["case"]
        K = args.steps
        value = job_rate(case.batch, K, world, r["total_ms"])
        peaks = r["peaks"]
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            cpu = cpu_oracle_rate(case)
        traffic = traffic_record()
        extra = None
        if world == 1 and args.workload_steps > 0:
            import torch
            extra = run_workloads(args, torch.device("cuda", 0), peaks)
        line = {
            "metric": "HISA indexer top-k selections/s (decode, 32K context)",
            "value": value, "unit": "selections/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": r["total_ms"] / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD["name"], "batch": case.batch, "L": 32768,
                       "H_I": case.H, "d_I": case.d, "B": case.B, "m": case.m, "k": case.k,
                       "key_dtype": "bf16", "parallelism": f"replicas x{world}" if world > 1 else "1 gpu",
                       "step": "hisa_decode_step: 64 keys appended (trailing block means updated) + "
                               "64 rows selected at the new last positions (= hisa_append + hisa_select)",
                       "launch": "each timed step replayed from a CUDA graph captured from the same calls",
                       "l2": "flushed between timed steps (256 MiB write, outside the timed events)"},
            "clocks": r["clocks"],
            "gpu_launches": r["launches"],
            "roofline": {"kernel": "token_score (stage 2: gather + tcgen05 scoring)",
                         "bound": "hbm", "achieved": r["achieved"], "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": r["achieved"] / peaks["hbm_gbs"],
                         "traffic": traffic, "peak_source": peaks["source"],
                         "algorithmic_bytes_per_launch": r["tok_bytes"]},
            "kernels": r["kernels"],
            "kernels_note": "per-launch times from a separate pass of the same steps, replayed from "
                            "CUDA graphs with an event pair around every launch (L2 flushed "
                            "between steps)",
            "pool": {"GB/s": r["pool_gbs"], "frac": r["pool_gbs"] / peaks["hbm_gbs"],
                     "ms": r["pool_ms"]},
            "flat_scan": {"ms_per_select": r["flat_ms"], "hisa_ms_per_select": r["hisa_sel_ms"],
                          "speedup": r["flat_ms"] / r["hisa_sel_ms"],
                          "flat_selections_per_s": case.batch / (r["flat_ms"] / 1e3),
                          "mean_iou_hisa_vs_flat": r["mean_iou"]},
            "e2e": r["e2e"],
            "workloads": extra,
            "cpu_baseline": cpu,
            "wall_s_timed_region": r["wall"],
        }
        print(json.dumps(line), flush=True)
        return 0
    finally:
        if world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
