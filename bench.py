"""Benchmark of the Double Sparsity decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config I]

One step = one decode token for every sequence of a layer, in one launch
(ds_decode_step): the new token's heavy channels are appended to the label
cache, then query gather, approximate scores, top-k and exact attention over
the selected K/V rows. The default workload is the
Llama-2-7B-shaped layer (batch 8, 32 MHA heads, head_dim 128, 4096 cached
tokens, 16 bf16 heavy channels, top-256). Inputs are seeded synthetic tensors.

Timing: the step captured in a CUDA graph, CUDA events on the launching stream, a 512 MiB
L2-flushing write before every timed step, max over ranks under torchrun
(weak scaling: every rank runs its own layer; no collective on the data path).
Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "sparse-decode attn tokens/s per layer; achieved HBM GB/s (% of B200 peak)"
UNIT = "tokens/s/layer"
NOMINAL_HBM_GBS = 8000.0
FLUSH_BYTES = 512 << 20
KERNEL_SOURCES = ["channel_token_sparse_b200/csrc/ds_decode_kernel.cuh",
                  "channel_token_sparse_b200/csrc/ds_common.cuh",
                  "channel_token_sparse_b200/csrc/ds_decode_bf16_fp.cu",
                  "channel_token_sparse_b200/csrc/ds_api.cu"]


# ----------------------------------------------------------- accounting

def algorithmic_bytes(wl: synth.Workload, out_esz: int = 2) -> dict:
    """Bytes the decode step must move: label cache (+ 4-bit scale/zero),
    the selected K and V rows, the query and the output."""
    esz = 4 if wl.kv_dtype == "f32" else 2
    rows = wl.b * wl.hkv
    if wl.label_dtype == "int4":
        lab_row = wl.c // 2 + 4
    else:
        lab_row = wl.c * esz
    k_eff = min(wl.topk, wl.s)
    label = rows * wl.s * lab_row
    kv = rows * k_eff * wl.d * esz * 2
    qo = wl.b * wl.hq * wl.d * (esz + out_esz)
    append = rows * (wl.d * esz + lab_row)  # new token: key row read, label row written
    dense = rows * wl.s * wl.d * esz * 2 + qo
    return {"label": label, "kv_selected": kv, "q_out": qo, "append": append,
            "total": label + kv + qo + append, "dense_total": dense}


def prefill_bytes(wl: synth.Workload) -> int:
    """Prefill label build over s-1 tokens: every 32-byte sector of the key
    rows is read (heavy channels are spread over the row) and the label rows
    are written."""
    esz = 4 if wl.kv_dtype == "f32" else 2
    lab_row = wl.c // 2 + 4 if wl.label_dtype == "int4" else wl.c * esz
    return wl.b * wl.hkv * (wl.s - 1) * (wl.d * esz + lab_row)


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_index: int):
    """DRAM bytes per decode launch from a committed ncu summary, if it was
    taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(str(workload_index))
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# -------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read only)."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            props = torch.cuda.get_device_properties(device_index)
            bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            try:  # NVML numbers devices independently of CUDA_VISIBLE_DEVICES: match by PCI id
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:  # noqa: BLE001
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.reasons_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = str(e)
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.reasons_fn(self.h)
                self.samples.append((mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.ok:
            self.t.join()

    def summary(self) -> dict:
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [m for m, _ in self.samples]
        mask = 0
        for _, r in self.samples:
            mask |= r
        reasons = [n for b, n in self.REASONS.items() if mask & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz)}


# ------------------------------------------------------------ distributed

def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(batch_per_rank: int, world: int, steps: int, max_seconds: float) -> float:
    """Whole-job decode tokens/s per layer: every rank decodes batch_per_rank
    tokens per step."""
    return batch_per_rank * world * steps / max_seconds


# ------------------------------------------------------------ our arm

def build_state(wl: synth.Workload, dev, rank: int):
    import torch

    import channel_token_sparse_b200 as ds
    if wl.s * wl.b * wl.hkv * wl.d <= (1 << 28):
        di = synth.decode_inputs(wl, seed_offset=rank)
        q, k, v = (_dev(x, wl.kv_dtype, dev) for x in (di.q, di.k, di.v))
    else:
        q, k, v = synth.decode_inputs_torch(wl, dev, seed_offset=rank)
    idx = torch.from_numpy(np.ascontiguousarray(synth.outlier_channels(wl)[:, : wl.c], np.int32)).to(dev)
    if idx.shape[1] < wl.c:  # more heavy channels than planted: pad with the next unused ones
        full = []
        for g in range(wl.hkv):
            have = list(synth.outlier_channels(wl)[g])
            extra = [c for c in range(wl.d) if c not in have][: wl.c - len(have)]
            full.append(sorted(have + extra))
        idx = torch.tensor(full, dtype=torch.int32, device=dev)
    lab, sc, ze = ds.new_label_cache(k, wl.c, int4=wl.label_dtype == "int4")
    return dict(q=q, k=k, v=v, idx=idx, lab=lab, sc=sc, ze=ze)


def _dev(x: np.ndarray, dtype: str, dev):
    import torch
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).to(dev)


def rotation(wl, dev, kind: str, out_esz: int):
    """How many independent layer instances the timed steps cycle through.
    'rotate': enough copies that their working sets together exceed twice the
    L2, so no step finds its inputs in L2 from an earlier step (a workload
    whose own working set is that large needs one); tiny workloads, where 16
    copies would still fit, fall back to 'flush'."""
    import math

    import torch
    if kind != "rotate":
        return kind, 1
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    ws = algorithmic_bytes(wl, out_esz)["total"]
    r = max(1, math.ceil(2 * l2 / ws))
    if r > 16:
        return "flush", 1
    return "rotate", r


def _clone_state(st):
    return {n: (t.clone() if t is not None and hasattr(t, "clone") and n != "idx" else t) for n, t in st.items()}


def run_ours(args, wl, rank, local_rank, world):
    import torch

    import channel_token_sparse_b200 as ds

    ds.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    out_dtype = torch.bfloat16 if wl.kv_dtype == "bf16" else torch.float32
    timing, R = rotation(wl, dev, args.timing, 2 if out_dtype == torch.bfloat16 else 4)
    st0 = build_state(wl, dev, rank)
    states = [st0] + [_clone_state(st0) for _ in range(R - 1)]
    for st in states:
        st["out"] = torch.empty((wl.b, wl.hq, wl.d), dtype=out_dtype, device=dev)
    q, k, v, idx, lab, sc, ze, out = (st0[n] for n in ("q", "k", "v", "idx", "lab", "sc", "ze", "out"))
    pos = wl.s - 1
    flush = L2Flush(dev, args.flush)
    stream = torch.cuda.Stream(device=dev)

    # prefill: label cache for the first s-1 tokens (timed separately, after
    # one untimed call that loads the kernel)
    for st in states:
        ds.build_label_cache(st["k"], st["idx"], pos, st["lab"], st["sc"], st["ze"])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush()
    e0.record()
    ds.build_label_cache(k, idx, pos, lab, sc, ze)
    e1.record()
    torch.cuda.synchronize()
    prefill_ms = e0.elapsed_time(e1)

    def step_of(st):
        # one launch: label row of token s-1 (ds_append_label's work) + sparse decode
        return lambda: ds.decode_step(st["q"], st["k"], st["v"], st["lab"], st["idx"], wl.s, wl.topk,
                                      lscale=st["sc"], lzero=st["ze"], out=st["out"])

    graphs = []
    for st in states:
        fn = step_of(st)
        with torch.cuda.stream(stream):
            for _ in range(3):  # set kernel attributes before capture
                fn()
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        graphs.append(g)

    def one_step(i, evs=None):
        if timing == "flush":
            flush()  # untimed: evicts L2 (the step's inputs could otherwise stay in the 126 MB L2)
        if evs:
            evs[0].record()
        graphs[i % R].replay()
        if evs:
            evs[1].record()

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            one_step(i)
    torch.cuda.synchronize()

    sampler = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    if timing == "flush":
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        with sampler:
            wall0 = time.perf_counter()
            with torch.cuda.stream(stream):
                for i in range(args.steps):
                    one_step(i, evs[i])
            torch.cuda.synchronize()
            wall1 = time.perf_counter()
        step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    else:
        # back to back, cycling through the R layer instances; one event pair
        # around the K steps on the launching stream
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with sampler:
            wall0 = time.perf_counter()
            with torch.cuda.stream(stream):
                t0.record()
                for i in range(args.steps):
                    one_step(args.warmup + i)
                t1.record()
            torch.cuda.synchronize()
            wall1 = time.perf_counter()
        step_ms = [t0.elapsed_time(t1) / args.steps] * args.steps
    barrier()
    total_s = sum(step_ms) / 1e3
    max_s = reduce_max(total_s, dev)

    # end to end through the public API with host buffers: one H2D copy of the
    # new query and the new token's K/V rows (packed side by side in one pinned
    # buffer), the decode step that writes those rows into the caches itself
    # (ds_decode_step_kv), and the D2H copy of the output
    esz = 2 if wl.kv_dtype == "bf16" else 4
    nq, nkv = q.numel(), wl.b * wl.hkv * wl.d
    host_in = torch.empty(nq + 2 * nkv, dtype=q.dtype).pin_memory()
    host_in[:nq].copy_(q.reshape(-1).cpu())
    host_in[nq:nq + nkv].copy_(k[:, :, pos].reshape(-1).cpu())
    host_in[nq + nkv:].copy_(v[:, :, pos].reshape(-1).cpu())
    dev_in = torch.empty_like(host_in, device=dev)
    dq = dev_in[:nq].view(q.shape)
    dk = dev_in[nq:nq + nkv].view(wl.b, wl.hkv, wl.d)
    dv = dev_in[nq + nkv:].view(wl.b, wl.hkv, wl.d)
    hout = torch.empty_like(out, device="cpu").pin_memory()

    def e2e_step(i):
        st = states[i % R]
        dev_in.copy_(host_in, non_blocking=True)
        ds.decode_step_kv(dq, dk, dv, st["k"], st["v"], st["lab"], st["idx"], wl.s, wl.topk, lscale=st["sc"],
                          lzero=st["ze"], out=st["out"])
        hout.copy_(st["out"], non_blocking=True)

    e2e_ms = []
    with torch.cuda.stream(stream):
        if timing == "flush":
            for i in range(args.warmup + args.steps):
                flush()
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                e2e_step(i)
                b_.record()
                if i >= args.warmup:
                    e2e_ms.append((a, b_))
        else:
            for i in range(args.warmup):
                e2e_step(i)
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for i in range(args.steps):
                e2e_step(args.warmup + i)
            b_.record()
            e2e_ms.append((a, b_))
    torch.cuda.synchronize()
    e2e_s = sum(a.elapsed_time(b_) for a, b_ in e2e_ms) / 1e3
    e2e_max = reduce_max(e2e_s, dev)
    h2d = host_in.numel() * host_in.element_size()
    d2h = out.numel() * out.element_size()

    # dense baseline on the same cache: our dense kernel and torch SDPA
    dense_ms, sdpa_ms = dense_baselines(wl, q, k, v, out, flush if timing == "flush" else None, stream)
    offload = offload_timing(wl, q, k, v, idx, lab, sc, ze, out, flush, stream) if args.offload else None

    res = dict(step_ms=step_ms, total_s=total_s, max_s=max_s, timing=timing, rotate=R,
               wall_s=wall1 - wall0, e2e_s=e2e_max, h2d=h2d, d2h=d2h, prefill_ms=prefill_ms,
               clocks=sampler.summary(), dense_ms=dense_ms, sdpa_ms=sdpa_ms, offload=offload,
               plan=ds.plan(wl.b, wl.hq, wl.hkv, wl.s, wl.d, wl.c, wl.topk,
                            ds.DS_BF16 if wl.kv_dtype == "bf16" else ds.DS_F32,
                            ds.DS_INT4 if wl.label_dtype == "int4" else
                            (ds.DS_BF16 if wl.kv_dtype == "bf16" else ds.DS_F32)),
               out_esz=out.element_size(), host=(q, k, v, idx, lab, sc, ze))
    return res


class L2Flush:
    """Evicts L2 between timed steps by writing FLUSH_BYTES (> the 126 MB L2).
    'write_read' (default) = a fill kernel over FLUSH_BYTES, then a reduction
    that reads another FLUSH_BYTES: the written lines are written back to HBM
    before the timed region instead of during the step, and L2 is left holding
    only clean lines of the flush buffer. 'copy' = a device-to-device copy of
    FLUSH_BYTES/2; 'fill' = the fill kernel alone (both leave up to an L2 of
    dirty flush data, whose write-back the next step then pays for)."""

    def __init__(self, dev, kind: str):
        import torch
        self.kind = kind
        if kind == "copy":
            self.src = torch.empty(FLUSH_BYTES // 2, dtype=torch.uint8, device=dev)
            self.dst = torch.empty_like(self.src)
        else:
            self.buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
            if kind == "write_read":
                self.rd = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        if self.kind == "copy":
            self.dst.copy_(self.src)
        else:
            self.buf.zero_()
            if self.kind == "write_read":
                self.rd.sum()


def dense_baselines(wl, q, k, v, out, flush, stream, reps=20):
    """Dense decode over the same cache (ds_dense_decode and torch SDPA), in
    ms per call: with `flush`, the median of single calls after an L2 flush;
    without, the mean of back-to-back calls (their K+V exceed the L2)."""
    import torch
    import torch.nn.functional as F

    import channel_token_sparse_b200 as ds

    def timed(fn):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
            ts = []
            if flush is None:
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                for _ in range(reps):
                    fn()
                b_.record()
            else:
                for _ in range(reps):
                    flush()
                    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record()
                    fn()
                    b_.record()
                    ts.append((a, b_))
        torch.cuda.synchronize()
        if flush is None:
            return a.elapsed_time(b_) / reps
        return statistics.median(a.elapsed_time(b_) for a, b_ in ts)

    dense_ms = timed(lambda: ds.dense_decode(q, k, v, wl.s, out=out))
    sdpa_ms = None
    try:
        kk, vv = k[:, :, : wl.s], v[:, :, : wl.s]
        qq = q[:, :, None, :]
        sdpa_ms = timed(lambda: F.scaled_dot_product_attention(qq, kk, vv, enable_gqa=wl.hq != wl.hkv))
    except Exception:  # noqa: BLE001
        pass
    return dense_ms, sdpa_ms


def offload_timing(wl, q, k, v, idx, lab, sc, ze, out, flush, stream, reps=20):
    """Double Sparsity's offloading mode: the same decode step with the K/V
    caches in pinned host memory (label cache, query and output on the GPU),
    the selected rows crossing the host link; and dense decode over the same
    host caches (every row crosses). Medians of `reps` launches (ms)."""
    import torch

    import channel_token_sparse_b200 as ds

    kh, vh = k.cpu().pin_memory(), v.cpu().pin_memory()

    def timed(fn):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
            ts = []
            for _ in range(reps):
                flush()
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b_.record()
                ts.append((a, b_))
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b_) for a, b_ in ts)

    sparse_ms = timed(lambda: ds.decode_step(q, kh, vh, lab, idx, wl.s, wl.topk, lscale=sc, lzero=ze, out=out))
    dense_ms = timed(lambda: ds.dense_decode(q, kh, vh, wl.s, out=out))
    del kh, vh
    return sparse_ms, dense_ms


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ------------------------------------------------------------ CPU oracle

def oracle_sample(wl: synth.Workload, host, budget_s: float, max_rows: int | None = None):
    """Time the CPU oracle on (b, kv head) rows of the same workload until
    `budget_s` seconds have passed (at least one row). Returns (seconds per
    full step, rows timed)."""
    import oracle
    q, k, v, idx, lab, sc, ze = host
    G = wl.g
    rows = [(b, g) for b in range(wl.b) for g in range(wl.hkv)]
    done, t_used = 0, 0.0
    for (b, g) in rows:
        if max_rows is not None and done >= max_rows:
            break
        qr = q[b:b + 1, g * G:(g + 1) * G]
        kr = np.ascontiguousarray(k[b:b + 1, g:g + 1])
        vr = np.ascontiguousarray(v[b:b + 1, g:g + 1])
        ir = np.ascontiguousarray(idx[g:g + 1])
        t0 = time.perf_counter()
        labr = oracle.build_label(kr, wl.kv_dtype, wl.label_dtype, ir, wl.s)  # prefill + append
        oracle.sparse_decode(qr, kr, vr, wl.kv_dtype, labr, wl.label_dtype, ir, wl.s, wl.topk)
        t_used += time.perf_counter() - t0
        done += 1
        if t_used >= budget_s:
            break
    per_row = t_used / done
    return per_row * len(rows), done


def host_arrays(wl, state_tensors):
    import torch
    out = []
    for t in state_tensors:
        if t is None:
            out.append(None)
        elif t.dtype == torch.bfloat16:
            out.append(t.view(torch.int16).cpu().numpy().view(np.uint16))
        elif t.dtype == torch.int16:
            out.append(t.cpu().numpy().view(np.uint16))
        else:
            out.append(t.cpu().numpy())
    return out


def run_reference(args, wl):
    """The oracle as the reference arm: each step is a bounded sample (a
    fixed number of (b, kv head) rows) of the same workload on host cores."""
    import oracle
    oracle.build()
    di = synth.decode_inputs(wl)
    idx = np.ascontiguousarray(synth.outlier_channels(wl)[:, : wl.c], np.int32)
    host = (di.q, di.k, di.v, idx, None, None, None)
    rows_per_step = max(1, min(wl.b * wl.hkv, args.ref_rows))
    for _ in range(args.warmup):
        oracle_sample(wl, host, 0.0, max_rows=rows_per_step)
    t_total = 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle_sample(wl, host, float("inf"), max_rows=rows_per_step)
        t_total += time.perf_counter() - t0
    frac = rows_per_step / (wl.b * wl.hkv)
    value = wl.b * frac * args.steps / t_total
    sample = f"{rows_per_step} of {wl.b * wl.hkv} (batch, kv-head) rows per step"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {**workload_config(wl, None), "l2": "not applicable (CPU oracle)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def workload_config(wl, plan):
    cfg = {"workload": wl.name, "batch": wl.b, "q_heads": wl.hq, "kv_heads": wl.hkv, "head_dim": wl.d,
           "seq_len": wl.s, "heavy_channels": wl.c, "label": wl.label_dtype, "topk": wl.topk,
           "kv_dtype": wl.kv_dtype}
    if plan:
        cfg["cluster_ctas"], cfg["tokens_per_cta"], cfg["smem_bytes"] = plan
    return cfg


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=1, help="workload index (0-4)")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--ref-rows", type=int, default=8, help="rows per reference-arm step")
    ap.add_argument("--label", default=None, choices=["f32", "bf16", "int4"],
                    help="override the workload's label cache dtype (measurement variants)")
    ap.add_argument("--offload", action="store_true",
                    help="also time the step with the K/V caches in pinned host memory")
    ap.add_argument("--timing", default="rotate", choices=["rotate", "flush"],
                    help="rotate: back-to-back steps cycling through enough layer instances that the "
                         "inputs exceed the L2; flush: one step per event pair after an L2 flush")
    ap.add_argument("--flush", default="write_read", choices=["write_read", "copy", "fill"],
                    help="L2 eviction between timed steps: fill then read (default), D2D copy, or fill kernel")
    args = ap.parse_args()
    wl = synth.workload(args.config)
    if args.label and args.label != wl.label_dtype:
        if args.label != "int4" and args.label != wl.kv_dtype:
            raise SystemExit("an fp label cache has the key cache's dtype")
        wl = dataclasses.replace(wl, label_dtype=args.label, name=f"{wl.name}, {args.label} label")
    rank, local_rank, world = dist_env()

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, wl)
        return

    import torch
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        r = run_ours(args, wl, rank, local_rank, world)
        line = None
        if rank == 0:
            line = report(args, wl, r, world)
        barrier()
        if line:
            print(json.dumps(line))
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


def l2_note(args, r) -> str:
    if r["timing"] == "rotate":
        return (f"inputs larger than L2: the {args.steps} timed steps run back to back, cycling through "
                f"{r['rotate']} independent layer instances (own q, K, V, label cache and output) whose "
                f"working sets together exceed twice the L2; one event pair around the K steps")
    return (f"flushed before every timed step: {FLUSH_BYTES >> 20} MiB written by "
            + ("a device-to-device copy" if args.flush == "copy" else "a fill kernel")
            + (f", then {FLUSH_BYTES >> 20} MiB read (flush data written back before the step)"
               if args.flush == "write_read" else ""))


def report(args, wl, r, world):
    ab = algorithmic_bytes(wl, r["out_esz"])
    peaks = measured_peaks()
    value = job_value(wl.b, world, args.steps, r["max_s"])
    dec_avg_s = sum(r["step_ms"]) / len(r["step_ms"]) / 1e3  # the step is one launch of the kernel
    achieved = ab["total"] / dec_avg_s / 1e9
    cpu = None
    if world == 1:
        host = host_arrays(wl, r["host"])
        t_step, rows = oracle_sample(wl, host, args.cpu_budget)
        cpu = {"value": wl.b / t_step, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{rows} of {wl.b * wl.hkv} (batch, kv-head) rows of one step "
                         f"(label build + scores + top-k + attention), scaled to the full step"}
    dense_s = r["dense_ms"] / 1e3
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * r["max_s"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.kv_dtype, "data": "synthetic (seeded N(0,1) "
        "Q/K/V with planted outlier channels)",
        "config": {**workload_config(wl, r["plan"]), "parallelism": f"dp{world} (independent layers per rank)",
                   "l2": l2_note(args, r)},
        "hbm_gbs": achieved, "pct_of_nominal_hbm": 100 * achieved / NOMINAL_HBM_GBS,
        "pct_of_measured_hbm": 100 * achieved / peaks["hbm_gbs"],
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"],
                     "traffic": (recorded_traffic(args.config)
                                 if wl.label_dtype == synth.workload(args.config).label_dtype else None), "kernel": "ds_decode_kernel",
                     "algorithmic_bytes_per_launch": ab["total"], "avg_launch_us": dec_avg_s * 1e6},
        "step_us": dec_avg_s * 1e6,
        "cpu_baseline": cpu,
        "e2e": {"value": job_value(wl.b, world, args.steps, r["e2e_s"]), "unit": UNIT,
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": args.steps,
        "clocks": r["clocks"],
        "dense_baseline": {"ds_dense_decode_us": r["dense_ms"] * 1e3,
                           "torch_sdpa_us": None if r["sdpa_ms"] is None else r["sdpa_ms"] * 1e3,
                           "dense_bytes": ab["dense_total"],
                           "speedup_vs_faster_dense": min(x for x in (r["dense_ms"], r["sdpa_ms"]) if x)
                           / 1e3 / dec_avg_s,
                           "byte_ratio": ab["dense_total"] / ab["total"],
                           "dense_hbm_gbs": ab["dense_total"] / dense_s / 1e9},
        "prefill_label_build": {"us": r["prefill_ms"] * 1e3,
                                "gbs": prefill_bytes(wl) / (r["prefill_ms"] / 1e3) / 1e9},
        "wall_s_timed_region": r["wall_s"],
    }
    if r["offload"]:
        sp_ms, dn_ms = r["offload"]
        esz = 2 if wl.kv_dtype == "bf16" else 4
        link = wl.b * wl.hkv * (2 * min(wl.topk, wl.s) + 1) * wl.d * esz
        line["offload"] = {"kv_in": "pinned host memory", "sparse_step_us": sp_ms * 1e3,
                           "tokens_per_s": wl.b / (sp_ms / 1e3), "host_link_bytes": link,
                           "host_link_gbs": link / (sp_ms / 1e3) / 1e9,
                           "dense_us": dn_ms * 1e3, "dense_host_link_bytes": 2 * wl.b * wl.hkv * wl.s * wl.d * esz,
                           "speedup_vs_dense": dn_ms / sp_ms}
    return line


if __name__ == "__main__":
    main()
