"""Benchmark of the Double Sparsity decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config I] [--also I,J,...]

One step = one decode token for every sequence of a layer, in one launch
(ds_decode_step): the new token's heavy channels are appended to the label
cache, then query gather, approximate scores, top-k and exact attention over
the selected K/V rows. Inputs are seeded synthetic tensors.

The headline workload is the largest single-GPU one: batch 32, 32 MHA heads,
head_dim 128, 16384 cached tokens, a 32-channel 4-bit label cache, top-1024
(873 MB of label, selected K/V and q/out per step). The JSON line nests the
same record for the other workloads under "configs" (Llama-2-7B layer,
Llama-3-8B GQA layer, 256K context).

Timing: the step captured in a CUDA graph, K steps back to back between one
pair of CUDA events on the launching stream, cycling through enough
independent layer instances that the inputs exceed the L2; max over ranks
under torchrun (weak scaling: every rank runs its own layer; no collective on
the data path). Rank 0 prints one JSON line.
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
CHAIN_STEPS = 8  # at least this many consecutive steps per captured graph
KERNEL_SOURCES = ["channel_token_sparse_b200/csrc/ds_decode_kernel.cuh",
                  "channel_token_sparse_b200/csrc/ds_common.cuh",
                  "channel_token_sparse_b200/csrc/ds_decode_bf16_fp.cu",
                  "channel_token_sparse_b200/csrc/ds_decode_bf16_i4.cu",
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

    def __init__(self, device_index: int, period_s: float = 0.0005):
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

def heavy_channels(wl: synth.Workload) -> np.ndarray:
    """idx [Hkv, C] int32: the planted channels, padded (when C is larger)
    with the lowest unplanted ones, ascending."""
    planted = synth.outlier_channels(wl)
    if planted.shape[1] >= wl.c:
        return np.ascontiguousarray(planted[:, : wl.c], np.int32)
    full = []
    for g in range(wl.hkv):
        have = list(planted[g])
        extra = [c for c in range(wl.d) if c not in have][: wl.c - len(have)]
        full.append(sorted(have + extra))
    return np.asarray(full, np.int32)


def build_state(wl: synth.Workload, dev, rank: int):
    import torch

    import channel_token_sparse_b200 as ds
    if wl.s * wl.b * wl.hkv * wl.d <= (1 << 28):
        di = synth.decode_inputs(wl, seed_offset=rank)
        q, k, v = (_dev(x, wl.kv_dtype, dev) for x in (di.q, di.k, di.v))
    else:
        q, k, v = synth.decode_inputs_torch(wl, dev, seed_offset=rank)
    idx = torch.from_numpy(heavy_channels(wl)).to(dev)
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

    # consecutive steps (layer instances in turn) are also captured together,
    # M of them in one graph, as a decode loop launches its layers: the steps
    # then run back to back without a graph launch between each two
    M = R * -(-CHAIN_STEPS // R)
    chain = torch.cuda.CUDAGraph()
    with torch.cuda.graph(chain, stream=stream):
        for j in range(M):
            step_of(states[j % R])()

    def one_step(i, evs=None):
        if timing == "flush":
            flush()  # untimed: evicts L2 (the step's inputs could otherwise stay in the 126 MB L2)
        if evs:
            evs[0].record()
        graphs[i % R].replay()
        if evs:
            evs[1].record()

    def run_steps(start, count):
        """Launch exactly `count` steps, instances start % R, (start + 1) % R, ..."""
        i, end = start, start + count
        while i < end and i % M:
            graphs[i % R].replay()
            i += 1
        while i + M <= end:
            chain.replay()
            i += M
        while i < end:
            graphs[i % R].replay()
            i += 1

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            one_step(i)
        if timing != "flush":
            chain.replay()  # warm the chained graph too
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
                run_steps(args.warmup, args.steps)
                t1.record()
            torch.cuda.synchronize()
            wall1 = time.perf_counter()
        step_ms = [t0.elapsed_time(t1) / args.steps] * args.steps
    barrier()
    total_s = sum(step_ms) / 1e3
    max_s = reduce_max(total_s, dev)

    # end to end through the public API with host buffers: one call per step,
    # ds_decode_step_kv with the new query and the new token's K/V rows in
    # pinned host memory and the output written to pinned host memory; the
    # kernel reads those inputs over the host link, writes the rows into the
    # caches, runs the step and writes the output back over the link
    pin = lambda t: t.contiguous().cpu().pin_memory()
    host_q, host_kn, host_vn = pin(q), pin(k[:, :, pos]), pin(v[:, :, pos])
    hout = torch.empty_like(out, device="cpu").pin_memory()

    # a serving loop prepares the call once per layer (ds.PreparedDecodeStepKV:
    # arguments checked and converted once) and then makes one C-ABI call per step
    with torch.cuda.stream(stream):
        prepared = [ds.PreparedDecodeStepKV(host_q, host_kn, host_vn, st["k"], st["v"], st["lab"], st["idx"],
                                            wl.s, wl.topk, lscale=st["sc"], lzero=st["ze"], out=hout)
                    for st in states]

    def e2e_step(i):
        prepared[i % R]()

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
    h2d = sum(t.numel() * t.element_size() for t in (host_q, host_kn, host_vn))
    d2h = hout.numel() * hout.element_size()

    # dense baseline on the same cache: our dense kernel and torch SDPA
    dense_ms, sdpa_ms = dense_baselines(wl, q, k, v, out, flush if timing == "flush" else None, stream)
    offload = offload_timing(wl, q, k, v, idx, lab, sc, ze, out, flush, stream) if args.offload else None

    res = dict(step_ms=step_ms, total_s=total_s, max_s=max_s, timing=timing, rotate=R, chain=M,
               wall_s=wall1 - wall0, e2e_s=e2e_max, h2d=h2d, d2h=d2h, prefill_ms=prefill_ms,
               clocks=sampler.summary(), dense_ms=dense_ms, sdpa_ms=sdpa_ms, offload=offload,
               plan=ds.plan(wl.b, wl.hq, wl.hkv, wl.s, wl.d, wl.c, wl.topk,
                            ds.DS_BF16 if wl.kv_dtype == "bf16" else ds.DS_F32,
                            ds.DS_INT4 if wl.label_dtype == "int4" else
                            (ds.DS_BF16 if wl.kv_dtype == "bf16" else ds.DS_F32)),
               out_esz=out.element_size(), rows=DeviceRows(wl, q, k, v, idx))
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

class DeviceRows:
    """Host copies of single (b, kv head) rows of the device-resident
    workload, fetched on demand (the multi-GB caches are never copied whole)."""

    def __init__(self, wl, q, k, v, idx):
        self.wl, self.q, self.k, self.v = wl, q, k, v
        self.idx = idx.cpu().numpy()

    @staticmethod
    def _np(t):
        import torch
        t = t.contiguous().cpu()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    def row(self, b, g):
        wl, G = self.wl, self.wl.g
        return (self._np(self.q[b:b + 1, g * G:(g + 1) * G]), self._np(self.k[b:b + 1, g:g + 1, : wl.s]),
                self._np(self.v[b:b + 1, g:g + 1, : wl.s]), np.ascontiguousarray(self.idx[g:g + 1]))


class SynthRows:
    """Rows drawn on the host (the reference arm: no GPU, no full workload)."""

    def __init__(self, wl):
        self.wl = wl
        self.idx = heavy_channels(wl)

    def row(self, b, g):
        q, k, v = synth.decode_row_inputs(self.wl, b, g)
        return q, k, v, np.ascontiguousarray(self.idx[g:g + 1])


def oracle_row(wl, row):
    """One (b, kv head) row of a step on the oracle: label build (prefill and
    append) and the sparse decode."""
    import oracle
    qr, kr, vr, ir = row
    labr = oracle.build_label(kr, wl.kv_dtype, wl.label_dtype, ir, wl.s)
    oracle.sparse_decode(qr, kr, vr, wl.kv_dtype, labr, wl.label_dtype, ir, wl.s, wl.topk)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def _row_list(wl):
    return [(b, g) for b in range(wl.b) for g in range(wl.hkv)]


def oracle_single(wl, rows_src, budget_s: float):
    """The oracle on one thread, rows in order (each fetched untimed) until
    `budget_s` seconds of oracle time. Returns (seconds per full step, rows)."""
    import oracle
    oracle.build()
    t_used, done = 0.0, 0
    rows = _row_list(wl)
    for (b, g) in rows:
        row = rows_src.row(b, g)
        t0 = time.perf_counter()
        oracle_row(wl, row)
        t_used += time.perf_counter() - t0
        done += 1
        if t_used >= budget_s:
            break
    return t_used / done * len(rows), done


def oracle_parallel(wl, rows_src, budget_s: float, threads: int, max_bytes: int = 2 << 30):
    """The oracle on `threads` host threads at once (ctypes releases the GIL
    while the C code runs). M rows are fetched first (untimed; at most
    2 * threads and at most `max_bytes` of host copies), then the threads
    take rows 0, 1, ..., M-1, 0, ... until `budget_s` seconds of wall time.
    Returns (seconds per full step, rows timed, threads used)."""
    import concurrent.futures as cf
    import itertools
    import oracle
    oracle.build()
    oracle._load()  # load once before the threads start
    esz = 4 if wl.kv_dtype == "f32" else 2
    row_bytes = 2 * wl.s * wl.d * esz
    rows = _row_list(wl)
    m = max(1, min(len(rows), 2 * threads, max_bytes // row_bytes))
    data = [rows_src.row(b, g) for (b, g) in rows[:m]]
    used = min(threads, m)
    counter = itertools.count()
    t_start = time.perf_counter()
    deadline = t_start + budget_s

    def worker():
        n = 0
        while True:
            i = next(counter)
            if n > 0 and time.perf_counter() >= deadline:
                return n
            if i >= m and time.perf_counter() >= deadline:
                return n
            oracle_row(wl, data[i % m])
            n += 1

    with cf.ThreadPoolExecutor(max_workers=used) as ex:
        done = sum(f.result() for f in [ex.submit(worker) for _ in range(used)])
    wall = time.perf_counter() - t_start
    return wall / done * len(rows), done, used


def cpu_baseline(wl, rows_src, budget_s: float) -> dict:
    """The oracle timed on this host: all host threads, and one thread."""
    threads = os.cpu_count() or 1
    tn, rowsn, used = oracle_parallel(wl, rows_src, budget_s, threads)
    t1, rows1 = oracle_single(wl, rows_src, budget_s)
    nrows = wl.b * wl.hkv
    return {"value": wl.b / tn, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"{rowsn} (batch, kv-head) rows of one step (label build + scores + top-k + "
                      f"attention; {nrows} rows per step) on {used} threads for about {budget_s:g} s, "
                      f"scaled to the full step",
            "cpu_model": cpu_model(), "host_threads": threads,
            "single_thread": {"value": wl.b / t1, "unit": UNIT, "cores": 1,
                              "sample": f"{rows1} of {nrows} rows on 1 thread, scaled to the full step"}}


def run_reference(args, wl):
    """The oracle as the reference arm: each step is a bounded sample (one
    (b, kv head) row per host thread, drawn on the host once) of the same
    workload, processed by all host threads at once."""
    import concurrent.futures as cf
    import oracle
    oracle.build()
    oracle._load()
    threads = os.cpu_count() or 1
    src = SynthRows(wl)
    rows = _row_list(wl)
    esz = 4 if wl.kv_dtype == "f32" else 2
    cap = max(1, (2 << 30) // (2 * wl.s * wl.d * esz))
    per_step = max(1, min(len(rows), threads, cap, args.ref_rows or len(rows)))
    data = [src.row(b, g) for (b, g) in rows[:per_step]]
    used = min(threads, per_step)

    def one_step(ex):
        list(ex.map(lambda r: oracle_row(wl, r), data))

    with cf.ThreadPoolExecutor(max_workers=used) as ex:
        for _ in range(args.warmup):
            one_step(ex)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            one_step(ex)
        t_total = time.perf_counter() - t0
    frac = per_step / len(rows)
    value = wl.b * frac * args.steps / t_total
    sample = (f"{per_step} of {len(rows)} (batch, kv-head) rows per step (label build + scores + top-k + "
              f"attention), one per thread")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {**workload_config(wl, None), "l2": "not applicable (CPU oracle)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle", "sample": sample,
                             "cpu_model": cpu_model()},
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

DEFAULT_CONFIG = 2          # the largest single-GPU workload is the headline
DEFAULT_ALSO = (1, 3, 4)    # nested records


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=None,
                    help=f"headline workload index (0-4; default {DEFAULT_CONFIG})")
    ap.add_argument("--also", default=None,
                    help="comma-separated workload indices measured after the headline and nested under "
                         "'configs' (default: the other full-size workloads; '' for none)")
    ap.add_argument("--cpu-budget", type=float, default=8.0,
                    help="seconds of oracle time per cpu_baseline leg (headline; nested records use half)")
    ap.add_argument("--ref-rows", type=int, default=0,
                    help="rows per reference-arm step (0: one per host thread)")
    ap.add_argument("--label", default=None, choices=["f32", "bf16", "int4"],
                    help="override the headline workload's label cache dtype (measurement variants)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the headline workload's batch (smaller cases for profiling)")
    ap.add_argument("--offload", action="store_true",
                    help="also time the step with the K/V caches in pinned host memory")
    ap.add_argument("--timing", default="rotate", choices=["rotate", "flush"],
                    help="rotate: back-to-back steps cycling through enough layer instances that the "
                         "inputs exceed the L2; flush: one step per event pair after an L2 flush")
    ap.add_argument("--flush", default="write_read", choices=["write_read", "copy", "fill"],
                    help="L2 eviction between timed steps: fill then read (default), D2D copy, or fill kernel")
    args = ap.parse_args()
    head = DEFAULT_CONFIG if args.config is None else args.config
    if args.also is None:
        also = [i for i in DEFAULT_ALSO if i != head] if args.config is None else []
    else:
        also = [int(x) for x in args.also.split(",") if x.strip()]
    wl = synth.workload(head)
    if args.label and args.label != wl.label_dtype:
        if args.label != "int4" and args.label != wl.kv_dtype:
            raise SystemExit("an fp label cache has the key cache's dtype")
        wl = dataclasses.replace(wl, label_dtype=args.label, name=f"{wl.name}, {args.label} label")
    if args.batch and args.batch != wl.b:
        wl = dataclasses.replace(wl, b=args.batch, name=wl.name.replace(f"b{wl.b} ", f"b{args.batch} ", 1))
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
        line = report(args, wl, r, world, head, args.cpu_budget) if rank == 0 else None
        del r
        torch.cuda.empty_cache()
        nested = {}
        for i in also:
            wl_i = synth.workload(i)
            r_i = run_ours(args, wl_i, rank, local_rank, world)
            if rank == 0:
                rec = report(args, wl_i, r_i, world, i, args.cpu_budget / 2)
                nested[wl_i.name] = {k: rec[k] for k in NESTED_KEYS if k in rec}
            del r_i
            torch.cuda.empty_cache()
        barrier()
        if line:
            if nested:
                line["configs"] = nested
            print(json.dumps(line))
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


NESTED_KEYS = ("value", "unit", "ms_per_step", "steps", "config", "hbm_gbs", "roofline", "step_us",
               "cpu_baseline", "e2e", "gpu_launches", "clocks", "dense_baseline", "prefill_label_build",
               "offload")


def l2_note(args, r) -> str:
    if r["timing"] == "rotate":
        return (f"inputs larger than L2: the {args.steps} timed steps run back to back, cycling through "
                f"{r['rotate']} independent layer instances (own q, K, V, label cache and output) whose "
                f"working sets together exceed twice the L2, launched as CUDA graphs of {r['chain']} "
                f"consecutive steps; one event pair around the K steps")
    return (f"flushed before every timed step: {FLUSH_BYTES >> 20} MiB written by "
            + ("a device-to-device copy" if args.flush == "copy" else "a fill kernel")
            + (f", then {FLUSH_BYTES >> 20} MiB read (flush data written back before the step)"
               if args.flush == "write_read" else ""))


def report(args, wl, r, world, index, cpu_budget):
    ab = algorithmic_bytes(wl, r["out_esz"])
    peaks = measured_peaks()
    value = job_value(wl.b, world, args.steps, r["max_s"])
    dec_avg_s = sum(r["step_ms"]) / len(r["step_ms"]) / 1e3  # the step is one launch of the kernel
    achieved = ab["total"] / dec_avg_s / 1e9
    cpu = cpu_baseline(wl, r["rows"], cpu_budget) if world == 1 else None
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
                     "traffic": (recorded_traffic(index)
                                 if wl.label_dtype == synth.workload(index).label_dtype else None),
                     "kernel": "ds_decode_kernel",
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
        "prefill_label_build": {"us": r["prefill_ms"] * 1e3, "bytes": prefill_bytes(wl),
                                "gbs": prefill_bytes(wl) / (r["prefill_ms"] / 1e3) / 1e9,
                                "frac": prefill_bytes(wl) / (r["prefill_ms"] / 1e3) / 1e9 / peaks["hbm_gbs"]},
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
