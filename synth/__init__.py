"""Seeded synthetic inputs for Double Sparsity decode attention.

This module only draws random tensors and lays them out; it holds none of the
method's arithmetic (no scores, no selection, no attention, no quantisation).
Both the CUDA path and the CPU oracle are fed from it, so that they see the same
bytes.

Recipe (the pages describe Llama-2-7B / Llama-3-8B / Qwen-shaped layers whose
keys carry a few large "outlier" channels per head; no weights or datasets are
available, so these shapes stand in for them):

* Q, K, V ~ N(0, 1), drawn in float32 from numpy's PCG64 generator seeded with
  ``1000 * config_index + tensor_id``.
* Per kv head ``g`` a set of ``n_outlier`` distinct channels is drawn (seeded);
  those channels are multiplied by ``outlier_scale`` in K and in every query
  head of the group. V is left plain.
* The float32 draws are rounded to bfloat16 (round to nearest even) when the
  workload is bf16; bf16 tensors are stored as ``uint16`` bit patterns.

Layouts: ``q [B, Hq, D]``, ``k, v [B, Hkv, S_cap, D]`` (rows past ``S`` are
zero), calibration windows ``q_win [N, Hq, W, D]`` and keys ``k [N, Hkv, S, D]``.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# tensor ids mixed into the seed
_T_Q, _T_K, _T_V, _T_OUT, _T_QWIN, _T_KCAL, _T_QNEW, _T_KNEW, _T_VNEW = range(1, 10)


@dataclass(frozen=True)
class Workload:
    """One decode-attention workload: shapes, dtypes and sparsity settings."""

    name: str
    index: int          # seed base: 1000 * index
    b: int
    hq: int
    hkv: int
    d: int
    s: int
    c: int              # heavy channels per kv head
    topk: int
    kv_dtype: str       # "f32" | "bf16"
    label_dtype: str    # "f32" | "bf16" | "int4"
    n_outlier: int
    outlier_scale: float
    calib_samples: int = 1
    calib_w: int = 32
    calib_s: int = 0    # 0 -> min(s, 4096)
    extra: dict = field(default_factory=dict)

    @property
    def g(self) -> int:
        return self.hq // self.hkv

    @property
    def rows(self) -> int:
        return self.b * self.hkv


# The five workloads. Sizes follow the decode configurations the pages study:
# a tiny fp32 case, a Llama-2-7B-shaped MHA layer, a 32-channel 4-bit label
# cache at 1/16 token sparsity, a Llama-3-8B-shaped GQA layer and a 256K context.
WORKLOADS = [
    Workload("tiny-fp32 b1 h2 d64 s512 c8 k32", 0, 1, 2, 2, 64, 512, 8, 32,
             "f32", "f32", 8, 8.0, calib_samples=4, calib_w=32, calib_s=512),
    Workload("llama2-7b mha b8 h32 d128 s4096 c16 k256", 1, 8, 32, 32, 128, 4096, 16, 256,
             "bf16", "bf16", 16, 6.0),
    Workload("mha b32 h32 d128 s16384 c32-int4 k1024", 2, 32, 32, 32, 128, 16384, 32, 1024,
             "bf16", "int4", 16, 6.0),
    Workload("llama3-8b gqa b4 hq32 hkv8 d128 s32768 c16 k2048", 3, 4, 32, 8, 128, 32768, 16, 2048,
             "bf16", "bf16", 16, 6.0),
    Workload("long-context b1 h32 d128 s262144 c16 k16384", 4, 1, 32, 32, 128, 262144, 16, 16384,
             "bf16", "bf16", 16, 6.0),
]


def workload(i: int) -> Workload:
    return WORKLOADS[i]


def custom(name: str = "custom", index: int = 90, **kw) -> Workload:
    """A workload with explicit sizes (parity and edge-case tests)."""
    base = dict(b=1, hq=2, hkv=2, d=64, s=512, c=8, topk=32, kv_dtype="f32",
                label_dtype="f32", n_outlier=8, outlier_scale=8.0)
    base.update(kw)
    return Workload(name, index, **base)


# ---------------------------------------------------------------- primitives

def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal(shape, seed: int) -> np.ndarray:
    return rng(seed).standard_normal(size=shape, dtype=np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16, nearest-even, returning the uint16 bit pattern.
    Inputs are finite draws (no NaN handling needed)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return f32_to_bf16_bits(x)
    raise ValueError(dtype)


def storage_to_f32(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return x.astype(np.float32)
    if dtype == "bf16":
        return bf16_bits_to_f32(x)
    raise ValueError(dtype)


def outlier_channels(wl: Workload) -> np.ndarray:
    """[Hkv, n_outlier] int32, sorted ascending, distinct within a head."""
    r = rng(1000 * wl.index + _T_OUT)
    out = np.empty((wl.hkv, wl.n_outlier), dtype=np.int32)
    for g in range(wl.hkv):
        out[g] = np.sort(r.choice(wl.d, size=wl.n_outlier, replace=False))
    return out


def _plant_kv(x: np.ndarray, chans: np.ndarray, scale: float) -> None:
    """x [..., Hkv, T, D] in place: scale each kv head's outlier channels."""
    for g in range(chans.shape[0]):
        x[..., g, :, chans[g]] *= np.float32(scale)


def _plant_q(x: np.ndarray, chans: np.ndarray, scale: float, group: int) -> None:
    """x [..., Hq, (T,) D] in place: scale the outlier channels of q heads h in group h // G."""
    for h in range(x.shape[-2] if x.ndim == 3 else x.shape[-3]):
        g = h // group
        if x.ndim == 3:
            x[:, h, chans[g]] *= np.float32(scale)
        else:
            x[..., h, :, chans[g]] *= np.float32(scale)


@dataclass
class DecodeInputs:
    wl: Workload
    s_cap: int
    q: np.ndarray       # [B, Hq, D] storage
    k: np.ndarray       # [B, Hkv, S_cap, D] storage
    v: np.ndarray       # [B, Hkv, S_cap, D] storage
    outliers: np.ndarray


def decode_inputs(wl: Workload, s_cap: int | None = None, seed_offset: int = 0) -> DecodeInputs:
    """Q, K, V for one decode step over a cache holding ``wl.s`` tokens."""
    s_cap = wl.s if s_cap is None else s_cap
    base = 1000 * wl.index + 100 * seed_offset
    chans = outlier_channels(wl)
    q = normal((wl.b, wl.hq, wl.d), base + _T_Q)
    _plant_q(q, chans, wl.outlier_scale, wl.g)
    kshape = (wl.b, wl.hkv, s_cap, wl.d)
    k = np.zeros(kshape, dtype=np.float32)
    v = np.zeros(kshape, dtype=np.float32)
    k[:, :, : wl.s] = normal((wl.b, wl.hkv, wl.s, wl.d), base + _T_K)
    v[:, :, : wl.s] = normal((wl.b, wl.hkv, wl.s, wl.d), base + _T_V)
    _plant_kv(k, chans, wl.outlier_scale)
    return DecodeInputs(wl, s_cap, to_storage(q, wl.kv_dtype), to_storage(k, wl.kv_dtype),
                        to_storage(v, wl.kv_dtype), chans)


def new_token(wl: Workload, step: int = 0):
    """K and V rows [B, Hkv, D] and a query [B, Hq, D] for one appended decode token."""
    chans = outlier_channels(wl)
    base = 1000 * wl.index + 7 * step
    kn = normal((wl.b, wl.hkv, 1, wl.d), base + _T_KNEW)
    vn = normal((wl.b, wl.hkv, 1, wl.d), base + _T_VNEW)
    qn = normal((wl.b, wl.hq, wl.d), base + _T_QNEW)
    _plant_kv(kn, chans, wl.outlier_scale)
    _plant_q(qn, chans, wl.outlier_scale, wl.g)
    return (to_storage(kn[:, :, 0], wl.kv_dtype), to_storage(vn[:, :, 0], wl.kv_dtype),
            to_storage(qn, wl.kv_dtype))


def decode_row_inputs(wl: Workload, b: int, g: int, seed_offset: int = 0):
    """The query heads of kv head g ([1, G, D]) and that head's K and V
    ([1, 1, S, D]) for batch entry b, drawn on the host with the recipe of
    :func:`decode_inputs` (N(0, 1), the planted channels scaled in K and q)
    from a seed of their own: one row of a workload too large to draw whole."""
    chans = outlier_channels(wl)[g:g + 1]
    base = 1000 * wl.index + 100 * seed_offset + 10_000_000 + 4 * (b * wl.hkv + g)
    q = normal((1, wl.g, wl.d), base + 0)
    q[:, :, chans[0]] *= np.float32(wl.outlier_scale)
    k = normal((1, 1, wl.s, wl.d), base + 1)
    v = normal((1, 1, wl.s, wl.d), base + 2)
    _plant_kv(k, chans, wl.outlier_scale)
    return to_storage(q, wl.kv_dtype), to_storage(k, wl.kv_dtype), to_storage(v, wl.kv_dtype)


@dataclass
class CalibInputs:
    wl: Workload
    q_win: np.ndarray   # [N, Hq, W, D] storage
    k: np.ndarray       # [N, Hkv, S, D] storage
    outliers: np.ndarray


def calib_inputs(wl: Workload) -> CalibInputs:
    """Calibration samples: observation-window queries and full keys, with the
    same planted outlier channels as the decode inputs (the static-channel
    premise)."""
    chans = outlier_channels(wl)
    n = wl.calib_samples
    s = wl.calib_s if wl.calib_s else min(wl.s, 4096)
    qw = normal((n, wl.hq, wl.calib_w, wl.d), 1000 * wl.index + _T_QWIN)
    kc = normal((n, wl.hkv, s, wl.d), 1000 * wl.index + _T_KCAL)
    _plant_q(qw, chans, wl.outlier_scale, wl.g)
    _plant_kv(kc, chans, wl.outlier_scale)
    return CalibInputs(wl, to_storage(qw, wl.kv_dtype), to_storage(kc, wl.kv_dtype), chans)


# ------------------------------------------------------------ device inputs

def decode_inputs_torch(wl: Workload, device, s_cap: int | None = None, seed_offset: int = 0):
    """Same recipe as :func:`decode_inputs`, drawn on ``device`` with torch's
    seeded generator (for the multi-GB workloads, where drawing on the host is
    slow). Returns torch tensors (q, k, v) in the workload's dtype; rows past
    ``wl.s`` are zero. The oracle gets host copies of the rows it checks."""
    import torch

    s_cap = wl.s if s_cap is None else s_cap
    dt = torch.float32 if wl.kv_dtype == "f32" else torch.bfloat16
    gen = torch.Generator(device=device)
    gen.manual_seed(1000 * wl.index + 100 * seed_offset + 50)
    chans = torch.from_numpy(outlier_channels(wl)).to(device=device, dtype=torch.long)
    scale = torch.ones((wl.hkv, wl.d), device=device)
    scale.scatter_(1, chans, wl.outlier_scale)
    q = torch.randn((wl.b, wl.hq, wl.d), generator=gen, device=device)
    q *= scale.repeat_interleave(wl.g, 0)[None]
    k = torch.zeros((wl.b, wl.hkv, s_cap, wl.d), dtype=dt, device=device)
    v = torch.zeros((wl.b, wl.hkv, s_cap, wl.d), dtype=dt, device=device)
    for bb in range(wl.b):  # one batch entry at a time bounds the fp32 temporaries
        kk = torch.randn((wl.hkv, wl.s, wl.d), generator=gen, device=device)
        kk *= scale[:, None, :]
        k[bb, :, : wl.s] = kk.to(dt)
        v[bb, :, : wl.s] = torch.randn((wl.hkv, wl.s, wl.d), generator=gen, device=device).to(dt)
        del kk
    return q.to(dt), k, v
