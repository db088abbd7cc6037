"""B200-native Double Sparsity decode attention.

Thin ctypes binding over ``libds.so`` (C ABI declared in ``include/ds.h``).
This module only marshals arguments: every step runs in the library's CUDA
kernels. PyTorch supplies device memory and the current stream.

There is no fallback: importing works without a GPU (so the ABI can be
inspected), but calling an entry point needs ``libds.so`` (``build()``) and a
CUDA device, and raises otherwise.

Layouts (see include/ds.h): q [B, Hq, D]; k, v [B, Hkv, S_cap, D];
idx [Hkv, C] int32; label [B, Hkv, S_cap, C] (dtype of k) or, 4-bit,
[B, Hkv, S_cap, C/2] uint8 with fp16 lscale / lzero [B, Hkv, S_cap].
"""

from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libds.so")

DS_OK, DS_ERR_INVALID_ARG, DS_ERR_UNSUPPORTED, DS_ERR_CUDA, DS_ERR_WORKSPACE, DS_ERR_TIMEOUT = range(6)
DS_F32, DS_BF16, DS_F16, DS_INT4 = range(4)
DS_FALLBACK_PER_ENTRY, DS_FALLBACK_BATCH = range(2)
DS_CRIT_LEANK_RATIO, DS_CRIT_Q_OUTLIER, DS_CRIT_K_OUTLIER, DS_CRIT_QK_OUTLIER, DS_CRIT_QK_CHUNKED = range(5)

# every C-ABI entry point: name -> (restype, argtypes)
_vp, _i, _f, _sz = C.c_void_p, C.c_int, C.c_float, C.c_size_t
SIGNATURES = {
    "ds_status_string": (C.c_char_p, [_i]),
    "ds_last_error": (C.c_char_p, []),
    "ds_calibrate_workspace_size": (_i, [_i, _i, _i, _i, _i, _i, C.POINTER(_sz)]),
    "ds_calibrate_channels": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]),
    "ds_calibrate_channels_noalloc": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp]),
    "ds_decode_step_kv": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                               _i, _f, _vp, _i, _vp, _vp, _vp]),
    "ds_build_label_cache_paged": (_i, [_vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _i, _vp,
                                        _vp, _vp]),
    "ds_decode_step_paged": (_i, [_vp, _vp, _vp, _i, _vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _vp, _i, _i, _i,
                                  _i, _i, _i, _i, _i, _i, _i, _f, _vp, _i, _vp, _vp, _vp]),
    "ds_calibrate_channels_criterion": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp, _vp,
                                             _vp, _sz, _vp]),
    "ds_build_label_cache": (_i, [_vp, _i, _vp, _i, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp, _vp]),
    "ds_append_label": (_i, [_vp, _i, _vp, _i, _i, _i, _i, _i, _i, _vp, _i, _vp, _vp, _vp]),
    "ds_sparse_decode": (_i, [_vp, _vp, _vp, _i, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                              _f, _vp, _i, _vp, _vp, _vp]),
    "ds_decode_step": (_i, [_vp, _vp, _vp, _i, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i,
                            _f, _vp, _i, _vp, _vp, _vp]),
    "ds_decode_step_varlen": (_i, [_vp, _vp, _vp, _i, _vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i,
                                   _i, _i, _i, _f, _vp, _i, _vp, _vp, _vp]),
    "ds_sparse_decode_plan": (_i, [_i, _i, _i, _i, _i, _i, _i, _i, _i, C.POINTER(_i), C.POINTER(_i),
                                   C.POINTER(_i)]),
    "ds_sparse_decode_set_cluster": (None, [_i]),
    "ds_sparse_decode_tune": (_i, [C.c_char_p, _i]),
    "ds_check_device": (_i, [_vp]),
    "ds_selftest_bounded_wait": (_i, [_i, _vp]),
    "ds_sparse_decode_workspace": (_i, [_i, _i, _i, _i, _i, _i, _i, C.POINTER(_sz)]),
    "ds_dense_decode": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _vp, _i, _vp]),
}

_lib = None


class DSError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{status_string(status) if _lib else status}: {msg}")
        self.status = status


def build(force: bool = False) -> str:
    """Compile libds.so for sm_100a (nvcc) if it is missing or stale."""
    from . import buildlib as _b
    return _b.build(force=force)


def lib():
    """The loaded libds.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run channel_token_sparse_b200.build() first")
        _lib = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(_lib, name)
            fn.restype = res
            fn.argtypes = args
    return _lib


def status_string(st: int) -> str:
    return lib().ds_status_string(st).decode()


def last_error() -> str:
    return lib().ds_last_error().decode()


def _check(st: int):
    if st != DS_OK:
        raise DSError(st, last_error())


# ------------------------------------------------------------------ helpers

def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


_mapped = {}  # host address of a pinned tensor -> its device-mapped address


def _ptr_kv(t):
    """Device address of a tensor the kernels may read (or write) over the
    host link: a CUDA tensor, or a pinned host tensor mapped into the
    device's address space (DS-Offload keeps K/V there; a decode step may also
    take its new rows and query from there and write its output there)."""
    if t is None:
        return None
    if t.is_cuda:
        return C.c_void_p(t.data_ptr())
    if not t.is_pinned():
        raise ValueError("a tensor in host memory must be pinned")
    hp = t.data_ptr()
    dp = _mapped.get(hp)
    if dp is None:
        from cuda.bindings import runtime as rt
        err, dp = rt.cudaHostGetDevicePointer(hp, 0)
        if err != rt.cudaError_t.cudaSuccess:
            raise ValueError(f"pinned host tensor is not mapped for the device: {err}")
        dp = int(dp)
        if len(_mapped) > 4096:
            _mapped.clear()
        _mapped[hp] = dp
    return C.c_void_p(dp)


def _need_cuda_or_pinned(*ts):
    for t in ts:
        if not (t.is_cuda or t.is_pinned()):
            raise ValueError("key/value caches must be CUDA tensors or pinned host tensors")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _stream(stream=None):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return C.c_void_p(s.cuda_stream)


def _kv_dtype(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return DS_F32
    if t.dtype == torch.bfloat16:
        return DS_BF16
    raise TypeError(f"unsupported k/v dtype {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must be CUDA tensors")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def set_cluster(n: int) -> None:
    """Force CTAs per (b, kv head) cluster (1..16, power of two); 0 = automatic."""
    lib().ds_sparse_decode_set_cluster(int(n))


def check_device(stream=None) -> None:
    """Raise DSError(DS_ERR_TIMEOUT) if a kernel gave up a bounded wait since
    the last check (synchronises the stream)."""
    _check(lib().ds_check_device(_stream(stream)))


def tune(name: str, value: int) -> None:
    """Set a decode tuning knob ("scan_prefetch", "i4_ring");
    a negative value restores its default."""
    _check(lib().ds_sparse_decode_tune(name.encode(), int(value)))


def plan(b, hq, hkv, s, d, c, topk, kv_dtype=DS_BF16, label_dtype=DS_BF16):
    """(cluster size, tokens per CTA, shared memory bytes) of ds_sparse_decode."""
    n, ch, sm = C.c_int(), C.c_int(), C.c_int()
    _check(lib().ds_sparse_decode_plan(b, hq, hkv, s, d, c, topk, kv_dtype, label_dtype,
                                       C.byref(n), C.byref(ch), C.byref(sm)))
    return n.value, ch.value, sm.value


def sparse_decode_workspace(b, hq, hkv, s, d, c, topk) -> int:
    """Device scratch bytes ds_sparse_decode needs for a shape (0: on chip)."""
    out = C.c_size_t()
    _check(lib().ds_sparse_decode_workspace(b, hq, hkv, s, d, c, topk, C.byref(out)))
    return out.value


# -------------------------------------------------------------- entry points

def calibrate_workspace_size(n, hq, hkv, w, s, d) -> int:
    out = C.c_size_t()
    _check(lib().ds_calibrate_workspace_size(n, hq, hkv, w, s, d, C.byref(out)))
    return out.value


def calibrate_channels(q_win, k, c: int, ratio_out=None, idx_out=None, ws=None, stream=None):
    """Heavy channels idx [Hkv, C] (and ratio r [Hkv, D]) from q_win [N, Hq, W, D],
    k [N, Hkv, S, D]. Returns (idx, ratio)."""
    torch = _torch()
    _need_cuda(q_win, k)
    n, hq, w, d = q_win.shape
    _, hkv, s, _ = k.shape
    if idx_out is None:
        idx_out = torch.empty((hkv, c), dtype=torch.int32, device=k.device)
    if ratio_out is None:
        ratio_out = torch.empty((hkv, d), dtype=torch.float32, device=k.device)
    nbytes = calibrate_workspace_size(n, hq, hkv, w, s, d)
    if ws is None:
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=k.device)
    _check(lib().ds_calibrate_channels(_ptr(q_win), _ptr(k), _kv_dtype(k), n, hq, hkv, w, s, d, c,
                                       _ptr(ratio_out), _ptr(idx_out), _ptr(ws), ws.numel(),
                                       _stream(stream)))
    return idx_out, ratio_out


def calibrate_channels_criterion(q_win, k, c: int, criterion: int, chunk: int = 0, score_out=None,
                                 idx_out=None, ws=None, stream=None):
    """Heavy channels ranked by one of the DS_CRIT_* criteria. Returns (idx, score)."""
    torch = _torch()
    _need_cuda(q_win, k)
    n, hq, w, d = q_win.shape
    _, hkv, s, _ = k.shape
    if idx_out is None:
        idx_out = torch.empty((hkv, c), dtype=torch.int32, device=k.device)
    if score_out is None:
        score_out = torch.empty((hkv, d), dtype=torch.float32, device=k.device)
    nbytes = calibrate_workspace_size(n, hq, hkv, w, s, d)
    if ws is None:
        ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=k.device)
    _check(lib().ds_calibrate_channels_criterion(_ptr(q_win), _ptr(k), _kv_dtype(k), n, hq, hkv, w, s, d,
                                                 c, int(criterion), int(chunk), _ptr(score_out),
                                                 _ptr(idx_out), _ptr(ws), ws.numel(), _stream(stream)))
    return idx_out, score_out


def calibrate_channels_noalloc(q_win, k, c: int, ratio_out, idx_out, stream=None):
    """ds_calibrate_channels with the library's fixed scratch instead of a
    workspace (for callers that cannot allocate device memory); the outputs
    must be provided."""
    _need_cuda(q_win, k, ratio_out, idx_out)
    n, hq, w, d = q_win.shape
    _, hkv, s, _ = k.shape
    _check(lib().ds_calibrate_channels_noalloc(_ptr(q_win), _ptr(k), _kv_dtype(k), n, hq, hkv, w, s, d, c,
                                               _ptr(ratio_out), _ptr(idx_out), _stream(stream)))
    return idx_out, ratio_out


def _label_args(label, lscale, lzero, kdt):
    torch = _torch()
    if label.dtype == torch.uint8:
        if lscale is None or lzero is None:
            raise ValueError("4-bit label needs lscale and lzero")
        return DS_INT4
    return kdt


def build_label_cache(k, idx, s: int, label, lscale=None, lzero=None, stream=None):
    """Fill label rows [0, s) from the key cache k [B, Hkv, S_cap, D] (device,
    or pinned host memory)."""
    _need_cuda_or_pinned(k)
    _need_cuda(idx, label, lscale, lzero)
    b, hkv, s_cap, d = k.shape
    c = idx.shape[1]
    kdt = _kv_dtype(k)
    _check(lib().ds_build_label_cache(_ptr_kv(k), kdt, _ptr(idx), b, hkv, s, s_cap, d, c, _ptr(label),
                                      _label_args(label, lscale, lzero, kdt), _ptr(lscale),
                                      _ptr(lzero), _stream(stream)))


def append_label(k, idx, pos: int, label, lscale=None, lzero=None, stream=None):
    """Fill label row `pos` from k[:, :, pos]."""
    _need_cuda_or_pinned(k)
    _need_cuda(idx, label, lscale, lzero)
    b, hkv, s_cap, d = k.shape
    c = idx.shape[1]
    kdt = _kv_dtype(k)
    _check(lib().ds_append_label(_ptr_kv(k), kdt, _ptr(idx), b, hkv, pos, s_cap, d, c, _ptr(label),
                                 _label_args(label, lscale, lzero, kdt), _ptr(lscale), _ptr(lzero),
                                 _stream(stream)))


def new_label_cache(k, c: int, int4: bool = False):
    """Allocate (uninitialised) label storage matching a key cache (torch)."""
    torch = _torch()
    b, hkv, s_cap, d = k.shape
    if int4:
        return (torch.empty((b, hkv, s_cap, c // 2), dtype=torch.uint8, device=k.device),
                torch.empty((b, hkv, s_cap), dtype=torch.int16, device=k.device),
                torch.empty((b, hkv, s_cap), dtype=torch.int16, device=k.device))
    return torch.empty((b, hkv, s_cap, c), dtype=k.dtype, device=k.device), None, None


def sparse_decode(q, k, v, label, idx, s: int, topk: int, lscale=None, lzero=None, out=None,
                  out_dtype=None, sm_scale: float = 0.0, sel_out=None, score_out=None, stream=None):
    """One Double Sparsity decode step; returns out [B, Hq, D]."""
    torch = _torch()
    _need_cuda_or_pinned(k, v)
    _need_cuda(q, label, idx, lscale, lzero, out, sel_out, score_out)
    b, hq, d = q.shape
    _, hkv, s_cap, _ = k.shape
    c = idx.shape[1]
    kdt = _kv_dtype(k)
    if out is None:
        out = torch.empty((b, hq, d), dtype=out_dtype or torch.float32, device=q.device)
    odt = DS_F32 if out.dtype == torch.float32 else DS_BF16
    _check(lib().ds_sparse_decode(_ptr(q), _ptr_kv(k), _ptr_kv(v), kdt, _ptr(label),
                                  _label_args(label, lscale, lzero, kdt), _ptr(lscale), _ptr(lzero),
                                  _ptr(idx), b, hq, hkv, s, s_cap, d, c, topk, float(sm_scale),
                                  _ptr(out), odt, _ptr(sel_out), _ptr(score_out), _stream(stream)))
    return out


def decode_step(q, k, v, label, idx, s: int, topk: int, lscale=None, lzero=None, out=None,
                out_dtype=None, sm_scale: float = 0.0, sel_out=None, score_out=None, stream=None):
    """append_label(pos = s - 1) followed by sparse_decode, in one launch;
    returns out [B, Hq, D]."""
    torch = _torch()
    _need_cuda_or_pinned(k, v)
    _need_cuda(q, label, idx, lscale, lzero, out, sel_out, score_out)
    b, hq, d = q.shape
    _, hkv, s_cap, _ = k.shape
    c = idx.shape[1]
    kdt = _kv_dtype(k)
    if out is None:
        out = torch.empty((b, hq, d), dtype=out_dtype or torch.float32, device=q.device)
    odt = DS_F32 if out.dtype == torch.float32 else DS_BF16
    _check(lib().ds_decode_step(_ptr(q), _ptr_kv(k), _ptr_kv(v), kdt, _ptr(label),
                                _label_args(label, lscale, lzero, kdt), _ptr(lscale), _ptr(lzero),
                                _ptr(idx), b, hq, hkv, s, s_cap, d, c, topk, float(sm_scale),
                                _ptr(out), odt, _ptr(sel_out), _ptr(score_out), _stream(stream)))
    return out


def decode_step_kv(q, k_new, v_new, k, v, label, idx, s: int, topk: int, lscale=None, lzero=None, out=None,
                   out_dtype=None, sm_scale: float = 0.0, sel_out=None, score_out=None, stream=None):
    """decode_step that first writes the new token's rows k_new, v_new
    [B, Hkv, D] into k, v at position s - 1 (in the same launch); returns
    out [B, Hq, D]. q, k_new, v_new and out may be pinned host tensors: the
    kernel then reads the step's inputs and writes its output over the host
    link itself, so a step from host buffers is this one call."""
    torch = _torch()
    _need_cuda_or_pinned(k, v, q, k_new, v_new)
    if out is not None:
        _need_cuda_or_pinned(out)
    _need_cuda(label, idx, lscale, lzero, sel_out, score_out)
    b, hq, d = q.shape
    _, hkv, s_cap, _ = k.shape
    c = idx.shape[1]
    kdt = _kv_dtype(k)
    if k_new.dtype != k.dtype or v_new.dtype != v.dtype:
        raise TypeError("k_new / v_new must have the caches' dtype")
    if out is None:
        out = torch.empty((b, hq, d), dtype=out_dtype or torch.float32, device=label.device)
    odt = DS_F32 if out.dtype == torch.float32 else DS_BF16
    _check(lib().ds_decode_step_kv(_ptr_kv(q), _ptr_kv(k_new), _ptr_kv(v_new), _ptr_kv(k), _ptr_kv(v), kdt,
                                   _ptr(label), _label_args(label, lscale, lzero, kdt), _ptr(lscale), _ptr(lzero),
                                   _ptr(idx), b, hq, hkv, s, s_cap, d, c, topk, float(sm_scale),
                                   _ptr_kv(out), odt, _ptr(sel_out), _ptr(score_out), _stream(stream)))
    return out


class PreparedDecodeStepKV:
    """decode_step_kv with every argument checked and converted once.

    A serving loop decodes token after token into the same caches, label
    cache and (pinned host or device) buffers; only their contents and the
    token count change. Preparing the call keeps the per-step host cost to
    one C-ABI call: ``step()`` enqueues one step (ds_decode_step_kv) on the
    stream that was current at preparation (or `stream`), and
    ``step.set_length(s)`` moves to another token count."""

    _S_ARG = 14  # position of `s` in the ds_decode_step_kv argument list

    def __init__(self, q, k_new, v_new, k, v, label, idx, s: int, topk: int, lscale=None, lzero=None,
                 out=None, out_dtype=None, sm_scale: float = 0.0, stream=None):
        torch = _torch()
        _need_cuda_or_pinned(k, v, q, k_new, v_new)
        _need_cuda(label, idx, lscale, lzero)
        b, hq, d = q.shape
        _, hkv, s_cap, _ = k.shape
        c = idx.shape[1]
        kdt = _kv_dtype(k)
        if k_new.dtype != k.dtype or v_new.dtype != v.dtype:
            raise TypeError("k_new / v_new must have the caches' dtype")
        if out is None:
            out = torch.empty((b, hq, d), dtype=out_dtype or torch.float32, device=label.device)
        _need_cuda_or_pinned(out)
        odt = DS_F32 if out.dtype == torch.float32 else DS_BF16
        self.out = out
        self._keep = (q, k_new, v_new, k, v, label, idx, lscale, lzero, out)  # keep the memory alive
        self._args = [_ptr_kv(q), _ptr_kv(k_new), _ptr_kv(v_new), _ptr_kv(k), _ptr_kv(v), kdt, _ptr(label),
                      _label_args(label, lscale, lzero, kdt), _ptr(lscale), _ptr(lzero), _ptr(idx), b, hq, hkv,
                      int(s), s_cap, d, c, int(topk), float(sm_scale), _ptr_kv(out), odt, None, None,
                      _stream(stream)]
        assert self._args[self._S_ARG - 1] == hkv and self._args[self._S_ARG + 1] == s_cap  # layout check
        self._fn = lib().ds_decode_step_kv

    def set_length(self, s: int) -> None:
        self._args[self._S_ARG] = int(s)

    def __call__(self):
        st = self._fn(*self._args)
        if st != DS_OK:
            raise DSError(st, last_error())
        return self.out


def decode_step_varlen(q, k, v, label, idx, seq_lens, s_max: int, topk: int, lscale=None, lzero=None, out=None,
                       out_dtype=None, sm_scale: float = 0.0, sel_out=None, score_out=None,
                       sparse_threshold: int = 0, fallback: int = DS_FALLBACK_PER_ENTRY, stream=None):
    """decode_step with a per-batch-entry token count seq_lens [B] (int32,
    device) and the short-entry fallback rule; returns out [B, Hq, D]."""
    torch = _torch()
    _need_cuda_or_pinned(k, v)
    _need_cuda(q, label, idx, seq_lens, lscale, lzero, out, sel_out, score_out)
    b, hq, d = q.shape
    _, hkv, s_cap, _ = k.shape
    c = idx.shape[1]
    kdt = _kv_dtype(k)
    if out is None:
        out = torch.empty((b, hq, d), dtype=out_dtype or torch.float32, device=q.device)
    odt = DS_F32 if out.dtype == torch.float32 else DS_BF16
    _check(lib().ds_decode_step_varlen(_ptr(q), _ptr_kv(k), _ptr_kv(v), kdt, _ptr(label),
                                       _label_args(label, lscale, lzero, kdt), _ptr(lscale), _ptr(lzero),
                                       _ptr(idx), _ptr(seq_lens), int(sparse_threshold), int(fallback),
                                       b, hq, hkv, s_max, s_cap, d, c, topk,
                                       float(sm_scale), _ptr(out), odt, _ptr(sel_out), _ptr(score_out),
                                       _stream(stream)))
    return out


def build_label_cache_paged(k_pool, idx, block_table, s: int, label, lscale=None, lzero=None, stream=None):
    """Fill label rows [0, s) (label [B, Hkv, S_cap, ...]) from a paged key
    pool k_pool [num_blocks, Hkv, page, D] through block_table [B, max_blocks]."""
    _need_cuda_or_pinned(k_pool)
    _need_cuda(idx, block_table, label, lscale, lzero)
    num_blocks, hkv, page, d = k_pool.shape
    b, max_blocks = block_table.shape
    s_cap = label.shape[2]
    c = idx.shape[1]
    kdt = _kv_dtype(k_pool)
    _check(lib().ds_build_label_cache_paged(_ptr_kv(k_pool), kdt, _ptr(idx), _ptr(block_table), max_blocks, page,
                                            num_blocks, b, hkv, s, s_cap, d, c, _ptr(label),
                                            _label_args(label, lscale, lzero, kdt), _ptr(lscale), _ptr(lzero),
                                            _stream(stream)))


def decode_step_paged(q, k_pool, v_pool, label, idx, block_table, s_max: int, topk: int, seq_lens=None,
                      lscale=None, lzero=None, out=None, out_dtype=None, sm_scale: float = 0.0, sel_out=None,
                      score_out=None, sparse_threshold: int = 0, fallback: int = DS_FALLBACK_PER_ENTRY,
                      stream=None):
    """decode_step(_varlen) over paged pools k_pool/v_pool [num_blocks, Hkv,
    page, D] with block_table [B, max_blocks]; returns out [B, Hq, D]."""
    torch = _torch()
    _need_cuda_or_pinned(k_pool, v_pool)
    _need_cuda(q, label, idx, block_table, seq_lens, lscale, lzero, out, sel_out, score_out)
    b, hq, d = q.shape
    num_blocks, hkv, page, _ = k_pool.shape
    max_blocks = block_table.shape[1]
    s_cap = label.shape[2]
    c = idx.shape[1]
    kdt = _kv_dtype(k_pool)
    if out is None:
        out = torch.empty((b, hq, d), dtype=out_dtype or torch.float32, device=q.device)
    odt = DS_F32 if out.dtype == torch.float32 else DS_BF16
    _check(lib().ds_decode_step_paged(_ptr(q), _ptr_kv(k_pool), _ptr_kv(v_pool), kdt, _ptr(label),
                                      _label_args(label, lscale, lzero, kdt), _ptr(lscale), _ptr(lzero),
                                      _ptr(idx), _ptr(block_table), max_blocks, page, num_blocks, _ptr(seq_lens),
                                      int(sparse_threshold), int(fallback), b, hq, hkv, s_max, s_cap, d, c, topk,
                                      float(sm_scale), _ptr(out), odt, _ptr(sel_out), _ptr(score_out),
                                      _stream(stream)))
    return out


def dense_decode(q, k, v, s: int, out=None, out_dtype=None, sm_scale: float = 0.0, stream=None):
    """Dense decode attention over tokens [0, s) (measurement baseline)."""
    torch = _torch()
    _need_cuda_or_pinned(k, v)
    _need_cuda(q, out)
    b, hq, d = q.shape
    _, hkv, s_cap, _ = k.shape
    if out is None:
        out = torch.empty((b, hq, d), dtype=out_dtype or torch.float32, device=q.device)
    odt = DS_F32 if out.dtype == torch.float32 else DS_BF16
    _check(lib().ds_dense_decode(_ptr(q), _ptr_kv(k), _ptr_kv(v), _kv_dtype(k), b, hq, hkv, s, s_cap, d,
                                 float(sm_scale), _ptr(out), odt, _stream(stream)))
    return out
