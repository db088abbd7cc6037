"""CPU oracle for Double Sparsity decode attention -- TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 C implementation (``ds_oracle.c``) of what the decode path
computes, wrapped with ctypes. Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import this package. It shares no code with
the CUDA library (``channel_token_sparse_b200``) and neither imports the other.

Every function takes numpy arrays in the storage layout of the CUDA library
(bf16 as uint16 bit patterns) and returns numpy arrays.

Sources: "大模型稀疏化技术原理：Double Sparsity" (joto.ai blog), sections 离线校准
and 在线前向计算 steps 1-3; "K通道静态性量化方法解析" (aitangshan.cn) §1.1 for the
calibration ratio. Each C function states the reading it takes.
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ds_oracle.c")
_LIB = os.path.join(_HERE, "libds_oracle.so")
_DT = {"f32": 0, "bf16": 1, "f16": 2}

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C11, no fused multiply-add contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", _LIB, _SRC, "-lm"])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        vp, i, d = C.c_void_p, C.c_int, C.c_double
        _lib.oracle_calibrate.argtypes = [vp, vp, i, i, i, i, i, i, i, i, vp, vp]
        _lib.oracle_calibrate_criterion.argtypes = [vp, vp, i, i, i, i, i, i, i, i, i, i, vp, vp]
        _lib.oracle_label_copy.argtypes = [vp, i, vp, i, i, i, i, i, i, i, vp]
        _lib.oracle_label_int4.argtypes = [vp, i, vp, i, i, i, i, i, i, i, vp, vp, vp]
        _lib.oracle_label_int4_values.argtypes = [vp, vp, vp, i, i, i, i, vp]
        _lib.oracle_scores.argtypes = [vp, i, vp, vp, i, i, i, i, i, i, vp]
        _lib.oracle_topk.argtypes = [vp, i, i, i, vp]
        _lib.oracle_attention.argtypes = [vp, vp, vp, i, vp, i, i, i, i, i, i, d, vp]
        for f in (_lib.oracle_calibrate, _lib.oracle_calibrate_criterion, _lib.oracle_label_copy, _lib.oracle_label_int4,
                  _lib.oracle_label_int4_values, _lib.oracle_scores, _lib.oracle_topk,
                  _lib.oracle_attention):
            f.restype = C.c_int
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def calibrate(q_win: np.ndarray, k: np.ndarray, dtype: str, c: int):
    """Channel importance ratio r [Hkv, D] and heavy channels idx [Hkv, C].

    q_win [N, Hq, W, D], k [N, Hkv, S, D] in storage format."""
    n, hq, w, d = q_win.shape
    n2, hkv, s, d2 = k.shape
    assert n == n2 and d == d2
    ratio = np.zeros((hkv, d), dtype=np.float64)
    idx = np.zeros((hkv, c), dtype=np.int32)
    _check(_load().oracle_calibrate(_p(q_win), _p(k), _DT[dtype], n, hq, hkv, w, s, d, c,
                                    _p(ratio), _p(idx)), "calibrate")
    return ratio, idx


CRITERIA = {"leank": 0, "q": 1, "k": 2, "qk": 3, "qk_chunked": 4}


def calibrate_criterion(q_win: np.ndarray, k: np.ndarray, dtype: str, c: int, criterion: str,
                        chunk: int = 0):
    """Channel score [Hkv, D] under one outlier criterion and the heavy
    channels idx [Hkv, C]; criterion in CRITERIA, chunk for "qk_chunked"."""
    n, hq, w, d = q_win.shape
    n2, hkv, s, d2 = k.shape
    assert n == n2 and d == d2
    score = np.zeros((hkv, d), dtype=np.float64)
    idx = np.zeros((hkv, c), dtype=np.int32)
    _check(_load().oracle_calibrate_criterion(_p(q_win), _p(k), _DT[dtype], n, hq, hkv, w, s, d, c,
                                              CRITERIA[criterion], int(chunk), _p(score), _p(idx)),
           "calibrate_criterion")
    return score, idx


def label_copy(k: np.ndarray, dtype: str, idx: np.ndarray, s: int, t_begin: int = 0,
               label: np.ndarray | None = None):
    """fp label cache [B, Hkv, S_cap, C] (storage dtype of k); rows [t_begin, s) filled."""
    b, hkv, s_cap, d = k.shape
    c = idx.shape[1]
    if label is None:
        label = np.zeros((b, hkv, s_cap, c), dtype=k.dtype)
    _check(_load().oracle_label_copy(_p(k), _DT[dtype], _p(np.ascontiguousarray(idx, np.int32)),
                                     b, hkv, t_begin, s, s_cap, d, c, _p(label)), "label_copy")
    return label


def label_int4(k: np.ndarray, dtype: str, idx: np.ndarray, s: int, t_begin: int = 0,
               out=None):
    """4-bit label cache: payload [B, Hkv, S_cap, C/2] uint8, scale and zero
    [B, Hkv, S_cap] as fp16 bit patterns (uint16)."""
    b, hkv, s_cap, d = k.shape
    c = idx.shape[1]
    if out is None:
        out = (np.zeros((b, hkv, s_cap, c // 2), np.uint8), np.zeros((b, hkv, s_cap), np.uint16),
               np.zeros((b, hkv, s_cap), np.uint16))
    lab, sc, ze = out
    _check(_load().oracle_label_int4(_p(k), _DT[dtype], _p(np.ascontiguousarray(idx, np.int32)),
                                     b, hkv, t_begin, s, s_cap, d, c, _p(lab), _p(sc), _p(ze)),
           "label_int4")
    return lab, sc, ze


def label_values(label, label_dtype: str, s: int, c: int) -> np.ndarray:
    """Label cache as doubles [rows, S, C]. ``label`` is the fp array or the
    (payload, scale, zero) triple of the 4-bit cache."""
    if label_dtype == "int4":
        lab, sc, ze = label
        rows = lab.shape[0] * lab.shape[1]
        s_cap = lab.shape[2]
        out = np.zeros((rows, s, c), np.float64)
        _check(_load().oracle_label_int4_values(_p(lab), _p(sc), _p(ze), rows, s, s_cap, c, _p(out)),
               "label_int4_values")
        return out
    b, hkv, s_cap, cc = label.shape
    assert cc == c
    x = label[:, :, :s, :].reshape(b * hkv, s, c)
    if label_dtype == "bf16":
        x = (x.astype(np.uint32) << 16).view(np.float32)
    return np.ascontiguousarray(x, dtype=np.float64)


def scores(q: np.ndarray, qdtype: str, lab_values: np.ndarray, idx: np.ndarray, hkv: int):
    """Approximate scores [B, Hkv, S] (fp64)."""
    b, hq, d = q.shape
    rows, s, c = lab_values.shape
    assert rows == b * hkv
    out = np.zeros((b, hkv, s), np.float64)
    _check(_load().oracle_scores(_p(q), _DT[qdtype], _p(lab_values),
                                 _p(np.ascontiguousarray(idx, np.int32)), b, hq, hkv, s, d, c,
                                 _p(out)), "scores")
    return out


def topk(scores_: np.ndarray, k: int) -> np.ndarray:
    """Top-k token indices per row, ascending, padded with -1: [..., k] int32."""
    lead = scores_.shape[:-1]
    s = scores_.shape[-1]
    sc = np.ascontiguousarray(scores_.reshape(-1, s), np.float64)
    sel = np.zeros((sc.shape[0], k), np.int32)
    _check(_load().oracle_topk(_p(sc), sc.shape[0], s, k, _p(sel)), "topk")
    return sel.reshape(*lead, k)


def attention(q, k, v, dtype: str, sel: np.ndarray, hkv: int, sm_scale: float | None = None):
    """Exact softmax attention over the selected tokens: out [B, Hq, D] fp64."""
    b, hq, d = q.shape
    s_cap = k.shape[2]
    if sm_scale is None or sm_scale <= 0:
        sm_scale = 1.0 / np.sqrt(d)
    sel = np.ascontiguousarray(sel, np.int32)
    kk = sel.shape[-1]
    out = np.zeros((b, hq, d), np.float64)
    _check(_load().oracle_attention(_p(q), _p(k), _p(v), _DT[dtype], _p(sel), kk, b, hq, hkv,
                                    s_cap, d, float(sm_scale), _p(out)), "attention")
    return out


def build_label(k, kv_dtype: str, label_dtype: str, idx, s: int):
    if label_dtype == "int4":
        return label_int4(k, kv_dtype, idx, s)
    assert label_dtype == kv_dtype, "an fp label cache has the key cache's dtype"
    return label_copy(k, kv_dtype, idx, s)


def sparse_decode(q, k, v, kv_dtype: str, label, label_dtype: str, idx, s: int, topk_: int,
                  sm_scale: float | None = None):
    """The whole decode step: (out [B,Hq,D], sel [B,Hkv,k], scores [B,Hkv,S])."""
    b, hkv = k.shape[0], k.shape[1]
    c = idx.shape[1]
    lv = label_values(label, label_dtype, s, c)
    sc = scores(q, kv_dtype, lv, idx, hkv)
    sel = topk(sc, topk_)
    out = attention(q, k, v, kv_dtype, sel, hkv, sm_scale)
    return out, sel, sc
