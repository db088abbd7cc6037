"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/ds.h declares, rejects bad arguments before launching
anything, and plans launches as documented."""

import ctypes as C
import os
import re

import pytest

import channel_token_sparse_b200 as ds

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    ds.build()
    return ds.lib()


def header_functions():
    with open(os.path.join(ROOT, "include", "ds.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"DS_API\s+[\w\s\*]+?\b(ds_\w+)\s*\(", text)))


def test_header_symbols_exported(lib):
    names = header_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
        assert n in ds.SIGNATURES, n
    assert set(ds.SIGNATURES) == set(names)


def test_status_strings(lib):
    assert ds.status_string(ds.DS_OK) == "DS_OK"
    assert ds.status_string(ds.DS_ERR_WORKSPACE) == "DS_ERR_WORKSPACE"


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def _decode(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, kvdt=ds.DS_BF16, label=FAKE, label_dt=ds.DS_BF16, lscale=None,
             lzero=None, idx=FAKE, b=1, hq=32, hkv=32, s=4096, s_cap=4096, d=128, c=16, topk=256,
             sm_scale=0.0, out=FAKE, out_dt=ds.DS_F32, sel_out=None, score_out=None)
    a.update(kw)
    # force an invalid topk unless the test sets its own fault, so nothing can launch
    return lib.ds_sparse_decode(a["q"], a["k"], a["v"], a["kvdt"], a["label"], a["label_dt"],
                                a["lscale"], a["lzero"], a["idx"], a["b"], a["hq"], a["hkv"], a["s"],
                                a["s_cap"], a["d"], a["c"], a["topk"], a["sm_scale"], a["out"],
                                a["out_dt"], a["sel_out"], a["score_out"], None)


@pytest.mark.parametrize("fault,expect", [
    (dict(q=None), ds.DS_ERR_INVALID_ARG),
    (dict(label=None), ds.DS_ERR_INVALID_ARG),
    (dict(hq=30, hkv=8), ds.DS_ERR_INVALID_ARG),
    (dict(hq=32, hkv=2), ds.DS_ERR_UNSUPPORTED),          # group of 16 heads
    (dict(d=96), ds.DS_ERR_UNSUPPORTED),
    (dict(c=12), ds.DS_ERR_UNSUPPORTED),
    (dict(c=128, d=64), ds.DS_ERR_UNSUPPORTED),
    (dict(s=0), ds.DS_ERR_INVALID_ARG),
    (dict(s=5000, s_cap=4096), ds.DS_ERR_INVALID_ARG),
    (dict(topk=0), ds.DS_ERR_INVALID_ARG),
    (dict(k=FAKE + 8), ds.DS_ERR_INVALID_ARG),            # misaligned
    (dict(out_dt=ds.DS_BF16, kvdt=ds.DS_F32, label_dt=ds.DS_F32), ds.DS_ERR_INVALID_ARG),
    (dict(label_dt=ds.DS_F32), ds.DS_ERR_INVALID_ARG),    # label dtype != k dtype
    (dict(label_dt=ds.DS_INT4), ds.DS_ERR_INVALID_ARG),   # 4-bit without scale/zero
    (dict(kvdt=ds.DS_F16, label_dt=ds.DS_F16), ds.DS_ERR_UNSUPPORTED),
    (dict(s=600000, s_cap=600000, topk=10), ds.DS_ERR_UNSUPPORTED),  # > 16 CTAs x 32768 tokens
])
def test_decode_validation(lib, fault, expect):
    st = _decode(lib, **fault)
    assert st == expect, ds.last_error()
    assert ds.last_error()


def test_label_and_calibration_validation(lib):
    st = lib.ds_build_label_cache(FAKE, ds.DS_BF16, FAKE, 1, 2, 10, 8, 128, 16, FAKE, ds.DS_BF16,
                                  None, None, None)
    assert st == ds.DS_ERR_INVALID_ARG  # s > s_cap
    st = lib.ds_append_label(FAKE, ds.DS_BF16, FAKE, 1, 2, 8, 8, 128, 16, FAKE, ds.DS_BF16,
                             None, None, None)
    assert st == ds.DS_ERR_INVALID_ARG  # pos == s_cap
    st = lib.ds_build_label_cache(FAKE, ds.DS_BF16, None, 1, 2, 8, 8, 128, 16, FAKE, ds.DS_BF16,
                                  None, None, None)
    assert st == ds.DS_ERR_INVALID_ARG  # idx NULL
    need = ds.calibrate_workspace_size(4, 2, 2, 32, 512, 64)
    assert need == 4 * 2 * (2 * 64 + 1) * 8
    st = lib.ds_calibrate_channels(FAKE, FAKE, ds.DS_F32, 4, 2, 2, 32, 512, 64, 8, None, FAKE, FAKE,
                                   need - 8, None)
    assert st == ds.DS_ERR_WORKSPACE
    st = lib.ds_calibrate_channels(FAKE, FAKE, ds.DS_F32, 4, 2, 2, 32, 512, 64, 65, None, FAKE, FAKE,
                                   need, None)
    assert st == ds.DS_ERR_INVALID_ARG  # c > d


def test_plan_choices(lib):
    ds.set_cluster(0)
    # one wave of 2 CTAs per SM on 148 SMs: rows * N <= 296
    assert ds.plan(8, 32, 32, 4096, 128, 16, 256)[0] == 1          # 256 rows
    assert ds.plan(32, 32, 32, 16384, 128, 32, 1024, ds.DS_BF16, ds.DS_INT4)[0] == 1
    assert ds.plan(4, 32, 8, 32768, 128, 16, 2048)[0] == 8         # 32 rows
    n, chunk, smem = ds.plan(1, 32, 32, 262144, 128, 16, 16384)
    assert (n, chunk) == (8, 32768) and smem <= 227 * 1024
    n, chunk, _ = ds.plan(1, 2, 2, 512, 64, 8, 32, ds.DS_F32, ds.DS_F32)
    assert n * chunk >= 512 and chunk >= 256
    # the four benchmark layers keep two CTAs per SM: (228 KiB - 2 KiB) / 2 of
    # shared memory each at most
    for shape in ((8, 32, 32, 4096, 128, 16, 256, ds.DS_BF16, ds.DS_BF16),
                  (32, 32, 32, 16384, 128, 32, 1024, ds.DS_BF16, ds.DS_INT4),
                  (4, 32, 8, 32768, 128, 16, 2048, ds.DS_BF16, ds.DS_BF16),
                  (1, 32, 32, 262144, 128, 16, 16384, ds.DS_BF16, ds.DS_BF16)):
        assert ds.plan(*shape)[2] <= (228 - 2) * 1024 // 2, shape
    ds.set_cluster(16)
    try:
        assert ds.plan(8, 32, 32, 4096, 128, 16, 256)[:2] == (16, 256)
    finally:
        ds.set_cluster(0)


def test_sparse_decode_workspace(lib):
    # every supported shape keeps its per-step scratch on chip
    for shape in [(8, 32, 32, 4096, 128, 16, 256), (32, 32, 32, 16384, 128, 32, 1024),
                  (4, 32, 8, 32768, 128, 16, 2048), (1, 32, 32, 262144, 128, 16, 16384),
                  (1, 2, 2, 512, 64, 8, 32)]:
        assert ds.sparse_decode_workspace(*shape) == 0
    out = C.c_size_t(12345)
    for bad, expect in [((1, 30, 8, 512, 64, 8, 32), ds.DS_ERR_INVALID_ARG),   # hq % hkv
                        ((1, 2, 2, 512, 96, 8, 32), ds.DS_ERR_UNSUPPORTED),    # head_dim
                        ((1, 2, 2, 512, 64, 12, 32), ds.DS_ERR_UNSUPPORTED),   # channels
                        ((1, 2, 2, 512, 64, 8, 0), ds.DS_ERR_INVALID_ARG),     # topk
                        ((1, 2, 2, 0, 64, 8, 32), ds.DS_ERR_INVALID_ARG)]:     # s
        assert lib.ds_sparse_decode_workspace(*bad, C.byref(out)) == expect
        assert out.value == 12345  # untouched on failure
    assert lib.ds_sparse_decode_workspace(1, 2, 2, 512, 64, 8, 32, None) == ds.DS_ERR_INVALID_ARG
