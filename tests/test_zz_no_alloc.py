"""The allocation-free calibration entry point.

Some callers cannot allocate device memory: plugins whose host framework
owns every allocation, or runtimes with a fixed device budget. ds_calibrate_channels_noalloc serves them with a
fixed scratch array inside the library instead of a caller workspace. This
test calls it through the C ABI twice in a row (the shared scratch keeps the
previous call's contents, so the second call checks that it is cleared) and
compares both results with ds_calibrate_channels: channel indices equal,
ratios within the tolerance the other calibration tests use.

This file is named so that pytest collects it last.
"""

import ctypes as C

import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import channel_token_sparse_b200 as ds  # noqa: E402


def _inputs(index, hq, hkv, d, c, s, n_samples, kv_dtype):
    wl = synth.custom(b=1, hq=hq, hkv=hkv, d=d, s=s, c=c, kv_dtype=kv_dtype, label_dtype=kv_dtype,
                      n_outlier=c, outlier_scale=6.0, index=index, calib_samples=n_samples, calib_w=32,
                      calib_s=s)
    ci = synth.calib_inputs(wl)

    def dev(x):
        if kv_dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(x)).cuda()

    return wl, dev(ci.q_win), dev(ci.k)


def _noalloc(q_win, k, c):
    n, hq, w, d = q_win.shape
    _, hkv, s, _ = k.shape
    idx = torch.full((hkv, c), -1, dtype=torch.int32, device="cuda")
    ratio = torch.full((hkv, d), -1.0, dtype=torch.float32, device="cuda")
    dt = ds.DS_BF16 if k.dtype == torch.bfloat16 else ds.DS_F32
    st = ds.lib().ds_calibrate_channels_noalloc(
        C.c_void_p(q_win.data_ptr()), C.c_void_p(k.data_ptr()), dt, n, hq, hkv, w, s, d, c,
        C.c_void_p(ratio.data_ptr()), C.c_void_p(idx.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ds.DS_OK, ds.last_error()
    return idx, ratio


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ds.build()
    ds.lib()


@pytest.mark.parametrize("index,hq,hkv,d,c,s,n_samples,kv_dtype", [
    (81, 2, 2, 64, 8, 512, 4, "f32"),
    (82, 32, 8, 128, 16, 1024, 2, "bf16"),
])
def test_noalloc_matches_workspace_entry_point_twice(index, hq, hkv, d, c, s, n_samples, kv_dtype):
    wl, q_win, k = _inputs(index, hq, hkv, d, c, s, n_samples, kv_dtype)
    idx_ref, ratio_ref = ds.calibrate_channels(q_win, k, c)
    for _ in range(2):
        idx, ratio = _noalloc(q_win, k, c)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx_ref)
        np.testing.assert_allclose(ratio.cpu().numpy(), ratio_ref.cpu().numpy(), rtol=2e-5, atol=1e-7)


def test_noalloc_call_takes_no_device_memory():
    """After a first call (which looks up the scratch array's address), calls
    change neither torch's allocations nor the device's free memory."""
    wl, q_win, k = _inputs(83, 8, 4, 128, 16, 512, 2, "bf16")
    idx, ratio = _noalloc(q_win, k, 16)  # first call in this context
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        n, hq, w, d = q_win.shape
        _, hkv, s, _ = k.shape
        st = ds.lib().ds_calibrate_channels_noalloc(
            C.c_void_p(q_win.data_ptr()), C.c_void_p(k.data_ptr()), ds.DS_BF16, n, hq, hkv, w, s, d, 16,
            C.c_void_p(ratio.data_ptr()), C.c_void_p(idx.data_ptr()),
            C.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == ds.DS_OK, ds.last_error()
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == alloc0
    assert free1 == free0


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    # 8 samples x 128 kv heads x (2*128+1) doubles > 1 MiB: refused before any launch
    q = torch.empty(16, dtype=torch.float32, device="cuda")
    out = torch.empty(16, dtype=torch.int32, device="cuda")
    st = ds.lib().ds_calibrate_channels_noalloc(
        C.c_void_p(q.data_ptr()), C.c_void_p(q.data_ptr()), ds.DS_F32, 8, 128, 128, 32, 64, 128, 16,
        None, C.c_void_p(out.data_ptr()), None)
    assert st == ds.DS_ERR_WORKSPACE
    assert "scratch" in ds.last_error()
