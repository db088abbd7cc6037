"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars: label cache, 4-bit codes, scale/zero bits and channel indices bit-exact;
approximate scores within 1e-3 relative; the top-k set exact except tokens
within 1e-4 relative of the k-th score; outputs within max-abs 2e-3 of the
oracle's attention over the GPU's selected set.
"""

import dataclasses

import numpy as np
import pytest

import oracle
import synth
from dshelp import (OUT_ATOL, check_scores, check_selection, oracle_row_slices, to_dev, to_host)

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import channel_token_sparse_b200 as ds  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ds.build()
    ds.lib()
    yield
    ds.set_cluster(0)


def _idx_random(wl, seed=1):
    r = np.random.default_rng(seed)
    return np.stack([np.sort(r.choice(wl.d, wl.c, replace=False)) for _ in range(wl.hkv)]).astype(np.int32)


def _gpu_label(kd, idxd, s, wl):
    lab, sc, ze = ds.new_label_cache(kd, wl.c, int4=wl.label_dtype == "int4")
    lab.zero_()
    if sc is not None:
        sc.zero_(); ze.zero_()
    ds.build_label_cache(kd, idxd, s, lab, sc, ze)
    return lab, sc, ze


def _host_label(lab, sc, ze, wl):
    if wl.label_dtype == "int4":
        return (lab.cpu().numpy(), to_host(sc, "bf16"), to_host(ze, "bf16"))
    return to_host(lab, wl.kv_dtype)


def run_decode_case(wl, s_cap=None, idx=None, cluster=0, q_override=None, topk=None, check_label=True):
    """Full decode step on the GPU vs the oracle, on every (b, kv head) row."""
    topk = wl.topk if topk is None else topk
    di = synth.decode_inputs(wl, s_cap=s_cap)
    q = di.q if q_override is None else q_override
    idx = _idx_random(wl) if idx is None else idx
    qd, kd, vd = to_dev(q, wl.kv_dtype), to_dev(di.k, wl.kv_dtype), to_dev(di.v, wl.kv_dtype)
    idxd = torch.from_numpy(idx).cuda()
    lab, sc, ze = _gpu_label(kd, idxd, wl.s, wl)
    ds.set_cluster(cluster)
    try:
        sel = torch.full((wl.b, wl.hkv, topk), -7, dtype=torch.int32, device="cuda")
        scores = torch.zeros((wl.b, wl.hkv, wl.s), dtype=torch.float32, device="cuda")
        out = ds.sparse_decode(qd, kd, vd, lab, idxd, wl.s, topk, lscale=sc, lzero=ze,
                               sel_out=sel, score_out=scores)
        torch.cuda.synchronize()
    finally:
        ds.set_cluster(0)
    ref_label = oracle.build_label(di.k, wl.kv_dtype, wl.label_dtype, idx, wl.s)
    if check_label:
        got = _host_label(lab, sc, ze, wl)
        if wl.label_dtype == "int4":
            for a, b_ in zip(got, ref_label):
                assert np.array_equal(a, b_), "4-bit label not bit-exact"
        else:
            assert np.array_equal(got, ref_label), "label not bit-exact"
    o_ref, sel_ref, s_ref = oracle.sparse_decode(q, di.k, di.v, wl.kv_dtype, ref_label, wl.label_dtype,
                                                 idx, wl.s, topk)
    s_gpu = scores.cpu().numpy()
    sel_gpu = sel.cpu().numpy()
    check_scores(s_gpu, s_ref)
    check_selection(sel_gpu.reshape(-1, topk), sel_ref.reshape(-1, topk), s_ref.reshape(-1, wl.s),
                    topk, wl.s)
    o_on_gpu_sel = oracle.attention(q, di.k, di.v, wl.kv_dtype, sel_gpu, wl.hkv)
    err = np.abs(out.cpu().numpy() - o_on_gpu_sel).max()
    assert err <= OUT_ATOL, f"output max-abs error {err}"
    return out, sel_gpu, sel_ref, o_ref


# --------------------------------------------------------------- label cache

@pytest.mark.parametrize("kv,label", [("f32", "f32"), ("bf16", "bf16"), ("bf16", "int4"), ("f32", "int4")])
@pytest.mark.parametrize("d,c", [(64, 8), (128, 32)])
def test_label_build_and_append_bit_exact(kv, label, d, c):
    wl = synth.custom(b=3, hq=6, hkv=3, d=d, s=1000, c=c, kv_dtype=kv, label_dtype=label,
                      n_outlier=4, index=61)
    di = synth.decode_inputs(wl, s_cap=1037)
    idx = _idx_random(wl, 3)
    kd, idxd = to_dev(di.k, kv), torch.from_numpy(idx).cuda()
    lab, sc, ze = _gpu_label(kd, idxd, wl.s, wl)
    torch.cuda.synchronize()
    ref = oracle.build_label(di.k, kv, label, idx, wl.s)
    got = _host_label(lab, sc, ze, wl)
    if label == "int4":
        for a, b_ in zip(got, ref):
            assert np.array_equal(a, b_)
    else:
        assert np.array_equal(got, ref)
    # append token 1020 (beyond s) into a fresh cache: only that row changes
    lab2, sc2, ze2 = ds.new_label_cache(kd, c, int4=label == "int4")
    lab2.zero_()
    if sc2 is not None:
        sc2.zero_(); ze2.zero_()
    ds.append_label(kd, idxd, 1020, lab2, sc2, ze2)
    torch.cuda.synchronize()
    got2 = _host_label(lab2, sc2, ze2, wl)
    kfull = di.k.copy()
    if label == "int4":
        r2 = oracle.label_int4(kfull, kv, idx, 1021, t_begin=1020)
        for a, b_ in zip(got2, r2):
            assert np.array_equal(a, b_)
    else:
        r2 = oracle.label_copy(kfull, kv, idx, 1021, t_begin=1020)
        assert np.array_equal(got2, r2)


@pytest.mark.parametrize("kv,label,d,c", [("bf16", "bf16", 128, 16), ("bf16", "int4", 128, 32),
                                          ("f32", "f32", 64, 8), ("f32", "int4", 64, 8), ("bf16", "int4", 128, 8),
                                          ("bf16", "bf16", 64, 64), ("bf16", "int4", 128, 128),
                                          ("f32", "f32", 128, 32)])
def test_pipelined_label_build_bit_exact(kv, label, d, c):
    """Prefill builds large enough for the pipelined (bulk-copy ring) label
    kernel: every row bit-exact against the oracle, a ragged last block per
    row, an odd cache capacity, and rows past s left untouched."""
    wl = synth.custom(b=4, hq=8, hkv=8, d=d, s=5000, c=c, kv_dtype=kv, label_dtype=label,
                      n_outlier=min(8, c), index=66)
    di = synth.decode_inputs(wl, s_cap=5003)
    idx = _idx_random(wl, 9)
    kd, idxd = to_dev(di.k, kv), torch.from_numpy(idx).cuda()
    lab, sc, ze = ds.new_label_cache(kd, c, int4=label == "int4")
    lab.fill_(7 if label == "int4" else 3)
    if sc is not None:
        sc.fill_(5); ze.fill_(5)
    ds.build_label_cache(kd, idxd, wl.s, lab, sc, ze)
    ds.check_device()
    got = _host_label(lab, sc, ze, wl)
    ref = oracle.build_label(di.k, kv, label, idx, wl.s)
    if label == "int4":
        for a, b_ in zip(got, ref):
            assert np.array_equal(a[:, :, : wl.s], b_[:, :, : wl.s])
        assert np.all(got[0][:, :, wl.s:] == 7) and np.all(got[1][:, :, wl.s:] == 5)
    else:
        assert np.array_equal(got[:, :, : wl.s], ref[:, :, : wl.s])
        assert torch.all(lab[:, :, wl.s:] == 3)


@pytest.mark.parametrize("kv,c", [("bf16", 32), ("f32", 16), ("bf16", 64)])
def test_pipelined_int4_half_way_codes(kv, c):
    """4-bit prefill build where many quotients (x - zero) / scale are exact
    half-integers: each heavy row spans [0, 15 h] with h a power of two, so
    scale = h exactly and odd multiples of h / 2 sit half-way between two
    codes. Rounding must be half to even, as the IEEE quotient gives; the
    kernel's reciprocal shortcut has to fall back to the division there."""
    wl = synth.custom(b=4, hq=8, hkv=8, d=128, s=1000, c=c, kv_dtype=kv, label_dtype="int4",
                      n_outlier=min(8, c), index=67)
    di = synth.decode_inputs(wl, s_cap=1000)
    idx = _idx_random(wl, 11)
    r = np.random.default_rng(5)
    k = synth.storage_to_f32(di.k, kv).copy()
    for g in range(wl.hkv):
        h = 2.0 ** r.integers(-4, 3, size=(wl.b, wl.s))
        m = r.integers(0, 31, size=(wl.b, wl.s, c)).astype(np.float64)  # multiples of h / 2 in [0, 15 h]
        m[:, :, 0], m[:, :, 1] = 0, 30
        k[:, g, :, idx[g]] = np.moveaxis(m * h[:, :, None] / 2, 2, 0)
    kst = synth.to_storage(k.astype(np.float32), kv)
    assert np.array_equal(synth.storage_to_f32(kst, kv), k.astype(np.float32))  # exact in the key dtype
    kd, idxd = to_dev(kst, kv), torch.from_numpy(idx).cuda()
    lab, sc, ze = _gpu_label(kd, idxd, wl.s, wl)
    ds.check_device()
    got = _host_label(lab, sc, ze, wl)
    ref = oracle.build_label(kst, kv, "int4", idx, wl.s)
    for a, b_ in zip(got, ref):
        assert np.array_equal(a, b_)


def test_bounded_wait_self_test_reports_timeout():
    """A kernel wait that runs out is recorded and reported, and the context
    stays usable: a transaction barrier nothing completes, waited on for about
    50 us; then a normal launch still runs."""
    ds.check_device()  # clears any earlier record
    st = ds.lib().ds_selftest_bounded_wait(50, None)
    assert st == ds.DS_OK
    with pytest.raises(ds.DSError) as e:
        ds.check_device()
    assert e.value.status == ds.DS_ERR_TIMEOUT
    ds.check_device()  # cleared by the read
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float(x.sum()) == 1023 * 1024 / 2
    assert ds.lib().ds_selftest_bounded_wait(0, None) == ds.DS_ERR_INVALID_ARG


# ----------------------------------------------------------------- decode

@pytest.mark.parametrize("cluster", [0, 1, 2, 4, 8, 16])
def test_decode_cluster_sizes_bf16(cluster):
    wl = synth.custom(b=2, hq=8, hkv=4, d=128, s=3001, c=16, topk=200, kv_dtype="bf16",
                      label_dtype="bf16", n_outlier=16, outlier_scale=6.0, index=62)
    run_decode_case(wl, s_cap=3072, cluster=cluster)


@pytest.mark.parametrize("cluster", [0, 2, 16])
def test_decode_int4(cluster):
    wl = synth.custom(b=3, hq=4, hkv=4, d=128, s=2500, c=32, topk=160, kv_dtype="bf16",
                      label_dtype="int4", n_outlier=16, outlier_scale=6.0, index=63)
    run_decode_case(wl, cluster=cluster)


@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (8, 4), (16, 2)])
def test_decode_gqa_groups_f32(hq, hkv):
    wl = synth.custom(b=2, hq=hq, hkv=hkv, d=64, s=777, c=8, topk=50, n_outlier=8, index=64)
    run_decode_case(wl, cluster=2)


def test_decode_c64_d128_and_bf16_out():
    wl = synth.custom(b=1, hq=4, hkv=4, d=128, s=1500, c=64, topk=300, kv_dtype="bf16",
                      label_dtype="bf16", n_outlier=16, outlier_scale=6.0, index=65)
    out, sel_gpu, _, _ = run_decode_case(wl, cluster=4)
    di = synth.decode_inputs(wl)
    idx = _idx_random(wl)
    qd, kd, vd = (to_dev(x, "bf16") for x in (di.q, di.k, di.v))
    idxd = torch.from_numpy(idx).cuda()
    lab, _, _ = _gpu_label(kd, idxd, wl.s, wl)
    ob = ds.sparse_decode(qd, kd, vd, lab, idxd, wl.s, wl.topk, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    np.testing.assert_allclose(ob.float().cpu().numpy(), out.cpu().numpy(), atol=1e-2, rtol=1e-2)


@pytest.mark.parametrize("kv,d", [("f32", 64), ("bf16", 128)])
def test_full_channels_all_tokens_equals_dense(kv, d):
    """C = D and k = S: the GPU step is dense softmax attention."""
    wl = synth.custom(b=2, hq=4, hkv=2, d=d, s=600, c=d, topk=600, kv_dtype=kv, label_dtype=kv,
                      n_outlier=8, index=66)
    idx = np.tile(np.arange(d, dtype=np.int32), (2, 1))
    out, sel_gpu, _, o_ref = run_decode_case(wl, idx=idx, cluster=2)
    assert np.array_equal(sel_gpu, np.tile(np.arange(600), (2, 2, 1)))
    assert np.abs(out.cpu().numpy() - o_ref).max() <= OUT_ATOL


def test_topk_at_least_s_selects_all_and_pads():
    wl = synth.custom(b=1, hq=2, hkv=2, d=64, s=100, c=8, topk=130, index=67)
    _, sel_gpu, _, _ = run_decode_case(wl)
    assert np.array_equal(sel_gpu[..., :100], np.tile(np.arange(100), (1, 2, 1)))
    assert np.all(sel_gpu[..., 100:] == -1)


@pytest.mark.parametrize("s,topk", [(1, 1), (2, 1), (33, 1), (64, 63), (5000, 4999)])
def test_small_and_extreme_k(s, topk):
    wl = synth.custom(b=2, hq=2, hkv=2, d=64, s=s, c=8, topk=topk, index=68)
    run_decode_case(wl, cluster=0)
    if s >= 64:
        run_decode_case(wl, cluster=4)


@pytest.mark.parametrize("cluster", [1, 8])
def test_all_scores_equal_takes_lowest_indices(cluster):
    """q = 0 makes every approximate score 0: the selection is the first k
    tokens (ties to the lower index) and the output the mean of their V."""
    wl = synth.custom(b=1, hq=2, hkv=2, d=64, s=2000, c=8, topk=300, index=69)
    q0 = np.zeros((1, 2, 64), np.float32)
    _, sel_gpu, sel_ref, _ = run_decode_case(wl, q_override=q0, cluster=cluster)
    assert np.array_equal(sel_gpu, sel_ref)
    assert np.array_equal(sel_gpu[0, 0], np.arange(300))


def test_planted_ties_across_ctas():
    """Integer-valued label rows give many exactly equal scores spread over
    several CTAs: the tie-break must take the lowest indices cluster-wide."""
    wl = synth.custom(b=1, hq=1, hkv=1, d=64, s=4096, c=8, topk=1000, index=70)
    di = synth.decode_inputs(wl)
    r = np.random.default_rng(4)
    di.k[:] = np.float32(r.integers(-2, 3, size=di.k.shape))
    q = np.ones((1, 1, 64), np.float32)
    idx = np.arange(8, dtype=np.int32)[None]
    qd, kd, vd = to_dev(q, "f32"), to_dev(di.k, "f32"), to_dev(di.v, "f32")
    idxd = torch.from_numpy(idx).cuda()
    lab, _, _ = _gpu_label(kd, idxd, wl.s, wl)
    for cl in (1, 4, 16):
        ds.set_cluster(cl)
        sel = torch.empty((1, 1, 1000), dtype=torch.int32, device="cuda")
        ds.sparse_decode(qd, kd, vd, lab, idxd, wl.s, 1000, sel_out=sel)
        torch.cuda.synchronize()
        ds.set_cluster(0)
        ref_lab = oracle.label_copy(di.k, "f32", idx, wl.s)
        _, sel_ref, _ = oracle.sparse_decode(q, di.k, di.v, "f32", ref_lab, "f32", idx, wl.s, 1000)
        assert np.array_equal(sel.cpu().numpy(), sel_ref), f"cluster {cl}"


def test_dense_decode_matches_oracle():
    wl = synth.custom(b=2, hq=8, hkv=2, d=128, s=2049, c=16, kv_dtype="bf16", label_dtype="bf16",
                      index=71)
    di = synth.decode_inputs(wl, s_cap=2100)
    qd, kd, vd = (to_dev(x, "bf16") for x in (di.q, di.k, di.v))
    for cl in (0, 1, 8):
        ds.set_cluster(cl)
        out = ds.dense_decode(qd, kd, vd, wl.s)
        torch.cuda.synchronize()
        ds.set_cluster(0)
        sel = np.tile(np.arange(wl.s, dtype=np.int32), (2, 2, 1))
        ref = oracle.attention(di.q, di.k, di.v, "bf16", sel, 2)
        assert np.abs(out.cpu().numpy() - ref).max() <= OUT_ATOL


def test_stream_and_repeat_determinism():
    wl = synth.custom(b=2, hq=4, hkv=4, d=128, s=3000, c=16, topk=100, kv_dtype="bf16",
                      label_dtype="bf16", index=72)
    di = synth.decode_inputs(wl)
    idx = _idx_random(wl)
    qd, kd, vd = (to_dev(x, "bf16") for x in (di.q, di.k, di.v))
    idxd = torch.from_numpy(idx).cuda()
    lab, _, _ = _gpu_label(kd, idxd, wl.s, wl)
    s1 = torch.cuda.Stream()
    with torch.cuda.stream(s1):
        a = ds.sparse_decode(qd, kd, vd, lab, idxd, wl.s, wl.topk)
        b_ = ds.sparse_decode(qd, kd, vd, lab, idxd, wl.s, wl.topk)
    torch.cuda.synchronize()
    assert torch.equal(a, b_)


# ------------------------------------------------------------ calibration

@pytest.mark.parametrize("wl_i", [0, 1, 3])
def test_calibration_matches_oracle_and_recovers_outliers(wl_i):
    wl = synth.workload(wl_i)
    if wl_i:
        wl = synth.custom(b=1, hq=wl.hq, hkv=wl.hkv, d=wl.d, s=1024, c=wl.c, kv_dtype=wl.kv_dtype,
                          label_dtype=wl.label_dtype, n_outlier=wl.n_outlier,
                          outlier_scale=wl.outlier_scale, index=wl.index, calib_samples=2,
                          calib_w=32, calib_s=1024)
    ci = synth.calib_inputs(wl)
    r_ref, i_ref = oracle.calibrate(ci.q_win, ci.k, wl.kv_dtype, wl.c)
    qw, kc = to_dev(ci.q_win, wl.kv_dtype), to_dev(ci.k, wl.kv_dtype)
    idx, ratio = ds.calibrate_channels(qw, kc, wl.c)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), i_ref)
    assert np.array_equal(i_ref, ci.outliers)
    np.testing.assert_allclose(ratio.cpu().numpy(), r_ref, rtol=2e-5, atol=1e-7)


# ------------------------------------------------------ full-size configs

def _full_config(i, rows_to_check, label_dtype=None):
    wl = synth.workload(i)
    if label_dtype:
        wl = dataclasses.replace(wl, label_dtype=label_dtype)
    if i == 0:
        # heavy channels from calibration on the 4 samples (= the planted set, pinned on CPU)
        run_decode_case(wl, idx=synth.outlier_channels(wl))
        return
    q, k, v = synth.decode_inputs_torch(wl, "cuda")
    if wl.c == wl.n_outlier:
        idx = synth.outlier_channels(wl)
    else:
        # 32 channels: the 16 planted ones plus 16 chosen by the oracle's calibration
        # on one seeded sample; the GPU calibration must agree bit for bit
        cw = synth.custom(b=1, hq=wl.hq, hkv=wl.hkv, d=wl.d, s=1024, c=wl.c, kv_dtype=wl.kv_dtype,
                          label_dtype=wl.label_dtype, n_outlier=wl.n_outlier,
                          outlier_scale=wl.outlier_scale, index=wl.index, calib_samples=1,
                          calib_s=1024)
        ci = synth.calib_inputs(cw)
        _, idx = oracle.calibrate(ci.q_win, ci.k, wl.kv_dtype, wl.c)
        idx_t, _ = ds.calibrate_channels(to_dev(ci.q_win, wl.kv_dtype), to_dev(ci.k, wl.kv_dtype), wl.c)
        assert np.array_equal(idx_t.cpu().numpy(), idx)
        assert all(set(ci.outliers[g]) <= set(idx[g]) for g in range(wl.hkv))
    idxd = torch.from_numpy(np.ascontiguousarray(idx, np.int32)).cuda()
    lab, sc, ze = ds.new_label_cache(k, wl.c, int4=wl.label_dtype == "int4")
    ds.build_label_cache(k, idxd, wl.s, lab, sc, ze)
    sel = torch.empty((wl.b, wl.hkv, wl.topk), dtype=torch.int32, device="cuda")
    scores = torch.empty((wl.b, wl.hkv, wl.s), dtype=torch.float32, device="cuda")
    out = ds.sparse_decode(q, k, v, lab, idxd, wl.s, wl.topk, lscale=sc, lzero=ze, sel_out=sel,
                           score_out=scores, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ds.check_device()
    G = wl.g
    if rows_to_check == "all":
        rows_to_check = [(b, g) for b in range(wl.b) for g in range(wl.hkv)]
    # caches up to 1 GiB are copied to the host once, larger ones row by row
    whole = k.numel() * k.element_size() * 2 <= (1 << 30)
    if whole:
        kh, vh, qh = (to_host(t, wl.kv_dtype) for t in (k, v, q))
    for (b, g) in rows_to_check:
        if whole:
            kr = np.ascontiguousarray(kh[b:b + 1, g:g + 1])
            vr = np.ascontiguousarray(vh[b:b + 1, g:g + 1])
            qr = np.ascontiguousarray(qh[b:b + 1, g * G:(g + 1) * G])
        else:
            kr = to_host(k[b:b + 1, g:g + 1].contiguous(), wl.kv_dtype)
            vr = to_host(v[b:b + 1, g:g + 1].contiguous(), wl.kv_dtype)
            qr = to_host(q[b:b + 1, g * G:(g + 1) * G].contiguous(), wl.kv_dtype)
        ir = np.ascontiguousarray(idx[g:g + 1], np.int32)
        ref_lab = oracle.build_label(kr, wl.kv_dtype, wl.label_dtype, ir, wl.s)
        if wl.label_dtype == "int4":
            got = (lab[b:b + 1, g:g + 1].cpu().numpy(), to_host(sc[b:b + 1, g:g + 1], "bf16"),
                   to_host(ze[b:b + 1, g:g + 1], "bf16"))
            for a, b_ in zip(got, ref_lab):
                assert np.array_equal(a, b_)
        else:
            assert np.array_equal(to_host(lab[b:b + 1, g:g + 1].contiguous(), wl.kv_dtype), ref_lab)
        _, sel_ref, s_ref = oracle.sparse_decode(qr, kr, vr, wl.kv_dtype, ref_lab, wl.label_dtype, ir,
                                                 wl.s, wl.topk)
        check_scores(scores[b, g].cpu().numpy()[None], s_ref[0, 0][None])
        sg = sel[b, g].cpu().numpy()[None]
        check_selection(sg, sel_ref[0], s_ref[0], wl.topk, wl.s)
        o = oracle.attention(qr, kr, vr, wl.kv_dtype, sg[None], 1)
        err = np.abs(out[b, g * G:(g + 1) * G].cpu().numpy() - o[0]).max()
        assert err <= OUT_ATOL, (b, g, err)
    # properties at every row: exactly min(k, s) distinct ascending in-range tokens
    sa = sel.cpu().numpy().reshape(-1, wl.topk)
    assert np.all(np.diff(sa, axis=1) > 0) and sa.min() >= 0 and sa.max() < wl.s
    assert torch.isfinite(out).all()


# Rows of the 32-channel layer (1024 one-CTA rows): both ends, both sides of
# the staggered first wave's halves (CTAs 0-147 and 148-295 on 148 SMs), the
# first rows of the later waves, and the middle.
_C2_ROWS = [divmod(r, 32) for r in (0, 1, 147, 148, 149, 295, 296, 297, 511, 512, 700, 1022, 1023)]


@pytest.mark.parametrize("i,rows", [
    (0, None),
    (1, "all"),
    (2, _C2_ROWS),
    (3, "all"),
    (4, [(0, 0), (0, 1), (0, 15), (0, 16), (0, 30), (0, 31)]),
])
def test_full_size_configs(i, rows):
    """Every workload at its full size against the oracle: every row of the
    Llama-2-7B and GQA layers; on the two multi-GB ones, rows spread over the
    launch (first and last, both halves of the staggered first wave, later
    waves, the middle). Scores, selection and output row by row; label bits
    of each checked row."""
    _full_config(i, rows)


@pytest.mark.parametrize("i,rows", [
    (1, [(0, 0), (5, 9)]),
    (3, [(1, 2)]),
    (4, [(0, 5)]),
])
def test_int4_labels_at_bf16_label_shapes(i, rows):
    """The 4-bit label cache (16 channels: 8 payload bytes + fp16 scale and
    zero per token) on the Llama-2-7B, GQA and 256K shapes."""
    _full_config(i, rows, label_dtype="int4")


# ------------------------------------------------------- fused decode step

@pytest.mark.parametrize("kv,label,d,c,hq,hkv,s,topk,cluster", [
    ("bf16", "bf16", 128, 16, 8, 4, 3001, 200, 0),
    ("bf16", "bf16", 128, 16, 8, 4, 3001, 200, 4),
    ("bf16", "int4", 128, 32, 4, 4, 2500, 160, 0),
    ("bf16", "int4", 128, 32, 4, 4, 2500, 160, 16),
    ("f32", "f32", 64, 8, 4, 2, 777, 50, 2),
    ("f32", "int4", 64, 16, 2, 2, 300, 400, 0),   # k >= s: select all
])
def test_decode_step_equals_append_then_decode(kv, label, d, c, hq, hkv, s, topk, cluster):
    """ds_decode_step = ds_append_label(s - 1) + ds_sparse_decode, bit for bit,
    and it matches the oracle."""
    wl = synth.custom(b=2, hq=hq, hkv=hkv, d=d, s=s, c=c, topk=topk, kv_dtype=kv, label_dtype=label,
                      n_outlier=min(16, c), outlier_scale=6.0, index=73)
    di = synth.decode_inputs(wl, s_cap=s + 5)
    idx = _idx_random(wl, 7)
    qd, kd, vd = (to_dev(x, kv) for x in (di.q, di.k, di.v))
    idxd = torch.from_numpy(idx).cuda()
    lab1, sc1, ze1 = _gpu_label(kd, idxd, s - 1, wl)      # prefill of s - 1 tokens only
    lab2, sc2, ze2 = _gpu_label(kd, idxd, s, wl)          # prefill of all s tokens
    ds.set_cluster(cluster)
    try:
        sel1 = torch.full((wl.b, hkv, topk), -7, dtype=torch.int32, device="cuda")
        sel2 = sel1.clone()
        s1 = torch.zeros((wl.b, hkv, s), dtype=torch.float32, device="cuda")
        s2 = s1.clone()
        o1 = ds.decode_step(qd, kd, vd, lab1, idxd, s, topk, lscale=sc1, lzero=ze1, sel_out=sel1, score_out=s1)
        o2 = ds.sparse_decode(qd, kd, vd, lab2, idxd, s, topk, lscale=sc2, lzero=ze2, sel_out=sel2, score_out=s2)
        torch.cuda.synchronize()
    finally:
        ds.set_cluster(0)
    assert torch.equal(lab1, lab2)
    if sc1 is not None:
        assert torch.equal(sc1, sc2) and torch.equal(ze1, ze2)
    assert torch.equal(s1, s2) and torch.equal(sel1, sel2) and torch.equal(o1, o2)
    ref_label = oracle.build_label(di.k, kv, label, idx, s)
    got = _host_label(lab1, sc1, ze1, wl)
    if label == "int4":
        for a, b_ in zip(got, ref_label):
            assert np.array_equal(a, b_)
    else:
        assert np.array_equal(got, ref_label)
    _, sel_ref, s_ref = oracle.sparse_decode(di.q, di.k, di.v, kv, ref_label, label, idx, s, topk)
    check_scores(s1.cpu().numpy(), s_ref)
    sg = sel1.cpu().numpy()
    check_selection(sg.reshape(-1, topk), sel_ref.reshape(-1, topk), s_ref.reshape(-1, s), topk, s)
    o_ref = oracle.attention(di.q, di.k, di.v, kv, sg, hkv)
    assert np.abs(o1.cpu().numpy() - o_ref).max() <= OUT_ATOL


@pytest.mark.parametrize("cluster,s,topk", [(1, 600, 100), (1, 3000, 700), (2, 3000, 700), (1, 2048, 1)])
def test_exact_ties_small_buckets(cluster, s, topk):
    """Integer label values make many exactly tied scores with small 16-bit
    buckets (the in-bucket rank path for single-CTA rows, radix passes
    otherwise); the selection must match the oracle's lowest-index rule."""
    wl = synth.custom(b=1, hq=2, hkv=2, d=64, s=s, c=8, topk=topk, index=74)
    di = synth.decode_inputs(wl)
    r = np.random.default_rng(6)
    di.k[:] = np.float32(r.integers(-8, 9, size=di.k.shape))
    q = np.ones((1, 2, 64), np.float32)
    idx = np.tile(np.arange(8, dtype=np.int32), (2, 1))
    qd, kd, vd = to_dev(q, "f32"), to_dev(di.k, "f32"), to_dev(di.v, "f32")
    idxd = torch.from_numpy(idx).cuda()
    lab, _, _ = _gpu_label(kd, idxd, wl.s, wl)
    ds.set_cluster(cluster)
    try:
        sel = torch.empty((1, 2, topk), dtype=torch.int32, device="cuda")
        out = ds.sparse_decode(qd, kd, vd, lab, idxd, wl.s, topk, sel_out=sel)
        torch.cuda.synchronize()
    finally:
        ds.set_cluster(0)
    ref_lab = oracle.label_copy(di.k, "f32", idx, wl.s)
    _, sel_ref, _ = oracle.sparse_decode(q, di.k, di.v, "f32", ref_lab, "f32", idx, wl.s, topk)
    assert np.array_equal(sel.cpu().numpy(), sel_ref)
    o_ref = oracle.attention(q, di.k, di.v, "f32", sel_ref, 2)
    assert np.abs(out.cpu().numpy() - o_ref).max() <= OUT_ATOL
