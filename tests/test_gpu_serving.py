"""Serving-shaped variants of the CUDA path, against the CPU oracle:

- per-batch-entry sequence lengths (ds_decode_step_varlen), each row checked
  against the oracle run on that entry alone with its own length, including
  rows short enough that every token is attended, and the threshold rule for
  short entries (per entry, or for the whole batch as SGLang states it);
- key/value caches in pinned host memory read by the kernels over the host
  link (Double Sparsity's offloading mode), bit-identical to device caches;
- paged K/V pools with a block table, bit-identical to the dense layout;
- the decode step that writes the new token's K/V rows itself;
- the channel criteria of ds_calibrate_channels_criterion (Q-, K-, QK-outlier,
  chunked QK norm, LeanK ratio): channel indices bit-exact.
"""

import numpy as np
import pytest

import oracle
import synth
from dshelp import OUT_ATOL, check_scores, check_selection, to_dev, to_host

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


def _label_alloc(kd, wl):
    lab, sc, ze = ds.new_label_cache(kd, wl.c, int4=wl.label_dtype == "int4")
    lab.zero_()
    if sc is not None:
        sc.zero_(); ze.zero_()
    return lab, sc, ze


def _sl(t, b):
    return None if t is None else t[b:b + 1]


def _host_label_row(lab, sc, ze, wl, b):
    if wl.label_dtype == "int4":
        return (lab[b:b + 1].cpu().numpy(), to_host(sc[b:b + 1], "bf16"), to_host(ze[b:b + 1], "bf16"))
    return to_host(lab[b:b + 1].contiguous(), wl.kv_dtype)


# --------------------------------------------------- per-entry lengths

VARLEN_CASES = [
    # kv, label, d, c, hq, hkv, s_max, topk, seq_lens, cluster
    ("f32", "f32", 64, 8, 4, 2, 3000, 256, [3000, 1700, 257, 100], 0),
    ("f32", "f32", 64, 8, 4, 2, 3000, 256, [3000, 1700, 257, 100], 4),
    ("bf16", "bf16", 128, 16, 8, 8, 5000, 300, [4999, 1, 300, 2047], 0),
    ("bf16", "int4", 128, 32, 8, 2, 4096, 512, [513, 4096, 64, 3333], 2),
    ("bf16", "bf16", 128, 16, 4, 4, 2000, 64, [2000, 65, 1999, 1000], 1),
]


@pytest.mark.parametrize("kv,label,d,c,hq,hkv,s_max,topk,seq_lens,cluster", VARLEN_CASES)
def test_varlen_rows_match_oracle_per_entry(kv, label, d, c, hq, hkv, s_max, topk, seq_lens, cluster):
    """Entry b attends its own first seq_lens[b] tokens: label row
    seq_lens[b] - 1 is appended, scores, selection and output equal the
    oracle's decode step on that entry alone, and nothing past the entry's
    length is written."""
    b = len(seq_lens)
    s_cap = s_max + 8
    wl = synth.custom(b=b, hq=hq, hkv=hkv, d=d, s=s_max, c=c, topk=topk, kv_dtype=kv, label_dtype=label,
                      n_outlier=min(16, c), outlier_scale=6.0, index=81)
    di = synth.decode_inputs(wl, s_cap=s_cap)
    idx = _idx_random(wl, 9)
    qd, kd, vd = (to_dev(x, kv) for x in (di.q, di.k, di.v))
    idxd = torch.from_numpy(idx).cuda()
    lab, sc, ze = _label_alloc(kd, wl)
    for bb, sb in enumerate(seq_lens):            # prefill of each entry's first sb - 1 tokens
        if sb > 1:
            ds.build_label_cache(kd[bb:bb + 1], idxd, sb - 1, lab[bb:bb + 1], _sl(sc, bb), _sl(ze, bb))
    lens = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    sel = torch.full((b, hkv, topk), -7, dtype=torch.int32, device="cuda")
    scores = torch.full((b, hkv, s_max), 12345.0, dtype=torch.float32, device="cuda")
    ds.set_cluster(cluster)
    try:
        out = ds.decode_step_varlen(qd, kd, vd, lab, idxd, lens, s_max, topk, lscale=sc, lzero=ze,
                                    sel_out=sel, score_out=scores)
        torch.cuda.synchronize()
    finally:
        ds.set_cluster(0)
    out_h, sel_h, sc_h = out.cpu().numpy(), sel.cpu().numpy(), scores.cpu().numpy()
    for bb, sb in enumerate(seq_lens):
        kb = np.ascontiguousarray(di.k[bb:bb + 1])
        vb = np.ascontiguousarray(di.v[bb:bb + 1])
        qb = np.ascontiguousarray(di.q[bb:bb + 1])
        ref_label = oracle.build_label(kb, kv, label, idx, sb)
        got = _host_label_row(lab, sc, ze, wl, bb)
        if label == "int4":
            for a, r in zip(got, ref_label):
                assert np.array_equal(a, r), f"entry {bb}: 4-bit label rows differ"
        else:
            assert np.array_equal(got, ref_label), f"entry {bb}: label rows differ"
        _, sel_ref, s_ref = oracle.sparse_decode(qb, kb, vb, kv, ref_label, label, idx, sb, topk)
        check_scores(sc_h[bb:bb + 1, :, :sb], s_ref)
        assert np.all(sc_h[bb, :, sb:] == 12345.0), f"entry {bb}: scores written past its length"
        check_selection(sel_h[bb].reshape(-1, topk), sel_ref.reshape(-1, topk), s_ref.reshape(-1, sb),
                        topk, sb)
        if sb <= topk:
            assert np.array_equal(sel_h[bb], sel_ref[0]), f"entry {bb}: all-token selection"
        o_ref = oracle.attention(qb, kb, vb, kv, sel_h[bb:bb + 1], hkv)
        err = np.abs(out_h[bb:bb + 1] - o_ref).max()
        assert err <= OUT_ATOL, f"entry {bb}: output max-abs error {err}"


def _expected_all_tokens(seq_lens, topk, threshold, rule):
    """Which entries attend every token (the SGLang threshold rule of the
    Double Sparsity page, per entry or for the whole batch)."""
    if rule == ds.DS_FALLBACK_BATCH:
        whole = max(seq_lens) < threshold or min(seq_lens) < topk
        return [whole or sb <= topk for sb in seq_lens]
    return [sb <= topk or sb < threshold for sb in seq_lens]


@pytest.mark.parametrize("seq_lens,threshold,rule", [
    ([3000, 1700, 900, 100], 1000, ds.DS_FALLBACK_PER_ENTRY),
    ([3000, 1700, 900, 200], 0, ds.DS_FALLBACK_BATCH),      # shortest < topk: the batch goes dense
    ([3000, 1700, 900, 300], 3500, ds.DS_FALLBACK_BATCH),   # longest < threshold: dense
    ([3000, 1700, 900, 300], 2000, ds.DS_FALLBACK_BATCH),   # neither: every entry sparse
])
def test_fallback_rule(seq_lens, threshold, rule):
    kv, label, d, c, hq, hkv, s_max, topk = "bf16", "bf16", 128, 16, 8, 4, 3000, 256
    b = len(seq_lens)
    wl = synth.custom(b=b, hq=hq, hkv=hkv, d=d, s=s_max, c=c, topk=topk, kv_dtype=kv, label_dtype=label,
                      n_outlier=16, outlier_scale=6.0, index=84)
    di = synth.decode_inputs(wl, s_cap=s_max + 8)
    idx = _idx_random(wl, 12)
    qd, kd, vd = (to_dev(x, kv) for x in (di.q, di.k, di.v))
    idxd = torch.from_numpy(idx).cuda()
    lab, sc, ze = _label_alloc(kd, wl)
    for bb, sb in enumerate(seq_lens):
        ds.build_label_cache(kd[bb:bb + 1], idxd, sb - 1, lab[bb:bb + 1])
    lens = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    sel = torch.full((b, hkv, topk), -7, dtype=torch.int32, device="cuda")
    out = ds.decode_step_varlen(qd, kd, vd, lab, idxd, lens, s_max, topk, sel_out=sel,
                                sparse_threshold=threshold, fallback=rule)
    torch.cuda.synchronize()
    out_h, sel_h = out.cpu().numpy(), sel.cpu().numpy()
    for bb, (sb, dense) in enumerate(zip(seq_lens, _expected_all_tokens(seq_lens, topk, threshold, rule))):
        kb, vb, qb = (np.ascontiguousarray(x[bb:bb + 1]) for x in (di.k, di.v, di.q))
        ref_label = oracle.build_label(kb, kv, label, idx, sb)
        if dense:
            every = np.broadcast_to(np.arange(sb, dtype=np.int32), (1, hkv, sb)).copy()
            o_ref = oracle.attention(qb, kb, vb, kv, every, hkv)
            want = np.full((hkv, topk), -1, np.int32)
            if sb <= topk:
                want[:, :sb] = np.arange(sb)
            assert np.array_equal(sel_h[bb], want), f"entry {bb}: sel_out of an all-token row"
        else:
            _, sel_ref, s_ref = oracle.sparse_decode(qb, kb, vb, kv, ref_label, label, idx, sb, topk)
            check_selection(sel_h[bb].reshape(-1, topk), sel_ref.reshape(-1, topk), s_ref.reshape(-1, sb),
                            topk, sb)
            o_ref = oracle.attention(qb, kb, vb, kv, sel_h[bb:bb + 1], hkv)
        err = np.abs(out_h[bb:bb + 1] - o_ref).max()
        assert err <= OUT_ATOL, f"entry {bb} (all tokens: {dense}): output max-abs error {err}"


def test_varlen_uniform_lengths_equal_decode_step():
    """All entries at s_max: bit-identical to ds_decode_step."""
    wl = synth.custom(b=3, hq=8, hkv=4, d=128, s=4000, c=16, topk=256, kv_dtype="bf16",
                      label_dtype="bf16", n_outlier=16, outlier_scale=6.0, index=82)
    di = synth.decode_inputs(wl, s_cap=4008)
    idx = _idx_random(wl, 10)
    qd, kd, vd = (to_dev(x, "bf16") for x in (di.q, di.k, di.v))
    idxd = torch.from_numpy(idx).cuda()
    lab1, _, _ = _label_alloc(kd, wl)
    ds.build_label_cache(kd, idxd, wl.s - 1, lab1)
    lab2 = lab1.clone()
    lens = torch.full((wl.b,), wl.s, dtype=torch.int32, device="cuda")
    sel1 = torch.empty((wl.b, wl.hkv, wl.topk), dtype=torch.int32, device="cuda")
    sel2 = torch.empty_like(sel1)
    o1 = ds.decode_step(qd, kd, vd, lab1, idxd, wl.s, wl.topk, sel_out=sel1)
    o2 = ds.decode_step_varlen(qd, kd, vd, lab2, idxd, lens, wl.s, wl.topk, sel_out=sel2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(sel1, sel2) and torch.equal(lab1, lab2)


def test_varlen_rejects_missing_lengths():
    q = torch.zeros((1, 2, 64), device="cuda")
    k = torch.zeros((1, 2, 64, 64), device="cuda")
    lab = torch.zeros((1, 2, 64, 8), device="cuda")
    idx = torch.zeros((2, 8), dtype=torch.int32, device="cuda")
    out = torch.zeros((1, 2, 64), device="cuda")
    lens = torch.full((1,), 64, dtype=torch.int32, device="cuda")

    def call(seq_lens, threshold=0, rule=ds.DS_FALLBACK_PER_ENTRY):
        return ds.lib().ds_decode_step_varlen(q.data_ptr(), k.data_ptr(), k.data_ptr(), ds.DS_F32, lab.data_ptr(),
                                              ds.DS_F32, None, None, idx.data_ptr(), seq_lens, threshold, rule,
                                              1, 2, 2, 64, 64, 64, 8, 16, 0.0, out.data_ptr(), ds.DS_F32, None,
                                              None, torch.cuda.current_stream().cuda_stream)
    assert call(None) == ds.DS_ERR_INVALID_ARG
    assert call(lens.data_ptr(), threshold=-1) == ds.DS_ERR_INVALID_ARG
    assert call(lens.data_ptr(), rule=5) == ds.DS_ERR_INVALID_ARG


# ------------------------------------------------------ offloaded caches

@pytest.mark.parametrize("kv,label", [("bf16", "bf16"), ("f32", "int4"), ("bf16", "int4")])
def test_host_resident_kv_equals_device_kv(kv, label):
    """Key/value caches in pinned host memory: the label build, the fused
    decode step and dense decode give the same bits as with device caches."""
    wl = synth.custom(b=2, hq=8, hkv=2, d=128, s=6000, c=16, topk=384, kv_dtype=kv, label_dtype=label,
                      n_outlier=16, outlier_scale=6.0, index=83)
    di = synth.decode_inputs(wl, s_cap=6016)
    idx = _idx_random(wl, 11)
    qd, kd, vd = (to_dev(x, kv) for x in (di.q, di.k, di.v))
    kh, vh = kd.cpu().pin_memory(), vd.cpu().pin_memory()
    assert kh.is_pinned() and not kh.is_cuda
    idxd = torch.from_numpy(idx).cuda()
    labd, scd, zed = _label_alloc(kd, wl)
    labh, sch, zeh = _label_alloc(kd, wl)
    ds.build_label_cache(kd, idxd, wl.s - 1, labd, scd, zed)
    ds.build_label_cache(kh, idxd, wl.s - 1, labh, sch, zeh)
    seld = torch.empty((wl.b, wl.hkv, wl.topk), dtype=torch.int32, device="cuda")
    selh = torch.empty_like(seld)
    od = ds.decode_step(qd, kd, vd, labd, idxd, wl.s, wl.topk, lscale=scd, lzero=zed, sel_out=seld)
    oh = ds.decode_step(qd, kh, vh, labh, idxd, wl.s, wl.topk, lscale=sch, lzero=zeh, sel_out=selh)
    dd = ds.dense_decode(qd, kd, vd, wl.s)
    dh = ds.dense_decode(qd, kh, vh, wl.s)
    torch.cuda.synchronize()
    assert torch.equal(labd, labh)
    if scd is not None:
        assert torch.equal(scd, sch) and torch.equal(zed, zeh)
    assert torch.equal(seld, selh) and torch.equal(od, oh) and torch.equal(dd, dh)
    ref_label = oracle.build_label(di.k, kv, label, idx, wl.s)
    _, sel_ref, s_ref = oracle.sparse_decode(di.q, di.k, di.v, kv, ref_label, label, idx, wl.s, wl.topk)
    sg = selh.cpu().numpy()
    check_selection(sg.reshape(-1, wl.topk), sel_ref.reshape(-1, wl.topk), s_ref.reshape(-1, wl.s),
                    wl.topk, wl.s)
    o_ref = oracle.attention(di.q, di.k, di.v, kv, sg, wl.hkv)
    assert np.abs(oh.cpu().numpy() - o_ref).max() <= OUT_ATOL


def test_unpinned_host_cache_is_rejected():
    k = torch.zeros((1, 2, 64, 64))
    q = torch.zeros((1, 2, 64), device="cuda")
    lab = torch.zeros((1, 2, 64, 8), device="cuda")
    idx = torch.zeros((2, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        ds.sparse_decode(q, k, k, lab, idx, 64, 16)


# ---------------------------------------------------- channel criteria

CRITERIA = [("leank", ds.DS_CRIT_LEANK_RATIO, 0), ("q", ds.DS_CRIT_Q_OUTLIER, 0),
            ("k", ds.DS_CRIT_K_OUTLIER, 0), ("qk", ds.DS_CRIT_QK_OUTLIER, 0),
            ("qk_chunked", ds.DS_CRIT_QK_CHUNKED, 100), ("qk_chunked", ds.DS_CRIT_QK_CHUNKED, 1)]


def _calib_case(wl_i):
    wl = synth.workload(wl_i)
    if wl_i:
        wl = synth.custom(b=1, hq=wl.hq, hkv=wl.hkv, d=wl.d, s=1024, c=wl.c, kv_dtype=wl.kv_dtype,
                          label_dtype=wl.label_dtype, n_outlier=wl.n_outlier,
                          outlier_scale=wl.outlier_scale, index=wl.index, calib_samples=2,
                          calib_w=32, calib_s=1024)
    return wl, synth.calib_inputs(wl)


@pytest.mark.parametrize("name,crit,chunk", CRITERIA)
@pytest.mark.parametrize("wl_i", [0, 3])
def test_criteria_match_oracle(wl_i, name, crit, chunk):
    wl, ci = _calib_case(wl_i)
    sc_ref, i_ref = oracle.calibrate_criterion(ci.q_win, ci.k, wl.kv_dtype, wl.c, name, chunk)
    qw, kc = to_dev(ci.q_win, wl.kv_dtype), to_dev(ci.k, wl.kv_dtype)
    idx, score = ds.calibrate_channels_criterion(qw, kc, wl.c, crit, chunk)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), i_ref)
    assert np.array_equal(i_ref, ci.outliers)     # planted in Q and K: every criterion finds them
    rtol = 2e-5 if name == "leank" else 1e-6
    np.testing.assert_allclose(score.cpu().numpy(), sc_ref, rtol=rtol, atol=1e-7)


def test_criteria_separate_query_and_key_outliers_on_gpu():
    """Outliers planted only in K (resp. Q) are found by the K (resp. Q) criterion."""
    r = np.random.default_rng(24)
    q = r.standard_normal((2, 4, 16, 64)).astype(np.float32)
    k = r.standard_normal((2, 2, 700, 64)).astype(np.float32)
    kch, qch = [3, 9, 17, 30, 41, 50, 58, 63], [1, 12, 20, 25, 33, 44, 47, 60]
    k[..., kch] *= 8
    q[..., qch] *= 8
    qd, kd = torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda()
    ik, _ = ds.calibrate_channels_criterion(qd, kd, 8, ds.DS_CRIT_K_OUTLIER)
    iq, _ = ds.calibrate_channels_criterion(qd, kd, 8, ds.DS_CRIT_Q_OUTLIER)
    torch.cuda.synchronize()
    assert ik.cpu().numpy().tolist() == [kch, kch]
    assert iq.cpu().numpy().tolist() == [qch, qch]
    for name, crit in (("k", ds.DS_CRIT_K_OUTLIER), ("q", ds.DS_CRIT_Q_OUTLIER)):
        _, i_ref = oracle.calibrate_criterion(q, k, "f32", 8, name)
        i_gpu, _ = ds.calibrate_channels_criterion(qd, kd, 8, crit)
        assert np.array_equal(i_gpu.cpu().numpy(), i_ref)


def test_criteria_reject_bad_arguments():
    q = torch.zeros((1, 2, 4, 64), device="cuda")
    k = torch.zeros((1, 2, 32, 64), device="cuda")
    with pytest.raises(ds.DSError):
        ds.calibrate_channels_criterion(q, k, 8, ds.DS_CRIT_QK_CHUNKED, 0)
    with pytest.raises(ds.DSError):
        ds.calibrate_channels_criterion(q, k, 8, 7)


# --------------------------------------------------------------- paged K/V

def _to_pool(x, page, seed):
    """Scatter a dense cache [B, Hkv, S_cap, D] into a pool [num_blocks, Hkv,
    page, D] of shuffled blocks (plus unused ones); returns (pool, table)."""
    b, hkv, s_cap, d = x.shape
    mb = (s_cap + page - 1) // page
    nblk = b * mb + 5
    perm = torch.from_numpy(np.random.default_rng(seed).permutation(nblk)[: b * mb].astype(np.int32))
    table = perm.view(b, mb).cuda()
    pool = torch.zeros((nblk, hkv, page, d), dtype=x.dtype, device=x.device)
    pad = torch.zeros((b, hkv, mb * page, d), dtype=x.dtype, device=x.device)
    pad[:, :, :s_cap] = x
    blocks = pad.view(b, hkv, mb, page, d).permute(0, 2, 1, 3, 4).reshape(b * mb, hkv, page, d)
    pool[perm.long().cuda()] = blocks
    return pool, table


@pytest.mark.parametrize("kv,label,page,varlen,cluster", [
    ("bf16", "bf16", 16, False, 0), ("bf16", "int4", 64, True, 0), ("f32", "f32", 8, True, 2),
    ("bf16", "bf16", 1, False, 4), ("bf16", "bf16", 256, True, 1)])
def test_paged_kv_equals_dense_layout(kv, label, page, varlen, cluster):
    """The paged pools give the same bits as the dense caches holding the
    same values: label build, decode step (per-entry lengths too)."""
    b, hq, hkv, d, c, s, topk = 3, 8, 4, 128, 16 if label != "int4" else 32, 3000, 256
    if kv == "f32":
        d, c = 64, 8
    wl = synth.custom(b=b, hq=hq, hkv=hkv, d=d, s=s, c=c, topk=topk, kv_dtype=kv, label_dtype=label,
                      n_outlier=min(16, c), outlier_scale=6.0, index=85)
    di = synth.decode_inputs(wl, s_cap=s + 8)
    idx = _idx_random(wl, 13)
    qd, kd, vd = (to_dev(x, kv) for x in (di.q, di.k, di.v))
    idxd = torch.from_numpy(idx).cuda()
    kp, table = _to_pool(kd, page, 5)
    vp, table_v = _to_pool(vd, page, 5)
    assert torch.equal(table, table_v)
    lab1, sc1, ze1 = _label_alloc(kd, wl)
    lab2, sc2, ze2 = _label_alloc(kd, wl)
    ds.build_label_cache(kd, idxd, s - 1, lab1, sc1, ze1)
    ds.build_label_cache_paged(kp, idxd, table, s - 1, lab2, sc2, ze2)
    torch.cuda.synchronize()
    assert torch.equal(lab1, lab2)
    if sc1 is not None:
        assert torch.equal(sc1, sc2) and torch.equal(ze1, ze2)
    lens = torch.tensor([s, 1700, 200][:b], dtype=torch.int32, device="cuda") if varlen else None
    sel1 = torch.full((b, hkv, topk), -7, dtype=torch.int32, device="cuda")
    sel2 = sel1.clone()
    ds.set_cluster(cluster)
    try:
        if varlen:
            o1 = ds.decode_step_varlen(qd, kd, vd, lab1, idxd, lens, s, topk, lscale=sc1, lzero=ze1, sel_out=sel1)
        else:
            o1 = ds.decode_step(qd, kd, vd, lab1, idxd, s, topk, lscale=sc1, lzero=ze1, sel_out=sel1)
        o2 = ds.decode_step_paged(qd, kp, vp, lab2, idxd, table, s, topk, seq_lens=lens, lscale=sc2, lzero=ze2,
                                  sel_out=sel2)
        torch.cuda.synchronize()
    finally:
        ds.set_cluster(0)
    assert torch.equal(lab1, lab2) and torch.equal(sel1, sel2) and torch.equal(o1, o2)
    if not varlen:      # and the oracle agrees
        ref_label = oracle.build_label(di.k, kv, label, idx, s)
        _, sel_ref, s_ref = oracle.sparse_decode(di.q, di.k, di.v, kv, ref_label, label, idx, s, topk)
        sg = sel2.cpu().numpy()
        check_selection(sg.reshape(-1, topk), sel_ref.reshape(-1, topk), s_ref.reshape(-1, s), topk, s)
        o_ref = oracle.attention(di.q, di.k, di.v, kv, sg, hkv)
        assert np.abs(o2.cpu().numpy() - o_ref).max() <= OUT_ATOL


def test_paged_rejects_bad_tables():
    q = torch.zeros((1, 2, 64), device="cuda")
    pool = torch.zeros((4, 2, 16, 64), device="cuda")
    lab = torch.zeros((1, 2, 64, 8), device="cuda")
    idx = torch.zeros((2, 8), dtype=torch.int32, device="cuda")
    table = torch.zeros((1, 4), dtype=torch.int32, device="cuda")
    with pytest.raises(ds.DSError):      # 4 blocks of 16 cannot hold 65 tokens
        ds.decode_step_paged(q, pool, pool, torch.zeros((1, 2, 80, 8), device="cuda"), idx, table, 65, 16)
    with pytest.raises(ds.DSError):      # page size not a power of two
        ds.decode_step_paged(q, torch.zeros((4, 2, 12, 64), device="cuda"), torch.zeros((4, 2, 12, 64), device="cuda"),
                             lab, idx, table, 40, 16)
    ds.decode_step_paged(q, pool, pool, lab, idx, table, 64, 16)   # valid
    torch.cuda.synchronize()


# -------------------------------------------- new token's rows in the launch

@pytest.mark.parametrize("kv,label,cluster", [("bf16", "bf16", 0), ("bf16", "int4", 4), ("f32", "f32", 2),
                                              ("bf16", "bf16", 16)])
def test_decode_step_kv_equals_copy_then_step(kv, label, cluster):
    """ds_decode_step_kv writes the new token's K/V rows into the caches and
    then runs the step: the same bits as copying them in and calling
    ds_decode_step (caches, label cache, selection, output)."""
    b, hq, hkv, d, c, s, topk = 3, 8, 4, 128 if kv == "bf16" else 64, 16, 5000, 300
    if label == "int4":
        c = 32
    if kv == "f32":
        c = 8
    wl = synth.custom(b=b, hq=hq, hkv=hkv, d=d, s=s, c=c, topk=topk, kv_dtype=kv, label_dtype=label,
                      n_outlier=min(16, c), outlier_scale=6.0, index=86)
    di = synth.decode_inputs(wl, s_cap=s + 8)
    idx = _idx_random(wl, 14)
    qd, kd, vd = (to_dev(x, kv) for x in (di.q, di.k, di.v))
    idxd = torch.from_numpy(idx).cuda()
    k_new, v_new = kd[:, :, s - 1].clone(), vd[:, :, s - 1].clone()
    k1, v1 = kd.clone(), vd.clone()
    k1[:, :, s - 1] = 0
    v1[:, :, s - 1] = 0
    lab1, sc1, ze1 = _label_alloc(kd, wl)
    ds.build_label_cache(kd, idxd, s - 1, lab1, sc1, ze1)
    lab2 = lab1.clone()
    sc2, ze2 = (None, None) if sc1 is None else (sc1.clone(), ze1.clone())
    sel1 = torch.empty((b, hkv, topk), dtype=torch.int32, device="cuda")
    sel2 = torch.empty_like(sel1)
    ds.set_cluster(cluster)
    try:
        o1 = ds.decode_step_kv(qd, k_new, v_new, k1, v1, lab1, idxd, s, topk, lscale=sc1, lzero=ze1, sel_out=sel1)
        o2 = ds.decode_step(qd, kd, vd, lab2, idxd, s, topk, lscale=sc2, lzero=ze2, sel_out=sel2)
        torch.cuda.synchronize()
    finally:
        ds.set_cluster(0)
    assert torch.equal(k1, kd) and torch.equal(v1, vd)
    assert torch.equal(lab1, lab2) and torch.equal(sel1, sel2) and torch.equal(o1, o2)
    if sc1 is not None:
        assert torch.equal(sc1, sc2) and torch.equal(ze1, ze2)


@pytest.mark.parametrize("kv,label,cluster,out_dtype", [("bf16", "bf16", 0, "bf16"), ("bf16", "int4", 4, "f32"),
                                                        ("f32", "f32", 2, "f32")])
def test_decode_step_kv_from_host_buffers(kv, label, cluster, out_dtype):
    """A decode step straight from pinned host buffers: the kernel reads the
    query and the new token's K/V rows over the host link and writes the
    output there, giving the same bits as the step on device copies."""
    b, hq, hkv, d, c, s, topk = 2, 8, 4, 128 if kv == "bf16" else 64, 16, 3000, 200
    if label == "int4":
        c = 32
    if kv == "f32":
        c = 8
    wl = synth.custom(b=b, hq=hq, hkv=hkv, d=d, s=s, c=c, topk=topk, kv_dtype=kv, label_dtype=label,
                      n_outlier=min(16, c), outlier_scale=6.0, index=87)
    di = synth.decode_inputs(wl, s_cap=s + 8)
    idxd = torch.from_numpy(_idx_random(wl, 15)).cuda()
    qd, kd, vd = (to_dev(x, kv) for x in (di.q, di.k, di.v))
    k_new, v_new = kd[:, :, s - 1].clone(), vd[:, :, s - 1].clone()
    odt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
    caches = []
    for _ in range(2):
        k1, v1 = kd.clone(), vd.clone()
        k1[:, :, s - 1] = 0
        v1[:, :, s - 1] = 0
        lab, sc, ze = _label_alloc(kd, wl)
        ds.build_label_cache(kd, idxd, s - 1, lab, sc, ze)
        caches.append((k1, v1, lab, sc, ze))
    qh, knh, vnh = (t.cpu().pin_memory() for t in (qd, k_new, v_new))
    oh = torch.full((b, hq, d), float("nan"), dtype=odt).pin_memory()
    od = torch.empty((b, hq, d), dtype=odt, device="cuda")
    ds.set_cluster(cluster)
    try:
        k1, v1, lab, sc, ze = caches[0]
        ds.decode_step_kv(qh, knh, vnh, k1, v1, lab, idxd, s, topk, lscale=sc, lzero=ze, out=oh)
        k2, v2, lab2, sc2, ze2 = caches[1]
        ds.decode_step_kv(qd, k_new, v_new, k2, v2, lab2, idxd, s, topk, lscale=sc2, lzero=ze2, out=od)
        torch.cuda.synchronize()
    finally:
        ds.set_cluster(0)
    assert torch.equal(k1, k2) and torch.equal(v1, v2) and torch.equal(lab, lab2)
    assert torch.equal(oh, od.cpu())
    with pytest.raises(ValueError):  # pageable host memory is refused
        ds.decode_step_kv(qd.cpu(), k_new, v_new, k1, v1, lab, idxd, s, topk, lscale=sc, lzero=ze, out=od)


def test_prepared_decode_step_equals_call():
    """PreparedDecodeStepKV (arguments bound once) gives the bits of
    decode_step_kv, from host buffers, and follows set_length."""
    b, hq, hkv, d, c, s, topk = 2, 8, 4, 128, 16, 2500, 128
    wl = synth.custom(b=b, hq=hq, hkv=hkv, d=d, s=s, c=c, topk=topk, kv_dtype="bf16", label_dtype="bf16",
                      n_outlier=16, outlier_scale=6.0, index=88)
    di = synth.decode_inputs(wl, s_cap=s + 8)
    idxd = torch.from_numpy(_idx_random(wl, 16)).cuda()
    qd, kd, vd = (to_dev(x, "bf16") for x in (di.q, di.k, di.v))
    outs = []
    for length in (s, s - 300):
        k_new, v_new = kd[:, :, length - 1].clone(), vd[:, :, length - 1].clone()
        runs = []
        for mode in ("call", "prepared"):
            k1, v1 = kd.clone(), vd.clone()
            lab, _, _ = _label_alloc(kd, wl)
            ds.build_label_cache(kd, idxd, length - 1, lab)
            qh, knh, vnh = (t.cpu().pin_memory() for t in (qd, k_new, v_new))
            oh = torch.zeros((b, hq, d), dtype=torch.bfloat16).pin_memory()
            if mode == "call":
                ds.decode_step_kv(qh, knh, vnh, k1, v1, lab, idxd, length, topk, out=oh)
            else:
                step = ds.PreparedDecodeStepKV(qh, knh, vnh, k1, v1, lab, idxd, s, topk, out=oh)
                step.set_length(length)
                step()
            torch.cuda.synchronize()
            runs.append((oh.clone(), lab.clone()))
        assert torch.equal(runs[0][0], runs[1][0]) and torch.equal(runs[0][1], runs[1][1])
        outs.append(runs[0][0])
    assert not torch.equal(outs[0], outs[1])
