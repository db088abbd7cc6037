"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- hand-worked values (tests/golden), closed forms, library
routines, brute force on tiny inputs, or invariants of the method -- so that a
dropped term, a wrong sign or index, or a transposed operand fails one of them.

Sources: "大模型稀疏化技术原理：Double Sparsity" (joto.ai blog), sections 离线校准
and 在线前向计算; "K通道静态性量化方法解析" (aitangshan.cn) §1.1.
"""

import itertools
import json
import os

import numpy as np
import pytest

import oracle
import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def textbook_attention(q, k, v, G, scale):
    """Dense softmax attention, written independently of the oracle:
    out[b,h] = softmax(scale * K[b,h//G] q[b,h]) V[b,h//G]."""
    b, hq, d = q.shape
    out = np.zeros((b, hq, d))
    for bb in range(b):
        for h in range(hq):
            kk, vv = k[bb, h // G], v[bb, h // G]
            logits = kk @ q[bb, h] * scale
            w = np.exp(logits - logits.max())
            out[bb, h] = (w / w.sum()) @ vv
    return out


def _f64(x, dtype):
    return synth.storage_to_f32(x, dtype).astype(np.float64)


# ------------------------------------------------------------------ pipeline

@pytest.mark.parametrize("kv_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (8, 2)])
def test_full_channels_all_tokens_is_dense_attention(kv_dtype, hq, hkv):
    """With every channel heavy (C = D) and k = S, the decode step is plain
    dense softmax attention (step 3 uses full Q/K/V over the selected tokens)."""
    wl = synth.custom(b=2, hq=hq, hkv=hkv, d=64, s=40, c=64, topk=40, kv_dtype=kv_dtype,
                      label_dtype=kv_dtype, n_outlier=4, outlier_scale=4.0, index=91)
    di = synth.decode_inputs(wl, s_cap=48)
    idx = np.tile(np.arange(wl.d, dtype=np.int32), (hkv, 1))
    lab = oracle.build_label(di.k, kv_dtype, kv_dtype, idx, wl.s)
    out, sel, _ = oracle.sparse_decode(di.q, di.k, di.v, kv_dtype, lab, kv_dtype, idx, wl.s, wl.topk)
    q, k, v = (_f64(x, kv_dtype) for x in (di.q, di.k, di.v))
    ref = textbook_attention(q, k[:, :, : wl.s], v[:, :, : wl.s], hq // hkv, 1 / np.sqrt(wl.d))
    assert np.array_equal(sel, np.tile(np.arange(wl.s), (wl.b, hkv, 1)))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_attention_over_subset_matches_dense_on_gathered_rows():
    """Attention over a selected set equals dense attention on the cache built
    from only those rows (catches a wrong token index in the gather)."""
    wl = synth.custom(b=1, hq=4, hkv=2, d=64, s=64, index=92)
    di = synth.decode_inputs(wl)
    r = np.random.default_rng(5)
    sel = np.stack([np.sort(r.choice(wl.s, 10, replace=False)) for _ in range(wl.hkv)])[None]
    out = oracle.attention(di.q, di.k, di.v, "f32", sel.astype(np.int32), wl.hkv)
    q, k, v = (_f64(x, "f32") for x in (di.q, di.k, di.v))
    ks = np.stack([k[0, g, sel[0, g]] for g in range(wl.hkv)])[None]
    vs = np.stack([v[0, g, sel[0, g]] for g in range(wl.hkv)])[None]
    np.testing.assert_allclose(out, textbook_attention(q, ks, vs, 2, 1 / 8.0), atol=1e-12)


def test_attention_invariants():
    """Equal keys give uniform weights (output = mean of V); one dominant logit
    returns that token's V; a custom sm_scale is honoured."""
    d, s = 64, 16
    r = np.random.default_rng(3)
    q = r.standard_normal((1, 1, d)).astype(np.float32)
    krow = r.standard_normal(d).astype(np.float32)
    k = np.tile(krow, (1, 1, s, 1)).astype(np.float32)
    v = r.standard_normal((1, 1, s, d)).astype(np.float32)
    sel = np.arange(s, dtype=np.int32)[None, None]
    out = oracle.attention(q, k, v, "f32", sel, 1)
    np.testing.assert_allclose(out[0, 0], v[0, 0].astype(np.float64).mean(0), atol=1e-12)
    k2 = r.standard_normal((1, 1, s, d)).astype(np.float32)
    k2[0, 0, 7] = q[0, 0] * 50
    out2 = oracle.attention(q, k2, v, "f32", sel, 1)
    np.testing.assert_allclose(out2[0, 0], v[0, 0, 7], atol=1e-9)
    # sm_scale: scaling q by a and sm_scale by 1/a leaves the output unchanged
    out3 = oracle.attention((q * 2).astype(np.float32), k2, v, "f32", sel, 1, sm_scale=0.5 / np.sqrt(d))
    np.testing.assert_allclose(out3, out2, atol=1e-12)


# ------------------------------------------------------------------- scores

@pytest.mark.parametrize("hq,hkv", [(2, 2), (8, 2)])
def test_scores_equal_masked_query_dot_keys(hq, hkv):
    """Step 2 written another way: the approximate score is the dot product of
    the group-summed query, with non-heavy channels zeroed, with the full key."""
    wl = synth.custom(b=2, hq=hq, hkv=hkv, d=64, s=33, c=8, index=93)
    di = synth.decode_inputs(wl)
    r = np.random.default_rng(11)
    idx = np.stack([np.sort(r.choice(wl.d, wl.c, replace=False)) for _ in range(hkv)]).astype(np.int32)
    lab = oracle.label_copy(di.k, "f32", idx, wl.s)
    sc = oracle.scores(di.q, "f32", oracle.label_values(lab, "f32", wl.s, wl.c), idx, hkv)
    q, k = _f64(di.q, "f32"), _f64(di.k, "f32")
    G = hq // hkv
    for bb in range(wl.b):
        for g in range(hkv):
            mask = np.zeros(wl.d)
            mask[idx[g]] = 1.0
            qsum = q[bb, g * G:(g + 1) * G].sum(0) * mask
            np.testing.assert_allclose(sc[bb, g], k[bb, g, : wl.s] @ qsum, rtol=1e-13, atol=1e-12)


def test_scores_full_channels_equal_qk():
    wl = synth.custom(b=1, hq=4, hkv=4, d=64, s=20, c=64, index=94)
    di = synth.decode_inputs(wl)
    idx = np.tile(np.arange(64, dtype=np.int32), (4, 1))
    lab = oracle.label_copy(di.k, "f32", idx, wl.s)
    sc = oracle.scores(di.q, "f32", oracle.label_values(lab, "f32", wl.s, 64), idx, 4)
    q, k = _f64(di.q, "f32"), _f64(di.k, "f32")
    np.testing.assert_allclose(sc[0], np.einsum("hd,htd->ht", q[0], k[0]), rtol=1e-13, atol=1e-12)


# -------------------------------------------------------------------- top-k

def test_topk_hand_cases():
    for case in _gold("topk_hand.json")["cases"]:
        sel = oracle.topk(np.array([case["scores"]], np.float64), case["k"])
        assert sel[0].tolist() == case["sel"], case


def test_topk_brute_force_tiny():
    """Enumerate every k-subset: exactly one has every member ranked above every
    non-member under (score desc, index asc), and it is the oracle's."""
    r = np.random.default_rng(7)
    for trial in range(60):
        s = int(r.integers(1, 9))
        k = int(r.integers(1, s + 1))
        sc = r.integers(-3, 4, size=s).astype(np.float64)  # many ties
        sel = oracle.topk(sc[None], k)[0]
        winners = []
        for sub in itertools.combinations(range(s), k):
            out = [u for u in range(s) if u not in sub]
            if all(sc[t] > sc[u] or (sc[t] == sc[u] and t < u) for t in sub for u in out):
                winners.append(list(sub))
        assert len(winners) == 1
        assert sel.tolist() == winners[0]


def test_topk_matches_library_lexsort():
    r = np.random.default_rng(8)
    sc = r.standard_normal((5, 300))
    sc[:, ::7] = 0.25  # plant ties
    sel = oracle.topk(sc, 40)
    for i in range(5):
        order = np.lexsort((np.arange(300), -sc[i]))
        assert sel[i].tolist() == sorted(order[:40].tolist())


def test_topk_planted_ranks():
    r = np.random.default_rng(9)
    perm = r.permutation(1000)
    sc = perm.astype(np.float64)[None]  # token t has rank 999 - perm[t]
    sel = oracle.topk(sc, 100)[0]
    assert sel.tolist() == sorted(np.nonzero(perm >= 900)[0].tolist())


# -------------------------------------------------------------- calibration

def test_calibration_hand_cases():
    for case in _gold("calib_hand.json")["cases"]:
        q = np.array(case["q"], np.float32)[None, None]       # [N=1, Hq=1, W, D]
        k = np.array(case["k"], np.float32)[None, None]       # [N=1, Hkv=1, S, D]
        ratio, idx = oracle.calibrate(q, k, "f32", case["c"])
        np.testing.assert_allclose(ratio[0], case["ratio"], rtol=1e-14)
        assert idx[0].tolist() == case["idx"]


def test_calibration_closed_forms():
    """r_i * ||QK^T||_F = ||Q[i]|| ||K[i]|| (rank-one closed form, also equal to
    the spectral norm of the outer product), and ||QK^T||_F^2 equals the Gram
    identity sum((Q^T Q) * (K^T K))."""
    r = np.random.default_rng(12)
    q = r.standard_normal((1, 1, 6, 5)).astype(np.float32)
    k = r.standard_normal((1, 1, 9, 5)).astype(np.float32)
    ratio, _ = oracle.calibrate(q, k, "f32", 2)
    Q, K = q[0, 0].astype(np.float64), k[0, 0].astype(np.float64)
    den_lib = np.linalg.norm(Q @ K.T, "fro")
    den_gram = np.sqrt(np.sum((Q.T @ Q) * (K.T @ K)))
    assert abs(den_lib - den_gram) < 1e-12 * den_lib
    for i in range(5):
        closed = np.linalg.norm(Q[:, i]) * np.linalg.norm(K[:, i])
        spectral = np.linalg.norm(np.outer(Q[:, i], K[:, i]), 2)
        np.testing.assert_allclose(ratio[0, i] * den_lib, closed, rtol=1e-12)
        np.testing.assert_allclose(closed, spectral, rtol=1e-12)


def test_calibration_invariants():
    """r is scale-invariant in Q and K, averaging identical samples changes
    nothing, and a GQA group behaves like one head whose window stacks the
    group's query windows."""
    r = np.random.default_rng(13)
    q = r.standard_normal((1, 2, 4, 8)).astype(np.float32)
    k = r.standard_normal((1, 1, 12, 8)).astype(np.float32)
    ra, ia = oracle.calibrate(q, k, "f32", 3)
    rb, _ = oracle.calibrate((q * 4).astype(np.float32), (k * 0.5).astype(np.float32), "f32", 3)
    np.testing.assert_allclose(ra, rb, rtol=1e-12)
    rc, _ = oracle.calibrate(np.concatenate([q, q]), np.concatenate([k, k]), "f32", 3)
    np.testing.assert_allclose(ra, rc, rtol=1e-12)
    stacked = q.reshape(1, 1, 8, 8)  # heads 0 and 1 windows stacked
    rd, idd = oracle.calibrate(stacked, k, "f32", 3)
    np.testing.assert_allclose(ra, rd, rtol=1e-12)
    assert ia.tolist() == idd.tolist()


def test_calibration_recovers_planted_outliers():
    """The pages' premise: a few channels dominate QK^T and are found offline.
    The tiny workload plants 8 channels per head (x8) in Q and K."""
    wl = synth.workload(0)
    ci = synth.calib_inputs(wl)
    _, idx = oracle.calibrate(ci.q_win, ci.k, wl.kv_dtype, wl.c)
    assert np.array_equal(idx, ci.outliers)


def test_calibration_zero_keys_give_zero_ratio():
    q = np.ones((1, 1, 2, 4), np.float32)
    k = np.zeros((1, 1, 3, 4), np.float32)
    ratio, idx = oracle.calibrate(q, k, "f32", 2)
    assert np.all(ratio == 0) and idx[0].tolist() == [0, 1]


# -------------------------------------------------------------- label cache

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_label_copy_is_gather(dtype):
    wl = synth.custom(b=2, hq=4, hkv=2, d=64, s=30, c=8, kv_dtype=dtype, label_dtype=dtype, index=95)
    di = synth.decode_inputs(wl, s_cap=37)
    r = np.random.default_rng(1)
    idx = np.stack([np.sort(r.choice(64, 8, replace=False)) for _ in range(2)]).astype(np.int32)
    lab = oracle.label_copy(di.k, dtype, idx, wl.s)
    for g in range(2):
        assert np.array_equal(lab[:, g, : wl.s], di.k[:, g, : wl.s][..., idx[g]])
    assert not lab[:, :, wl.s:].any()
    # appending token t alone reproduces the same row
    app = np.zeros_like(lab)
    app = oracle.label_copy(di.k, dtype, idx, 11, t_begin=10, label=app)
    assert np.array_equal(app[:, :, 10], lab[:, :, 10]) and not app[:, :, :10].any()


def test_int4_hand_cases():
    for case in _gold("int4_hand.json")["cases"]:
        x = np.array(case["x"], np.float32)
        c = len(x)
        k = x[None, None, None, :]  # [1,1,1,c], channels in order
        lab, sc, ze = oracle.label_int4(np.ascontiguousarray(k), "f32",
                                        np.arange(c, dtype=np.int32)[None], 1)
        assert int(sc[0, 0, 0]) == case["scale_bits"], case["note"]
        assert int(ze[0, 0, 0]) == case["zero_bits"], case["note"]
        assert lab[0, 0, 0].tolist() == case["payload"], case["note"]


def test_int4_properties():
    """Scale/zero are numpy's fp16 rounding of (max-min)/15 and of min; the
    minimum maps to code 0 and the maximum to 15 (up to fp16 rounding); the
    round trip is within half a step plus the zero's rounding; the payload of
    32 channels is 16 bytes, 1/16 of a 128-channel bf16 key row."""
    wl = synth.custom(b=2, hq=2, hkv=2, d=128, s=50, c=32, kv_dtype="bf16", label_dtype="int4",
                      n_outlier=16, outlier_scale=6.0, index=96)
    di = synth.decode_inputs(wl)
    r = np.random.default_rng(2)
    idx = np.stack([np.sort(r.choice(128, 32, replace=False)) for _ in range(2)]).astype(np.int32)
    lab, sc, ze = oracle.label_int4(di.k, "bf16", idx, wl.s)
    assert lab.shape[-1] * 16 == wl.d * 2  # 16 B payload vs 256 B key row
    k = synth.storage_to_f32(di.k, "bf16")
    vals = oracle.label_values((lab, sc, ze), "int4", wl.s, 32).reshape(2, 2, wl.s, 32)
    for bb in range(2):
        for g in range(2):
            x = k[bb, g, : wl.s][:, idx[g]]
            mn, mx = x.min(1), x.max(1)
            exp_s = ((mx - mn) / np.float32(15)).astype(np.float16).view(np.uint16)
            exp_z = mn.astype(np.float16).view(np.uint16)
            assert np.array_equal(sc[bb, g, : wl.s], exp_s)
            assert np.array_equal(ze[bb, g, : wl.s], exp_z)
            step = exp_s.view(np.float16).astype(np.float64)
            z = exp_z.view(np.float16).astype(np.float64)
            err = np.abs(vals[bb, g] - x)
            bound = step[:, None] / 2 + np.abs(z - mn)[:, None] + 1e-6 * np.abs(x)
            assert np.all(err <= bound + step[:, None] * 0.01)
            nib = np.stack([lab[bb, g, : wl.s] & 15, lab[bb, g, : wl.s] >> 4], -1).reshape(wl.s, 32)
            tmin = np.argmin(x, 1)
            tmax = np.argmax(x, 1)
            assert np.all(nib[np.arange(wl.s), tmin] <= 1)
            assert np.all(nib[np.arange(wl.s), tmax] >= 14)


def test_int4_scores_equal_dequantised_dot():
    """Scores over a 4-bit cache use the dequantised values scale*n + zero."""
    wl = synth.custom(b=1, hq=2, hkv=1, d=64, s=20, c=16, label_dtype="int4", index=97)
    di = synth.decode_inputs(wl)
    idx = np.arange(0, 64, 4, dtype=np.int32)[None]
    lab, sc, ze = oracle.label_int4(di.k, "f32", idx, wl.s)
    vals = oracle.label_values((lab, sc, ze), "int4", wl.s, 16)
    s = oracle.scores(di.q, "f32", vals, idx, 1)
    nib = np.stack([lab & 15, lab >> 4], -1).reshape(1, 1, wl.s, 16).astype(np.float64)
    deq = nib * sc.view(np.float16).astype(np.float64)[..., :, None] + \
        ze.view(np.float16).astype(np.float64)[..., :, None]
    qsum = di.q[0].astype(np.float64).sum(0)[idx[0]]
    np.testing.assert_allclose(s[0, 0], deq[0, 0] @ qsum, rtol=1e-12, atol=1e-12)


# ------------------------------------------------- calibration criteria

_CRIT = ("q", "k", "qk", "qk_chunked")


def test_criteria_hand_cases():
    for case in _gold("calib_criteria_hand.json")["cases"]:
        q = np.array(case["q"], np.float32)[None, None]
        k = np.array(case["k"], np.float32)[None, None]
        for name, key in (("q", "q_outlier"), ("k", "k_outlier"), ("qk", "qk_outlier"),
                          ("qk_chunked", "qk_chunked"), ("leank", "leank")):
            if key not in case:
                continue
            score, idx = oracle.calibrate_criterion(q, k, "f32", case["c"], name, case["chunk"])
            np.testing.assert_allclose(score[0], case[key]["score"], rtol=1e-14)
            assert idx[0].tolist() == case[key]["idx"], name


def _stack_group(q_win, g, G):
    """[N, Hq, W, D] -> per sample the group's windows stacked, [N, G*W, D]."""
    n, hq, w, d = q_win.shape
    return q_win[:, g * G:(g + 1) * G].reshape(n, G * w, d).astype(np.float64)


def test_criteria_match_library_norms():
    """Column norms and outer-product norms from numpy, averaged over samples,
    with a GQA group of two query heads per kv head."""
    r = np.random.default_rng(21)
    n, hq, hkv, w, s, d = 3, 4, 2, 5, 37, 16
    q = r.standard_normal((n, hq, w, d)).astype(np.float32)
    k = r.standard_normal((n, hkv, s, d)).astype(np.float32)
    G = hq // hkv
    for g in range(hkv):
        Qs, Ks = _stack_group(q, g, G), k[:, g].astype(np.float64)
        want = {
            "q": np.mean([np.linalg.norm(Qs[j], axis=0) for j in range(n)], axis=0),
            "k": np.mean([np.linalg.norm(Ks[j], axis=0) for j in range(n)], axis=0),
            "qk": np.mean([[np.linalg.norm(np.outer(Qs[j][:, i], Ks[j][:, i]), "fro") for i in range(d)]
                           for j in range(n)], axis=0),
            "qk_chunked": np.mean([[sum(np.linalg.norm(np.outer(Qs[j][:, i], Ks[j][t0:t0 + 10, i]), "fro")
                                        for t0 in range(0, s, 10)) for i in range(d)]
                                   for j in range(n)], axis=0),
        }
        for name in _CRIT:
            score, idx = oracle.calibrate_criterion(q, k, "f32", 5, name, 10)
            np.testing.assert_allclose(score[g], want[name], rtol=1e-12)
            top = sorted(np.lexsort((np.arange(d), -want[name]))[:5].tolist())
            assert idx[g].tolist() == top, name


def test_chunked_criterion_limits():
    """One chunk spanning the context equals the QK-outlier score; chunks of
    one token give ||Q[:,i]|| * sum_t |K[t,i]| (closed form)."""
    r = np.random.default_rng(22)
    q = r.standard_normal((2, 1, 4, 8)).astype(np.float32)
    k = r.standard_normal((2, 1, 13, 8)).astype(np.float32)
    a, _ = oracle.calibrate_criterion(q, k, "f32", 3, "qk")
    b, _ = oracle.calibrate_criterion(q, k, "f32", 3, "qk_chunked", 13)
    c, _ = oracle.calibrate_criterion(q, k, "f32", 3, "qk_chunked", 1000)
    np.testing.assert_allclose(a, b, rtol=1e-14)
    np.testing.assert_allclose(a, c, rtol=1e-14)
    one, _ = oracle.calibrate_criterion(q, k, "f32", 3, "qk_chunked", 1)
    Q, K = q[:, 0].astype(np.float64), k[:, 0].astype(np.float64)
    closed = np.mean(np.linalg.norm(Q, axis=1) * np.abs(K).sum(axis=1), axis=0)
    np.testing.assert_allclose(one[0], closed, rtol=1e-12)


def test_leank_criterion_and_single_sample_qk_ranking():
    """Criterion "leank" is the LeanK ratio; with one sample the ratio is the
    QK-outlier score over a per-head constant, so both rank alike."""
    r = np.random.default_rng(23)
    q = r.standard_normal((1, 2, 6, 16)).astype(np.float32)
    k = r.standard_normal((1, 1, 20, 16)).astype(np.float32)
    ra, ia = oracle.calibrate(q, k, "f32", 6)
    rb, ib = oracle.calibrate_criterion(q, k, "f32", 6, "leank")
    np.testing.assert_array_equal(ra, rb)
    assert ia.tolist() == ib.tolist()
    sq, iq = oracle.calibrate_criterion(q, k, "f32", 6, "qk")
    Qs, K = q[0].reshape(12, 16).astype(np.float64), k[0, 0].astype(np.float64)
    np.testing.assert_allclose(sq[0], ra[0] * np.linalg.norm(Qs @ K.T, "fro"), rtol=1e-12)
    assert iq.tolist() == ia.tolist()


def test_criteria_separate_query_and_key_outliers():
    """Outliers planted only in K are found by the K criterion and missed by
    the Q criterion, and the other way round (catches swapped operands)."""
    r = np.random.default_rng(24)
    q = r.standard_normal((2, 2, 8, 32)).astype(np.float32)
    k = r.standard_normal((2, 1, 64, 32)).astype(np.float32)
    kch, qch = [3, 9, 17, 30], [1, 12, 20, 25]
    k[..., kch] *= 8
    q[..., qch] *= 8
    _, ik = oracle.calibrate_criterion(q, k, "f32", 4, "k")
    _, iq = oracle.calibrate_criterion(q, k, "f32", 4, "q")
    assert ik[0].tolist() == kch and iq[0].tolist() == qch


def test_criteria_reject_bad_arguments():
    q = np.ones((1, 1, 2, 4), np.float32)
    k = np.ones((1, 1, 3, 4), np.float32)
    with pytest.raises(Exception):
        oracle.calibrate_criterion(q, k, "f32", 2, "qk_chunked", 0)
