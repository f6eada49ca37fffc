"""Pins for the fp64 oracle: things the pages and the mathematics fix.

Each ``pin_*`` takes an oracle namespace so that the mutation tests at the
bottom can run the same pins against copies of the oracle with a planted
mistake (a dropped ReLU, a transposed operand, the wrong tie-break, ...) and
check that at least one pin catches each mistake.
"""
import json
import math
import os
import types

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle as ORC
from dsa_inputs import CONFIGS, gen_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def e4m3_codes(values) -> np.ndarray:
    """Encode exactly representable values to e4m3 bytes (torch's cast)."""
    t = torch.tensor(values, dtype=torch.float32)
    codes = t.to(torch.float8_e4m3fn)
    assert torch.equal(codes.float(), t), "value not exact in e4m3"
    return codes.view(torch.uint8).numpy()


def real_oracle():
    return types.SimpleNamespace(index_scores=ORC.index_scores, topk_select=ORC.topk_select,
                                 sparse_mla=ORC.sparse_mla, dense_causal_mqa=ORC.dense_causal_mqa,
                                 decode_e4m3=ORC.decode_e4m3,
                                 indexer_kl_target=ORC.indexer_kl_target,
                                 index_scores_dequantised=ORC.index_scores_dequantised,
                                 indexer_kl_score_grad=ORC.indexer_kl_score_grad,
                                 sparse_mla_backward=ORC.sparse_mla_backward,
                                 indexer_backward=ORC.indexer_backward)


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------


def pin_three_token(orc):
    """Hand-worked example (golden file): scores, top-1/top-2, attention closed form."""
    g = json.load(open(os.path.join(GOLDEN, "three_token.json")))
    keys = e4m3_codes(g["keys"])
    ones_k = np.ones(len(g["keys"]), np.float32)
    for row in g["rows"]:
        t = row["t"]
        n = t + 1
        sc = orc.index_scores(e4m3_codes(row["q"]), np.ones(g["H_I"], np.float32),
                              np.asarray(row["w"], np.float32), keys[:n], ones_k[:n])
        assert np.array_equal(sc, np.asarray(row["scores"], np.float64)), (t, sc)
        assert list(orc.topk_select(sc, 1)) == row["top1"], t
        assert list(orc.topk_select(sc, 2)) == row["top2"], t
    ln3 = math.log(3.0)
    kv = np.array([[0.0, 0.0], [ln3, 1.0]])
    out, lse = orc.sparse_mla(np.array([[1.0, 0.0]]), kv, np.array([0, 1]), 1.0, 2)
    assert np.allclose(out[0], [0.75 * ln3, 0.75], rtol=0, atol=1e-15), out
    assert abs(lse[0] - math.log(4.0)) < 1e-15
    # the same through bf16 storage: r = bf16(ln 3) replaces ln 3 in the closed form
    r = float(torch.tensor(ln3).to(torch.bfloat16).float())
    kvb = torch.tensor([[0.0, 0.0], [ln3, 1.0]]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    qb = torch.tensor([[1.0, 0.0]]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    out, _ = orc.sparse_mla(qb, kvb, np.array([0, 1]), 1.0, 2)
    er = math.exp(r)
    assert np.allclose(out[0], [r * er / (1 + er), er / (1 + er)], rtol=0, atol=1e-15)


def pin_e4m3_table(orc):
    """Decode table against the bit format's landmarks and torch's e4m3 cast."""
    codes = np.arange(256, dtype=np.uint8)
    vals = orc.decode_e4m3(codes)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(vals), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(vals[ok], ref[ok])
    assert vals[0x7E] == 448.0 and vals[0x38] == 1.0 and vals[0x08] == 2.0 ** -6
    assert vals[0x01] == 2.0 ** -9 and vals[0x80] == 0.0 and vals[0xBE] == -1.75
    assert np.isnan(vals[0x7F]) and np.isnan(vals[0xFF])


def _random_indexer(seed, H_I=4, d_I=32, n=50, qsign=None, ksign=None):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((H_I, d_I)).astype(np.float32)
    kk = rng.standard_normal((n, d_I)).astype(np.float32)
    if qsign is not None:
        q = np.abs(q) * qsign
    if ksign is not None:
        kk = np.abs(kk) * ksign
    qc = torch.from_numpy(q / np.abs(q).max(1, keepdims=True) * 448).to(torch.float8_e4m3fn)
    kc = torch.from_numpy(kk / np.abs(kk).max(1, keepdims=True) * 448).to(torch.float8_e4m3fn)
    qs = rng.uniform(0.5, 2.0, H_I).astype(np.float32)
    ks = rng.uniform(0.5, 2.0, n).astype(np.float32)
    w = rng.uniform(0.1, 1.0, H_I).astype(np.float32)
    return (qc.view(torch.uint8).numpy(), qs, w, kc.view(torch.uint8).numpy(), ks,
            qc.double().numpy(), kc.double().numpy())


def pin_indexer_closed_forms(orc):
    """Eq. 1 closed forms: all dots > 0 -> one GEMV; all dots <= 0 -> 0; w scaling."""
    qc, qs, w, kc, ks, qd, kd = _random_indexer(1, qsign=1.0, ksign=1.0)
    sc = orc.index_scores(qc, qs, w, kc, ks)
    assert (qd @ kd.T > 0).all()
    gemv = ks.astype(np.float64) * (kd @ ((w.astype(np.float64) * qs) @ qd))
    assert np.allclose(sc, gemv, rtol=1e-13, atol=0)
    qc, qs, w, kc, ks, _, _ = _random_indexer(2, qsign=1.0, ksign=-1.0)
    assert np.array_equal(orc.index_scores(qc, qs, w, kc, ks), np.zeros(kc.shape[0]))
    qc, qs, w, kc, ks, _, _ = _random_indexer(3)
    a = orc.index_scores(qc, qs, w, kc, ks)
    b = orc.index_scores(qc, qs, (w * 4.0).astype(np.float32), kc, ks)
    assert np.allclose(b, 4.0 * a, rtol=1e-14, atol=0)
    assert np.array_equal(orc.topk_select(a, 7), orc.topk_select(b, 7))


def pin_indexer_mixed_signs(orc):
    """Mixed-sign dots: the ReLU keeps only the positive per-head dots.

    Two heads, one key: head 0 dot = +3, head 1 dot = -5, w = (2, 7), scales
    s^q = (0.5, 4), s^k = 0.25  ->  I = 0.25 * (2 * 0.5 * 3 + 7 * 4 * 0) = 0.75.
    Head 1 with a negative weight would not change that either.
    """
    q = e4m3_codes([[1, 2, 0], [-1, -2, 0]])
    kk = e4m3_codes([[1, 1, 0]])
    sc = orc.index_scores(q, np.array([0.5, 4.0], np.float32), np.array([2.0, 7.0], np.float32),
                          kk, np.array([0.25], np.float32))
    assert sc.tolist() == [0.75]
    sc = orc.index_scores(q, np.array([0.5, 4.0], np.float32), np.array([2.0, -7.0], np.float32),
                          kk, np.array([0.25], np.float32))
    assert sc.tolist() == [0.75]
    # and a key whose dots flip sign per head picks the other head
    kk2 = e4m3_codes([[-1, -1, 0]])
    sc = orc.index_scores(q, np.array([0.5, 4.0], np.float32), np.array([2.0, 7.0], np.float32),
                          kk2, np.array([0.25], np.float32))
    assert sc.tolist() == [0.25 * 7 * 4 * 3]


def pin_topk_bruteforce(orc):
    """Selection by explicit rank: rank(s) = #greater + #equal with lower index."""
    rng = np.random.default_rng(5)
    for trial in range(40):
        n = int(rng.integers(1, 60))
        k = int(rng.integers(1, 40))
        sc = rng.integers(0, 6, n).astype(np.float64)   # many exact ties
        if trial % 3 == 0:
            sc = rng.standard_normal(n)
        got = orc.topk_select(sc, k)
        sel = []
        for s in range(n):
            rank = int((sc > sc[s]).sum() + (sc[:s] == sc[s]).sum())
            if rank < k:
                sel.append(s)
        expect = sel + [-1] * (k - len(sel))
        assert list(got) == expect, (n, k, sc, got)


def pin_topk_properties(orc):
    rng = np.random.default_rng(6)
    for n in (1, 2, 3, 31, 32, 33, 100):
        sc = rng.standard_normal(n)
        for k in (1, 32, 64):
            idx = orc.topk_select(sc, k)
            v = idx[idx >= 0]
            assert len(v) == min(k, n)
            assert len(set(v.tolist())) == len(v)
            assert (v < n).all() and (np.diff(v) > 0).all()
            assert (idx[len(v):] == -1).all()


def pin_attention_special_cases(orc):
    rng = np.random.default_rng(7)
    kv = rng.standard_normal((20, 12))
    q = rng.standard_normal((3, 12))
    # one key: output is that key's value part, exactly
    out, lse = orc.sparse_mla(q, kv, np.array([-1, 5, -1]), 0.3, 8)
    assert np.array_equal(out, np.broadcast_to(kv[5, :8], (3, 8)))
    assert np.allclose(lse, 0.3 * (q @ kv[5]), rtol=0, atol=1e-14)
    # equal logits: mean of the selected values
    out, lse = orc.sparse_mla(np.zeros((2, 12)), kv, np.array([1, 4, 9]), 1.0, 8)
    assert np.allclose(out, np.broadcast_to(kv[[1, 4, 9], :8].mean(0), (2, 8)), rtol=0, atol=1e-15)
    assert np.allclose(lse, math.log(3.0), rtol=0, atol=1e-15)
    # lse against the library log-sum-exp
    sel = np.array([0, 3, 7, 8, 19])
    _, lse = orc.sparse_mla(q, kv, sel, 0.7, 8)
    assert np.allclose(lse, logsumexp(0.7 * (q @ kv[sel].T), axis=1), rtol=0, atol=1e-13)
    # no valid key: zeros and -inf
    out, lse = orc.sparse_mla(q, kv, np.array([-1, -1]), 0.7, 8)
    assert np.array_equal(out, np.zeros((3, 8))) and np.isneginf(lse).all()


def pin_dense_equivalence(orc):
    """k >= every causal key count: sparse attention equals dense causal attention."""
    rng = np.random.default_rng(8)
    Lq, Lk, H, Dqk, Dv = 7, 10, 3, 12, 8
    q = rng.standard_normal((Lq, H, Dqk))
    kv = rng.standard_normal((Lk, Dqk))
    q_pos0 = Lk - Lq
    dense, dlse = orc.dense_causal_mqa(q, kv, 0.4, Dv, q_pos0)
    for t in range(Lq):
        p = q_pos0 + t
        sc = rng.standard_normal(p + 1)
        idx = orc.topk_select(sc, 16)
        out, lse = orc.sparse_mla(q[t], kv, idx, 0.4, Dv)
        assert np.allclose(out, dense[t], rtol=0, atol=1e-13)
        assert np.allclose(lse, dlse[t], rtol=0, atol=1e-13)


def pin_invariances(orc):
    """Non-selected rows cannot matter."""
    cfg = CONFIGS["tiny"]
    inp = ORC.numpy_inputs(gen_inputs(cfg, "cpu"))
    b, t = 0, 200
    n = t + 1
    sc = orc.index_scores(inp["qI"][b, t], inp["qI_scale"][b, t], inp["w"][b, t],
                          inp["kI"][b, :n], inp["kI_scale"][b, :n])
    idx = orc.topk_select(sc, cfg.k)
    out, lse = orc.sparse_mla(inp["q"][b, t], inp["kv"][b], idx, cfg.sm_scale, cfg.Dv)
    notsel = np.setdiff1d(np.arange(n), idx)
    kv2 = inp["kv"][b].copy()
    big = torch.full((len(notsel), cfg.Dqk), 1.0e4).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    kv2[notsel] = big
    out2, lse2 = orc.sparse_mla(inp["q"][b, t], kv2, idx, cfg.sm_scale, cfg.Dv)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)
    # permuting the indexer keys (and scales) of non-selected positions keeps the set
    perm = np.random.default_rng(9).permutation(notsel)
    kI2 = inp["kI"][b, :n].copy()
    ks2 = inp["kI_scale"][b, :n].copy()
    kI2[notsel] = kI2[perm]
    ks2[notsel] = ks2[perm]
    sc2 = orc.index_scores(inp["qI"][b, t], inp["qI_scale"][b, t], inp["w"][b, t], kI2, ks2)
    assert np.array_equal(orc.topk_select(sc2, cfg.k), idx)


def _golden_value(v):
    """Evaluate a fixture entry: a number or an expression in ln(), ln3 and fractions."""
    if isinstance(v, (int, float)):
        return float(v)
    return float(eval(v, {"__builtins__": {}}, {"ln": math.log, "ln3": math.log(3.0)}))


def pin_kl_golden(orc):
    """Hand-worked KL targets over two keys (tests/golden/kl_two_keys.json)."""
    g = json.load(open(os.path.join(GOLDEN, "kl_two_keys.json")))
    kv = np.array([[_golden_value(x) for x in g["keys"]["c0"]],
                   [_golden_value(x) for x in g["keys"]["c1"]]])
    for case in g["cases"]:
        q = np.array([[_golden_value(x) for x in row] for row in case["q"]])
        idx = np.array(case.get("idx", [0, 1]))
        sc = np.array([_golden_value(x) for x in case["scores"]])
        p, kl = orc.indexer_kl_target(q, kv, idx, sc, g["sm_scale"])
        assert np.allclose(p, [_golden_value(x) for x in case["p"]], rtol=0, atol=1e-15), case["note"]
        assert abs(kl - _golden_value(case["kl"])) < 1e-15, case["note"]


def pin_kl_properties(orc):
    """Gibbs' inequality, invariances, and the dense-warm-up reading checked against
    the separately written dense attention (linearity of the head average)."""
    cfg = CONFIGS["tiny"]
    inp = ORC.numpy_inputs(gen_inputs(cfg, "cpu"))
    rng = np.random.default_rng(21)
    b = 0
    for t in (0, 5, 40, 255):
        n = t + 1
        idx = rng.permutation(n)[: min(n, cfg.k)]
        sc = rng.standard_normal(idx.shape[0]) * 3.0
        p, kl = orc.indexer_kl_target(inp["q"][b, t], inp["kv"][b], idx, sc, cfg.sm_scale)
        assert kl >= -1e-15 and abs(p.sum() - 1.0) < 1e-12 and (p > 0).all()
        # shifting the scores changes nothing; permuting the set permutes p
        p2, kl2 = orc.indexer_kl_target(inp["q"][b, t], inp["kv"][b], idx, sc + 17.0, cfg.sm_scale)
        assert abs(kl2 - kl) < 1e-12 and np.allclose(p2, p, rtol=0, atol=1e-15)
        perm = rng.permutation(idx.shape[0])
        p3, kl3 = orc.indexer_kl_target(inp["q"][b, t], inp["kv"][b], idx[perm], sc[perm], cfg.sm_scale)
        assert abs(kl3 - kl) < 1e-12 and np.allclose(p3, p[perm], rtol=0, atol=1e-15)
    # dense warm-up: the set is every causal key; sum_s p_s c_s[:Dv] must be the head
    # mean of the dense attention outputs of the independently written routine
    Lq = 12
    dense, _ = orc.dense_causal_mqa(inp["q"][b, :Lq], inp["kv"][b, :Lq], cfg.sm_scale, cfg.Dv)
    c = ORC.to_f64(inp["kv"][b, :Lq])
    for t in range(Lq):
        idx = np.arange(t + 1)
        p, kl = orc.indexer_kl_target(inp["q"][b, t], inp["kv"][b], idx, np.zeros(t + 1), cfg.sm_scale)
        assert np.allclose(p @ c[: t + 1, : cfg.Dv], dense[t].mean(axis=0), rtol=0, atol=1e-13)
        # equal scores: r is uniform, so KL = sum p ln p + ln n
        assert abs(kl - (float(np.sum(p * np.log(p))) + math.log(t + 1))) < 1e-13


def _fd_grad(f, x, eps=1e-6):
    """Central differences of the scalar function f() in every element of x (x is
    perturbed in place and restored)."""
    g = np.zeros_like(x)
    for i in np.ndindex(*x.shape):
        old = x[i]
        x[i] = old + eps
        fp = f()
        x[i] = old - eps
        fm = f()
        x[i] = old
        g[i] = (fp - fm) / (2 * eps)
    return g


def pin_mla_backward_finite_differences(orc):
    """The attention gradients against central differences of the forward, for the
    loss sum(dout * out), on a set with a padded slot and keys outside the set."""
    rng = np.random.default_rng(31)
    H, Dqk, Dv, n, scale = 3, 6, 4, 7, 0.7
    q = rng.standard_normal((H, Dqk))
    kv = rng.standard_normal((n, Dqk))
    idx = np.array([5, 0, -1, 2, 6])
    dout = rng.standard_normal((H, Dv))

    def loss():
        return float(np.sum(dout * orc.sparse_mla(q, kv, idx, scale, Dv)[0]))

    dq, dkv = orc.sparse_mla_backward(q, kv, idx, dout, scale, Dv)
    assert np.allclose(dq, _fd_grad(loss, q), rtol=1e-6, atol=1e-8)
    assert np.allclose(dkv, _fd_grad(loss, kv), rtol=1e-6, atol=1e-8)
    assert not dkv[[1, 3, 4]].any()


def pin_mla_backward_closed_forms(orc):
    """One selected key: out = c_s[:Dv] whatever q is, so dq = 0 and the row receives
    sum_h dout[h] on its value columns and nothing on the others. Adding one vector
    to the columns past Dv of every selected row adds the same logit to each key of
    a head, which the softmax ignores, so those columns of dkv sum to 0 over the
    set. An empty set gives zeros."""
    rng = np.random.default_rng(32)
    H, Dqk, Dv, n = 4, 10, 6, 9
    q = rng.standard_normal((H, Dqk))
    kv = rng.standard_normal((n, Dqk))
    dout = rng.standard_normal((H, Dv))
    dq, dkv = orc.sparse_mla_backward(q, kv, np.array([4, -1, -1]), dout, 0.5, Dv)
    want = np.zeros((n, Dqk))
    want[4, :Dv] = dout.sum(axis=0)
    assert np.allclose(dq, 0.0, rtol=0, atol=1e-14)
    assert np.allclose(dkv, want, rtol=0, atol=1e-14)
    idx = rng.permutation(n)[:6]
    dq, dkv = orc.sparse_mla_backward(q, kv, idx, dout, 0.5, Dv)
    assert np.allclose(dkv[:, Dv:].sum(axis=0), 0.0, rtol=0, atol=1e-13)
    assert np.abs(dkv[:, Dv:]).max() > 1e-3
    dq, dkv = orc.sparse_mla_backward(q, kv, np.array([-1, n]), dout, 0.5, Dv)
    assert not dq.any() and not dkv.any()


def pin_indexer_backward_finite_differences(orc):
    """Indexer gradients against central differences of Eq. 1 on the dequantised
    values (loss sum_j dI_j I[idx_j]); heads with every dot <= 0 get nothing."""
    qc, qs, w, kc, ks, qd, kd = _random_indexer(41, H_I=3, d_I=5, n=8)
    qf = qd * qs.astype(np.float64)[:, None]
    kf = kd * ks.astype(np.float64)[:, None]
    wf = w.astype(np.float64)
    idx = np.array([6, -1, 1, 3, 0])
    dI = np.random.default_rng(42).standard_normal(idx.shape[0])
    ok = idx >= 0

    def loss():
        return float(np.sum(dI[ok] * orc.index_scores_dequantised(qf, wf, kf)[idx[ok]]))

    dq, dk, dw = orc.indexer_backward(qc, qs, w, kc, ks, idx, dI)
    x = qf @ kf[idx[ok]].T
    assert (np.abs(x) > 1e-3).all()          # no dot near the ReLU kink
    assert np.allclose(dq, _fd_grad(loss, qf), rtol=1e-6, atol=1e-8)
    assert np.allclose(dk, _fd_grad(loss, kf), rtol=1e-6, atol=1e-8)
    assert np.allclose(dw, _fd_grad(loss, wf), rtol=1e-6, atol=1e-8)
    qc, qs, w, kc, ks, _, _ = _random_indexer(43, qsign=1.0, ksign=-1.0)
    dq, dk, dw = orc.indexer_backward(qc, qs, w, kc, ks, np.arange(10), np.ones(10))
    assert not dq.any() and not dk.any() and not dw.any()


def pin_gradients_golden(orc):
    """Hand-worked gradients (tests/golden/sparse_stage_gradients.json): the attention
    backward on two keys, the indexer backward on the three-token example's last
    row, and the KL score gradient."""
    g = json.load(open(os.path.join(GOLDEN, "sparse_stage_gradients.json")))
    a = g["attention"]
    kv = np.array([[_golden_value(x) for x in row] for row in a["keys"]])
    for case in a["cases"]:
        q = np.array([[_golden_value(x) for x in row] for row in case["q"]])
        dout = np.array([[_golden_value(x) for x in row] for row in case["dout"]])
        dq, dkv = orc.sparse_mla_backward(q, kv, np.array(a["idx"]), dout, a["sm_scale"], case["Dv"])
        want_q = np.array([[_golden_value(x) for x in row] for row in case["dq"]])
        want_kv = np.array([[_golden_value(x) for x in row] for row in case["dkv"]])
        assert np.allclose(dq, want_q, rtol=0, atol=1e-14), case["note"]
        assert np.allclose(dkv, want_kv, rtol=0, atol=1e-14), case["note"]
    ix = g["indexer"]
    keys = e4m3_codes(ix["keys"])
    q = e4m3_codes(ix["q"])
    one_q = np.ones(len(ix["q"]), np.float32)
    one_k = np.ones(len(ix["keys"]), np.float32)
    for case in ix["cases"]:
        dq, dk, dw = orc.indexer_backward(q, one_q, np.asarray(ix["w"], np.float32), keys, one_k,
                                          np.array(ix["idx"]), np.asarray(case["dI"], np.float64))
        assert dw.tolist() == case["dw"], (case, dw)
        assert dq.tolist() == case["dq"], (case, dq)
        assert dk.tolist() == case["dk"], (case, dk)
    for case in g["kl_score_grad"]:
        idx = np.array(case.get("idx", list(range(len(case["p"])))))
        grad = orc.indexer_kl_score_grad(np.array([_golden_value(x) for x in case["p"]]),
                                         np.array([_golden_value(x) for x in case["scores"]]), idx, 2)
        assert np.allclose(grad, [_golden_value(x) for x in case["grad"]], rtol=0, atol=1e-15), \
            case["note"]


def pin_code_dots_exact(orc):
    """The indexer backward decides its ReLU mask on dots of e4m3 codes in float64,
    which must be exact: every e4m3 value times 2^9 is an integer, so the dot times
    2^18 is an integer sum, checked here with Python integers on the extreme codes."""
    rng = np.random.default_rng(45)
    table = orc.decode_e4m3(np.arange(256, dtype=np.uint8))
    finite = np.flatnonzero(np.isfinite(table)).astype(np.uint8)
    for d_I in (32, 128):
        a = rng.choice(finite, size=(6, d_I))
        b = rng.choice(finite, size=(9, d_I))
        a[0] = 0x7E              # 448, the largest code, in every column
        b[0] = 0x7E
        b[1] = 0x01              # the smallest subnormal, 2^-9
        got = orc.decode_e4m3(a) @ orc.decode_e4m3(b).T
        ia = (orc.decode_e4m3(a) * 512).astype(np.int64)
        ib = (orc.decode_e4m3(b) * 512).astype(np.int64)
        for i in range(a.shape[0]):
            for j in range(b.shape[0]):
                exact = sum(int(x) * int(y) for x, y in zip(ia[i], ib[j]))
                assert got[i, j] * 2.0 ** 18 == exact, (d_I, i, j)


def pin_kl_score_grad_finite_differences(orc):
    """r - p against central differences of KL(p || r) in the selected scores (p does
    not depend on them); slots outside the set get 0 and the gradient sums to 0."""
    cfg = CONFIGS["tiny"]
    inp = ORC.numpy_inputs(gen_inputs(cfg, "cpu"))
    rng = np.random.default_rng(44)
    t = 60
    idx = np.concatenate([rng.permutation(t + 1)[:20], [-1, -1]])
    sc = rng.standard_normal(idx.shape[0]) * 2.0

    def kl():
        return orc.indexer_kl_target(inp["q"][0, t], inp["kv"][0], idx, sc, cfg.sm_scale)[1]

    p, _ = orc.indexer_kl_target(inp["q"][0, t], inp["kv"][0], idx, sc, cfg.sm_scale)
    g = orc.indexer_kl_score_grad(p, sc, idx, inp["kv"].shape[1])
    assert np.allclose(g, _fd_grad(kl, sc), rtol=1e-6, atol=1e-9)
    assert g[-2:].tolist() == [0.0, 0.0] and abs(g.sum()) < 1e-14


PINS = [pin_three_token, pin_e4m3_table, pin_indexer_closed_forms, pin_indexer_mixed_signs,
        pin_topk_bruteforce, pin_topk_properties, pin_attention_special_cases,
        pin_dense_equivalence, pin_invariances, pin_kl_golden, pin_kl_properties,
        pin_mla_backward_finite_differences, pin_mla_backward_closed_forms,
        pin_indexer_backward_finite_differences, pin_code_dots_exact, pin_gradients_golden,
        pin_kl_score_grad_finite_differences]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(real_oracle())


def test_tiny_forward_properties():
    """The tiny workload end to end on the CPU: causality, set sizes, finiteness."""
    cfg = CONFIGS["tiny"]
    inp = ORC.numpy_inputs(gen_inputs(cfg, "cpu"))
    res = ORC.forward_rows(inp, cfg, 0, range(cfg.Lq))
    for t, (idx, out, lse) in enumerate(zip(res["idx"], res["out"], res["lse"])):
        v = idx[idx >= 0]
        assert len(v) == min(cfg.k, t + 1)
        assert v.max() <= t and len(set(v.tolist())) == len(v)
        assert np.isfinite(out).all() and np.isfinite(lse).all()


def test_generator_is_seeded_and_shaped():
    cfg = CONFIGS["tiny"]
    a = gen_inputs(cfg, "cpu")
    b = gen_inputs(cfg, "cpu")
    for name in a:
        assert torch.equal(a[name], b[name])
    assert a["qI"].shape == (1, 256, 4, 32) and a["qI"].dtype == torch.uint8
    assert a["kv"].shape == (1, 256, 80) and a["kv"].dtype == torch.bfloat16
    assert a["w"].dtype == torch.float32
    # per-row absmax scaling: every row reaches +-448 in code space
    vals = a["qI"].view(torch.float8_e4m3fn).float().abs().amax(-1)
    assert torch.all(vals == 448.0)


def test_output_gradient_is_seeded_bf16_normal():
    from dsa_inputs import output_gradient
    a = output_gradient((2, 3, 8, 64), seed=5)
    b = output_gradient((2, 3, 8, 64), seed=5)
    c = output_gradient((2, 3, 8, 64), seed=6)
    assert a.dtype == torch.bfloat16 and a.shape == (2, 3, 8, 64)
    assert torch.equal(a, b) and not torch.equal(a, c)
    x = output_gradient((1 << 16,), seed=7, std=2.0).double()
    assert abs(x.mean().item()) < 0.05 and abs(x.std().item() - 2.0) < 0.05


def test_random_key_sets_look_like_selections():
    from dsa_inputs import random_key_sets, random_scores
    idx = random_key_sets(2, 40, 16, 5, seed=3)
    assert idx.shape == (2, 40, 16) and idx.dtype == torch.int32
    for b in range(2):
        for t in range(40):
            row = idx[b, t].numpy()
            m = min(16, 5 + t + 1)
            v = row[:m]
            assert (row[m:] == -1).all() and (v >= 0).all() and (v <= 5 + t).all()
            assert (np.diff(v) > 0).all()                       # ascending and unique
            if m == 5 + t + 1:
                assert np.array_equal(v, np.arange(m))          # short rows keep every key
    assert torch.equal(idx, random_key_sets(2, 40, 16, 5, seed=3))
    holes = random_key_sets(1, 40, 16, 5, seed=3, holes=0.5).numpy()
    kept = holes[holes >= 0]
    assert 0 < kept.size < (idx[0] >= 0).sum().item() and (kept <= 5 + 39).all()
    sc = random_scores((3, 4), seed=9, std=2.0)
    assert sc.dtype == torch.float32 and torch.equal(sc, random_scores((3, 4), seed=9, std=2.0))


# ---------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin
# ---------------------------------------------------------------------------


def _mut_no_relu(qI, qs, w, kI, ks):
    q = ORC.decode_e4m3(qI) * ORC.to_f64(qs)[:, None]
    kk = ORC.decode_e4m3(kI) * ORC.to_f64(ks)[:, None]
    return ORC.to_f64(w) @ (q @ kk.T)


def _mut_relu_after_sum(qI, qs, w, kI, ks):
    q = ORC.decode_e4m3(qI) * ORC.to_f64(qs)[:, None]
    kk = ORC.decode_e4m3(kI) * ORC.to_f64(ks)[:, None]
    return np.maximum(ORC.to_f64(w) @ (q @ kk.T), 0.0)


def _mut_no_qscale(qI, qs, w, kI, ks):
    return ORC.index_scores(qI, np.ones_like(qs), w, kI, ks)


def _mut_weights_reversed(qI, qs, w, kI, ks):
    return ORC.index_scores(qI, qs, np.asarray(w)[::-1].copy(), kI, ks)


def _mut_ties_high(scores, k):
    n = scores.shape[0]
    out = np.full(k, -1, dtype=np.int64)
    if n <= k:
        out[:n] = np.arange(n)
        return out
    order = n - 1 - np.argsort(-scores[::-1], kind="stable")
    out[:] = np.sort(order[:k])
    return out


def _mut_topk_smallest(scores, k):
    return ORC.topk_select(-np.asarray(scores), k)


def _mut_values_tail(q, kv, idx, sm_scale, Dv):
    kvf = ORC.to_f64(kv)
    shifted = np.concatenate([kvf[:, -Dv:], kvf[:, Dv:]], axis=1)
    return ORC.sparse_mla(q, shifted, idx, sm_scale, Dv)


def _mut_no_scale(q, kv, idx, sm_scale, Dv):
    return ORC.sparse_mla(q, kv, idx, 1.0, Dv)


def _mut_lse_log2(q, kv, idx, sm_scale, Dv):
    out, lse = ORC.sparse_mla(q, kv, idx, sm_scale, Dv)
    return out, lse / math.log(2.0)


def _mut_e4m3_bias8(codes):
    return ORC.decode_e4m3(codes) * 0.5


def _mut_kl_reversed(q, kv, idx, sc, sm_scale):
    """KL(r || p) instead of KL(p || r)."""
    p, _ = ORC.indexer_kl_target(q, kv, idx, sc, sm_scale)
    ok = np.asarray(idx) >= 0
    s = np.asarray(sc, dtype=np.float64)[ok]
    r = np.exp(s - s.max())
    r /= r.sum()
    return p, float(np.sum(r * (np.log(r) - np.log(p[ok]))))


def _mut_kl_head_max(q, kv, idx, sc, sm_scale):
    """Aggregate heads by their largest weight instead of the sum."""
    qf = ORC.to_f64(q)
    ok = np.asarray(idx) >= 0
    c = ORC.to_f64(kv[np.asarray(idx)[ok]])
    z = sm_scale * (qf @ c.T)
    a = np.exp(z - z.max(axis=1, keepdims=True))
    a /= a.sum(axis=1, keepdims=True)
    agg = a.max(axis=0)
    p = agg / agg.sum()
    s = np.asarray(sc, dtype=np.float64)[ok]
    log_r = s - (s.max() + np.log(np.exp(s - s.max()).sum()))
    out = np.zeros(len(idx))
    out[ok] = p
    return out, float(np.sum(p * (np.log(p) - log_r)))


def _mut_kl_raw_scores(q, kv, idx, sc, sm_scale):
    """Uses the index scores as log-probabilities without normalising them."""
    p, _ = ORC.indexer_kl_target(q, kv, idx, sc, sm_scale)
    ok = np.asarray(idx) >= 0
    s = np.asarray(sc, dtype=np.float64)[ok]
    pp = p[ok]
    nz = pp > 0
    return p, float(np.sum(pp[nz] * (np.log(pp[nz]) - s[nz])))


def _mut_kl_no_scale(q, kv, idx, sc, sm_scale):
    return ORC.indexer_kl_target(q, kv, idx, sc, 1.0)


def _mut_mla_bwd_no_out_term(q, kv, idx, dout, sm_scale, Dv):
    """Drops the dout . out term of the softmax Jacobian."""
    qf = ORC.to_f64(q)
    idx = np.asarray(idx)
    valid = idx[(idx >= 0) & (idx < kv.shape[0])]
    dq = np.zeros_like(qf)
    dkv = np.zeros((kv.shape[0], qf.shape[1]))
    if valid.size == 0:
        return dq, dkv
    c = ORC.to_f64(kv[valid])
    z = sm_scale * (qf @ c.T)
    a = np.exp(z - z.max(axis=1, keepdims=True))
    a /= a.sum(axis=1, keepdims=True)
    dz = a * (ORC.to_f64(dout) @ c[:, :Dv].T)
    dc = sm_scale * (dz.T @ qf)
    dc[:, :Dv] += a.T @ ORC.to_f64(dout)
    np.add.at(dkv, valid, dc)
    return sm_scale * (dz @ c), dkv


def _mut_mla_bwd_no_value_grad(q, kv, idx, dout, sm_scale, Dv):
    """Forgets that the value part of a latent row is the same row as its key."""
    dq, dkv = ORC.sparse_mla_backward(q, kv, idx, dout, sm_scale, Dv)
    valid = np.asarray(idx)[(np.asarray(idx) >= 0) & (np.asarray(idx) < kv.shape[0])]
    qf = ORC.to_f64(q)
    c = ORC.to_f64(kv[valid])
    z = sm_scale * (qf @ c.T)
    a = np.exp(z - z.max(axis=1, keepdims=True))
    a /= a.sum(axis=1, keepdims=True)
    np.add.at(dkv[:, :Dv], valid, -(a.T @ ORC.to_f64(dout)))
    return dq, dkv


def _mut_mla_bwd_transposed_dq(q, kv, idx, dout, sm_scale, Dv):
    """Scales dq by 1/sm_scale instead of sm_scale."""
    dq, dkv = ORC.sparse_mla_backward(q, kv, idx, dout, sm_scale, Dv)
    return dq / (sm_scale * sm_scale), dkv


def _mut_idx_bwd_no_w(qI, qs, w, kI, ks, idx, dI):
    """Leaves the head weight out of the ReLU branch gradient."""
    return ORC.indexer_backward(qI, qs, np.ones_like(np.asarray(w, np.float64)), kI, ks, idx, dI)[:2] + \
        (ORC.indexer_backward(qI, qs, w, kI, ks, idx, dI)[2],)


def _mut_idx_bwd_dw_no_relu(qI, qs, w, kI, ks, idx, dI):
    """dw from the raw dots, without the ReLU."""
    dq, dk, _ = ORC.indexer_backward(qI, qs, w, kI, ks, idx, dI)
    q = ORC.decode_e4m3(qI) * ORC.to_f64(qs)[:, None]
    kk = ORC.decode_e4m3(kI) * ORC.to_f64(ks)[:, None]
    ok = np.asarray(idx) >= 0
    return dq, dk, (q @ kk[np.asarray(idx)[ok]].T) @ np.asarray(dI, np.float64)[ok]


def _mut_kl_grad_sign(p, sc, idx, n_keys):
    return -ORC.indexer_kl_score_grad(p, sc, idx, n_keys)


MUTANTS = {
    "mla_bwd_no_out_term": dict(sparse_mla_backward=_mut_mla_bwd_no_out_term),
    "mla_bwd_no_value_grad": dict(sparse_mla_backward=_mut_mla_bwd_no_value_grad),
    "mla_bwd_dq_wrong_scale": dict(sparse_mla_backward=_mut_mla_bwd_transposed_dq),
    "idx_bwd_no_head_weight": dict(indexer_backward=_mut_idx_bwd_no_w),
    "idx_bwd_dw_no_relu": dict(indexer_backward=_mut_idx_bwd_dw_no_relu),
    "kl_grad_sign": dict(indexer_kl_score_grad=_mut_kl_grad_sign),
    "kl_reversed": dict(indexer_kl_target=_mut_kl_reversed),
    "kl_heads_by_max": dict(indexer_kl_target=_mut_kl_head_max),
    "kl_unnormalised_scores": dict(indexer_kl_target=_mut_kl_raw_scores),
    "kl_no_softmax_scale": dict(indexer_kl_target=_mut_kl_no_scale),
    "no_relu": dict(index_scores=_mut_no_relu),
    "relu_after_head_sum": dict(index_scores=_mut_relu_after_sum),
    "dropped_q_scale": dict(index_scores=_mut_no_qscale),
    "weights_reversed": dict(index_scores=_mut_weights_reversed),
    "ties_to_highest": dict(topk_select=_mut_ties_high),
    "selects_smallest": dict(topk_select=_mut_topk_smallest),
    "values_from_tail": dict(sparse_mla=_mut_values_tail),
    "no_softmax_scale": dict(sparse_mla=_mut_no_scale),
    "lse_base2": dict(sparse_mla=_mut_lse_log2),
    "e4m3_wrong_bias": dict(decode_e4m3=_mut_e4m3_bias8),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    orc = real_oracle()
    for attr, fn in MUTANTS[name].items():
        setattr(orc, attr, fn)
    caught = []
    for pin in PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
