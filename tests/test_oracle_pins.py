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
                                 indexer_kl_target=ORC.indexer_kl_target)


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


PINS = [pin_three_token, pin_e4m3_table, pin_indexer_closed_forms, pin_indexer_mixed_signs,
        pin_topk_bruteforce, pin_topk_properties, pin_attention_special_cases,
        pin_dense_equivalence, pin_invariances, pin_kl_golden, pin_kl_properties]


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


MUTANTS = {
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
