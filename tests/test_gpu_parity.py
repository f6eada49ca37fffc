"""GPU parity: every kernel of the path against the fp64 oracle, through the C ABI.

Small cases are compared element by element in full; the full-size workloads
are compared on sampled query rows (the oracle computes them one by one), with
``dsa_forward`` run in the launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import oracle as ORC
import sparse_attention_long_scores_b200 as dsa
from dsa_inputs import CONFIGS, gen_inputs, sample_rows
from parity import bf16_to_f64, check_attention, check_scores, check_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    from sparse_attention_long_scores_b200.build import build
    build()
    torch.cuda.set_device(0)
    yield
    torch.cuda.synchronize()


def _u16(t):
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def _np(t):
    t = t.detach().to("cpu").contiguous()
    return _u16(t) if t.dtype == torch.bfloat16 else t.numpy()


class Rows:
    """Oracle evaluation of single query rows, copying only the slices it needs."""

    def __init__(self, cfg, inp):
        self.cfg, self.inp = cfg, inp
        self._seq = {}

    def seq(self, b):
        if b not in self._seq:
            self._seq = {b: (_np(self.inp["kI"][b]), _np(self.inp["kI_scale"][b]))}
        return self._seq[b]

    def scores(self, b, t):
        cfg, inp = self.cfg, self.inp
        n = cfg.q_pos0 + t + 1
        kI, ks = self.seq(b)
        return ORC.index_scores(_np(inp["qI"][b, t]), _np(inp["qI_scale"][b, t]),
                                _np(inp["w"][b, t]), kI[:n], ks[:n])

    def attention(self, b, t, idx):
        """Oracle attention of row (b, t) over the key set ``idx`` (int array)."""
        idx = np.asarray(idx)
        v = idx[(idx >= 0) & (idx < self.cfg.Lk)]
        if v.size == 0:
            return ORC.sparse_mla(_np(self.inp["q"][b, t]), np.zeros((1, self.cfg.Dqk), np.uint16),
                                  np.array([-1]), self.cfg.sm_scale, self.cfg.Dv)
        rows = _np(self.inp["kv"][b][torch.as_tensor(v, device=self.inp["kv"].device)])
        return ORC.sparse_mla(_np(self.inp["q"][b, t]), rows, np.arange(v.size), self.cfg.sm_scale,
                              self.cfg.Dv)


def _forward(cfg, inp, ws=None):
    p = dsa.Problem.from_config(cfg)
    out = torch.empty((cfg.B, cfg.Lq, cfg.H, cfg.Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((cfg.B, cfg.Lq, cfg.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.B, cfg.Lq, cfg.k), dtype=torch.int32, device="cuda")
    dsa.forward(p, inp, out=out, lse=lse, idx_out=idx, ws=ws)
    dsa.check_status()
    return out, lse, idx


# ---------------------------------------------------------------------------
# tiny workload: everything, every row
# ---------------------------------------------------------------------------


def test_tiny_all_stages_full():
    cfg = CONFIGS["tiny"]
    inp = gen_inputs(cfg, "cuda")
    host = ORC.numpy_inputs(inp)
    # indexer: the whole score matrix, -inf above the diagonal
    sc = dsa.indexer_scores(inp["qI"], inp["qI_scale"], inp["kI"], inp["kI_scale"], inp["w"])
    dsa.check_status()
    sc_h = sc.cpu().numpy()
    ref = ORC.forward_rows(host, cfg, 0, range(cfg.Lq))
    for t in range(cfg.Lq):
        check_scores(sc_h[0, t, :t + 1], ref["scores"][t], f"t={t}")
        assert np.all(np.isneginf(sc_h[0, t, t + 1:]))
    # top-k on the GPU scores
    idx = dsa.topk_select(sc, cfg.k)
    dsa.check_status()
    idx_h = idx.cpu().numpy()
    for t in range(cfg.Lq):
        check_selection(idx_h[0, t], ref["scores"][t], ref["idx"][t], cfg.k, t, f"t={t}")
    # sparse MLA on the oracle's selection
    ref_idx = torch.as_tensor(np.stack(ref["idx"])[None].astype(np.int32), device="cuda")
    out, lse = dsa.sparse_mla_fwd(inp["q"], inp["kv"], ref_idx, cfg.sm_scale, cfg.Dv)
    dsa.check_status()
    check_attention(bf16_to_f64(out[0]), np.stack(ref["out"]), lse[0].cpu().numpy(),
                    np.stack(ref["lse"]), "mla")
    # fused forward: selection, then attention over the GPU's own selection
    out, lse, idx = _forward(cfg, inp)
    idx_h = idx.cpu().numpy()
    rows = Rows(cfg, inp)
    ro, rl = [], []
    for t in range(cfg.Lq):
        check_selection(idx_h[0, t], ref["scores"][t], ref["idx"][t], cfg.k, t, f"fwd t={t}")
        o, l = rows.attention(0, t, idx_h[0, t])
        ro.append(o)
        rl.append(l)
    check_attention(bf16_to_f64(out[0]), np.stack(ro), lse[0].cpu().numpy(), np.stack(rl), "fwd")


@pytest.mark.parametrize("L", [1, 2, 3, 31, 32, 33, 257, 300])
def test_tiny_odd_lengths(L):
    cfg = CONFIGS["tiny"].with_(Lq=L, Lk=L, name="tiny")
    inp = gen_inputs(cfg, "cuda", seed=77 + L)
    host = ORC.numpy_inputs(inp)
    ref = ORC.forward_rows(host, cfg, 0, range(L))
    sc = dsa.indexer_scores(inp["qI"], inp["qI_scale"], inp["kI"], inp["kI_scale"], inp["w"])
    out, lse, idx = _forward(cfg, inp)
    sc_h, idx_h = sc.cpu().numpy(), idx.cpu().numpy()
    rows = Rows(cfg, inp)
    ro, rl = [], []
    for t in range(L):
        check_scores(sc_h[0, t, :t + 1], ref["scores"][t], f"L={L} t={t}")
        check_selection(idx_h[0, t], ref["scores"][t], ref["idx"][t], cfg.k, t, f"L={L} t={t}")
        o, l = rows.attention(0, t, idx_h[0, t])
        ro.append(o)
        rl.append(l)
    check_attention(bf16_to_f64(out[0]), np.stack(ro), lse[0].cpu().numpy(), np.stack(rl), f"L={L}")


def test_tiny_decode_and_batch():
    """Batched decode shape on tiny dims: B=5, Lq=1 against 300 cached keys, plus a
    chunked prefill continuation (q_pos0 > 0, Lq = 40)."""
    for cfg in (CONFIGS["tiny"].with_(B=5, Lq=1, Lk=300, q_pos0=299, mode="decode"),
                CONFIGS["tiny"].with_(B=2, Lq=40, Lk=100, q_pos0=60)):
        inp = gen_inputs(cfg, "cuda", seed=5)
        host = ORC.numpy_inputs(inp)
        out, lse, idx = _forward(cfg, inp)
        idx_h = idx.cpu().numpy()
        rows = Rows(cfg, inp)
        for b in range(cfg.B):
            ref = ORC.forward_rows(host, cfg, b, range(cfg.Lq))
            ro, rl = [], []
            for t in range(cfg.Lq):
                p = cfg.q_pos0 + t
                check_selection(idx_h[b, t], ref["scores"][t], ref["idx"][t], cfg.k, p, f"b={b} t={t}")
                o, l = rows.attention(b, t, idx_h[b, t])
                ro.append(o)
                rl.append(l)
            check_attention(bf16_to_f64(out[b]), np.stack(ro), lse[b].cpu().numpy(), np.stack(rl),
                            f"b={b}")


# ---------------------------------------------------------------------------
# top-k edge cases
# ---------------------------------------------------------------------------


@pytest.mark.parametrize("Lk,k,levels", [(3000, 2048, 4), (5000, 64, 0), (70000, 2048, 0),
                                          (70000, 256, 3), (40000, 32, 1)])
def test_topk_exact_ties_and_long_rows(Lk, k, levels):
    """Scores with many exact ties (levels > 0 distinct values) must select the
    lowest indices exactly; long rows exercise the global-memory path."""
    g = torch.Generator(device="cuda").manual_seed(Lk + k)
    B, Lq = 1, 3
    q_pos0 = Lk - Lq
    if levels:
        sc = torch.randint(0, levels, (B, Lq, Lk), generator=g, device="cuda").float()
        sc[..., ::7] = -0.0 if levels == 1 else sc[..., ::7]
    else:
        sc = torch.randn((B, Lq, Lk), generator=g, device="cuda")
    idx = dsa.topk_select(sc, k, q_pos0=q_pos0)
    dsa.check_status()
    sc_h = sc.cpu().double().numpy()
    idx_h = idx.cpu().numpy()
    for t in range(Lq):
        p = q_pos0 + t
        ref = ORC.topk_select(sc_h[0, t, :p + 1], k)
        assert np.array_equal(idx_h[0, t], ref), f"t={t}"


# ---------------------------------------------------------------------------
# full-size workloads on sampled rows
# ---------------------------------------------------------------------------


def _check_big(cfg, n_rows, score_blocks=2, all_rows=False):
    """Sampled rows of a full-size workload, run in the benchmark's launch
    configuration: selection and attention of ``n_rows`` rows per sequence, and
    the indexer scores of ``score_blocks`` blocks of 8 rows per sequence through
    the public score entry point. With ``all_rows`` every row's scores (the whole
    causal score matrix, one launch) and every row's selection are checked too."""
    inp = gen_inputs(cfg, "cuda")
    out, lse, idx = _forward(cfg, inp)
    rows = Rows(cfg, inp)
    samples = sample_rows(cfg, n_rows)
    n_band = 0
    if all_rows:
        sc_all = dsa.indexer_scores(inp["qI"], inp["qI_scale"], inp["kI"], inp["kI_scale"], inp["w"],
                                    q_pos0=cfg.q_pos0)
        dsa.check_status()
        idx_all = idx.cpu().numpy()
        for b in range(cfg.B):
            sc_h = sc_all[b].cpu().numpy()
            for t in range(cfg.Lq):
                p = cfg.q_pos0 + t
                ref_sc = rows.scores(b, t)
                check_scores(sc_h[t, :p + 1], ref_sc, f"{cfg.name} all-row scores b={b} t={t}")
                n_band += check_selection(idx_all[b, t], ref_sc, ORC.topk_select(ref_sc, cfg.k), cfg.k, p,
                                          f"{cfg.name} all-row selection b={b} t={t}")
            del sc_h
        del sc_all
        torch.cuda.empty_cache()
    for b in range(cfg.B):
        ro, rl, go, gl = [], [], [], []
        for t in samples:
            p = cfg.q_pos0 + t
            gidx = idx[b, t].cpu().numpy()
            if not all_rows:
                if p + 1 > cfg.k:
                    sc = rows.scores(b, t)
                    ref_idx = ORC.topk_select(sc, cfg.k)
                else:
                    sc, ref_idx = None, ORC.topk_select(np.zeros(p + 1), cfg.k)
                n_band += check_selection(gidx, sc, ref_idx, cfg.k, p, f"{cfg.name} b={b} t={t}")
            o, l = rows.attention(b, t, gidx)
            ro.append(o)
            rl.append(l)
            go.append(bf16_to_f64(out[b, t]))
            gl.append(lse[b, t].cpu().numpy())
        check_attention(np.stack(go), np.stack(ro), np.stack(gl), np.stack(rl), f"{cfg.name} b={b}")
    # indexer scores on blocks of rows through the public score entry point
    for b in range(min(cfg.B, 2)):
        for t0 in [samples[len(samples) // 2], samples[-1] - 7][:score_blocks]:
            t0 = max(0, min(t0, cfg.Lq - 8))
            nq = min(8, cfg.Lq)
            sl = slice(t0, t0 + nq)
            qpos = cfg.q_pos0 + t0
            sc = dsa.indexer_scores(inp["qI"][b:b + 1, sl].contiguous(),
                                    inp["qI_scale"][b:b + 1, sl].contiguous(), inp["kI"][b:b + 1],
                                    inp["kI_scale"][b:b + 1], inp["w"][b:b + 1, sl].contiguous(),
                                    q_pos0=qpos)
            sc_h = sc.cpu().numpy()
            for i in range(nq):
                t = t0 + i
                p = cfg.q_pos0 + t
                check_scores(sc_h[0, i, :p + 1], rows.scores(b, t), f"{cfg.name} scores b={b} t={t}")
    del inp, out, lse, idx
    torch.cuda.empty_cache()
    return n_band


def test_prefill_8k():
    """Every row's scores and selection; attention on 512 rows."""
    _check_big(CONFIGS["prefill_8k"], 512, all_rows=True)


def test_prefill_32k_batch2():
    _check_big(CONFIGS["prefill_32k"], 64)


def test_prefill_128k():
    _check_big(CONFIGS["prefill_128k"], 64)


def test_decode_128k():
    cfg = CONFIGS["decode_128k"]
    inp = gen_inputs(cfg, "cuda")
    out, lse, idx = _forward(cfg, inp)
    rows = Rows(cfg, inp)
    # the single-token indexer variant that decode runs, score for score: one query
    # row per sequence at position Lk - 1 against all 131072 cached keys
    sc_gpu = dsa.indexer_scores(inp["qI"], inp["qI_scale"], inp["kI"], inp["kI_scale"], inp["w"],
                                q_pos0=cfg.q_pos0)
    dsa.check_status()
    assert tuple(sc_gpu.shape) == (cfg.B, 1, cfg.Lk)
    sc_gpu = sc_gpu.cpu().numpy()
    go, gl, ro, rl = [], [], [], []
    for b in range(cfg.B):
        gidx = idx[b, 0].cpu().numpy()
        sc = rows.scores(b, 0)
        check_scores(sc_gpu[b, 0], sc, f"decode scores b={b}")
        check_selection(gidx, sc, ORC.topk_select(sc, cfg.k), cfg.k, cfg.q_pos0, f"decode b={b}")
        o, l = rows.attention(b, 0, gidx)
        ro.append(o)
        rl.append(l)
        go.append(bf16_to_f64(out[b, 0]))
        gl.append(lse[b, 0].cpu().numpy())
    check_attention(np.stack(go), np.stack(ro), np.stack(gl), np.stack(rl), "decode")


# ---------------------------------------------------------------------------
# invariances, determinism, bounded waits
# ---------------------------------------------------------------------------


def test_unselected_rows_do_not_matter_and_determinism():
    cfg = CONFIGS["tiny"].with_(Lq=200, Lk=200)
    inp = gen_inputs(cfg, "cuda", seed=11)
    out1, lse1, idx1 = _forward(cfg, inp)
    out2, lse2, idx2 = _forward(cfg, inp)
    assert torch.equal(out1, out2) and torch.equal(idx1, idx2) and torch.equal(lse1, lse2)
    t = cfg.Lq - 1
    sel = idx1[0, t][idx1[0, t] >= 0].long()
    mask = torch.ones(cfg.Lk, dtype=torch.bool, device="cuda")
    mask[sel] = False
    kv2 = inp["kv"].clone()
    kv2[0, mask] = 1.0e4
    o, l = dsa.sparse_mla_fwd(inp["q"][:, t:t + 1].contiguous(), kv2, idx1[:, t:t + 1].contiguous(),
                              cfg.sm_scale, cfg.Dv)
    o_ref, l_ref = dsa.sparse_mla_fwd(inp["q"][:, t:t + 1].contiguous(), inp["kv"],
                                      idx1[:, t:t + 1].contiguous(), cfg.sm_scale, cfg.Dv)
    assert torch.equal(o, o_ref) and torch.equal(l, l_ref)
    assert torch.equal(o[0, 0], out1[0, t])


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("prefill_8k", dict(Lq=2048, q_pos0=6144))])
def test_overlapped_schedule_matches_serial(name, kw):
    """dsa_forward runs the top-k of a score chunk on a side stream while the indexer
    scores the next half-size chunk; dsa_forward_profiled keeps the serial schedule with
    full-size chunks. Every score is computed the same way in both, so the selections
    and outputs must be identical."""
    cfg = CONFIGS[name].with_(**kw)
    inp = gen_inputs(cfg, "cuda", seed=23)
    out1, lse1, idx1 = _forward(cfg, inp)
    launches = dsa.last_launch_count()
    p = dsa.Problem.from_config(cfg)
    out2 = torch.empty_like(out1)
    prof = dsa.LaunchProfiler(4096)
    dsa.forward_profiled(p, inp, out2, prof)
    torch.cuda.synchronize()
    dsa.check_status()
    assert torch.equal(out1, out2)
    # the overlapped schedule splits the score chunks in two: more top-k launches
    assert launches > prof.n and dsa.last_launch_count() == prof.n


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("tiny", dict(B=3, Lq=37, Lk=301, q_pos0=264)),
                                     ("prefill_8k", dict(Lq=1000, q_pos0=7192)),
                                     ("decode_128k", dict(B=5))])
def test_fused_forward_matches_forward(name, kw):
    """dsa_forward_fused selects inside the indexer kernel (selector warps, one
    cooperative launch per score chunk); it computes every score and applies the
    selection rule exactly as dsa_forward does, so idx, out and lse are identical."""
    cfg = CONFIGS[name].with_(**kw)
    inp = gen_inputs(cfg, "cuda", seed=31)
    out1, lse1, idx1 = _forward(cfg, inp)
    p = dsa.Problem.from_config(cfg)
    out2 = torch.empty_like(out1)
    lse2 = torch.empty_like(lse1)
    idx2 = torch.empty_like(idx1)
    dsa.forward(p, inp, out=out2, lse=lse2, idx_out=idx2, fused=True)
    dsa.check_status()
    assert dsa.last_launch_count() >= 2
    assert torch.equal(idx1, idx2) and torch.equal(out1, out2) and torch.equal(lse1, lse2)


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("name,kw", [("tiny", {}), ("prefill_8k", dict(Lq=600, q_pos0=7592)),
                                     ("decode_128k", dict(B=4))])
def test_forward_returns_selected_scores(name, kw, fused):
    """sel_scores_out: the index score of every selected key, aligned with idx_out,
    written by the kernel that selects (every row is scored, short rows included).
    It must equal the materialised score matrix gathered at idx bit for bit, match
    the oracle on sampled rows, and leave the selection unchanged."""
    cfg = CONFIGS[name].with_(**kw)
    inp = gen_inputs(cfg, "cuda", seed=29)
    p = dsa.Problem.from_config(cfg)
    idx = torch.empty((cfg.B, cfg.Lq, cfg.k), dtype=torch.int32, device="cuda")
    sel = torch.full((cfg.B, cfg.Lq, cfg.k), float("nan"), dtype=torch.float32, device="cuda")
    out = dsa.forward(p, inp, idx_out=idx, sel_scores=sel, fused=fused)
    dsa.check_status()
    out2, _, idx2 = _forward(cfg, inp)
    assert torch.equal(idx, idx2) and torch.equal(out, out2)
    sc = dsa.indexer_scores(inp["qI"], inp["qI_scale"], inp["kI"], inp["kI_scale"], inp["w"],
                            q_pos0=cfg.q_pos0)
    dsa.check_status()
    valid = idx >= 0
    gathered = torch.where(valid, torch.gather(sc, 2, idx.clamp(min=0).long()), torch.zeros_like(sel))
    assert torch.equal(sel, gathered)
    rows = Rows(cfg, inp)
    idx_h, sel_h = idx.cpu().numpy(), sel.cpu().numpy()
    for b in range(cfg.B):
        for t in sorted({0, cfg.Lq // 2, cfg.Lq - 1}):
            v = idx_h[b, t][idx_h[b, t] >= 0]
            ref = rows.scores(b, t)
            check_scores(sel_h[b, t][: v.size], ref[v], f"{name} sel_scores b={b} t={t}")


@pytest.mark.parametrize("name,L,rows", [("tiny", 32, None), ("prefill_8k", 2048, (0, 1, 700, 2047))])
def test_short_context_is_dense_attention_without_indexer(name, L, rows):
    """L <= k: every row selects all of its causal keys without scores (the top-k of at
    most k candidates is all of them), so DSA is dense causal MQA and no indexer or
    score work is launched."""
    cfg = CONFIGS[name].with_(Lq=L, Lk=L, q_pos0=0)
    assert L <= cfg.k
    inp = gen_inputs(cfg, "cuda", seed=91)
    p = dsa.Problem.from_config(cfg)
    out = torch.empty((1, L, cfg.H, cfg.Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, L, cfg.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((1, L, cfg.k), dtype=torch.int32, device="cuda")
    prof = dsa.LaunchProfiler(64)
    dsa.forward_profiled(p, inp, out, prof, lse=lse, idx_out=idx)
    torch.cuda.synchronize()
    dsa.check_status()
    kinds = [k for k, _ in prof.durations()]
    assert "indexer" not in kinds and "sparse_mla" in kinds, kinds
    host = ORC.numpy_inputs(inp)
    idx_h = idx.cpu().numpy()
    check_rows = range(L) if rows is None else rows
    if rows is None:
        dense, dlse = ORC.dense_causal_mqa(host["q"][0], host["kv"][0], cfg.sm_scale, cfg.Dv)
    ro, rl = [], []
    for t in check_rows:
        assert np.array_equal(idx_h[0, t][: t + 1], np.arange(t + 1)) and (idx_h[0, t][t + 1:] == -1).all()
        if rows is None:
            ro.append(dense[t])
            rl.append(dlse[t])
        else:
            o, l = ORC.sparse_mla(host["q"][0, t], host["kv"][0], np.arange(t + 1), cfg.sm_scale, cfg.Dv)
            ro.append(o)
            rl.append(l)
    sel = list(check_rows)
    check_attention(bf16_to_f64(out[0, sel]), np.stack(ro), lse[0, sel].cpu().numpy(), np.stack(rl),
                    f"short {name}")


def test_sparse_mla_skips_invalid_indices():
    cfg = CONFIGS["tiny"].with_(Lq=4, Lk=64)
    inp = gen_inputs(cfg, "cuda", seed=3)
    idx = torch.full((1, 4, 32), -1, dtype=torch.int32, device="cuda")
    idx[0, 0, 5] = 7          # a lone valid key in the middle
    idx[0, 1, :3] = torch.tensor([1, 64, 2])   # 64 is out of range: skipped
    idx[0, 2, 0] = -5
    # row 3: no valid key at all
    out, lse = dsa.sparse_mla_fwd(inp["q"], inp["kv"], idx, cfg.sm_scale, cfg.Dv)
    dsa.check_status()
    rows = Rows(cfg, inp)
    for t in range(4):
        o, l = rows.attention(0, t, idx[0, t].cpu().numpy())
        check_attention(bf16_to_f64(out[0, t]), o, lse[0, t].cpu().numpy(), l, f"t={t}")
    assert torch.all(out[0, 2:] == 0) and torch.all(torch.isneginf(lse[0, 2:]))


def test_bounded_wait_reports_timeout():
    dsa.set_wait_limit_ns(20_000_000)   # 20 ms
    try:
        dsa.debug_wait_timeout()
        with pytest.raises(dsa.DsaError) as ei:
            dsa.check_status()
        assert ei.value.code == dsa.DSA_ERR_TIMEOUT
        assert "debug wait" in str(ei.value)
    finally:
        dsa.set_wait_limit_ns(2_000_000_000)
    dsa.check_status()   # cleared, context still usable
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


@pytest.mark.parametrize("tokens,Lk", [(6, 5000), (160, 3000)])
def test_mla_128_heads_every_row(tokens, Lk):
    """128-head / 576-wide attention on random selections, every row against the
    oracle: few tokens take the key-split path, many tokens the direct one. Row 0
    holds a short selection padded with -1, row 1 an out-of-range index."""
    cfg = CONFIGS["prefill_8k"].with_(B=1, Lq=tokens, Lk=Lk, q_pos0=Lk - tokens)
    inp = gen_inputs(cfg, "cuda", seed=tokens, only=("q", "kv"))
    g = torch.Generator(device="cuda").manual_seed(tokens + Lk)
    rows = [torch.sort(torch.randperm(Lk, generator=g, device="cuda")[:cfg.k]).values
            for _ in range(tokens)]
    idx = torch.stack(rows).view(1, tokens, cfg.k).to(torch.int32)
    idx[0, 0, 100:] = -1
    idx[0, 1, 7] = Lk + 5
    out, lse = dsa.sparse_mla_fwd(inp["q"], inp["kv"], idx.contiguous(), cfg.sm_scale, cfg.Dv)
    dsa.check_status()
    q_h, kv_h, idx_h = _np(inp["q"][0]), _np(inp["kv"][0]), idx[0].cpu().numpy()
    ro, rl = [], []
    for t in range(tokens):
        o, l = ORC.sparse_mla(q_h[t], kv_h, idx_h[t], cfg.sm_scale, cfg.Dv)
        ro.append(o)
        rl.append(l)
    check_attention(bf16_to_f64(out[0]), np.stack(ro), lse[0].cpu().numpy(), np.stack(rl),
                    f"mla128 tokens={tokens}")


@pytest.mark.parametrize("kw", [
    dict(B=2, Lq=5596, Lk=5596, q_pos0=0),      # blocks of 4096 + 1500 rows per sequence
    dict(B=1, Lq=4596, Lk=9000, q_pos0=4404),   # a 500-row remainder joins the first block
    dict(B=2, Lq=700, Lk=3000, q_pos0=2300),    # too short to pipeline
])
def test_host_entry_point_matches_device_forward(kw):
    """dsa_forward_host pipelines its copies with the compute by blocks of query rows,
    each block an ordinary forward over one sequence. Rows are independent, so out,
    lse and idx_out must equal one dsa_forward over the device tensors bit for bit."""
    cfg = CONFIGS["tiny"].with_(**kw)
    inp = gen_inputs(cfg, "cuda", seed=57)
    out1, lse1, idx1 = _forward(cfg, inp)
    p = dsa.Problem.from_config(cfg)
    host = {k: v.cpu().pin_memory() for k, v in inp.items()}
    dev = {k: torch.zeros_like(v) for k, v in inp.items()}   # staging, filled by the call
    h_out = torch.empty(tuple(out1.shape), dtype=torch.bfloat16).pin_memory()
    h_lse = torch.empty(tuple(lse1.shape), dtype=torch.float32).pin_memory()
    h_idx = torch.empty(tuple(idx1.shape), dtype=torch.int32).pin_memory()
    d_out, d_lse, d_idx = torch.empty_like(out1), torch.empty_like(lse1), torch.empty_like(idx1)
    ws = torch.empty(dsa.forward_workspace_size(p), dtype=torch.uint8, device="cuda")
    dsa.forward_host(p, host, dev, h_out, d_out, ws, host_lse=h_lse, dev_lse=d_lse,
                     host_idx=h_idx, dev_idx=d_idx)
    dsa.check_status()
    for k in inp:
        assert torch.equal(dev[k].cpu(), host[k]), k
    assert torch.equal(h_idx, idx1.cpu())
    assert torch.equal(h_lse, lse1.cpu())
    assert torch.equal(h_out, out1.cpu())
