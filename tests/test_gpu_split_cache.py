"""Decode with one sequence's key cache split over G devices, emulated on one GPU.

"DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models" (bud-325 paper
digest), "Key claims", section 2.1: the top-k over I[t,:] and attention over the
selected entries. The cache's keys are split into G shards in key order; the steps
each device would run (selection on its shard, the merge of the gathered candidates,
attention over its part of the merged set, the combine of the gathered partials) run
here one shard after another, and the "all-gather" of the candidates and partials is
a stack. The merged selection must equal the unsplit forward's bit for bit, and the
combined output must match the fp64 oracle's attention over that set.
"""
import numpy as np
import pytest
import torch

import oracle as ORC
import sparse_attention_long_scores_b200 as dsa
from dsa_inputs import CONFIGS, gen_inputs
from parity import check_attention, check_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_attention_long_scores_b200.build import build
    build()
    torch.cuda.set_device(0)


def _u16(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def _merge_reference(cs, ci, lo, k):
    """The definition: the k best (score, global index) pairs by score descending, then
    global index ascending, listed by ascending index and -1 padded."""
    G, R = cs.shape[0], cs.shape[1]
    idx = np.full((R, k), -1, np.int64)
    sel = np.zeros((R, k), np.float64)
    for r in range(R):
        pairs = [(float(cs[g, r, j]), int(lo[g] + ci[g, r, j])) for g in range(G)
                 for j in range(k) if ci[g, r, j] >= 0]
        best = sorted(pairs, key=lambda x: (-x[0], x[1]))[:k]
        best.sort(key=lambda x: x[1])
        for j, (sc, gi) in enumerate(best):
            idx[r, j], sel[r, j] = gi, sc
    return idx, sel


def test_topk_merge_ties_padding_and_short_rows():
    G, R, k = 3, 6, 32
    g = torch.Generator().manual_seed(5)
    lo = [0, 100, 1000]
    cs = torch.randint(0, 6, (G, R, k), generator=g).float() * 0.5   # many exact ties across shards
    ci = torch.sort(torch.randperm(90, generator=g)[:k]).values.int().repeat(G, R, 1)
    ci[1, 2, 20:] = -1                  # a shard with fewer candidates
    ci[:, 4, 5:] = -1                   # a row with 15 candidates in all (< k)
    cs[:, 5] = 1.0                      # a row of equal scores: the lowest indices win
    idx, sel = dsa.topk_merge(cs.cuda(), ci.cuda(), lo)
    ref_idx, ref_sel = _merge_reference(cs.numpy(), ci.numpy(), lo, k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert np.array_equal(sel.cpu().numpy().astype(np.float64), ref_sel)


def _emulate(cfg, inp, bounds):
    """Run the split-cache steps for shards [bounds[g], bounds[g+1]) on one GPU."""
    G = len(bounds) - 1
    lo = bounds[:-1]
    shards, cand_sc, cand_idx = [], [], []
    for g in range(G):
        a, b = bounds[g], bounds[g + 1]
        sh = {key: inp[key] for key in ("qI", "qI_scale", "w", "q")}
        sh["kI"] = inp["kI"][:, a:b].contiguous()
        sh["kI_scale"] = inp["kI_scale"][:, a:b].contiguous()
        sh["kv"] = inp["kv"][:, a:b].contiguous()
        p = dsa.Problem.from_config(cfg.with_(Lk=b - a, q_pos0=b - a - 1))
        idx = torch.empty((cfg.B, 1, cfg.k), dtype=torch.int32, device="cuda")
        sc = torch.empty((cfg.B, 1, cfg.k), dtype=torch.float32, device="cuda")
        dsa.select(p, sh, idx, sc)
        shards.append((p, sh))
        cand_sc.append(sc)
        cand_idx.append(idx)
    idx, _ = dsa.topk_merge(torch.stack(cand_sc), torch.stack(cand_idx), lo)
    outs, lses = [], []
    for g, (p, sh) in enumerate(shards):
        loc = dsa.index_localize(idx, lo[g], p.Lk)
        o, l = dsa.sparse_mla_fwd(sh["q"], sh["kv"], loc, cfg.sm_scale, cfg.Dv)
        outs.append(o)
        lses.append(l)
    out, lse = dsa.attn_combine(torch.stack(outs), torch.stack(lses))
    torch.cuda.synchronize()
    dsa.check_status()
    return out, lse, idx


CASES = [
    # tiny dimensions, three uneven shards
    (CONFIGS["tiny"].with_(mode="decode", B=3, Lq=1, Lk=700, q_pos0=699), [0, 250, 400, 700]),
    # full dimensions, a middle shard shorter than k, and a single shard
    (CONFIGS["decode_128k"].with_(B=2, Lk=9000, q_pos0=8999), [0, 4096, 5000, 9000]),
    (CONFIGS["decode_128k"].with_(B=2, Lk=5000, q_pos0=4999), [0, 5000]),
]


@pytest.mark.parametrize("cfg,bounds", CASES, ids=["tiny-3", "full-3", "full-1"])
def test_split_cache_decode_matches_unsplit(cfg, bounds):
    inp = gen_inputs(cfg, "cuda", seed=31)
    out, lse, idx = _emulate(cfg, inp, bounds)
    # the unsplit forward selects the same keys, bit for bit
    p = dsa.Problem.from_config(cfg)
    ref_idx = torch.empty((cfg.B, 1, cfg.k), dtype=torch.int32, device="cuda")
    dsa.forward(p, inp, idx_out=ref_idx)
    torch.cuda.synchronize()
    assert torch.equal(idx, ref_idx)
    host = ORC.numpy_inputs({key: v.cpu() for key, v in inp.items()})
    qn, kvn = _u16(inp["q"]), _u16(inp["kv"])
    for b in range(cfg.B):
        pos = cfg.Lk - 1
        sc = ORC.index_scores(host["qI"][b, 0], host["qI_scale"][b, 0], host["w"][b, 0],
                              host["kI"][b], host["kI_scale"][b])
        check_selection(idx[b, 0].cpu().numpy(), sc, ORC.topk_select(sc, cfg.k), cfg.k, pos,
                        f"b={b}")
        ro, rl = ORC.sparse_mla(qn[b, 0], kvn[b], idx[b, 0].cpu().numpy(), cfg.sm_scale, cfg.Dv)
        check_attention(out[b, 0].float().cpu().numpy(), ro, lse[b, 0].cpu().numpy(), rl,
                        f"b={b}")


def test_combine_of_empty_partials():
    """A shard that holds none of a row's keys contributes nothing; no shard at all
    gives zeros and lse = -inf."""
    G, R, H, Dv = 2, 3, 8, 64
    g = torch.Generator().manual_seed(9)
    po = torch.randn(G, R, H, Dv, generator=g).bfloat16()
    pl = torch.randn(G, R, H, generator=g)
    pl[1, 0] = -float("inf")          # row 0: only shard 0
    pl[:, 2] = -float("inf")          # row 2: no keys anywhere
    out, lse = dsa.attn_combine(po.cuda(), pl.cuda())
    out, lse = out.float().cpu(), lse.cpu()
    assert torch.equal(out[0], po[0, 0].float())
    assert torch.all(lse[0] == pl[0, 0])
    assert not out[2].any() and torch.all(torch.isneginf(lse[2]))
    w = torch.softmax(pl[:, 1].double(), dim=0)                  # [G, H]
    ref = (w[..., None] * po[:, 1].double()).sum(0)
    assert torch.allclose(out[1].double(), ref, atol=4e-3, rtol=4e-3)
    assert torch.allclose(lse[1].double(), torch.logsumexp(pl[:, 1].double(), 0), atol=1e-5)
