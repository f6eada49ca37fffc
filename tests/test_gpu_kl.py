"""GPU parity of the indexer alignment target (dsa_indexer_kl) against the fp64 oracle.

The target follows "DeepSeek-V3.2: Pushing the Frontier of Open Large Language
Models" (bud-325 paper digest): "Key claims", paper section 2.1.1 Eq. 3-4 (a KL loss
aligns the indexer with the head-aggregated main attention, given in words), and
"Method" (in the sparse stage the KL is taken on the selected tokens). Inputs are
seeded: latent rows and queries from the workload generator, key sets and index
scores from ``dsa_inputs.random_key_sets`` / ``random_scores``. The per-head lse the
kernel consumes comes from the CUDA forward (dsa_sparse_mla_fwd) over the same sets;
the oracle computes everything from scratch.
"""
import numpy as np
import pytest
import torch

import oracle as ORC
import sparse_attention_long_scores_b200 as dsa
from dsa_inputs import CONFIGS, gen_inputs, random_key_sets, random_scores
from parity import check_kl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_attention_long_scores_b200.build import build
    build()
    torch.cuda.set_device(0)


def _run(cfg, q, kv, idx, sel):
    """CUDA path: lse from the forward over idx, then the KL kernel."""
    qd, kvd, idxd, seld = (x.cuda() for x in (q, kv, idx, sel))
    _, lse = dsa.sparse_mla_fwd(qd, kvd, idxd, cfg.sm_scale, cfg.Dv)
    kl, p = dsa.indexer_kl(qd, kvd, idxd, lse, seld, cfg.sm_scale)
    torch.cuda.synchronize()
    dsa.check_status()
    return kl.cpu().numpy(), p.cpu().numpy()


def _check_rows(cfg, q, kv, idx, sel, rows, where):
    kl, p = _run(cfg, q, kv, idx, sel)
    qn = q.view(torch.int16).numpy().view(np.uint16)
    kvn = kv.view(torch.int16).numpy().view(np.uint16)
    worst = 0.0
    for b, t in rows:
        rp, rkl = ORC.indexer_kl_target(qn[b, t], kvn[b], idx[b, t].numpy(), sel[b, t].numpy(),
                                        cfg.sm_scale)
        worst = max(worst, check_kl(kl[b, t], p[b, t], rkl, rp, sel[b, t].numpy(), idx[b, t].numpy(),
                                    f"{where} b={b} t={t}"))
    return worst


def test_kl_tiny_every_row():
    cfg = CONFIGS["tiny"]
    inp = gen_inputs(cfg, "cpu")
    idx = random_key_sets(cfg.B, cfg.Lq, cfg.k, 0, seed=31)
    sel = random_scores((cfg.B, cfg.Lq, cfg.k), seed=32)
    _check_rows(cfg, inp["q"], inp["kv"], idx, sel, [(0, t) for t in range(cfg.Lq)], "tiny")


def test_kl_dense_warmup_sets_and_holes():
    # k covers every causal key (the dense warm-up reading), with a ragged last tile
    # (k = 96) and entries outside the set scattered through idx
    cfg = CONFIGS["tiny"].with_(Lq=90, Lk=90, k=96)
    inp = gen_inputs(cfg, "cpu", seed=41)
    idx = random_key_sets(1, 90, 96, 0, seed=42)
    sel = random_scores((1, 90, 96), seed=43, std=3.0)
    _check_rows(cfg, inp["q"], inp["kv"], idx, sel, [(0, t) for t in range(90)], "dense")
    holes = random_key_sets(1, 90, 96, 0, seed=44, holes=0.3)
    _check_rows(cfg, inp["q"], inp["kv"], holes, sel, [(0, t) for t in range(90)], "holes")


def test_kl_empty_and_single_key_rows():
    cfg = CONFIGS["tiny"].with_(Lq=4, Lk=64, q_pos0=60)
    inp = gen_inputs(cfg, "cpu", seed=51)
    idx = torch.full((1, 4, 32), -1, dtype=torch.int32)
    idx[0, 1, 0] = 7            # one key
    idx[0, 2, 31] = 60          # one key in the last slot
    idx[0, 3, :5] = torch.tensor([1, 3, 5, 7, 9], dtype=torch.int32)
    sel = random_scores((1, 4, 32), seed=52)
    kl, p = _run(cfg, inp["q"], inp["kv"], idx, sel)
    assert kl[0, 0] == 0.0 and (p[0, 0] == 0.0).all()          # empty set
    for t in (1, 2):                                            # one key: p = 1, KL = 0
        assert abs(kl[0, t]) < 1e-6 and abs(p[0, t].sum() - 1.0) < 1e-5
    _check_rows(cfg, inp["q"], inp["kv"], idx, sel, [(0, t) for t in range(4)], "edge")


def test_kl_prefill_8k_sampled_rows():
    cfg = CONFIGS["prefill_8k"].with_(Lq=256, q_pos0=8192 - 256)
    inp = gen_inputs(cfg, "cuda")
    q, kv = inp["q"].cpu(), inp["kv"].cpu()
    del inp
    idx = random_key_sets(1, cfg.Lq, cfg.k, cfg.q_pos0, seed=61)
    sel = random_scores((1, cfg.Lq, cfg.k), seed=62)
    rows = [(0, t) for t in (0, 1, 77, 128, 200, 255)]
    _check_rows(cfg, q, kv, idx, sel, rows, "8k")


def test_kl_p_is_a_distribution_at_full_size():
    # 2048-key sets over a 32K sequence: properties that hold at any size, every row
    cfg = CONFIGS["prefill_32k"].with_(B=1, Lq=512, q_pos0=32768 - 512)
    inp = gen_inputs(cfg, "cuda")
    idx = random_key_sets(1, cfg.Lq, cfg.k, cfg.q_pos0, seed=71).cuda()
    sel = random_scores((1, cfg.Lq, cfg.k), seed=72).cuda()
    _, lse = dsa.sparse_mla_fwd(inp["q"], inp["kv"], idx, cfg.sm_scale, cfg.Dv)
    kl, p = dsa.indexer_kl(inp["q"], inp["kv"], idx, lse, sel, cfg.sm_scale)
    torch.cuda.synchronize()
    dsa.check_status()
    ps = p.sum(-1)
    assert torch.all((ps - 1.0).abs() < 1e-3), float((ps - 1.0).abs().max())
    assert torch.all(kl >= -1e-4) and torch.all(torch.isfinite(kl))
    # one row against the oracle
    qn = inp["q"][0, 300].cpu().view(torch.int16).numpy().view(np.uint16)
    kvn = inp["kv"][0].cpu().view(torch.int16).numpy().view(np.uint16)
    rp, rkl = ORC.indexer_kl_target(qn, kvn, idx[0, 300].cpu().numpy(), sel[0, 300].cpu().numpy(),
                                    cfg.sm_scale)
    check_kl(kl[0, 300].item(), p[0, 300].cpu().numpy(), rkl, rp, sel[0, 300].cpu().numpy(),
             idx[0, 300].cpu().numpy(), "32k row 300")
