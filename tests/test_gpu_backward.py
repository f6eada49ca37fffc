"""GPU parity of the sparse-stage gradients against the fp64 oracle.

"DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models" (bud-325 paper
digest), "Method": in the sparse training stage the main model learns through the
attention over the top-k selected entries (``dsa_sparse_mla_bwd``), and the indexer
keeps learning the KL toward the main attention on the selected tokens, with its
input detached (``dsa_indexer_kl_grad`` then ``dsa_indexer_bwd``).

Inputs are seeded: queries, latent rows and indexer tensors from the workload
generator, key sets from ``dsa_inputs.random_key_sets`` (or the CUDA forward's own
selection at full size), output gradients from ``dsa_inputs.output_gradient`` and
index-score gradients from ``dsa_inputs.random_scores``. The forward's lse, which
the attention backward consumes, comes from the CUDA forward; the oracle recomputes
everything from the definitions.
"""
import numpy as np
import pytest
import torch

import oracle as ORC
import sparse_attention_long_scores_b200 as dsa
from dsa_inputs import CONFIGS, gen_inputs, output_gradient, random_key_sets, random_scores
from parity import (GRAD_ATT_ALL, GRAD_ATT_ROW, GRAD_IDX_ALL, GRAD_IDX_ROW, KL_GRAD_ATOL,
                    KL_GRAD_RTOL, check_grad)

pytestmark = pytest.mark.gpu

FULL = dict(H_I=64, d_I=128, H=128, Dqk=576, Dv=512, k=2048)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_attention_long_scores_b200.build import build
    build()
    torch.cuda.set_device(0)


def _u16(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def _attention_grads(cfg, inp, idx, dout, accumulate_twice=False):
    """CUDA path: forward over idx (for lse), then the backward."""
    q, kv, idxd, doutd = inp["q"].cuda(), inp["kv"].cuda(), idx.cuda(), dout.cuda()
    _, lse = dsa.sparse_mla_fwd(q, kv, idxd, cfg.sm_scale, cfg.Dv)
    dq, dkv = dsa.sparse_mla_bwd(q, kv, idxd, lse, doutd, cfg.sm_scale)
    if accumulate_twice:
        dq2, dkv2 = dsa.sparse_mla_bwd(q, kv, idxd, lse, doutd, cfg.sm_scale, dkv=dkv.clone(),
                                       accumulate_dkv=True)
    torch.cuda.synchronize()
    dsa.check_status()
    res = (dq.cpu().numpy(), dkv.cpu().numpy())
    if accumulate_twice:
        res += (dq2.cpu().numpy(), dkv2.cpu().numpy())
    return res


def _oracle_attention_grads(cfg, inp, idx, dout):
    qn, kvn, dn = _u16(inp["q"]), _u16(inp["kv"]), _u16(dout)
    idxn = idx.numpy()
    dq = np.zeros((cfg.B, cfg.Lq, cfg.H, cfg.Dqk))
    dkv = np.zeros((cfg.B, cfg.Lk, cfg.Dqk))
    for b in range(cfg.B):
        for t in range(cfg.Lq):
            g, gk = ORC.sparse_mla_backward(qn[b, t], kvn[b], idxn[b, t], dn[b, t], cfg.sm_scale,
                                            cfg.Dv)
            dq[b, t] = g
            dkv[b] += gk
    return dq, dkv


def _check_attention(cfg, inp, idx, dout, where):
    dq, dkv = _attention_grads(cfg, inp, idx, dout)
    rq, rkv = _oracle_attention_grads(cfg, inp, idx, dout)
    check_grad(dq, rq, GRAD_ATT_ROW, GRAD_ATT_ALL, f"{where} dq")
    check_grad(dkv, rkv, GRAD_ATT_ROW, GRAD_ATT_ALL, f"{where} dkv")
    # keys no row selected receive exactly nothing
    untouched = np.linalg.norm(rkv, axis=-1) == 0
    assert not dkv[untouched].any(), where
    return dq, dkv


def test_mla_backward_tiny_every_token():
    cfg = CONFIGS["tiny"]
    inp = gen_inputs(cfg, "cpu", seed=61)
    idx = random_key_sets(cfg.B, cfg.Lq, cfg.k, 0, seed=62)
    dout = output_gradient((cfg.B, cfg.Lq, cfg.H, cfg.Dv), seed=63)
    _check_attention(cfg, inp, idx, dout, "tiny")


def test_mla_backward_batch_holes_ragged_chunk_and_accumulate():
    # two sequences, decode-like positions, a fifth of the slots empty, 2 x 100 tokens
    # (chunks of 64 with a ragged last one); a second call that accumulates into dkv
    cfg = CONFIGS["tiny"].with_(B=2, Lq=100, Lk=300, q_pos0=200)
    inp = gen_inputs(cfg, "cpu", seed=64)
    idx = random_key_sets(cfg.B, cfg.Lq, cfg.k, cfg.q_pos0, seed=65, holes=0.2)
    dout = output_gradient((cfg.B, cfg.Lq, cfg.H, cfg.Dv), seed=66)
    dq, dkv, dq2, dkv2 = _attention_grads(cfg, inp, idx, dout, accumulate_twice=True)
    rq, rkv = _oracle_attention_grads(cfg, inp, idx, dout)
    check_grad(dq, rq, GRAD_ATT_ROW, GRAD_ATT_ALL, "batch dq")
    check_grad(dkv, rkv, GRAD_ATT_ROW, GRAD_ATT_ALL, "batch dkv")
    check_grad(dq2, rq, GRAD_ATT_ROW, GRAD_ATT_ALL, "batch dq (second call)")
    check_grad(dkv2, 2.0 * rkv, GRAD_ATT_ROW, GRAD_ATT_ALL, "batch dkv accumulated")


def test_mla_backward_empty_and_single_key_rows():
    # an empty set gives dq = 0; a single key gives dq = 0 and sum_h dout[h] on its
    # value columns (out = c_s[:Dv] whatever q is)
    cfg = CONFIGS["tiny"].with_(Lq=3, Lk=64, q_pos0=61)
    inp = gen_inputs(cfg, "cpu", seed=67)
    idx = torch.full((1, 3, cfg.k), -1, dtype=torch.int32)
    idx[0, 1, 5] = 9
    idx[0, 2, :4] = torch.tensor([2, 4, 8, 16], dtype=torch.int32)
    dout = output_gradient((1, 3, cfg.H, cfg.Dv), seed=68)
    dq, dkv = _attention_grads(cfg, inp, idx, dout)
    assert not dq[0, 0].any()
    assert np.abs(dq[0, 1]).max() < 1e-5
    d = dout[0, 1].float().numpy().astype(np.float64).sum(axis=0)
    assert np.allclose(dkv[0, 9, :cfg.Dv], d, rtol=1e-5, atol=1e-5)
    assert np.abs(dkv[0, 9, cfg.Dv:]).max() < 1e-5
    rq, rkv = _oracle_attention_grads(cfg, inp, idx, dout)
    check_grad(dq[0, 2], rq[0, 2], GRAD_ATT_ROW, GRAD_ATT_ALL, "four keys dq")
    check_grad(dkv, rkv, GRAD_ATT_ROW, GRAD_ATT_ALL, "empty/single dkv")


@pytest.mark.parametrize("holes", [0.0, 0.1])
def test_mla_backward_full_shapes(holes):
    # 128 heads, 576/512 latent rows, k = 2048: 70 tokens (a 64-token chunk and a
    # ragged 6), the first 17 with fewer than k candidates, every set sharing most keys
    cfg = CONFIGS["prefill_8k"].with_(B=1, Lq=70, Lk=2100, q_pos0=2030, **FULL)
    inp = gen_inputs(cfg, "cpu", seed=71)
    idx = random_key_sets(1, cfg.Lq, cfg.k, cfg.q_pos0, seed=72, holes=holes)
    dout = output_gradient((1, cfg.Lq, cfg.H, cfg.Dv), seed=73)
    _check_attention(cfg, inp, idx, dout, f"full holes={holes}")


def test_mla_backward_small_workspace_uses_short_chunks():
    """A workspace sized for 7 tokens (the recommended size of a 7-token call) makes
    dsa_sparse_mla_bwd and dsa_indexer_bwd work through 70 tokens in chunks of 7:
    the results must match the oracle, and the full-workspace call."""
    cfg = CONFIGS["prefill_8k"].with_(B=1, Lq=70, Lk=2100, q_pos0=2030, **FULL)
    inp = gen_inputs(cfg, "cpu", seed=75)
    idx = random_key_sets(1, cfg.Lq, cfg.k, cfg.q_pos0, seed=76, holes=0.1)
    dout = output_gradient((1, cfg.Lq, cfg.H, cfg.Dv), seed=77)
    q, kv, idxd, doutd = inp["q"].cuda(), inp["kv"].cuda(), idx.cuda(), dout.cuda()
    _, lse = dsa.sparse_mla_fwd(q, kv, idxd, cfg.sm_scale, cfg.Dv)
    small = lambda n: torch.empty(int(n), dtype=torch.uint8, device="cuda")
    ws7 = small(dsa.lib().dsa_sparse_mla_bwd_workspace_size(1, 7, cfg.H, cfg.Dqk, cfg.Dv, cfg.k))
    assert ws7.numel() < dsa.lib().dsa_sparse_mla_bwd_workspace_size(1, cfg.Lq, cfg.H, cfg.Dqk,
                                                                       cfg.Dv, cfg.k)
    dq7, dkv7 = dsa.sparse_mla_bwd(q, kv, idxd, lse, doutd, cfg.sm_scale, ws=ws7)
    dq, dkv = dsa.sparse_mla_bwd(q, kv, idxd, lse, doutd, cfg.sm_scale)
    torch.cuda.synchronize()
    dsa.check_status()
    rq, rkv = _oracle_attention_grads(cfg, inp, idx, dout)
    check_grad(dq7.cpu().numpy(), rq, GRAD_ATT_ROW, GRAD_ATT_ALL, "7-token chunks dq")
    check_grad(dkv7.cpu().numpy(), rkv, GRAD_ATT_ROW, GRAD_ATT_ALL, "7-token chunks dkv")
    # the chunking changes only summation orders
    check_grad(dq7.cpu().numpy(), dq.cpu().numpy().astype(np.float64), GRAD_ATT_ROW, GRAD_ATT_ALL,
               "7-token chunks dq vs full workspace")
    check_grad(dkv7.cpu().numpy(), dkv.cpu().numpy().astype(np.float64), GRAD_ATT_ROW, GRAD_ATT_ALL,
               "7-token chunks dkv vs full workspace")
    # the indexer backward with a 7-token workspace
    iinp, iidx, dI = _indexer_case(cfg, 78)
    wsi = small(dsa.lib().dsa_indexer_bwd_workspace_size(1, 7, cfg.H_I, cfg.d_I, cfg.k))
    args = [iinp[n].cuda() for n in ("qI", "qI_scale", "kI", "kI_scale", "w")]
    a7 = dsa.indexer_bwd(*args, iidx.cuda(), dI.cuda(), ws=wsi)
    af = dsa.indexer_bwd(*args, iidx.cuda(), dI.cuda())
    torch.cuda.synchronize()
    dsa.check_status()
    for j, name in enumerate(("dqI", "dkI", "dw")):
        check_grad(a7[j].cpu().numpy(), af[j].cpu().numpy().astype(np.float64), GRAD_IDX_ROW,
                   GRAD_IDX_ALL, f"7-token chunks {name} vs full workspace")


def test_mla_backward_prefill_32k_sampled_rows():
    """The bench workload (2 x 32K, the forward's own top-k sets): dq rows of sampled
    tokens against the oracle one by one, and for dkv a property that holds at any
    size - the columns past Dv of every token's key gradient sum to zero over its set
    (a common shift of those columns moves every logit of a head equally), so they
    sum to zero over all keys too."""
    cfg = CONFIGS["prefill_32k"]
    inp = gen_inputs(cfg, "cuda")
    p = dsa.Problem.from_config(cfg)
    out = torch.empty((cfg.B, cfg.Lq, cfg.H, cfg.Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((cfg.B, cfg.Lq, cfg.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((cfg.B, cfg.Lq, cfg.k), dtype=torch.int32, device="cuda")
    dsa.forward(p, inp, out=out, lse=lse, idx_out=idx)
    dout = output_gradient((cfg.B, cfg.Lq, cfg.H, cfg.Dv), seed=74, device="cuda")
    dq, dkv = dsa.sparse_mla_bwd(inp["q"], inp["kv"], idx, lse, dout, cfg.sm_scale)
    torch.cuda.synchronize()
    dsa.check_status()
    rope = dkv[:, :, cfg.Dv:].double()
    tot = rope.sum(dim=1).abs().max().item()
    scale = rope.abs().sum(dim=1).max().item()
    assert scale > 0 and tot <= 1e-3 * scale, (tot, scale)
    kvn = _u16(inp["kv"])
    for b, t in ((0, 1), (0, 2047), (0, 2048), (0, 20000), (1, 32767), (1, 9000)):
        g, _ = ORC.sparse_mla_backward(_u16(inp["q"][b, t]), kvn[b], idx[b, t].cpu().numpy(),
                                       _u16(dout[b, t]), cfg.sm_scale, cfg.Dv)
        check_grad(dq[b, t].cpu().numpy(), g, GRAD_ATT_ROW, GRAD_ATT_ALL, f"32k dq b={b} t={t}")


def _indexer_case(cfg, seed, holes=0.0):
    inp = gen_inputs(cfg, "cpu", seed=seed, only=("qI", "kI", "w"))
    idx = random_key_sets(cfg.B, cfg.Lq, cfg.k, cfg.q_pos0, seed=seed + 1, holes=holes)
    dI = random_scores((cfg.B, cfg.Lq, cfg.k), seed=seed + 2, std=1.0)
    return inp, idx, dI


def _check_indexer(cfg, inp, idx, dI, where):
    dev = {k: v.cuda() for k, v in inp.items()}
    dqI, dkI, dw = dsa.indexer_bwd(dev["qI"], dev["qI_scale"], dev["kI"], dev["kI_scale"], dev["w"],
                                   idx.cuda(), dI.cuda())
    torch.cuda.synchronize()
    dsa.check_status()
    w = inp["w"]
    wn = _u16(w) if w.dtype == torch.bfloat16 else w.numpy()
    rq = np.zeros((cfg.B, cfg.Lq, cfg.H_I, cfg.d_I))
    rk = np.zeros((cfg.B, cfg.Lk, cfg.d_I))
    rw = np.zeros((cfg.B, cfg.Lq, cfg.H_I))
    for b in range(cfg.B):
        for t in range(cfg.Lq):
            gq, gk, gw = ORC.indexer_backward(inp["qI"][b, t].numpy(), inp["qI_scale"][b, t].numpy(),
                                              wn[b, t], inp["kI"][b].numpy(),
                                              inp["kI_scale"][b].numpy(), idx[b, t].numpy(),
                                              dI[b, t].numpy())
            rq[b, t], rw[b, t] = gq, gw
            rk[b] += gk
    check_grad(dqI.cpu().numpy(), rq, GRAD_IDX_ROW, GRAD_IDX_ALL, f"{where} dqI")
    check_grad(dkI.cpu().numpy(), rk, GRAD_IDX_ROW, GRAD_IDX_ALL, f"{where} dkI")
    check_grad(dw.cpu().numpy(), rw, GRAD_IDX_ROW, GRAD_IDX_ALL, f"{where} dw")


def test_indexer_backward_tiny_every_token():
    cfg = CONFIGS["tiny"]
    inp, idx, dI = _indexer_case(cfg, 81)
    _check_indexer(cfg, inp, idx, dI, "tiny")


def test_indexer_backward_batch_with_holes():
    cfg = CONFIGS["tiny"].with_(B=2, Lq=100, Lk=300, q_pos0=200)
    inp, idx, dI = _indexer_case(cfg, 84, holes=0.2)
    _check_indexer(cfg, inp, idx, dI, "batch")


def test_indexer_backward_full_shapes():
    cfg = CONFIGS["prefill_8k"].with_(B=1, Lq=70, Lk=2100, q_pos0=2030, **FULL)
    inp, idx, dI = _indexer_case(cfg, 87)
    _check_indexer(cfg, inp, idx, dI, "full")


@pytest.mark.parametrize("name,kw", [("tiny", {}),
                                     ("prefill_8k", dict(B=1, Lq=40, Lk=2100, q_pos0=2060, **FULL))])
def test_kl_score_gradient(name, kw):
    """dsa_indexer_kl_grad on the p that dsa_indexer_kl returns, against r - p from the
    oracle with the same p; a padded row and an empty row included."""
    cfg = CONFIGS[name].with_(**kw)
    inp = gen_inputs(cfg, "cpu", seed=91, only=("q", "kv"))
    idx = random_key_sets(cfg.B, cfg.Lq, cfg.k, cfg.q_pos0, seed=92, holes=0.1)
    idx[0, 0] = -1
    sel = random_scores((cfg.B, cfg.Lq, cfg.k), seed=93, std=3.0)
    q, kv, idxd, seld = inp["q"].cuda(), inp["kv"].cuda(), idx.cuda(), sel.cuda()
    _, lse = dsa.sparse_mla_fwd(q, kv, idxd, cfg.sm_scale, cfg.Dv)
    _, p = dsa.indexer_kl(q, kv, idxd, lse, seld, cfg.sm_scale)
    dI = dsa.indexer_kl_grad(seld, p, idxd, cfg.Lk, loss_scale=0.5)
    torch.cuda.synchronize()
    dsa.check_status()
    pn, dn = p.cpu().numpy(), dI.cpu().numpy()
    for b in range(cfg.B):
        for t in range(cfg.Lq):
            ref = 0.5 * ORC.indexer_kl_score_grad(pn[b, t], sel[b, t].numpy(), idx[b, t].numpy(),
                                                  cfg.Lk)
            assert np.allclose(dn[b, t], ref, rtol=KL_GRAD_RTOL, atol=KL_GRAD_ATOL), (b, t)
    assert not dn[0, 0].any()
