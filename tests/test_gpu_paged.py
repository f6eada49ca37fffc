"""GPU parity of dsa_forward_paged: paged latent / index-key caches with per-sequence
lengths, against the fp64 oracle run on each sequence's logical data.

Each sequence's logical blocks are scattered over a shuffled pool of pages; query
row t of sequence b sits at position seq_lens[b] - Lq + t and its candidates are the
keys 0 .. that position of its own sequence ("DeepSeek-V3.2: Pushing the Frontier of
Open Large Language Models", bud-325 paper digest, Key claims section 2.1: the index
scores and the top-k selection run over the query's preceding tokens).
"""
import math

import numpy as np
import pytest
import torch

import oracle as ORC
import sparse_attention_long_scores_b200 as dsa
from dsa_inputs import CONFIGS, gen_inputs
from parity import bf16_to_f64, check_attention, check_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_attention_long_scores_b200.build import build
    build()
    torch.cuda.set_device(0)


def _paged_case(cfg, seq_lens, page_size, seed, shuffle=True):
    """Logical inputs of capacity Lk = max_blocks * page_size per sequence, and the
    same keys scattered over a pool of pages (plus unused pages)."""
    B = len(seq_lens)
    max_blocks = max(math.ceil(max(seq_lens) / page_size), 1)
    Lk = max_blocks * page_size
    c = cfg.with_(B=B, Lk=Lk, q_pos0=Lk - cfg.Lq)
    inp = gen_inputs(c, "cuda", seed=seed)
    used = [math.ceil(n / page_size) for n in seq_lens]
    num_pages = sum(used) + 3
    rng = np.random.default_rng(seed)
    perm = rng.permutation(num_pages) if shuffle else np.arange(num_pages)
    table = np.zeros((B, max_blocks), dtype=np.int32)
    pool_rows = []
    nxt = 0
    for b in range(B):
        for j in range(max_blocks):
            if j < used[b]:
                table[b, j] = perm[nxt]
                pool_rows.append((perm[nxt], b, j))
                nxt += 1
            else:
                table[b, j] = perm[-1]          # never read: beyond the sequence
    rows = num_pages * page_size
    kv = torch.zeros((rows, c.Dqk), dtype=torch.bfloat16, device="cuda")
    kI = torch.zeros((rows, c.d_I), dtype=torch.uint8, device="cuda")
    ks = torch.zeros((rows,), dtype=torch.float32, device="cuda")
    for pg, b, j in pool_rows:
        dst = slice(pg * page_size, (pg + 1) * page_size)
        src = slice(j * page_size, (j + 1) * page_size)
        kv[dst] = inp["kv"][b, src]
        kI[dst] = inp["kI"][b, src]
        ks[dst] = inp["kI_scale"][b, src]
    pinp = dict(inp, kv=kv, kI=kI, kI_scale=ks)
    return c, inp, pinp, torch.from_numpy(table).cuda(), torch.tensor(seq_lens, dtype=torch.int32,
                                                                       device="cuda")


def _run_paged(c, pinp, table, lens, page_size):
    p = dsa.Problem.from_config(c)
    out = torch.empty((c.B, c.Lq, c.H, c.Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((c.B, c.Lq, c.H), dtype=torch.float32, device="cuda")
    idx = torch.empty((c.B, c.Lq, c.k), dtype=torch.int32, device="cuda")
    dsa.forward_paged(p, pinp, table, lens, page_size, out=out, lse=lse, idx_out=idx)
    torch.cuda.synchronize()
    dsa.check_status()
    return out, lse, idx


def _check_against_oracle(c, inp, seq_lens, out, lse, idx, where):
    host = ORC.numpy_inputs(inp)
    idx_h = idx.cpu().numpy()
    for b, n_b in enumerate(seq_lens):
        cb = c.with_(B=1, Lk=n_b, q_pos0=n_b - c.Lq)
        hb = {k: v[b:b + 1] for k, v in host.items()}
        hb["kI"] = hb["kI"][:, :n_b]
        hb["kI_scale"] = hb["kI_scale"][:, :n_b]
        hb["kv"] = hb["kv"][:, :n_b]
        ref = ORC.forward_rows(hb, cb, 0, range(c.Lq))
        ro, rl = [], []
        for t in range(c.Lq):
            p = cb.q_pos0 + t
            check_selection(idx_h[b, t], ref["scores"][t], ref["idx"][t], c.k, p, f"{where} b={b} t={t}")
            o, l = ORC.sparse_mla(hb["q"][0, t], hb["kv"][0], idx_h[b, t], c.sm_scale, c.Dv)
            ro.append(o)
            rl.append(l)
        check_attention(bf16_to_f64(out[b]), np.stack(ro), lse[b].cpu().numpy(), np.stack(rl),
                        f"{where} b={b}")


def test_paged_decode_tiny_varlen():
    cfg = CONFIGS["tiny"].with_(Lq=1, mode="decode")
    lens = [1, 20, 129, 300, 500]
    c, inp, pinp, table, seq = _paged_case(cfg, lens, 128, seed=81)
    out, lse, idx = _run_paged(c, pinp, table, seq, 128)
    _check_against_oracle(c, inp, lens, out, lse, idx, "decode")


def test_paged_chunked_prefill_tiny_varlen():
    cfg = CONFIGS["tiny"].with_(Lq=40)
    lens = [40, 100, 400]
    c, inp, pinp, table, seq = _paged_case(cfg, lens, 128, seed=82)
    out, lse, idx = _run_paged(c, pinp, table, seq, 128)
    _check_against_oracle(c, inp, lens, out, lse, idx, "prefill")


def test_paged_decode_full_dims():
    cfg = CONFIGS["decode_128k"].with_(Lq=1)
    lens = [1000, 2048, 2049, 9000]
    c, inp, pinp, table, seq = _paged_case(cfg, lens, 256, seed=83)
    out, lse, idx = _run_paged(c, pinp, table, seq, 256)
    _check_against_oracle(c, inp, lens, out, lse, idx, "decode full")


def test_identity_pages_equal_the_unpaged_forward():
    # one page per block in order and every sequence full: the paged call is the
    # plain dsa_forward on the same rows, bit for bit
    cfg = CONFIGS["tiny"].with_(Lq=1, mode="decode")
    lens = [384, 384, 384]
    c, inp, pinp, table, seq = _paged_case(cfg, lens, 128, seed=84, shuffle=False)
    out_p, lse_p, idx_p = _run_paged(c, pinp, table, seq, 128)
    p = dsa.Problem.from_config(c)
    out = torch.empty_like(out_p)
    lse = torch.empty_like(lse_p)
    idx = torch.empty_like(idx_p)
    dsa.forward(p, inp, out=out, lse=lse, idx_out=idx)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_p) and torch.equal(out, out_p) and torch.equal(lse, lse_p)
