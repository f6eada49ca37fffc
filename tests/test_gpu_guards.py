"""Guard bands around every buffer the library writes.

compute-sanitizer is not available on the GPU pool, so out-of-bounds writes are
caught this way instead: each output and workspace handed to the C ABI is a
window of a larger allocation whose bytes before and after the window hold a
fixed pattern. After the call (and a device synchronisation) the pattern must be
intact: no kernel wrote outside the buffer it was given. The calls cover every
entry point that writes device memory, at shapes with ragged tails (row counts
and key counts that are not multiples of the tile sizes) and at full dimensions.
"""
import numpy as np
import pytest
import torch

import sparse_attention_long_scores_b200 as dsa
from dsa_inputs import CONFIGS, gen_inputs, output_gradient, random_key_sets, random_scores

pytestmark = pytest.mark.gpu

PRE = 256            # guard bytes before a window (keeps the window 256-byte aligned)
POST = 64 * 1024     # guard bytes after it
PATTERN = 0xA5


class Guarded:
    """Device buffers with a guard pattern on both sides."""

    def __init__(self):
        self.bufs = []

    def new(self, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        full = torch.full((PRE + nbytes + POST,), PATTERN, dtype=torch.uint8, device="cuda")
        view = full[PRE:PRE + nbytes].view(dtype).view(shape) if nbytes else \
            torch.empty(shape, dtype=dtype, device="cuda")
        self.bufs.append((full, nbytes))
        return view

    def bytes(self, n):
        return self.new((max(int(n), 1),), torch.uint8)

    def check(self, where):
        torch.cuda.synchronize()
        dsa.check_status()
        for i, (full, nbytes) in enumerate(self.bufs):
            pre = full[:PRE]
            post = full[PRE + nbytes:]
            bad_pre = int((pre != PATTERN).sum())
            bad_post = int((post != PATTERN).sum())
            assert bad_pre == 0 and bad_post == 0, (
                f"{where}: buffer {i} ({nbytes} bytes): {bad_pre} guard bytes before and "
                f"{bad_post} after it were overwritten")


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_attention_long_scores_b200.build import build
    build()
    torch.cuda.set_device(0)


@pytest.mark.parametrize("name,kw", [
    ("tiny", dict(Lq=257, Lk=257)),
    ("tiny", dict(B=3, Lq=37, Lk=301, q_pos0=264)),
    ("prefill_8k", dict(Lq=700, Lk=3001, q_pos0=2301)),
    ("decode_128k", dict(B=5, Lk=9001, q_pos0=9000)),
])
def test_forward_writes_stay_inside_buffers(name, kw):
    cfg = CONFIGS[name].with_(**kw)
    inp = gen_inputs(cfg, "cuda", seed=31)
    p = dsa.Problem.from_config(cfg)
    g = Guarded()
    out = g.new((cfg.B, cfg.Lq, cfg.H, cfg.Dv), torch.bfloat16)
    lse = g.new((cfg.B, cfg.Lq, cfg.H), torch.float32)
    idx = g.new((cfg.B, cfg.Lq, cfg.k), torch.int32)
    ws = g.bytes(dsa.forward_workspace_size(p))
    dsa.forward(p, inp, out=out, lse=lse, idx_out=idx, ws=ws)
    g.check(f"dsa_forward {name} {kw}")
    # without idx_out the selection lives in the workspace
    out2 = g.new((cfg.B, cfg.Lq, cfg.H, cfg.Dv), torch.bfloat16)
    dsa.forward(p, inp, out=out2, ws=ws)
    g.check(f"dsa_forward (idx in workspace) {name} {kw}")
    assert torch.equal(out, out2)


def test_stage_entry_points_write_inside_buffers():
    cfg = CONFIGS["prefill_8k"].with_(B=2, Lq=33, Lk=2305, q_pos0=2272)
    inp = gen_inputs(cfg, "cuda", seed=32)
    g = Guarded()
    sc = g.new((cfg.B, cfg.Lq, cfg.Lk), torch.float32)
    dsa.indexer_scores(inp["qI"], inp["qI_scale"], inp["kI"], inp["kI_scale"], inp["w"],
                       q_pos0=cfg.q_pos0, scores=sc)
    g.check("dsa_indexer_scores")
    idx = g.new((cfg.B, cfg.Lq, cfg.k), torch.int32)
    dsa.topk_select(sc, cfg.k, q_pos0=cfg.q_pos0, idx=idx)
    g.check("dsa_topk_select")
    out = g.new((cfg.B, cfg.Lq, cfg.H, cfg.Dv), torch.bfloat16)
    lse = g.new((cfg.B, cfg.Lq, cfg.H), torch.float32)
    ws = g.bytes(dsa.sparse_mla_workspace_size(cfg.B, cfg.Lq, cfg.Lk, cfg.H, cfg.Dqk, cfg.Dv, cfg.k))
    dsa.sparse_mla_fwd(inp["q"], inp["kv"], idx, cfg.sm_scale, cfg.Dv, out=out, lse=lse, ws=ws)
    g.check("dsa_sparse_mla_fwd")
    sel = random_scores((cfg.B, cfg.Lq, cfg.k), seed=33).cuda()
    p_out = g.new((cfg.B, cfg.Lq, cfg.k), torch.float32)
    kl = g.new((cfg.B, cfg.Lq), torch.float32)
    dsa.indexer_kl(inp["q"], inp["kv"], idx, lse, sel, cfg.sm_scale, p_out=p_out, kl_out=kl)
    g.check("dsa_indexer_kl")
    dI = g.new((cfg.B, cfg.Lq, cfg.k), torch.float32)
    dsa.indexer_kl_grad(sel, p_out, idx, cfg.Lk, dI=dI)
    g.check("dsa_indexer_kl_grad")


def test_decode_key_split_path_writes_inside_buffers():
    # few tokens: the attention splits keys and merges partials from the workspace
    cfg = CONFIGS["decode_128k"].with_(B=3, Lk=7001, q_pos0=7000)
    inp = gen_inputs(cfg, "cuda", seed=34, only=("q", "kv"))
    idx = random_key_sets(cfg.B, 1, cfg.k, cfg.q_pos0, seed=35, holes=0.05).cuda()
    g = Guarded()
    out = g.new((cfg.B, 1, cfg.H, cfg.Dv), torch.bfloat16)
    lse = g.new((cfg.B, 1, cfg.H), torch.float32)
    need = dsa.sparse_mla_workspace_size(cfg.B, 1, cfg.Lk, cfg.H, cfg.Dqk, cfg.Dv, cfg.k)
    assert need > 0   # the key-split path
    ws = g.bytes(need)
    dsa.sparse_mla_fwd(inp["q"], inp["kv"], idx, cfg.sm_scale, cfg.Dv, out=out, lse=lse, ws=ws)
    g.check("dsa_sparse_mla_fwd, key splits")


def test_gradients_write_inside_buffers():
    cfg = CONFIGS["prefill_8k"].with_(B=1, Lq=70, Lk=2100, q_pos0=2030)
    inp = gen_inputs(cfg, "cuda", seed=36)
    idx = random_key_sets(1, cfg.Lq, cfg.k, cfg.q_pos0, seed=37, holes=0.1).cuda()
    dout = output_gradient((1, cfg.Lq, cfg.H, cfg.Dv), seed=38).cuda()
    _, lse = dsa.sparse_mla_fwd(inp["q"], inp["kv"], idx, cfg.sm_scale, cfg.Dv)
    g = Guarded()
    dq = g.new((1, cfg.Lq, cfg.H, cfg.Dqk), torch.float32)
    dkv = g.new((1, cfg.Lk, cfg.Dqk), torch.float32)
    ws = g.bytes(dsa.lib().dsa_sparse_mla_bwd_workspace_size(1, cfg.Lq, cfg.H, cfg.Dqk, cfg.Dv, cfg.k))
    dsa.sparse_mla_bwd(inp["q"], inp["kv"], idx, lse, dout, cfg.sm_scale, dq=dq, dkv=dkv, ws=ws)
    g.check("dsa_sparse_mla_bwd")
    dI = random_scores((1, cfg.Lq, cfg.k), seed=39).cuda()
    dqI = g.new((1, cfg.Lq, cfg.H_I, cfg.d_I), torch.float32)
    dkI = g.new((1, cfg.Lk, cfg.d_I), torch.float32)
    dw = g.new((1, cfg.Lq, cfg.H_I), torch.float32)
    wsi = g.bytes(dsa.lib().dsa_indexer_bwd_workspace_size(1, cfg.Lq, cfg.H_I, cfg.d_I, cfg.k))
    dsa.indexer_bwd(inp["qI"], inp["qI_scale"], inp["kI"], inp["kI_scale"], inp["w"], idx, dI,
                    dqI=dqI, dkI=dkI, dw=dw, ws=wsi)
    g.check("dsa_indexer_bwd")


def test_paged_forward_writes_inside_buffers():
    cfg = CONFIGS["tiny"].with_(B=3, Lq=1, Lk=512, q_pos0=511, mode="decode")
    page = 128
    lens = torch.tensor([1, 300, 512], dtype=torch.int32)
    nblk = cfg.Lk // page
    pool_pages = cfg.B * nblk + 2
    gen = torch.Generator().manual_seed(40)
    perm = torch.randperm(pool_pages, generator=gen)[:cfg.B * nblk].view(cfg.B, nblk).to(torch.int32)
    base = gen_inputs(cfg.with_(B=1, Lk=pool_pages * page, q_pos0=pool_pages * page - 1), "cuda", seed=41)
    inp = gen_inputs(cfg, "cuda", seed=42)
    paged = dict(qI=inp["qI"], qI_scale=inp["qI_scale"], w=inp["w"], q=inp["q"],
                 kv=base["kv"][0], kI=base["kI"][0], kI_scale=base["kI_scale"][0])
    p = dsa.Problem.from_config(cfg)
    g = Guarded()
    out = g.new((cfg.B, 1, cfg.H, cfg.Dv), torch.bfloat16)
    lse = g.new((cfg.B, 1, cfg.H), torch.float32)
    idx = g.new((cfg.B, 1, cfg.k), torch.int32)
    ws = g.bytes(dsa.forward_paged_workspace_size(p))
    dsa.forward_paged(p, paged, perm.cuda(), lens.cuda(), page, out=out, lse=lse, idx_out=idx, ws=ws)
    g.check("dsa_forward_paged")
