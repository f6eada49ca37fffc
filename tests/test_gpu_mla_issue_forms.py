"""The sparse MLA kernel has two MMA issue forms: the whole issuer warp runs the
issue loop when a sequence has several query rows (prefill), one lane runs it when
each sequence has one row (decode). Both issue the same MMAs in the same order, so
the same (query row, selected keys) must give bit-identical output and lse either
way. With at least as many CTAs as SMs the launch uses one key split in both forms.
"""
import pytest
import torch

import sparse_attention_long_scores_b200 as dsa

pytestmark = pytest.mark.gpu

H, DQK, DV, K = 128, 576, 512, 2048
ROWS, LK = 96, 2304          # 96 rows x 2 value halves = 192 CTAs: one key split


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_attention_long_scores_b200.build import build
    build()
    torch.cuda.set_device(0)


def _inputs(seed: int):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(1, ROWS, H, DQK, generator=g) * 0.5).bfloat16()
    kv = (torch.randn(1, LK, DQK, generator=g) * 0.5).bfloat16()
    idx = torch.stack([torch.sort(torch.randperm(LK, generator=g)[:K]).values for _ in range(ROWS)])
    idx = idx.to(torch.int32).view(1, ROWS, K)
    idx[0, 5, K - 100:] = -1          # trailing padding: fewer tiles
    idx[0, 7, 1000:] = -1             # a row ending in mid-tile
    idx[0, 11, ::3] = -1              # invalid entries scattered through the row
    return q.cuda(), kv.cuda(), idx.cuda()


@pytest.mark.parametrize("seed", [1, 2])
def test_warp_and_single_lane_issue_agree_bit_for_bit(seed):
    q, kv, idx = _inputs(seed)
    scale = DQK ** -0.5
    # one sequence of ROWS query rows: the warp-wide issuer
    out_w, lse_w = dsa.sparse_mla_fwd(q, kv, idx, scale, DV)
    # ROWS sequences of one query row each (each with a copy of the same cache): one lane
    q1 = q.view(ROWS, 1, H, DQK).contiguous()
    kv1 = kv.expand(ROWS, LK, DQK).contiguous()
    idx1 = idx.view(ROWS, 1, K).contiguous()
    out_l, lse_l = dsa.sparse_mla_fwd(q1, kv1, idx1, scale, DV)
    torch.cuda.synchronize()
    dsa.check_status()
    assert torch.isfinite(out_w.float()).all()
    assert torch.equal(out_w.view(ROWS, 1, H, DV), out_l)
    assert torch.equal(lse_w.view(ROWS, 1, H), lse_l)
