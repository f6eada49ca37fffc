"""The allocation-free sparse-attention entry point, called through the C ABI.

dsa_sparse_mla_fwd_noalloc serves callers that cannot allocate device memory
or pass a workspace (for example a plugin inside a host framework that owns
all device memory). It keeps its key-split partials in a fixed array inside
the library. These checks compare it with dsa_sparse_mla_fwd on the same
inputs (bit for bit where both use the same key splits) and with the fp64
oracle, on calls in a row that use a small, a larger and again a smaller part
of the shared array, so that state left there by one call cannot leak into the
next.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as ORC
import sparse_attention_long_scores_b200 as dsa
from parity import bf16_to_f64, check_attention

pytestmark = pytest.mark.gpu


def _inputs(seed, B, Lq, Lk, k, H=128, Dqk=576):
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = (torch.randn((B, Lq, H, Dqk), generator=g, device="cuda")).to(torch.bfloat16)
    kv = (torch.randn((B, Lk, Dqk), generator=g, device="cuda")).to(torch.bfloat16)
    rows = [torch.sort(torch.randperm(Lk, generator=g, device="cuda")[:k]).values
            for _ in range(B * Lq)]
    idx = torch.stack(rows).view(B, Lq, k).to(torch.int32).contiguous()
    return q, kv, idx


def _noalloc(q, kv, idx, sm_scale, Dv=512):
    B, Lq, H, Dqk = q.shape
    Lk, k = kv.shape[1], idx.shape[2]
    out = torch.empty((B, Lq, H, Dv), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Lq, H), dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = dsa.lib().dsa_sparse_mla_fwd_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kv.data_ptr()),
        ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(lse.data_ptr()), B, Lq, Lk, H, Dqk, Dv, k, ctypes.c_float(sm_scale),
        stream)
    assert rc == dsa.DSA_OK, dsa.lib().dsa_last_error().decode()
    dsa.check_status()
    return out, lse


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_attention_long_scores_b200.build import build
    build()
    torch.cuda.set_device(0)


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    """Calls in a row that need a small, a large and then a small part of the
    shared array again (5, 2, 7 and 3 decode tokens, 8 key splits each): every
    output must equal the workspace entry point's bit for bit (the same kernels
    run with the same split count), and every row must match the fp64 oracle."""
    sm_scale = 1.0 / np.sqrt(192.0)
    for seed, B, Lq, Lk in ((11, 5, 1, 8192), (12, 2, 1, 4096), (14, 7, 1, 6000), (15, 3, 1, 5000)):
        q, kv, idx = _inputs(seed, B, Lq, Lk, 2048)
        assert dsa.sparse_mla_workspace_size(B, Lq, Lk, 128, 576, 512, 2048) > 0
        out_n, lse_n = _noalloc(q, kv, idx, sm_scale)
        out_r, lse_r = dsa.sparse_mla_fwd(q, kv, idx, sm_scale, 512)
        dsa.check_status()
        assert torch.equal(out_n, out_r) and torch.equal(lse_n, lse_r), f"noalloc B={B}: not bitwise"
        q_h = q.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        kv_h = kv.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
        idx_h = idx.cpu().numpy()
        ro, rl = [], []
        for b in range(B):
            o, l = ORC.sparse_mla(q_h[b, 0], kv_h[b], idx_h[b, 0], sm_scale, 512)
            ro.append(o)
            rl.append(l)
        check_attention(bf16_to_f64(out_n[:, 0]), np.stack(ro), lse_n[:, 0].cpu().numpy(),
                        np.stack(rl), f"noalloc vs oracle B={B}")


def test_noalloc_uses_fewer_splits_when_its_scratch_is_too_small():
    # 16 decode tokens: the recommended key splits need more partial-output bytes
    # than the 16 MiB built-in scratch holds, so the entry point splits less; the
    # result must still match the workspace entry point's within the tolerances
    B, Lk, k = 16, 4096, 2048
    need = dsa.sparse_mla_workspace_size(B, 1, Lk, 128, 576, 512, k)
    assert need > (16 << 20)
    sm_scale = 1.0 / np.sqrt(192.0)
    q, kv, idx = _inputs(13, B, 1, Lk, k)
    out_n, lse_n = _noalloc(q, kv, idx, sm_scale)
    out_r, lse_r = dsa.sparse_mla_fwd(q, kv, idx, sm_scale, 512)
    dsa.check_status()
    check_attention(bf16_to_f64(out_n), bf16_to_f64(out_r), lse_n.cpu().numpy(),
                    lse_r.cpu().numpy(), "noalloc, fewer splits")
    q_h = q.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    kv_h = kv.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    idx_h = idx.cpu().numpy()
    ro, rl = [], []
    for b in range(B):
        o, l = ORC.sparse_mla(q_h[b, 0], kv_h[b], idx_h[b, 0], sm_scale, 512)
        ro.append(o)
        rl.append(l)
    check_attention(bf16_to_f64(out_n[:, 0]), np.stack(ro), lse_n[:, 0].cpu().numpy(), np.stack(rl),
                    "noalloc, fewer splits, vs oracle")
