"""The host logic of the split-cache decode (decode_split_cache) as two gloo ranks on
the CPU: each rank holds one shard of the key cache; the candidates and the partial
attentions travel through the real process group's all-gather. The per-device
steps are stood in for by the fp64 oracle (this file's _OracleOps), so the test
checks the orchestration: shard offsets, gather order, the merge rule and the
combine, against the oracle's unsplit selection and attention.
"""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class _OracleOps:
    """The per-device steps in fp64 on the CPU (candidate scores travel as fp32)."""

    @staticmethod
    def select(p, inp, idx, sel):
        import oracle as ORC
        h = ORC.numpy_inputs(inp)
        for b in range(p.B):
            sc = ORC.index_scores(h["qI"][b, 0], h["qI_scale"][b, 0], h["w"][b, 0], h["kI"][b],
                                  h["kI_scale"][b])
            top = ORC.topk_select(sc, p.k)
            idx[b, 0] = torch.from_numpy(top.astype(np.int32))
            sel[b, 0] = torch.from_numpy(np.where(top >= 0, sc[np.maximum(top, 0)], 0.0))

    @staticmethod
    def merge(cs, ci, lo):
        G, B, _, k = cs.shape
        out = torch.full((B, 1, k), -1, dtype=torch.int32)
        for b in range(B):
            pairs = [(float(cs[g, b, 0, j]), int(lo[g]) + int(ci[g, b, 0, j])) for g in range(G)
                     for j in range(k) if ci[g, b, 0, j] >= 0]
            best = sorted(sorted(pairs, key=lambda x: (-x[0], x[1]))[:k], key=lambda x: x[1])
            out[b, 0, :len(best)] = torch.tensor([x[1] for x in best], dtype=torch.int32)
        return out

    @staticmethod
    def localize(idx, lo, length):
        return torch.where((idx >= lo) & (idx < lo + length), idx - lo, torch.full_like(idx, -1))

    @staticmethod
    def attend(q, kv, idx_local, sm_scale, Dv):
        import oracle as ORC
        B, _, H, _ = q.shape
        out = torch.zeros((B, 1, H, Dv), dtype=torch.float64)
        lse = torch.zeros((B, 1, H), dtype=torch.float64)
        h = ORC.numpy_inputs({"q": q, "kv": kv})
        for b in range(B):
            o, l = ORC.sparse_mla(h["q"][b, 0], h["kv"][b], idx_local[b, 0].numpy(), sm_scale, Dv)
            out[b, 0], lse[b, 0] = torch.from_numpy(o), torch.from_numpy(l)
        return out, lse

    @staticmethod
    def combine(part_out, part_lse):
        lse = torch.logsumexp(part_lse.double(), dim=0)
        w = torch.exp(part_lse.double() - lse)
        w = torch.nan_to_num(w, nan=0.0)
        return (w[..., None] * part_out.double()).sum(0), lse


BOUNDS = [0, 130, 300]


def _cfg():
    from dsa_inputs import CONFIGS
    return CONFIGS["tiny"].with_(mode="decode", B=2, Lq=1, Lk=300, q_pos0=299)


def _worker(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import sparse_attention_long_scores_b200 as dsa
    from dsa_inputs import gen_inputs
    try:
        cfg = _cfg()
        inp = gen_inputs(cfg, "cpu", seed=7)
        a, b = BOUNDS[rank], BOUNDS[rank + 1]
        sh = {key: inp[key] for key in ("qI", "qI_scale", "w", "q")}
        for key in ("kI", "kI_scale", "kv"):
            sh[key] = inp[key][:, a:b].contiguous()
        p = dsa.Problem.from_config(cfg.with_(Lk=b - a, q_pos0=b - a - 1))
        out, lse, idx = dsa.decode_split_cache(p, sh, BOUNDS[:-1], rank=rank, ops=_OracleOps)
        q.put((rank, out.numpy(), lse.numpy(), idx.numpy()))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_split_cache_two_gloo_ranks_match_unsplit_oracle():
    import oracle as ORC
    from dsa_inputs import gen_inputs

    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r[0], r[1:]) for r in (q.get(timeout=180) for _ in range(world)))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    out, lse, idx = res[0]
    for a, b in zip(res[0], res[1]):          # every rank ends with the same result
        assert np.array_equal(a, b)
    cfg = _cfg()
    h = ORC.numpy_inputs(gen_inputs(cfg, "cpu", seed=7))
    for b in range(cfg.B):
        sc = ORC.index_scores(h["qI"][b, 0], h["qI_scale"][b, 0], h["w"][b, 0], h["kI"][b],
                              h["kI_scale"][b])
        ref_idx = ORC.topk_select(sc, cfg.k)
        assert np.array_equal(idx[b, 0], ref_idx)
        ro, rl = ORC.sparse_mla(h["q"][b, 0], h["kv"][b], ref_idx, cfg.sm_scale, cfg.Dv)
        assert np.allclose(out[b, 0], ro, rtol=1e-9, atol=1e-12)
        assert np.allclose(lse[b, 0], rl, rtol=1e-9, atol=1e-12)
