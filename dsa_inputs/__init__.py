"""Seeded synthetic inputs for the DeepSeek Sparse Attention (DSA) forward path.

This module is shared by the tests, the benchmark and the oracle checks. It
only draws random numbers and packs them into the storage formats the method
consumes (FP8 e4m3 bytes with fp32 scales, bf16, fp32). It holds none of the
method's arithmetic: no index score, no selection, no attention.

Workload shapes follow the DSA description in "DeepSeek-V3.2: Pushing the
Frontier of Open Large Language Models" (bud-325 paper digest, "Key claims",
§2.1 Eq. 1-2 and "Method": H_I indexer heads in FP8, top-k = 2048, MLA in MQA
mode with one latent row shared by all query heads). The pages fix no tensor
dimension besides k; the dimensions below are the stated benchmark workloads.

Seeding: each workload has a base seed 1000 + its position in ``CONFIG_ORDER``.
``numpy.random.SeedSequence(base).spawn(5)`` gives one child per tensor in the
order qI, kI, w, q, kv. On the CPU each child drives a PCG64 generator; on a
CUDA device each child's first 64-bit state word seeds a torch Philox
generator. The two devices therefore give different (but each reproducible)
values; a test always feeds the *same bytes* to both the oracle and the
kernels, so this never affects parity.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch

E4M3_MAX = 448.0


@dataclass(frozen=True)
class DsaConfig:
    name: str
    mode: str            # "prefill" or "decode"
    B: int               # batch (sequences)
    Lq: int              # query rows per sequence
    Lk: int              # keys per sequence
    q_pos0: int          # absolute position of query row 0
    H_I: int             # indexer heads
    d_I: int             # indexer head dim
    k: int               # top-k
    H: int               # attention (query) heads
    Dqk: int             # latent key width (latent + rope)
    Dv: int              # value width (leading part of the latent row)
    sm_scale: float
    w_dtype: str         # "f32" or "bf16"
    qkv_std: float       # std of q and kv (normal)

    @property
    def tokens(self) -> int:
        return self.B * self.Lq

    def with_(self, **kw) -> "DsaConfig":
        return replace(self, **kw)


def _prefill(name, B, L, **kw) -> DsaConfig:
    base = dict(mode="prefill", B=B, Lq=L, Lk=L, q_pos0=0, H_I=64, d_I=128, k=2048,
                H=128, Dqk=576, Dv=512, sm_scale=1.0 / math.sqrt(192.0),
                w_dtype="bf16", qkv_std=0.5)
    base.update(kw)
    return DsaConfig(name=name, B=B, Lq=L, Lk=L, **{k: v for k, v in base.items()
                                                   if k not in ("B", "Lq", "Lk")})


CONFIGS = {
    # Tiny causal prefill: the oracle finishes it in seconds.
    "tiny": DsaConfig(name="tiny", mode="prefill", B=1, Lq=256, Lk=256, q_pos0=0,
                      H_I=4, d_I=32, k=32, H=8, Dqk=80, Dv=64,
                      sm_scale=1.0 / math.sqrt(80.0), w_dtype="f32", qkv_std=1.0),
    "prefill_8k": _prefill("prefill_8k", 1, 8192),
    "prefill_32k": _prefill("prefill_32k", 2, 32768),
    "prefill_128k": _prefill("prefill_128k", 1, 131072),
    # Decode: one new query token per sequence against a 131072-token cache
    # that already holds it (q_pos0 = Lk - 1).
    "decode_128k": DsaConfig(name="decode_128k", mode="decode", B=64, Lq=1, Lk=131072,
                             q_pos0=131071, H_I=64, d_I=128, k=2048, H=128, Dqk=576,
                             Dv=512, sm_scale=1.0 / math.sqrt(192.0), w_dtype="bf16",
                             qkv_std=1.0),
}
CONFIG_ORDER = ["tiny", "prefill_8k", "prefill_32k", "prefill_128k", "decode_128k"]
TENSOR_ORDER = ["qI", "kI", "w", "q", "kv"]


def child_seeds(cfg: DsaConfig, seed: int | None = None) -> dict:
    """One SeedSequence child per tensor, in the fixed tensor order."""
    base = 1000 + CONFIG_ORDER.index(cfg.name) if seed is None else seed
    kids = np.random.SeedSequence(base).spawn(len(TENSOR_ORDER))
    return dict(zip(TENSOR_ORDER, kids))


class _Source:
    """Normal / uniform draws from either numpy PCG64 (cpu) or torch Philox (cuda)."""

    def __init__(self, seq: np.random.SeedSequence, device: str):
        self.device = torch.device(device)
        if self.device.type == "cpu":
            self.rng = np.random.Generator(np.random.PCG64(seq))
            self.gen = None
        else:
            self.rng = None
            self.gen = torch.Generator(device=self.device)
            self.gen.manual_seed(int(seq.generate_state(1, np.uint64)[0] & ((1 << 63) - 1)))

    def normal(self, n: int) -> torch.Tensor:
        if self.rng is not None:
            return torch.from_numpy(self.rng.standard_normal(n, dtype=np.float32))
        return torch.randn(n, generator=self.gen, device=self.device, dtype=torch.float32)

    def uniform(self, n: int) -> torch.Tensor:
        if self.rng is not None:
            return torch.from_numpy(self.rng.random(n, dtype=np.float32))
        return torch.rand(n, generator=self.gen, device=self.device, dtype=torch.float32)


def quantize_e4m3_rows(x: torch.Tensor):
    """Per-row absmax scaling to FP8 e4m3 storage.

    x: float32 [..., d]. Returns (codes uint8 [..., d], scale float32 [...]) with
    x ~= decode(codes) * scale. scale = absmax / 448 (1.0 for an all-zero row);
    the cast rounds to nearest-even and values are clamped to +-448 first.
    """
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (x / scale.unsqueeze(-1)).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale.to(torch.float32)


def _fill_normal_bf16(src: _Source, shape, std: float, chunk: int = 1 << 27) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16, device=src.device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        flat[s:e] = (src.normal(e - s) * std).to(torch.bfloat16)
    return out


def _quantized_normal(src: _Source, rows: int, d: int, chunk_rows: int = 1 << 20):
    codes = torch.empty((rows, d), dtype=torch.uint8, device=src.device)
    scales = torch.empty((rows,), dtype=torch.float32, device=src.device)
    for s in range(0, rows, chunk_rows):
        e = min(rows, s + chunk_rows)
        x = src.normal((e - s) * d).view(e - s, d)
        c, sc = quantize_e4m3_rows(x)
        codes[s:e] = c
        scales[s:e] = sc
    return codes, scales


def gen_inputs(cfg: DsaConfig, device: str = "cpu", seed: int | None = None,
               only: tuple | None = None) -> dict:
    """Generate every input tensor of one workload.

    Returns a dict of torch tensors (contiguous):
      qI        uint8   [B, Lq, H_I, d_I]  e4m3 codes of the indexer queries
      qI_scale  float32 [B, Lq, H_I]       one scale per (token, indexer head) row
      kI        uint8   [B, Lk, d_I]       e4m3 codes of the indexer keys
      kI_scale  float32 [B, Lk]            one scale per key token
      w         float32 or bfloat16 [B, Lq, H_I]   per-head index weights ~ U(0,1)
      q         bfloat16 [B, Lq, H, Dqk]   attention queries
      kv        bfloat16 [B, Lk, Dqk]      latent rows; values are the first Dv columns
    ``only`` restricts generation to a subset of tensor names (the others are skipped,
    but the per-tensor seeds stay the same).
    """
    seeds = child_seeds(cfg, seed)
    want = set(TENSOR_ORDER if only is None else only)
    out = {}
    B, Lq, Lk = cfg.B, cfg.Lq, cfg.Lk
    if "qI" in want:
        c, s = _quantized_normal(_Source(seeds["qI"], device), B * Lq * cfg.H_I, cfg.d_I)
        out["qI"] = c.view(B, Lq, cfg.H_I, cfg.d_I)
        out["qI_scale"] = s.view(B, Lq, cfg.H_I)
    if "kI" in want:
        c, s = _quantized_normal(_Source(seeds["kI"], device), B * Lk, cfg.d_I)
        out["kI"] = c.view(B, Lk, cfg.d_I)
        out["kI_scale"] = s.view(B, Lk)
    if "w" in want:
        w = _Source(seeds["w"], device).uniform(B * Lq * cfg.H_I).view(B, Lq, cfg.H_I)
        out["w"] = w if cfg.w_dtype == "f32" else w.to(torch.bfloat16)
    if "q" in want:
        out["q"] = _fill_normal_bf16(_Source(seeds["q"], device), (B, Lq, cfg.H, cfg.Dqk),
                                     cfg.qkv_std)
    if "kv" in want:
        out["kv"] = _fill_normal_bf16(_Source(seeds["kv"], device), (B, Lk, cfg.Dqk),
                                      cfg.qkv_std)
    return out


def output_gradient(shape, seed: int, device: str = "cpu", std: float = 1.0) -> torch.Tensor:
    """Seeded N(0, std^2) bf16 stand-in for dL/d(out), the loss gradient that reaches
    the attention output in the sparse training stage. numpy PCG64 on the CPU, torch
    Philox on a CUDA device (the same seed gives different values on the two)."""
    return _fill_normal_bf16(_Source(np.random.SeedSequence(seed), device), shape, std)


def sample_rows(cfg: DsaConfig, n_per_seq: int = 64) -> list:
    """Query rows checked against the oracle at full size.

    Per sequence: rows around the top-k boundary (p+1 = k, k+1), an even stride
    over the rest, and the last row. Returns sorted unique local row indices t.
    """
    Lq, k = cfg.Lq, cfg.k
    t_edge = max(0, k - 1 - cfg.q_pos0)
    rows = {0, Lq - 1}
    for d in (-1, 0, 1):
        t = t_edge + d
        if 0 <= t < Lq:
            rows.add(t)
    rest = max(1, n_per_seq - len(rows))
    for i in range(rest):
        rows.add(int(round(i * (Lq - 1) / max(1, rest - 1))))
    return sorted(r for r in rows if 0 <= r < Lq)


def random_key_sets(B: int, Lq: int, k: int, q_pos0: int, seed: int, holes: float = 0.0) -> torch.Tensor:
    """Seeded random key sets shaped like a top-k selection: for query row t (absolute
    position p = q_pos0 + t) a uniformly random subset of the causal keys 0..p of size
    min(k, p + 1), ascending, padded with -1. With holes > 0 that fraction of the kept
    entries is replaced by -1 as well (entries outside the set may sit anywhere).
    Returns int32 [B, Lq, k] on the CPU."""
    rng = np.random.default_rng(seed)
    out = np.full((B, Lq, k), -1, dtype=np.int32)
    for b in range(B):
        for t in range(Lq):
            n = q_pos0 + t + 1
            m = min(k, n)
            sel = np.sort(rng.choice(n, size=m, replace=False)) if m < n else np.arange(n)
            if holes > 0.0:
                sel = np.where(rng.random(m) < holes, -1, sel)
            out[b, t, :m] = sel
    return torch.from_numpy(out)


def random_scores(shape, seed: int, std: float = 2.0) -> torch.Tensor:
    """Seeded N(0, std^2) fp32 values (stand-ins for index scores). CPU tensor."""
    rng = np.random.default_rng(seed)
    return torch.from_numpy((rng.standard_normal(shape) * std).astype(np.float32))
