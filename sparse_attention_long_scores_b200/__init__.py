"""Python binding of the sm_100a DeepSeek Sparse Attention forward library.

Thin ctypes layer over ``libdsa.so`` (C ABI in ``include/dsa.h``): it checks
tensor dtypes, shapes and devices, passes raw device pointers and the current
CUDA stream, and raises on a non-zero status. Every step of the path runs in
the library's CUDA kernels; there is no fallback. If the library is missing the
first call raises.

The computation ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language
Models", bud-325 paper digest, "Key claims", section 2.1 Eq. 1-2; "Method"):
    I[t,s] = sum_j w[t,j] * ReLU(q^I[t,j] . k^I[s])      (FP8 lightning indexer)
    S_t    = top-k_s I[t,s]                               (k = 2048)
    out[t] = softmax(sm_scale * q[t] . c_S^T) c_S[:, :Dv] (MLA, MQA mode)
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsa.so")

DSA_OK = 0
DSA_ERR_INVALID_ARG = -1
DSA_ERR_UNSUPPORTED_SHAPE = -2
DSA_ERR_WORKSPACE_TOO_SMALL = -3
DSA_ERR_CUDA = -4
DSA_ERR_TIMEOUT = -5
DSA_DTYPE_F32 = 0
DSA_DTYPE_BF16 = 1
DSA_MODE_PREFILL = 0
DSA_MODE_DECODE = 1

EXPORTED = [
    "dsa_last_error", "dsa_version", "dsa_indexer_scores", "dsa_topk_select",
    "dsa_sparse_mla_workspace_size", "dsa_sparse_mla_fwd", "dsa_forward_workspace_size",
    "dsa_forward", "dsa_forward_host", "dsa_forward_profiled", "dsa_check_status",
    "dsa_set_wait_limit_ns", "dsa_debug_wait_timeout", "dsa_sparse_mla_fwd_noalloc",
    "dsa_indexer_kl", "dsa_last_launch_count", "dsa_forward_paged_workspace_size",
    "dsa_forward_paged", "dsa_forward_fused", "dsa_sparse_mla_bwd_workspace_size", "dsa_sparse_mla_bwd",
    "dsa_indexer_kl_grad", "dsa_indexer_bwd_workspace_size", "dsa_indexer_bwd",
    "dsa_topk_merge_workspace_size", "dsa_topk_merge", "dsa_index_localize", "dsa_attn_combine",
]
KIND_NAMES = {1: "indexer", 2: "topk", 3: "sparse_mla", 4: "combine", 5: "indexer_topk"}


class DsaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"dsa error {code}: {msg}")
        self.code = code


class DsaProblem(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("B", ctypes.c_int), ("Lq", ctypes.c_int),
                ("Lk", ctypes.c_int), ("q_pos0", ctypes.c_int), ("H_I", ctypes.c_int),
                ("d_I", ctypes.c_int), ("H", ctypes.c_int), ("Dqk", ctypes.c_int),
                ("Dv", ctypes.c_int), ("k", ctypes.c_int), ("sm_scale", ctypes.c_float),
                ("w_dtype", ctypes.c_int)]


class DsaTensors(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("qI", "qI_scale", "kI", "kI_scale", "w", "q", "kv", "out", "lse", "idx_out",
                 "sel_scores_out")]


class DsaPagedCache(ctypes.Structure):
    _fields_ = [("block_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("max_blocks", ctypes.c_int), ("page_size", ctypes.c_int),
                ("num_pages", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load ``libdsa.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                           "(run python -m sparse_attention_long_scores_b200.build)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.dsa_last_error.restype = ctypes.c_char_p
    L.dsa_version.restype = ctypes.c_char_p
    L.dsa_indexer_scores.argtypes = [vp, vp, vp, vp, vp, i, vp, i, i, i, i, i, i, vp]
    L.dsa_topk_select.argtypes = [vp, vp, i, i, i, i, i, vp]
    L.dsa_sparse_mla_workspace_size.argtypes = [i, i, i, i, i, i, i]
    L.dsa_sparse_mla_workspace_size.restype = sz
    L.dsa_sparse_mla_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, ctypes.c_float,
                                     vp, sz, vp]
    L.dsa_sparse_mla_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i,
                                             ctypes.c_float, vp]
    L.dsa_sparse_mla_fwd_noalloc.restype = i
    L.dsa_indexer_kl.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, ctypes.c_float, vp]
    L.dsa_forward_workspace_size.argtypes = [ctypes.POINTER(DsaProblem)]
    L.dsa_forward_workspace_size.restype = sz
    L.dsa_forward.argtypes = [ctypes.POINTER(DsaProblem), ctypes.POINTER(DsaTensors), vp, sz, vp]
    L.dsa_forward_fused.argtypes = [ctypes.POINTER(DsaProblem), ctypes.POINTER(DsaTensors), vp, sz, vp]
    L.dsa_forward_paged_workspace_size.argtypes = [ctypes.POINTER(DsaProblem)]
    L.dsa_forward_paged_workspace_size.restype = sz
    L.dsa_forward_paged.argtypes = [ctypes.POINTER(DsaProblem), ctypes.POINTER(DsaTensors),
                                    ctypes.POINTER(DsaPagedCache), vp, sz, vp]
    L.dsa_forward_host.argtypes = [ctypes.POINTER(DsaProblem), ctypes.POINTER(DsaTensors),
                                   ctypes.POINTER(DsaTensors), vp, sz, vp]
    L.dsa_forward_profiled.argtypes = [ctypes.POINTER(DsaProblem), ctypes.POINTER(DsaTensors), vp,
                                       sz, vp, ctypes.POINTER(ctypes.c_void_p),
                                       ctypes.POINTER(ctypes.c_int), i, ctypes.POINTER(ctypes.c_int)]
    L.dsa_sparse_mla_bwd_workspace_size.argtypes = [i, i, i, i, i, i]
    L.dsa_sparse_mla_bwd_workspace_size.restype = sz
    L.dsa_sparse_mla_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i,
                                     ctypes.c_float, vp, sz, vp]
    L.dsa_indexer_kl_grad.argtypes = [vp, vp, vp, vp, i, i, i, i, ctypes.c_float, vp]
    L.dsa_indexer_bwd_workspace_size.argtypes = [i, i, i, i, i]
    L.dsa_indexer_bwd_workspace_size.restype = sz
    L.dsa_indexer_bwd.argtypes = [vp, vp, vp, vp, vp, i, vp, vp, vp, vp, vp, i, i, i, i, i, i, i,
                                  vp, sz, vp]
    L.dsa_topk_merge_workspace_size.argtypes = [i, i, i]
    L.dsa_topk_merge_workspace_size.restype = sz
    L.dsa_topk_merge.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_longlong), i, i, i, vp, vp, vp,
                                 sz, vp]
    L.dsa_index_localize.argtypes = [vp, vp, ctypes.c_longlong, i, i, vp]
    L.dsa_attn_combine.argtypes = [vp, vp, i, i, i, i, vp, vp, vp]
    L.dsa_check_status.argtypes = [vp]
    L.dsa_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    L.dsa_debug_wait_timeout.argtypes = [vp]
    for name in ("dsa_indexer_scores", "dsa_topk_select", "dsa_sparse_mla_fwd", "dsa_forward",
                 "dsa_forward_host", "dsa_forward_profiled", "dsa_check_status", "dsa_set_wait_limit_ns",
                 "dsa_debug_wait_timeout", "dsa_sparse_mla_bwd", "dsa_indexer_kl_grad",
                 "dsa_indexer_bwd", "dsa_topk_merge", "dsa_index_localize", "dsa_attn_combine"):
        getattr(L, name).restype = i
    _lib = L
    return L


def _check(code: int) -> None:
    if code != DSA_OK:
        raise DsaError(code, lib().dsa_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, shape=None, cuda=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if not cuda and t.is_cuda:
        raise ValueError(f"{name} must be in host memory")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _w_dtype(w: torch.Tensor) -> int:
    if w.dtype == torch.float32:
        return DSA_DTYPE_F32
    if w.dtype == torch.bfloat16:
        return DSA_DTYPE_BF16
    raise TypeError("w must be float32 or bfloat16")


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------


def indexer_scores(qI, qI_scale, kI, kI_scale, w, q_pos0: int = 0, scores=None, stream=None):
    """Lightning-indexer scores [B, Lq, Lk] fp32 (-inf above the causal limit)."""
    B, Lq, H_I, d_I = qI.shape
    Lk = kI.shape[1]
    _need(qI, "qI", torch.uint8, (B, Lq, H_I, d_I))
    _need(qI_scale, "qI_scale", torch.float32, (B, Lq, H_I))
    _need(kI, "kI", torch.uint8, (B, Lk, d_I))
    _need(kI_scale, "kI_scale", torch.float32, (B, Lk))
    _need(w, "w", w.dtype, (B, Lq, H_I))
    if scores is None:
        scores = torch.empty((B, Lq, Lk), dtype=torch.float32, device=qI.device)
    _need(scores, "scores", torch.float32, (B, Lq, Lk))
    _check(lib().dsa_indexer_scores(_ptr(qI), _ptr(qI_scale), _ptr(kI), _ptr(kI_scale), _ptr(w),
                                    _w_dtype(w), _ptr(scores), B, Lq, Lk, q_pos0, H_I, d_I,
                                    _stream(stream)))
    return scores


def topk_select(scores, k: int, q_pos0: int = 0, idx=None, stream=None):
    """Top-k key indices [B, Lq, k] int32, ascending, ties to the lowest index, -1 padded."""
    B, Lq, Lk = scores.shape
    _need(scores, "scores", torch.float32)
    if idx is None:
        idx = torch.empty((B, Lq, k), dtype=torch.int32, device=scores.device)
    _need(idx, "idx", torch.int32, (B, Lq, k))
    _check(lib().dsa_topk_select(_ptr(scores), _ptr(idx), B, Lq, Lk, q_pos0, k, _stream(stream)))
    return idx


def sparse_mla_workspace_size(B, Lq, Lk, H, Dqk, Dv, k) -> int:
    return int(lib().dsa_sparse_mla_workspace_size(B, Lq, Lk, H, Dqk, Dv, k))


def sparse_mla_fwd(q, kv, idx, sm_scale: float, Dv: int, out=None, lse=None, ws=None,
                   with_lse: bool = True, stream=None):
    """Sparse MQA attention over the selected latent rows; returns (out bf16, lse fp32|None)."""
    B, Lq, H, Dqk = q.shape
    Lk = kv.shape[1]
    k = idx.shape[2]
    _need(q, "q", torch.bfloat16)
    _need(kv, "kv", torch.bfloat16, (B, Lk, Dqk))
    _need(idx, "idx", torch.int32, (B, Lq, k))
    if out is None:
        out = torch.empty((B, Lq, H, Dv), dtype=torch.bfloat16, device=q.device)
    _need(out, "out", torch.bfloat16, (B, Lq, H, Dv))
    if lse is None and with_lse:
        lse = torch.empty((B, Lq, H), dtype=torch.float32, device=q.device)
    if lse is not None:
        _need(lse, "lse", torch.float32, (B, Lq, H))
    need = sparse_mla_workspace_size(B, Lq, Lk, H, Dqk, Dv, k)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().dsa_sparse_mla_fwd(_ptr(q), _ptr(kv), _ptr(idx), _ptr(out), _ptr(lse), B, Lq, Lk,
                                    H, Dqk, Dv, k, float(sm_scale), _ptr(ws), ws_bytes,
                                    _stream(stream)))
    return out, lse


def indexer_kl(q, kv, idx, lse, sel_scores, sm_scale: float, p_out=None, kl_out=None,
               with_p: bool = True, stream=None):
    """Indexer alignment target (forward): per query token KL(p || r) between the
    head-aggregated attention p over the key set idx and the softmax r of the index
    scores sel_scores over the same set; lse is the forward's per-head lse over that
    set. Returns (kl fp32 [B, Lq], p fp32 [B, Lq, k] | None)."""
    B, Lq, H, Dqk = q.shape
    Lk = kv.shape[1]
    k = idx.shape[2]
    _need(q, "q", torch.bfloat16)
    _need(kv, "kv", torch.bfloat16, (B, Lk, Dqk))
    _need(idx, "idx", torch.int32, (B, Lq, k))
    _need(lse, "lse", torch.float32, (B, Lq, H))
    _need(sel_scores, "sel_scores", torch.float32, (B, Lq, k))
    if kl_out is None:
        kl_out = torch.empty((B, Lq), dtype=torch.float32, device=q.device)
    _need(kl_out, "kl_out", torch.float32, (B, Lq))
    if p_out is None and with_p:
        p_out = torch.empty((B, Lq, k), dtype=torch.float32, device=q.device)
    if p_out is not None:
        _need(p_out, "p_out", torch.float32, (B, Lq, k))
    _check(lib().dsa_indexer_kl(_ptr(q), _ptr(kv), _ptr(idx), _ptr(lse), _ptr(sel_scores),
                                _ptr(p_out), _ptr(kl_out), B, Lq, Lk, H, Dqk, k,
                                float(sm_scale), _stream(stream)))
    return kl_out, p_out


def _workspace(nbytes: int, device):
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def sparse_mla_bwd(q, kv, idx, lse, dout, sm_scale: float, dq=None, dkv=None,
                   accumulate_dkv: bool = False, ws=None, stream=None):
    """Sparse-stage attention gradients: dq [B, Lq, H, Dqk] fp32 and dkv [B, Lk, Dqk]
    fp32 from dout = dL/d(out) [B, Lq, H, Dv] bf16, given the forward's idx and lse.
    dkv is overwritten unless accumulate_dkv. Returns (dq, dkv)."""
    B, Lq, H, Dqk = q.shape
    Lk = kv.shape[1]
    k = idx.shape[2]
    Dv = dout.shape[3]
    _need(q, "q", torch.bfloat16)
    _need(kv, "kv", torch.bfloat16, (B, Lk, Dqk))
    _need(idx, "idx", torch.int32, (B, Lq, k))
    _need(lse, "lse", torch.float32, (B, Lq, H))
    _need(dout, "dout", torch.bfloat16, (B, Lq, H, Dv))
    if dq is None:
        dq = torch.empty((B, Lq, H, Dqk), dtype=torch.float32, device=q.device)
    if dkv is None:
        dkv = torch.empty((B, Lk, Dqk), dtype=torch.float32, device=q.device)
    _need(dq, "dq", torch.float32, (B, Lq, H, Dqk))
    _need(dkv, "dkv", torch.float32, (B, Lk, Dqk))
    if ws is None:
        ws = _workspace(lib().dsa_sparse_mla_bwd_workspace_size(B, Lq, H, Dqk, Dv, k), q.device)
    _check(lib().dsa_sparse_mla_bwd(_ptr(q), _ptr(kv), _ptr(idx), _ptr(lse),
                                    _ptr(dout), _ptr(dq), _ptr(dkv), int(bool(accumulate_dkv)),
                                    B, Lq, Lk, H, Dqk, Dv, k, float(sm_scale), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream)))
    return dq, dkv


def indexer_kl_grad(sel_scores, p, idx, Lk: int, loss_scale: float = 1.0, dI=None, stream=None):
    """dI = loss_scale (softmax over the set of sel_scores - p) [B, Lq, k] fp32: the
    gradient of the KL alignment loss in the selected index scores."""
    B, Lq, k = idx.shape
    _need(idx, "idx", torch.int32)
    _need(sel_scores, "sel_scores", torch.float32, (B, Lq, k))
    _need(p, "p", torch.float32, (B, Lq, k))
    if dI is None:
        dI = torch.empty((B, Lq, k), dtype=torch.float32, device=idx.device)
    _need(dI, "dI", torch.float32, (B, Lq, k))
    _check(lib().dsa_indexer_kl_grad(_ptr(sel_scores), _ptr(p), _ptr(idx), _ptr(dI), B, Lq, int(Lk),
                                     k, float(loss_scale), _stream(stream)))
    return dI


def indexer_bwd(qI, qI_scale, kI, kI_scale, w, idx, dI, dqI=None, dkI=None, dw=None,
                accumulate_dkI: bool = False, ws=None, stream=None):
    """Indexer gradients with respect to the dequantised q^I [B, Lq, H_I, d_I], k^I
    [B, Lk, d_I] and the weights w [B, Lq, H_I] (all fp32), from dI = dL/dI at the
    selected slots [B, Lq, k]. dkI is overwritten unless accumulate_dkI. Returns
    (dqI, dkI, dw)."""
    B, Lq, H_I, d_I = qI.shape
    Lk = kI.shape[1]
    k = idx.shape[2]
    _need(qI, "qI", torch.uint8)
    _need(qI_scale, "qI_scale", torch.float32, (B, Lq, H_I))
    _need(kI, "kI", torch.uint8, (B, Lk, d_I))
    _need(kI_scale, "kI_scale", torch.float32, (B, Lk))
    if w.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError("w must be float32 or bfloat16")
    _need(w, "w", w.dtype, (B, Lq, H_I))
    _need(idx, "idx", torch.int32, (B, Lq, k))
    _need(dI, "dI", torch.float32, (B, Lq, k))
    dev = qI.device
    if dqI is None:
        dqI = torch.empty((B, Lq, H_I, d_I), dtype=torch.float32, device=dev)
    if dkI is None:
        dkI = torch.empty((B, Lk, d_I), dtype=torch.float32, device=dev)
    if dw is None:
        dw = torch.empty((B, Lq, H_I), dtype=torch.float32, device=dev)
    _need(dqI, "dqI", torch.float32, (B, Lq, H_I, d_I))
    _need(dkI, "dkI", torch.float32, (B, Lk, d_I))
    _need(dw, "dw", torch.float32, (B, Lq, H_I))
    if ws is None:
        ws = _workspace(lib().dsa_indexer_bwd_workspace_size(B, Lq, H_I, d_I, k), dev)
    wd = DSA_DTYPE_BF16 if w.dtype == torch.bfloat16 else DSA_DTYPE_F32
    _check(lib().dsa_indexer_bwd(_ptr(qI), _ptr(qI_scale), _ptr(kI), _ptr(kI_scale), _ptr(w), wd,
                                 _ptr(idx), _ptr(dI), _ptr(dqI), _ptr(dkI), _ptr(dw),
                                 int(bool(accumulate_dkI)), B, Lq, Lk, H_I, d_I, k, _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)))
    return dqI, dkI, dw


@dataclass
class Problem:
    B: int
    Lq: int
    Lk: int
    q_pos0: int
    H_I: int
    d_I: int
    H: int
    Dqk: int
    Dv: int
    k: int
    sm_scale: float
    w_dtype: int = DSA_DTYPE_BF16
    mode: int = DSA_MODE_PREFILL

    @classmethod
    def from_config(cls, cfg) -> "Problem":
        return cls(B=cfg.B, Lq=cfg.Lq, Lk=cfg.Lk, q_pos0=cfg.q_pos0, H_I=cfg.H_I, d_I=cfg.d_I,
                   H=cfg.H, Dqk=cfg.Dqk, Dv=cfg.Dv, k=cfg.k, sm_scale=cfg.sm_scale,
                   w_dtype=DSA_DTYPE_F32 if cfg.w_dtype == "f32" else DSA_DTYPE_BF16,
                   mode=DSA_MODE_DECODE if cfg.mode == "decode" else DSA_MODE_PREFILL)

    def c(self) -> DsaProblem:
        return DsaProblem(self.mode, self.B, self.Lq, self.Lk, self.q_pos0, self.H_I, self.d_I,
                          self.H, self.Dqk, self.Dv, self.k, self.sm_scale, self.w_dtype)


def forward_workspace_size(p: Problem) -> int:
    cp = p.c()
    n = int(lib().dsa_forward_workspace_size(ctypes.byref(cp)))
    if n == 0:
        raise DsaError(DSA_ERR_INVALID_ARG, lib().dsa_last_error().decode())
    return n


def _tensors(inp: dict, out, lse, idx_out, sel_scores=None) -> DsaTensors:
    return DsaTensors(*[None if x is None else x.data_ptr() for x in (
        inp["qI"], inp["qI_scale"], inp["kI"], inp["kI_scale"], inp["w"], inp["q"], inp["kv"],
        out, lse, idx_out, sel_scores)])


def _need_inputs(p: "Problem", inp: dict, prefix: str = "", cuda: bool = True) -> None:
    """Dtype, shape and contiguity of the seven input tensors of problem p."""
    _need(inp["qI"], prefix + "qI", torch.uint8, (p.B, p.Lq, p.H_I, p.d_I), cuda)
    _need(inp["qI_scale"], prefix + "qI_scale", torch.float32, (p.B, p.Lq, p.H_I), cuda)
    _need(inp["kI"], prefix + "kI", torch.uint8, (p.B, p.Lk, p.d_I), cuda)
    _need(inp["kI_scale"], prefix + "kI_scale", torch.float32, (p.B, p.Lk), cuda)
    _need(inp["w"], prefix + "w", torch.float32 if p.w_dtype == DSA_DTYPE_F32 else torch.bfloat16,
          (p.B, p.Lq, p.H_I), cuda)
    _need(inp["q"], prefix + "q", torch.bfloat16, (p.B, p.Lq, p.H, p.Dqk), cuda)
    _need(inp["kv"], prefix + "kv", torch.bfloat16, (p.B, p.Lk, p.Dqk), cuda)


def forward(p: Problem, inp: dict, out=None, lse=None, idx_out=None, ws=None, stream=None,
            sel_scores=None, fused: bool = False):
    """Whole DSA forward (indexer -> top-k -> sparse MLA) on device tensors.

    inp: dict with qI, qI_scale, kI, kI_scale, w, q, kv (see ``dsa_inputs.gen_inputs``).
    Returns out [B, Lq, H, Dv] bf16 (lse / idx_out are filled when given; sel_scores
    [B, Lq, k] fp32 receives the index score of every selected key and needs idx_out).
    fused: run dsa_forward_fused (top-k selection inside the indexer kernel).
    """
    dev = inp["q"].device
    _need_inputs(p, inp)
    if out is None:
        out = torch.empty((p.B, p.Lq, p.H, p.Dv), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, (p.B, p.Lq, p.H, p.Dv))
    if lse is not None:
        _need(lse, "lse", torch.float32, (p.B, p.Lq, p.H))
    if idx_out is not None:
        _need(idx_out, "idx_out", torch.int32, (p.B, p.Lq, p.k))
    if sel_scores is not None:
        _need(sel_scores, "sel_scores", torch.float32, (p.B, p.Lq, p.k))
    if ws is None:
        ws = torch.empty(forward_workspace_size(p), dtype=torch.uint8, device=dev)
    cp = p.c()
    ct = _tensors(inp, out, lse, idx_out, sel_scores)
    entry = lib().dsa_forward_fused if fused else lib().dsa_forward
    _check(entry(ctypes.byref(cp), ctypes.byref(ct), _ptr(ws), ws.numel() * ws.element_size(),
                 _stream(stream)))
    return out


def select(p: Problem, inp: dict, idx_out, sel_scores=None, ws=None, stream=None):
    """Selection only: dsa_forward with out = NULL (indexer and top-k; q and kv are not
    read). Fills idx_out [B, Lq, k] and, when given, sel_scores [B, Lq, k]."""
    dev = inp["qI"].device
    for name, t, dt, shape in (("qI", inp["qI"], torch.uint8, (p.B, p.Lq, p.H_I, p.d_I)),
                               ("qI_scale", inp["qI_scale"], torch.float32, (p.B, p.Lq, p.H_I)),
                               ("kI", inp["kI"], torch.uint8, (p.B, p.Lk, p.d_I)),
                               ("kI_scale", inp["kI_scale"], torch.float32, (p.B, p.Lk))):
        _need(t, name, dt, shape)
    _need(inp["w"], "w", torch.float32 if p.w_dtype == DSA_DTYPE_F32 else torch.bfloat16,
          (p.B, p.Lq, p.H_I))
    _need(idx_out, "idx_out", torch.int32, (p.B, p.Lq, p.k))
    if sel_scores is not None:
        _need(sel_scores, "sel_scores", torch.float32, (p.B, p.Lq, p.k))
    if ws is None:
        ws = torch.empty(forward_workspace_size(p), dtype=torch.uint8, device=dev)
    cp = p.c()
    ct = DsaTensors(*[None if x is None else x.data_ptr() for x in (
        inp["qI"], inp["qI_scale"], inp["kI"], inp["kI_scale"], inp["w"], None, None,
        None, None, idx_out, sel_scores)])
    _check(lib().dsa_forward(ctypes.byref(cp), ctypes.byref(ct), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)))
    return idx_out


def topk_merge(cand_scores, cand_idx, shard_lo, idx_out=None, sel_out=None, ws=None, stream=None):
    """The top-k of G shards' candidates (dsa_topk_merge): cand_scores [G, *rows, k] fp32,
    cand_idx [G, *rows, k] int32 shard-local (ascending, < 0 none), shard_lo: the first
    key of each shard. Returns (idx_out [*rows, k] global, sel_out [*rows, k])."""
    G = cand_scores.shape[0]
    rows_shape = tuple(cand_scores.shape[1:-1])
    k = cand_scores.shape[-1]
    R = 1
    for d in rows_shape:
        R *= d
    _need(cand_scores, "cand_scores", torch.float32)
    _need(cand_idx, "cand_idx", torch.int32, tuple(cand_scores.shape))
    if len(shard_lo) != G:
        raise ValueError("shard_lo needs one entry per shard")
    dev = cand_scores.device
    if idx_out is None:
        idx_out = torch.empty(rows_shape + (k,), dtype=torch.int32, device=dev)
    _need(idx_out, "idx_out", torch.int32, rows_shape + (k,))
    if sel_out is None:
        sel_out = torch.empty(rows_shape + (k,), dtype=torch.float32, device=dev)
    _need(sel_out, "sel_out", torch.float32, rows_shape + (k,))
    need = int(lib().dsa_topk_merge_workspace_size(G, R, k))
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    lo = (ctypes.c_longlong * G)(*[int(x) for x in shard_lo])
    _check(lib().dsa_topk_merge(_ptr(cand_scores), _ptr(cand_idx), lo, G, R, k, _ptr(idx_out),
                                _ptr(sel_out), _ptr(ws), ws.numel() * ws.element_size(),
                                _stream(stream)))
    return idx_out, sel_out


def index_localize(idx, lo: int, length: int, out=None, stream=None):
    """A shard's view of a selection: idx - lo where lo <= idx < lo + length, else -1."""
    _need(idx, "idx", torch.int32)
    if out is None:
        out = torch.empty_like(idx)
    _need(out, "out", torch.int32, tuple(idx.shape))
    _check(lib().dsa_index_localize(_ptr(idx), _ptr(out), idx.numel(), int(lo), int(length),
                                    _stream(stream)))
    return out


def attn_combine(part_out, part_lse, out=None, lse=None, stream=None):
    """lse-weighted combine of G partial attentions (dsa_attn_combine): part_out
    [G, *rows, H, Dv] bf16, part_lse [G, *rows, H] fp32 -> (out [*rows, H, Dv], lse)."""
    G, H, Dv = part_out.shape[0], part_out.shape[-2], part_out.shape[-1]
    rows_shape = tuple(part_out.shape[1:-2])
    R = 1
    for d in rows_shape:
        R *= d
    _need(part_out, "part_out", torch.bfloat16)
    _need(part_lse, "part_lse", torch.float32, (G,) + rows_shape + (H,))
    dev = part_out.device
    if out is None:
        out = torch.empty(rows_shape + (H, Dv), dtype=torch.bfloat16, device=dev)
    _need(out, "out", torch.bfloat16, rows_shape + (H, Dv))
    if lse is None:
        lse = torch.empty(rows_shape + (H,), dtype=torch.float32, device=dev)
    _need(lse, "lse", torch.float32, rows_shape + (H,))
    _check(lib().dsa_attn_combine(_ptr(part_out), _ptr(part_lse), G, R, H, Dv, _ptr(out), _ptr(lse),
                                  _stream(stream)))
    return out, lse


def _all_gather(t: torch.Tensor) -> torch.Tensor:
    """[G, *t.shape]: t from every rank of the default process group, in rank order."""
    import torch.distributed as dist
    parts = [torch.empty_like(t) for _ in range(dist.get_world_size())]
    dist.all_gather(parts, t.contiguous())
    return torch.stack(parts)


class _CudaSplitOps:
    """The per-device steps of decode_split_cache, on this library's kernels."""

    @staticmethod
    def select(p, inp, idx, sel):
        return select(p, inp, idx, sel)

    @staticmethod
    def merge(cand_scores, cand_idx, shard_lo):
        return topk_merge(cand_scores, cand_idx, shard_lo)[0]

    @staticmethod
    def localize(idx, lo, length):
        return index_localize(idx, lo, length)

    @staticmethod
    def attend(q, kv, idx_local, sm_scale, Dv):
        return sparse_mla_fwd(q, kv, idx_local, sm_scale, Dv)

    @staticmethod
    def combine(part_out, part_lse):
        return attn_combine(part_out, part_lse)


def decode_split_cache(p: Problem, inp: dict, shard_lo, rank=None, gather=None, ops=None):
    """Decode over key caches split across devices, one shard per rank.

    p: this rank's shard as a decode problem (Lq = 1, Lk = the shard's key count,
    q_pos0 = Lk - 1); inp: kI, kI_scale, kv of the shard and qI, qI_scale, w, q of the
    query rows (the same on every rank). shard_lo: the first key of every rank's shard,
    in rank order, the shards tiling the key range in that order. rank: this rank
    (default: torch.distributed's). gather(t) returns [G, *t.shape] from all ranks in
    rank order (default: torch.distributed all_gather). Every rank returns the same
    (out [B, 1, H, Dv] bf16, lse [B, 1, H] fp32, idx [B, 1, k] global key indices).
    """
    gather = gather or _all_gather
    ops = ops or _CudaSplitOps
    if rank is None:
        import torch.distributed as dist
        rank = dist.get_rank()
    dev = inp["q"].device
    cand_idx = torch.empty((p.B, p.Lq, p.k), dtype=torch.int32, device=dev)
    cand_sc = torch.empty((p.B, p.Lq, p.k), dtype=torch.float32, device=dev)
    ops.select(p, inp, cand_idx, cand_sc)
    idx = ops.merge(gather(cand_sc), gather(cand_idx), shard_lo)
    idx_local = ops.localize(idx, int(shard_lo[rank]), p.Lk)
    o, l = ops.attend(inp["q"], inp["kv"], idx_local, p.sm_scale, p.Dv)
    out, lse = ops.combine(gather(o), gather(l))
    return out, lse, idx


def forward_paged_workspace_size(p: Problem) -> int:
    cp = p.c()
    return int(lib().dsa_forward_paged_workspace_size(ctypes.byref(cp)))


def forward_paged(p: Problem, inp: dict, block_table, seq_lens, page_size: int, out=None,
                  lse=None, idx_out=None, ws=None, stream=None, sel_scores=None):
    """dsa_forward over a paged cache with per-sequence lengths.

    inp: qI, qI_scale, w, q as for ``forward`` ([B, Lq, ...]); kv, kI, kI_scale are
    pools of num_pages * page_size rows. block_table int32 [B, max_blocks], seq_lens
    int32 [B] (device). p.Lk must be max_blocks * page_size; p.q_pos0 is ignored.
    """
    dev = inp["q"].device
    _need(block_table, "block_table", torch.int32)
    _need(seq_lens, "seq_lens", torch.int32, (p.B,))
    B, max_blocks = block_table.shape
    rows = inp["kv"].shape[0]
    if rows % page_size:
        raise ValueError("pool rows must be a multiple of page_size")
    if out is None:
        out = torch.empty((p.B, p.Lq, p.H, p.Dv), dtype=torch.bfloat16, device=dev)
    if ws is None:
        ws = torch.empty(forward_paged_workspace_size(p), dtype=torch.uint8, device=dev)
    cp = p.c()
    ct = _tensors(inp, out, lse, idx_out, sel_scores)
    cc = DsaPagedCache(block_table.data_ptr(), seq_lens.data_ptr(), max_blocks, page_size,
                       rows // page_size)
    _check(lib().dsa_forward_paged(ctypes.byref(cp), ctypes.byref(ct), ctypes.byref(cc), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)))
    return out


class LaunchProfiler:
    """Events for ``forward_profiled``: one CUDA event around each kernel launch."""

    def __init__(self, max_launches: int = 4096):
        self.max = max_launches
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(max_launches + 1)]
        for e in self.events:      # torch creates the underlying event on first record
            e.record()
        self._ev = (ctypes.c_void_p * (max_launches + 1))(*[e.cuda_event for e in self.events])
        self._kinds = (ctypes.c_int * max_launches)()
        self.n = 0

    def durations(self):
        """[(kind name, ms)] of the last profiled call (synchronises)."""
        self.events[self.n].synchronize()
        return [(KIND_NAMES.get(self._kinds[i], "?"), self.events[i].elapsed_time(self.events[i + 1]))
                for i in range(self.n)]


def forward_profiled(p: Problem, inp: dict, out, prof: LaunchProfiler, lse=None, idx_out=None,
                     ws=None, stream=None):
    """``forward`` that records an event after every kernel launch into ``prof``."""
    if ws is None:
        ws = torch.empty(forward_workspace_size(p), dtype=torch.uint8, device=out.device)
    cp = p.c()
    ct = _tensors(inp, out, lse, idx_out)
    n = ctypes.c_int(0)
    rc = lib().dsa_forward_profiled(ctypes.byref(cp), ctypes.byref(ct), _ptr(ws),
                                    ws.numel() * ws.element_size(), _stream(stream), prof._ev,
                                    prof._kinds, prof.max, ctypes.byref(n))
    prof.n = n.value
    _check(rc)
    return out


def forward_host(p: Problem, host: dict, dev: dict, host_out, dev_out, ws, stream=None,
                 host_lse=None, dev_lse=None, host_idx=None, dev_idx=None):
    """dsa_forward on host tensors: H2D copies, forward, D2H copies of out (and of lse
    / idx_out when both their host and device tensors are given), synchronise. With
    Lq >= 1024 the library pipelines the copies with the compute by blocks of rows.
    Host and device tensors are checked for dtype, shape and contiguity first (the
    copies trust those sizes)."""
    extra = ((host_lse, dev_lse, "lse", torch.float32, (p.B, p.Lq, p.H)),
             (host_idx, dev_idx, "idx", torch.int32, (p.B, p.Lq, p.k)))
    _need_inputs(p, host, "host ", cuda=False)
    _need(host_out, "host out", torch.bfloat16, (p.B, p.Lq, p.H, p.Dv), cuda=False)
    for h, _, name, dt, shp in extra:
        if h is not None:
            _need(h, "host " + name, dt, shp, cuda=False)
    _need_inputs(p, dev, "device ")
    _need(dev_out, "device out", torch.bfloat16, (p.B, p.Lq, p.H, p.Dv))
    for _, d, name, dt, shp in extra:
        if d is not None:
            _need(d, "device " + name, dt, shp)
    if not ws.is_cuda:
        raise ValueError("ws must be on a CUDA device")
    cp = p.c()
    ch = _tensors(host, host_out, host_lse, host_idx)
    cd = _tensors(dev, dev_out, dev_lse, dev_idx)
    _check(lib().dsa_forward_host(ctypes.byref(cp), ctypes.byref(ch), ctypes.byref(cd), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)))
    return host_out


def last_launch_count() -> int:
    """Kernel launches of this thread's last forward call (see dsa_last_launch_count)."""
    return int(lib().dsa_last_launch_count())


def check_status(stream=None) -> None:
    """Synchronise and raise DsaError if a bounded device wait ran out."""
    _check(lib().dsa_check_status(_stream(stream)))


def set_wait_limit_ns(ns: int) -> None:
    _check(lib().dsa_set_wait_limit_ns(int(ns)))


def debug_wait_timeout(stream=None) -> None:
    _check(lib().dsa_debug_wait_timeout(_stream(stream)))
