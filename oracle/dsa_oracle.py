"""Plain fp64 CPU oracle for the DeepSeek Sparse Attention (DSA) path: the
forward and the gradients of its sparse training stage.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. The CUDA library
shares no code, table or constant with it, and it never reads a value the
CUDA path produced.

What it follows ("DeepSeek-V3.2: Pushing the Frontier of Open Large Language
Models", bud-325 paper digest):
  * "Key claims", §2.1 Eq. 1: the lightning-indexer score
        I[t,s] = sum_j w[t,j] * ReLU(q^I[t,j] . k^I[s])
    over H_I indexer heads, in FP8;
  * same passage, §2.1 Eq. 2 / Fig. 2: attention runs only on the top-k key-value
    entries selected by I[t,:], in MLA's MQA mode (one latent row shared by all
    query heads);
  * "Method": k = 2048, one latent vector per token shared by all heads;
  * "Key claims" (paper section 2.1.1, Eq. 3-4, in words) and "Method": the
    indexer is trained with a KL loss toward the head-aggregated main attention
    distribution, on the selected tokens in the sparse stage
    (``indexer_kl_target``, and its score gradient ``indexer_kl_score_grad``);
  * "Method": in the sparse stage the main model learns through the sparse
    attention and the indexer through its own detached inputs
    (``sparse_mla_backward``, ``indexer_backward``).
The eu.36kr.com article (section 02) adds that candidates are the query's
preceding tokens and that top-k index scores pick the entries that are read.

Readings where the pages are silent (each one is listed in the design notes):
  * candidates for query row t at absolute position p = q_pos0 + t are keys s <= p;
  * FP8 values carry positive fp32 scales: one per key row of k^I, one per
    (token, head) row of q^I. A positive scale commutes with ReLU, so
    I[t,s] = s^k[s] * sum_j w[t,j] * s^q[t,j] * max(0, qhat[t,j] . khat[s]);
  * ties at the k-th score go to the lowest key index; the selected set is
    returned in ascending key order, padded with -1 when fewer than k exist;
  * attention is exact softmax(sm_scale * q . c_s) over the selected rows with
    values c_s[:Dv]; lse is the natural-log log-sum-exp of the scaled logits;
    a row with no valid key gives zeros and lse = -inf.

Every function here is a direct transcription of those definitions in numpy
float64 with library primitives (matmul, argsort, exp) as single steps.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# Storage formats
# ---------------------------------------------------------------------------


def e4m3_table() -> np.ndarray:
    """Value of every FP8 E4M3 (OCP "fn" variant) byte, built from the bit layout.

    Layout S.EEEE.MMM, exponent bias 7, no infinities; S.1111.111 is NaN.
    Exponent field 0 is subnormal: value = (-1)^S * 2^(1-7) * M/8.
    """
    out = np.empty(256, dtype=np.float64)
    for b in range(256):
        sign = -1.0 if (b >> 7) & 1 else 1.0
        e = (b >> 3) & 0xF
        m = b & 0x7
        if e == 0xF and m == 0x7:
            out[b] = np.nan
        elif e == 0:
            out[b] = sign * (m / 8.0) * 2.0 ** (1 - 7)
        else:
            out[b] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


_E4M3 = e4m3_table()


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64 (exact: bf16 is the top half of fp32)."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


def to_f64(x: np.ndarray) -> np.ndarray:
    """Decode a stored array: uint16 means bf16 bits, floats are widened."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return decode_bf16(x)
    return x.astype(np.float64)


# ---------------------------------------------------------------------------
# Lightning indexer (Eq. 1)
# ---------------------------------------------------------------------------


def index_scores(qI: np.ndarray, qI_scale: np.ndarray, w: np.ndarray,
                 kI: np.ndarray, kI_scale: np.ndarray) -> np.ndarray:
    """I[s] for one query row against keys kI[0..n).

    qI: uint8 e4m3 codes [H_I, d_I]; qI_scale: [H_I]; w: [H_I] (f32 or bf16 bits)
    kI: uint8 e4m3 codes [n, d_I];   kI_scale: [n]
    Returns float64 [n]:  I[s] = sum_j w_j * ReLU(q^I_j . k^I_s), where the
    dequantised vectors are q^I_j = qhat_j * s^q_j and k^I_s = khat_s * s^k_s.
    """
    q = decode_e4m3(qI) * to_f64(qI_scale)[:, None]          # [H_I, d_I]
    kk = decode_e4m3(kI) * to_f64(kI_scale)[:, None]         # [n, d_I]
    return index_scores_dequantised(q, to_f64(w), kk)


def index_scores_dequantised(q: np.ndarray, w: np.ndarray, kk: np.ndarray) -> np.ndarray:
    """Eq. 1 on real-valued vectors: I[s] = sum_j w_j * ReLU(q_j . k_s).

    q: [H_I, d_I]; w: [H_I]; kk: [n, d_I]. Returns float64 [n].
    """
    dots = np.asarray(q, np.float64) @ np.asarray(kk, np.float64).T    # [H_I, n]
    return np.asarray(w, np.float64) @ np.maximum(dots, 0.0)


# ---------------------------------------------------------------------------
# Fine-grained token selection
# ---------------------------------------------------------------------------


def topk_select(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores, ties to the lowest index.

    scores: float64 [n], the candidates 0..n-1 of one query row. Returns int64
    [k]: the selected indices in ascending order, padded with -1 if n < k.
    """
    n = scores.shape[0]
    out = np.full(k, -1, dtype=np.int64)
    if n <= k:
        out[:n] = np.arange(n)
        return out
    order = np.argsort(-scores, kind="stable")   # stable: equal scores keep index order
    out[:] = np.sort(order[:k])
    return out


# ---------------------------------------------------------------------------
# Sparse MLA in MQA mode
# ---------------------------------------------------------------------------


def sparse_mla(q: np.ndarray, kv: np.ndarray, idx: np.ndarray, sm_scale: float, Dv: int):
    """Exact softmax attention of one query token over its selected latent rows.

    q: [H, Dqk] (bf16 bits or float); kv: [n_keys, Dqk] latent rows of the
    sequence (bf16 bits or float); idx: selected key indices, entries < 0 or
    >= n_keys are skipped. Every head attends to the same rows (MQA mode):
        z[h,s] = sm_scale * q[h] . c_s,  out[h] = sum_s softmax(z[h])_s * c_s[:Dv]
    Returns (out float64 [H, Dv], lse float64 [H]).
    """
    qf = to_f64(q)
    H = qf.shape[0]
    idx = np.asarray(idx)
    valid = idx[(idx >= 0) & (idx < kv.shape[0])]
    if valid.size == 0:
        return np.zeros((H, Dv)), np.full(H, -np.inf)
    c = to_f64(kv[valid])                                    # [n_sel, Dqk]
    z = sm_scale * (qf @ c.T)                                # [H, n_sel]
    m = z.max(axis=1, keepdims=True)
    p = np.exp(z - m)
    denom = p.sum(axis=1, keepdims=True)
    out = (p @ c[:, :Dv]) / denom
    lse = m[:, 0] + np.log(denom[:, 0])
    return out, lse


# ---------------------------------------------------------------------------
# Indexer alignment target (training objective, forward only)
# ---------------------------------------------------------------------------


def indexer_kl_target(q: np.ndarray, kv: np.ndarray, idx: np.ndarray, sel_scores: np.ndarray,
                      sm_scale: float):
    """KL divergence between the aggregated main-attention distribution and the
    lightning indexer's distribution over one query token's key set.

    Follows "DeepSeek-V3.2: Pushing the Frontier of Open Large Language Models"
    (bud-325 paper digest): "Key claims" (paper section 2.1.1, Eq. 3-4, given in
    words only) has a KL-divergence loss align the indexer output with the main
    attention distribution aggregated over heads; "Method" restricts that KL to
    the selected tokens in the sparse stage. The eu.36kr.com article (section 02)
    says the indexer learns to mimic the original attention's distribution.
    Reading (the pages print neither equation):
      * the key set is the valid entries of ``idx`` (all causal keys for the dense
        warm-up, the top-k set for the sparse stage);
      * main attention of head h: a[h,s] = softmax over the set of sm_scale q[h].c_s;
      * target p = sum_h a[h,:], L1-normalised over the set;
      * indexer distribution r = softmax over the set of sel_scores;
      * loss KL(p || r) = sum_s p_s (ln p_s - ln r_s), natural log; terms with
        p_s = 0 are 0.
    q: [H, Dqk]; kv: [n_keys, Dqk]; idx: [k] (entries < 0 or >= n_keys are not in
    the set); sel_scores: [k] index scores I[t, idx[j]] aligned with idx.
    Returns (p float64 [k] with 0 at the slots outside the set, kl float64).
    """
    qf = to_f64(q)
    idx = np.asarray(idx)
    ok = (idx >= 0) & (idx < kv.shape[0])
    p_out = np.zeros(idx.shape[0])
    if not ok.any():
        return p_out, 0.0
    c = to_f64(kv[idx[ok]])                                   # [n, Dqk]
    z = sm_scale * (qf @ c.T)                                 # [H, n]
    a = np.exp(z - z.max(axis=1, keepdims=True))
    a /= a.sum(axis=1, keepdims=True)                         # each head's attention
    agg = a.sum(axis=0)
    p = agg / agg.sum()                                       # L1-normalised aggregate
    sc = np.asarray(sel_scores, dtype=np.float64)[ok]
    log_r = sc - (sc.max() + np.log(np.exp(sc - sc.max()).sum()))
    nz = p > 0
    kl = float(np.sum(p[nz] * (np.log(p[nz]) - log_r[nz])))
    p_out[ok] = p
    return p_out, kl


def indexer_kl_score_grad(p: np.ndarray, sel_scores: np.ndarray, idx: np.ndarray,
                          n_keys: int) -> np.ndarray:
    """Gradient of KL(p || r) with respect to the selected index scores, p held fixed.

    The bud-325 digest ("Method") trains the indexer on the KL toward the main
    attention with the indexer's input detached from the main model's graph, so p
    is a constant for this loss. With r = softmax over the set of the scores,
    ln r_s = I_s - logsumexp(I) and sum_s p_s = 1 give
        d KL / d I_u = -p_u + sum_s p_s r_u = r_u - p_u.
    p, sel_scores, idx: [k] aligned slots; slots whose idx lies outside
    [0, n_keys) are not in the set and get 0. Returns float64 [k].
    """
    idx = np.asarray(idx)
    ok = (idx >= 0) & (idx < n_keys)
    g = np.zeros(idx.shape[0])
    if not ok.any():
        return g
    s = np.asarray(sel_scores, np.float64)[ok]
    r = np.exp(s - s.max())
    r /= r.sum()
    g[ok] = r - np.asarray(p, np.float64)[ok]
    return g


# ---------------------------------------------------------------------------
# Sparse training stage: gradients
# ---------------------------------------------------------------------------


def sparse_mla_backward(q: np.ndarray, kv: np.ndarray, idx: np.ndarray, dout: np.ndarray,
                        sm_scale: float, Dv: int):
    """Gradients of one query token's sparse attention with respect to its query
    and the latent rows, given dL/d(out).

    The bud-325 digest ("Method") trains the main model in the sparse stage through
    attention over the selected entries only, so the gradient is the ordinary
    softmax-attention gradient restricted to the set. With
    z[h,s] = sm_scale q[h].c_s, a = softmax_s(z), out[h] = sum_s a[h,s] c_s[:Dv]:
        dA[h,s] = dout[h] . c_s[:Dv]
        dz[h,s] = a[h,s] (dA[h,s] - dout[h] . out[h])        (softmax Jacobian)
        dq[h]   = sm_scale sum_s dz[h,s] c_s
        dc_s    = sm_scale sum_h dz[h,s] q[h], plus sum_h a[h,s] dout[h] on the
                  first Dv columns (the value part of the shared latent row).
    q: [H, Dqk]; kv: [n_keys, Dqk]; idx: [k] (entries outside [0, n_keys) are
    skipped; an index listed twice counts twice, as in the forward); dout: [H, Dv].
    Returns (dq float64 [H, Dqk], dkv float64 [n_keys, Dqk]).
    """
    qf = to_f64(q)
    H, Dqk = qf.shape
    idx = np.asarray(idx)
    valid = idx[(idx >= 0) & (idx < kv.shape[0])]
    dq = np.zeros((H, Dqk))
    dkv = np.zeros((kv.shape[0], Dqk))
    if valid.size == 0:
        return dq, dkv
    c = to_f64(kv[valid])                                    # [n, Dqk]
    do = to_f64(dout)                                        # [H, Dv]
    z = sm_scale * (qf @ c.T)                                # [H, n]
    a = np.exp(z - z.max(axis=1, keepdims=True))
    a /= a.sum(axis=1, keepdims=True)
    out = a @ c[:, :Dv]                                      # [H, Dv]
    dA = do @ c[:, :Dv].T                                    # [H, n]
    dz = a * (dA - np.sum(do * out, axis=1, keepdims=True))
    dq = sm_scale * (dz @ c)
    dc = sm_scale * (dz.T @ qf)                              # [n, Dqk]
    dc[:, :Dv] += a.T @ do
    np.add.at(dkv, valid, dc)
    return dq, dkv


def indexer_backward(qI: np.ndarray, qI_scale: np.ndarray, w: np.ndarray, kI: np.ndarray,
                     kI_scale: np.ndarray, idx: np.ndarray, dI: np.ndarray):
    """Gradients of L = sum_j dI[j] * I[idx[j]] (one query row) with respect to the
    dequantised indexer query q^I, the dequantised keys k^I and the weights w.

    The bud-325 digest ("Method") keeps training the indexer in the sparse stage
    on the KL over the selected tokens, with its input detached: the loss reaches
    only the indexer's own q^I, k^I and w. From Eq. 1, x[j,s] = q^I_j . k^I_s and
    I_s = sum_j w_j ReLU(x[j,s]):
        dw_j   = sum_s dI_s ReLU(x[j,s])
        g[j,s] = dI_s w_j [x[j,s] > 0]            (ReLU'(0) taken as 0)
        dq^I_j = sum_s g[j,s] k^I_s
        dk^I_s = sum_j g[j,s] q^I_j
    The FP8 rounding is passed through as the identity (gradients are with respect
    to the dequantised values q^I = s^q qhat and k^I = s^k khat).
    The positive scales factor out of the dot, x = s^q s^k (qhat . khat), and the
    dot of two rows of e4m3 codes is exact in float64 (each product needs at most
    8 significant bits and every partial sum is a multiple of 2^-18 below 2^25),
    so the ReLU mask is decided on that exact value.
    qI: uint8 [H_I, d_I]; qI_scale, w: [H_I]; kI: uint8 [n_keys, d_I]; kI_scale:
    [n_keys]; idx, dI: [k] aligned (slots outside [0, n_keys) skipped).
    Returns (dqI float64 [H_I, d_I], dkI float64 [n_keys, d_I], dw float64 [H_I]).
    """
    sq = to_f64(qI_scale)
    sk = to_f64(kI_scale)
    qh = decode_e4m3(qI)
    kh = decode_e4m3(kI)
    q = qh * sq[:, None]
    kk = kh * sk[:, None]
    wf = to_f64(w)
    idx = np.asarray(idx)
    ok = (idx >= 0) & (idx < kk.shape[0])
    valid = idx[ok]
    d = np.asarray(dI, np.float64)[ok]
    dk = np.zeros_like(kk)
    if valid.size == 0:
        return np.zeros_like(q), dk, np.zeros_like(wf)
    xhat = qh @ kh[valid].T                                  # [H_I, n], exact
    x = xhat * sq[:, None] * sk[valid][None, :]
    dw = np.maximum(x, 0.0) @ d
    g = (xhat > 0) * wf[:, None] * d[None, :]
    dq = g @ kk[valid]
    np.add.at(dk, valid, g.T @ q)
    return dq, dk, dw


def dense_causal_mqa(q: np.ndarray, kv: np.ndarray, sm_scale: float, Dv: int, q_pos0: int = 0):
    """Dense causal MQA attention, written independently of ``sparse_mla``.

    q: [Lq, H, Dqk]; kv: [Lk, Dqk]. Row t attends to keys 0..q_pos0+t with a
    per-key loop and a running (max, sum) pair. Used only to pin the sparse path:
    when k covers every causal key the two must agree.
    """
    qf = to_f64(q)
    cf = to_f64(kv)
    Lq, H, _ = qf.shape
    out = np.zeros((Lq, H, Dv))
    lse = np.zeros((Lq, H))
    for t in range(Lq):
        last = q_pos0 + t
        for h in range(H):
            mx = -np.inf
            tot = 0.0
            acc = np.zeros(Dv)
            for s in range(last + 1):
                zz = sm_scale * float(np.dot(qf[t, h], cf[s]))
                if zz > mx:
                    r = np.exp(mx - zz) if np.isfinite(mx) else 0.0
                    tot *= r
                    acc *= r
                    mx = zz
                e = np.exp(zz - mx)
                tot += e
                acc += e * cf[s, :Dv]
            out[t, h] = acc / tot
            lse[t, h] = mx + np.log(tot)
    return out, lse


# ---------------------------------------------------------------------------
# Whole forward on chosen rows
# ---------------------------------------------------------------------------


def forward_rows(inp: dict, cfg, b: int, rows, with_scores: bool = True) -> dict:
    """DSA forward for query rows ``rows`` of sequence ``b``.

    inp: dict of numpy arrays in storage format (see ``numpy_inputs``).
    Returns per-row lists: 'scores' (float64 [p+1]), 'idx' (int64 [k]),
    'out' (float64 [H, Dv]), 'lse' (float64 [H]).
    """
    res = {"scores": [], "idx": [], "out": [], "lse": []}
    for t in rows:
        p = cfg.q_pos0 + t
        n = p + 1
        if with_scores or n > cfg.k:
            sc = index_scores(inp["qI"][b, t], inp["qI_scale"][b, t], inp["w"][b, t],
                              inp["kI"][b, :n], inp["kI_scale"][b, :n])
        else:
            sc = None
        idx = topk_select(sc, cfg.k) if n > cfg.k else topk_select(np.zeros(n), cfg.k)
        out, lse = sparse_mla(inp["q"][b, t], inp["kv"][b], idx, cfg.sm_scale, cfg.Dv)
        res["scores"].append(sc)
        res["idx"].append(idx)
        res["out"].append(out)
        res["lse"].append(lse)
    return res


def numpy_inputs(tensors: dict) -> dict:
    """Torch tensors from the input generator -> numpy storage arrays.

    bf16 tensors become uint16 bit patterns, e4m3 stays uint8, fp32 stays fp32.
    Accepts tensors on any device (copies to host).
    """
    import torch

    out = {}
    for name, t in tensors.items():
        t = t.detach().to("cpu")
        if t.dtype == torch.bfloat16:
            out[name] = t.view(torch.int16).numpy().view(np.uint16)
        else:
            out[name] = t.numpy()
    return out
