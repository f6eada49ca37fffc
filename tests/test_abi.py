"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before touching a GPU (no device needed)."""
import ctypes
import math
import os
import re

import pytest

import sparse_attention_long_scores_b200 as dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def L():
    from sparse_attention_long_scores_b200.build import build
    build()
    return dsa.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(dsa_[a-z0-9_]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("dsa_indexer_scores", "dsa_topk_select", "dsa_sparse_mla_fwd", "dsa_forward",
              "dsa_forward_workspace_size", "dsa_last_error", "dsa_check_status"):
        assert n in names
    assert sorted(dsa.EXPORTED) == names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
    assert L.dsa_version().decode().startswith("dsa-b200")


FAKE = 0x10000   # aligned, never dereferenced: validation fails first


def test_indexer_rejects_bad_args(L):
    p = ctypes.c_void_p(FAKE)
    # unsupported indexer shape
    rc = L.dsa_indexer_scores(p, p, p, p, p, 0, p, 1, 8, 8, 0, 32, 64, None)
    assert rc == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    assert "unsupported" in L.dsa_last_error().decode()
    # null pointer
    rc = L.dsa_indexer_scores(None, p, p, p, p, 0, p, 1, 8, 8, 0, 4, 32, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG and "qI" in L.dsa_last_error().decode()
    # misaligned
    rc = L.dsa_indexer_scores(ctypes.c_void_p(FAKE + 4), p, p, p, p, 0, p, 1, 8, 8, 0, 4, 32, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG and "aligned" in L.dsa_last_error().decode()
    # causal window outside the keys
    rc = L.dsa_indexer_scores(p, p, p, p, p, 0, p, 1, 8, 8, 1, 4, 32, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG
    # bad w dtype
    rc = L.dsa_indexer_scores(p, p, p, p, p, 7, p, 1, 8, 8, 0, 4, 32, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG


def test_topk_rejects_bad_k(L):
    p = ctypes.c_void_p(FAKE)
    for k in (0, 16, 33, 8192):
        assert L.dsa_topk_select(p, p, 1, 8, 8, 0, k, None) == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    assert L.dsa_topk_select(p, None, 1, 8, 8, 0, 32, None) == dsa.DSA_ERR_INVALID_ARG


def test_sparse_mla_rejects_bad_args(L):
    p = ctypes.c_void_p(FAKE)
    rc = L.dsa_sparse_mla_fwd(p, p, p, p, None, 1, 4, 8, 16, 80, 64, 32, 0.1, None, 0, None)
    assert rc == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    rc = L.dsa_sparse_mla_fwd(p, p, p, p, None, 1, 4, 8, 8, 80, 64, 32, -1.0, None, 0, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG
    rc = L.dsa_sparse_mla_fwd(p, p, p, p, None, 1, 4, 8, 8, 80, 64, 32, float("nan"), None, 0, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG


def test_indexer_kl_rejects_bad_args(L):
    p = ctypes.c_void_p(FAKE)
    # (H, Dqk) outside the supported pair
    rc = L.dsa_indexer_kl(p, p, p, p, p, None, p, 1, 4, 8, 16, 80, 32, 0.1, None)
    assert rc == dsa.DSA_ERR_UNSUPPORTED_SHAPE and "unsupported" in L.dsa_last_error().decode()
    # k not a multiple of 32
    rc = L.dsa_indexer_kl(p, p, p, p, p, None, p, 1, 4, 8, 8, 80, 40, 0.1, None)
    assert rc == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    # missing lse (required), missing kl_out, misaligned scores, bad scale
    rc = L.dsa_indexer_kl(p, p, p, None, p, None, p, 1, 4, 8, 8, 80, 32, 0.1, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG and "lse" in L.dsa_last_error().decode()
    rc = L.dsa_indexer_kl(p, p, p, p, p, None, None, 1, 4, 8, 8, 80, 32, 0.1, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG and "kl_out" in L.dsa_last_error().decode()
    rc = L.dsa_indexer_kl(p, p, p, p, ctypes.c_void_p(FAKE + 8), None, p, 1, 4, 8, 8, 80, 32, 0.1, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG and "aligned" in L.dsa_last_error().decode()
    rc = L.dsa_indexer_kl(p, p, p, p, p, None, p, 1, 4, 8, 8, 80, 32, 0.0, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG


def test_backward_entry_points_reject_bad_args(L):
    """The sparse-stage gradient calls validate everything before any device work."""
    p = ctypes.c_void_p(FAKE)
    odd = ctypes.c_void_p(FAKE + 8)
    big = 1 << 40

    def mla(**kw):
        a = dict(q=p, kv=p, idx=p, lse=p, dout=p, dq=p, dkv=p, acc=0, B=1, Lq=4, Lk=8, H=8,
                 Dqk=80, Dv=64, k=32, scale=0.1, ws=p, ws_bytes=big)
        a.update(kw)
        return L.dsa_sparse_mla_bwd(*a.values(), None)

    for kw, code, text in ((dict(lse=None), dsa.DSA_ERR_INVALID_ARG, "lse"),
                           (dict(dq=odd), dsa.DSA_ERR_INVALID_ARG, "aligned"),
                           (dict(H=16), dsa.DSA_ERR_UNSUPPORTED_SHAPE, ""),
                           (dict(k=40), dsa.DSA_ERR_UNSUPPORTED_SHAPE, ""),
                           (dict(scale=0.0), dsa.DSA_ERR_INVALID_ARG, "sm_scale"),
                           (dict(Lq=0), dsa.DSA_ERR_INVALID_ARG, ""),
                           (dict(ws_bytes=4096), dsa.DSA_ERR_WORKSPACE_TOO_SMALL, "workspace")):
        rc = mla(**kw)
        assert rc == code and text in L.dsa_last_error().decode(), (kw, L.dsa_last_error())

    def idx_bwd(**kw):
        a = dict(qI=p, qs=p, kI=p, ks=p, w=p, wd=dsa.DSA_DTYPE_BF16, idx=p, dI=p, dqI=p, dkI=p, dw=p,
                 acc=0, B=1, Lq=4, Lk=8, H_I=4, d_I=32, k=32, ws=p, ws_bytes=big)
        a.update(kw)
        return L.dsa_indexer_bwd(*a.values(), None)

    for kw, code, text in ((dict(dw=None), dsa.DSA_ERR_INVALID_ARG, "dw"),
                           (dict(H_I=8), dsa.DSA_ERR_UNSUPPORTED_SHAPE, ""),
                           (dict(wd=7), dsa.DSA_ERR_INVALID_ARG, "w_dtype"),
                           (dict(k=0), dsa.DSA_ERR_UNSUPPORTED_SHAPE, ""),
                           (dict(ws_bytes=4096), dsa.DSA_ERR_WORKSPACE_TOO_SMALL, "workspace")):
        rc = idx_bwd(**kw)
        assert rc == code and text in L.dsa_last_error().decode(), (kw, L.dsa_last_error())

    assert L.dsa_indexer_kl_grad(p, None, p, p, 1, 4, 8, 32, 1.0, None) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_indexer_kl_grad(p, p, p, p, 1, 4, 8, 33, 1.0, None) == dsa.DSA_ERR_UNSUPPORTED_SHAPE
    assert L.dsa_indexer_kl_grad(p, p, p, p, 1, 4, 8, 32, math.nan, None) == dsa.DSA_ERR_INVALID_ARG


def test_forward_host_checks_host_tensors_before_any_copy():
    """dsa_forward_host's copies trust the tensor sizes, so the binding checks the
    host tensors' dtype, shape and contiguity before the call (no GPU needed: with
    valid host tensors the next check to fail is the device one)."""
    import torch
    from dsa_inputs import CONFIGS, gen_inputs
    cfg = CONFIGS["tiny"].with_(Lq=8, Lk=8)
    p = dsa.Problem.from_config(cfg)
    host = gen_inputs(cfg, "cpu", seed=3)
    out = torch.empty((1, 8, cfg.H, cfg.Dv), dtype=torch.bfloat16)
    ws = torch.empty(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="must be on a CUDA device"):
        dsa.forward_host(p, host, host, out, out, ws)
    bad = dict(host, q=host["q"][:, :4].contiguous())
    with pytest.raises(ValueError, match="host q has shape"):
        dsa.forward_host(p, bad, host, out, out, ws)
    bad = dict(host, kv=host["kv"].transpose(1, 2))
    with pytest.raises(ValueError, match="host kv must be contiguous"):
        dsa.forward_host(p, bad, host, out, out, ws)
    bad = dict(host, kI_scale=host["kI_scale"].double())
    with pytest.raises(TypeError, match="host kI_scale must be"):
        dsa.forward_host(p, bad, host, out, out, ws)
    with pytest.raises(ValueError, match="host out has shape"):
        dsa.forward_host(p, host, host, out[:, :4], out, ws)
    with pytest.raises(ValueError, match="host lse has shape"):
        dsa.forward_host(p, host, host, out, out, ws, host_lse=torch.empty(3))


C_PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "dsa.h"
int main(void) {
  /* host-only calls: version, sizes and argument validation (no device needed) */
  dsa_problem p;
  memset(&p, 0, sizeof p);
  p.mode = DSA_MODE_PREFILL; p.B = 1; p.Lq = 256; p.Lk = 256; p.H_I = 4; p.d_I = 32;
  p.H = 8; p.Dqk = 80; p.Dv = 64; p.k = 32; p.sm_scale = 0.1f; p.w_dtype = DSA_DTYPE_F32;
  if (dsa_forward_workspace_size(&p) == 0) return 1;
  if (dsa_sparse_mla_bwd_workspace_size(1, 256, 8, 80, 64, 32) == 0) return 2;
  int rc = dsa_sparse_mla_bwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 1, 256, 256, 8, 80,
                              64, 32, 0.1f, NULL, 0, NULL);
  if (rc != DSA_ERR_INVALID_ARG || strstr(dsa_last_error(), "q") == NULL) return 3;
  if (dsa_last_launch_count() != 0) return 4;
  printf("%s\n", dsa_version());
  return 0;
}
"""


def test_plain_c_program_uses_the_abi(L, tmp_path):
    """The boundary is plain C: a C99 program compiles against include/dsa.h, links
    to libdsa.so and makes host-only calls through it."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "abi.c"
    exe = tmp_path / "abi"
    src.write_text(C_PROGRAM)
    libdir = os.path.dirname(dsa.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir,
                    "-ldsa", "-Wl,-rpath," + libdir], check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert r.stdout.startswith("dsa-b200")


def test_backward_workspace_sizes(L):
    """Chunks of at most 64 tokens: the recommended workspace grows with the token
    count up to 64 and then stays flat. At the full shapes a token holds its gathered
    rows (k x 576 bf16), [q; dout] (256 x 576 bf16), [S; dP] (256 x k fp32) and
    [dz; P] (256 x k bf16): 5.8 MB."""
    f = L.dsa_sparse_mla_bwd_workspace_size
    sizes = [f(1, n, 128, 576, 512, 2048) for n in (1, 2, 64, 65, 65536)]
    assert sizes[0] < sizes[1] < sizes[2] == sizes[3] == sizes[4]
    per_token = (sizes[2] - sizes[0]) / 63
    expect = 2048 * 576 * 2 + 256 * 576 * 2 + 256 * 2048 * 4 + 256 * 2048 * 2
    assert abs(per_token - expect) < 4096, (per_token, expect)
    g = L.dsa_indexer_bwd_workspace_size
    assert 0 < g(1, 1, 64, 128, 2048) < g(2, 32768, 64, 128, 2048) == g(1, 64, 64, 128, 2048)
    assert f(0, 1, 8, 80, 64, 32) == 0 and g(1, 0, 4, 32, 32) == 0


def test_forward_paged_rejects_bad_cache(L):
    from dsa_inputs import CONFIGS
    p = dsa.Problem.from_config(CONFIGS["tiny"].with_(Lq=1, Lk=512, q_pos0=511))
    cp = p.c()
    t = dsa.DsaTensors(*([FAKE] * 8 + [None, None]))
    ws = ctypes.c_void_p(FAKE)
    assert L.dsa_forward_paged_workspace_size(ctypes.byref(cp)) > 0
    good = dict(block_table=FAKE, seq_lens=FAKE, max_blocks=4, page_size=128, num_pages=8)
    for change, code, text in ((dict(page_size=100), dsa.DSA_ERR_UNSUPPORTED_SHAPE, "page_size"),
                               (dict(max_blocks=3), dsa.DSA_ERR_INVALID_ARG, "max_blocks * page_size"),
                               (dict(block_table=None), dsa.DSA_ERR_INVALID_ARG, "block_table"),
                               (dict(num_pages=0), dsa.DSA_ERR_INVALID_ARG, "num_pages")):
        c = dsa.DsaPagedCache(**dict(good, **change))
        rc = L.dsa_forward_paged(ctypes.byref(cp), ctypes.byref(t), ctypes.byref(c), ws, 1 << 30, None)
        assert rc == code and text in L.dsa_last_error().decode(), (change, L.dsa_last_error())


def test_workspace_sizes(L):
    from dsa_inputs import CONFIGS
    for name, cfg in CONFIGS.items():
        p = dsa.Problem.from_config(cfg)
        n = dsa.forward_workspace_size(p)
        assert n > 0
        # never anywhere near the full score matrix
        full = cfg.B * cfg.Lq * cfg.Lk * 4
        idx = cfg.B * cfg.Lq * cfg.k * 4
        assert n < idx + max(full // 8, 256 << 20), name
    # a small decode batch splits keys (one wave of CTAs): needs a partial-output
    # buffer; 64 sequences already fill the SMs with one split
    d = CONFIGS["decode_128k"]
    assert dsa.sparse_mla_workspace_size(8, d.Lq, d.Lk, d.H, d.Dqk, d.Dv, d.k) > 0
    assert dsa.sparse_mla_workspace_size(d.B, d.Lq, d.Lk, d.H, d.Dqk, d.Dv, d.k) == 0
    pf = CONFIGS["prefill_32k"]
    assert dsa.sparse_mla_workspace_size(pf.B, pf.Lq, pf.Lk, pf.H, pf.Dqk, pf.Dv, pf.k) == 0


def test_forward_rejects_bad_problem(L):
    from dsa_inputs import CONFIGS
    p = dsa.Problem.from_config(CONFIGS["tiny"])
    p.k = 4096
    cp = p.c()
    assert L.dsa_forward_workspace_size(ctypes.byref(cp)) == 0
    assert "k = 4096" in L.dsa_last_error().decode()
    p = dsa.Problem.from_config(CONFIGS["tiny"])
    cp = p.c()
    t = dsa.DsaTensors(*([FAKE] * 8 + [None, None]))
    rc = L.dsa_forward(ctypes.byref(cp), ctypes.byref(t), ctypes.c_void_p(FAKE), 16, None)
    assert rc == dsa.DSA_ERR_WORKSPACE_TOO_SMALL
    t.kv = None
    rc = L.dsa_forward(ctypes.byref(cp), ctypes.byref(t), ctypes.c_void_p(FAKE), 1 << 30, None)
    assert rc == dsa.DSA_ERR_INVALID_ARG and "kv" in L.dsa_last_error().decode()


def test_wait_limit_validation(L):
    assert L.dsa_set_wait_limit_ns(0) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_set_wait_limit_ns(2_000_000_000) == dsa.DSA_OK


def test_no_cpu_fallback_in_binding():
    """The binding has no compute of its own: every entry calls into the library."""
    src = open(os.path.join(ROOT, "sparse_attention_long_scores_b200", "__init__.py")).read()
    assert "import oracle" not in src and "from oracle" not in src
    for banned in ("torch.topk", "torch.softmax", "torch.matmul", "@ ", "einsum"):
        assert banned not in src, banned


def test_recommended_workspace_passes_validation(L):
    """The recommended size passes validation and a tiny one does not. With fake
    device pointers a valid call gets past validation and then fails for want of
    a GPU, so this runs only where no GPU is visible."""
    import torch
    from dsa_inputs import CONFIGS
    if torch.cuda.is_available():
        pytest.skip("uses fake device pointers")
    for name, cfg in CONFIGS.items():
        p = dsa.Problem.from_config(cfg)
        cp = p.c()
        n = L.dsa_forward_workspace_size(ctypes.byref(cp))
        t = dsa.DsaTensors(*([FAKE] * 8 + [None, None]))
        rc = L.dsa_forward(ctypes.byref(cp), ctypes.byref(t), ctypes.c_void_p(FAKE), n, None)
        assert rc == dsa.DSA_ERR_CUDA, (name, rc, L.dsa_last_error().decode())
        rc = L.dsa_forward(ctypes.byref(cp), ctypes.byref(t), ctypes.c_void_p(FAKE), 64, None)
        assert rc == dsa.DSA_ERR_WORKSPACE_TOO_SMALL, name
