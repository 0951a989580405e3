"""C-ABI library checks that need no GPU: it loads, exports every symbol that
include/efla.h declares, and rejects bad arguments on the host before any CUDA
call (fake pointer values are never dereferenced on these paths)."""
import ctypes
import os
import re

import pytest

from delta_rule_linear_efla_b200 import efla

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from delta_rule_linear_efla_b200 import build

    build.build()
    return efla.load_library()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "efla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(efla_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    decl = declared_symbols()
    assert len(decl) >= 8
    for name in decl:
        assert hasattr(lib, name), name
    assert sorted(efla.ABI_SYMBOLS) == sorted(decl)


def test_status_strings_and_version(lib):
    assert efla.status_str(0) == "ok"
    assert "aligned" in efla.status_str(8)
    assert efla.status_str(99) == "unknown status"
    assert lib.efla_version() >= 100


BF16, F32 = efla.EFLA_BF16, efla.EFLA_F32
P = 0x10000  # a fake, 16-byte aligned address (never dereferenced below)


def _chunk(lib, **kw):
    a = dict(q=P, k=P, v=P, beta=P, S0=None, o=P, Sf=P, B=1, H=1, L=64, dk=64, dv=64, chunk=64,
             dt=BF16, odt=F32, ws=None, wsb=0, s=None)
    a.update(kw)
    return lib.efla_chunk_fwd(a["q"], a["k"], a["v"], a["beta"], a["S0"], a["o"], a["Sf"], a["B"],
                              a["H"], a["L"], a["dk"], a["dv"], a["chunk"], a["dt"], a["odt"],
                              a["ws"], a["wsb"], a["s"])


def test_chunk_fwd_host_errors(lib):
    assert _chunk(lib, dt=7) == 3                    # EFLA_ERR_DTYPE
    assert _chunk(lib, odt=2) == 3
    assert _chunk(lib, B=0) == 2                     # EFLA_ERR_SHAPE
    assert _chunk(lib, L=-1) == 2
    assert _chunk(lib, dk=0) == 2
    assert _chunk(lib, dk=129) == 4                  # EFLA_ERR_UNSUPPORTED
    assert _chunk(lib, chunk=48) == 4
    assert _chunk(lib, chunk=128) == 4
    assert _chunk(lib, q=None) == 1                  # EFLA_ERR_NULL
    assert _chunk(lib, o=None) == 1
    assert _chunk(lib, k=P + 2) == 8                 # EFLA_ERR_ALIGN
    assert _chunk(lib, S0=P + 4) == 8


def test_recurrent_step_host_errors(lib):
    f = lib.efla_recurrent_step
    assert f(P, P, P, P, P, P, 1, 1, 64, 64, 9, F32, None) == 3
    assert f(P, P, P, P, P, P, 1, 1, 64, 64, BF16, 9, None) == 3
    assert f(P, P, P, P, P, P, 0, 1, 64, 64, BF16, F32, None) == 2
    assert f(P, P, P, P, P, P, 1, 1, 300, 64, BF16, F32, None) == 4
    assert f(P, None, P, P, P, P, 1, 1, 64, 64, BF16, F32, None) == 1
    assert f(P, P, P, P, P + 8, P, 1, 1, 64, 64, BF16, F32, None) == 8   # S: 16-byte aligned
    assert f(P, P, P, P + 1, P, P, 1, 1, 64, 64, BF16, F32, None) == 8   # bf16: 2-byte aligned
    assert f(P, P, P, P, P, P + 2, 1, 1, 64, 64, BF16, F32, None) == 8   # fp32 o: 4-byte aligned


def test_alpha_host_errors(lib):
    f = lib.efla_alpha
    assert f(P, P, P, 1, 1, 4, 16, 5, None) == 3
    assert f(P, P, P, 1, 1, 4, 0, BF16, None) == 2
    assert f(P, P, P, 1, 1, 4, 512, BF16, None) == 4
    assert f(None, P, P, 1, 1, 4, 16, BF16, None) == 1
    assert f(P, P, P, 1, 1, 0, 16, BF16, None) == 0  # zero tokens: nothing to do


def test_workspace_query_is_host_only(lib):
    for wid_sizes in ((8, 8, 2048, 128, 128, 64), (1, 1, 64, 16, 16, 16), (4, 16, 4096, 128, 128, 64)):
        for dt in (BF16, F32):
            n = lib.efla_chunk_fwd_workspace_size(*wid_sizes, dt, F32)
            assert n >= 0
            path = lib.efla_chunk_fwd_path(*wid_sizes, dt, F32)
            assert path in (0, 1, 2)
            if path == 0:
                assert n == 0
    assert lib.efla_chunk_fwd_workspace_size(1, 1, 64, 16, 16, 48, BF16, F32) == 0


def test_binding_fails_loudly_without_cuda():
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    q = torch.zeros(1, 1, 4, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        efla.chunk_fwd(q, q, q, torch.zeros(1, 1, 4, dtype=torch.bfloat16))


def test_binding_raises_when_library_missing(tmp_path):
    with pytest.raises(RuntimeError):
        efla.load_library(str(tmp_path / "missing.so"))


def test_workspace_reserves_segment_state(lib):
    """Sizes that may run as sequence segments reserve eight segments' [S_in | H | P] fp32
    states per head after the Ta tiles; other sizes need only the Ta tiles (8 KiB per chunk)."""
    ta = 16 * 1024 * 64 * 64 * 2
    assert lib.efla_chunk_fwd_workspace_size(1, 16, 65536, 128, 128, 64, BF16, F32) == \
        ta + 16 * 8 * 3 * 128 * 128 * 4
    assert lib.efla_chunk_fwd_workspace_size(4, 16, 4096, 128, 128, 64, BF16, F32) == 4 * 16 * 64 * 8192
    assert lib.efla_chunk_fwd_workspace_size(1, 2, 4096, 128, 64, 64, BF16, F32) == 2 * 64 * 8192


def test_unknown_rule_is_refused_on_the_host(lib):
    P = ctypes.c_void_p(16)
    EFLA_ERR_RULE = 10
    assert lib.efla_alpha_rule(P, P, P, 1, 1, 4, 16, BF16, 2, None) == EFLA_ERR_RULE
    assert lib.efla_chunk_fwd_rule(P, P, P, P, None, P, None, 1, 1, 64, 16, 16, 64, BF16, F32, 7,
                                   None, 0, None) == EFLA_ERR_RULE
    assert lib.efla_recurrent_step_rule(P, P, P, P, P, P, 1, 1, 16, 16, BF16, F32, -1,
                                        None) == EFLA_ERR_RULE
    assert "rule" in lib.efla_status_str(EFLA_ERR_RULE).decode()


def test_selftest_budget_is_checked_on_the_host(lib):
    EFLA_ERR_SHAPE = 2
    assert lib.efla_selftest_bounded_wait(0, None) == EFLA_ERR_SHAPE
    assert lib.efla_selftest_bounded_wait(3_000_000_000, None) == EFLA_ERR_SHAPE


def test_bwd_workspace_size_and_alignment(lib):
    """The backward's workspace, every region rounded up to 256 bytes: eight fp32 coefficients per
    token; four ints of statistics per head; per (head, 16-column block) r of every token and the
    block's state every 64 tokens and at the end; the column blocks' shares of dq, dk and dbeta;
    and, where the tensor-core forward can run (bf16 inputs), its workspace, every token's u and the
    state after every 64-token block (fp16), and for the tensor-core backward the fp16 dO, every token's
    dU' and the state gradient after every block.  A workspace that is not 16-byte aligned is
    refused before any CUDA call."""
    up = lambda f: (f + 63) // 64 * 64
    B, H, L, dk, dv = 4, 16, 4096, 128, 128
    NS, NB, BH = 8, 64, B * H
    base = up(8 * BH * L) + up(4 * BH) + up(BH * NS * (L * 16 + (NB + 1) * dk * 16)) + \
        up(NS * BH * L * (2 * dk + 1))
    tc = lib.efla_chunk_fwd_workspace_size(B, H, L, dk, dv, 64, BF16, F32)
    tcb = 2 * (2 * BH * L * dv + BH * NB * dk * dv)  # fp16 dO, dU' and the chunks' state gradients
    saved = up(tc // 4) + up(BH * L * dv // 2) + up(BH * NB * dk * dv // 2) + (tcb + 3) // 4  # fp16 u, states
    assert lib.efla_bwd_workspace_size(B, H, L, dk, dv) == 4 * (base + saved)
    # ragged, no tensor-core forward (d_k = 8): dv = 20 takes two column blocks, L = 65 two blocks
    assert lib.efla_bwd_workspace_size(1, 1, 65, 8, 20) == \
        4 * (up(8 * 65) + up(4) + up(2 * (65 * 16 + 3 * 8 * 16)) + up(2 * 65 * 17))
    assert lib.efla_bwd_workspace_size(1, 1, 16, 129, 16) == 0
    P = ctypes.c_void_p(64)
    EFLA_ERR_ALIGN, EFLA_ERR_WORKSPACE = 8, 7
    args = [P, P, P, P, None, P, None, P, P, P, P, None, 1, 1, 16, 16, 16, F32, 0]
    need = lib.efla_bwd_workspace_size(1, 1, 16, 16, 16)
    assert lib.efla_bwd(*args, ctypes.c_void_p(64 + 4), need, None) == EFLA_ERR_ALIGN
    assert lib.efla_bwd(*args, P, need - 4, None) == EFLA_ERR_WORKSPACE


def test_kept_buffer_size_and_host_errors(lib):
    """The training-step pair's kept buffer is the backward workspace's tensor-core forward
    region, u and chunk states (every region rounded up to 256 bytes); sizes without a
    tensor-core backward have none, and the entry points refuse them before any CUDA call."""
    up = lambda f: (f + 63) // 64 * 64
    B, H, L, dk, dv = 4, 16, 4096, 128, 128
    BH, NB = B * H, 64
    tc = lib.efla_chunk_fwd_workspace_size(B, H, L, dk, dv, 64, BF16, F32)
    assert lib.efla_bwd_kept_size(B, H, L, dk, dv) == \
        4 * (up(tc // 4) + up(BH * L * dv // 2) + up(BH * NB * dk * dv // 2))
    assert lib.efla_bwd_kept_size(1, 1, 65, 8, 20) == 0
    assert lib.efla_bwd_kept_size(1, 1, 0, 64, 64) == 0
    P = ctypes.c_void_p(64)
    UNSUPPORTED, WORKSPACE, ALIGN = 4, 7, 8
    need = lib.efla_bwd_kept_size(1, 1, 64, 64, 64)
    fwd = [P, P, P, P, None, P, P, 1, 1, 64, 64, 64]
    assert lib.efla_chunk_fwd_keep(*fwd, F32, F32, 0, P, need, None) == UNSUPPORTED
    assert lib.efla_chunk_fwd_keep(*fwd, BF16, F32, 0, None, 0, None) == WORKSPACE
    assert lib.efla_chunk_fwd_keep(*fwd, BF16, F32, 0, P, need - 16, None) == WORKSPACE
    assert lib.efla_chunk_fwd_keep(*fwd, BF16, F32, 0, ctypes.c_void_p(72), need, None) == ALIGN
    bwd = [P, P, P, P, None, P, None, P, P, P, P, None, 1, 1, 64, 64, 64]
    ws = lib.efla_bwd_workspace_size(1, 1, 64, 64, 64)
    assert lib.efla_bwd_kept(*bwd, F32, 0, P, need, P, ws, None) == UNSUPPORTED
    assert lib.efla_bwd_kept(*bwd, BF16, 0, None, 0, P, ws, None) == WORKSPACE
