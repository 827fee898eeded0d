"""The C-ABI library loads, exports every entry point of include/libkda.h, and rejects bad
arguments on the host before anything is launched (no GPU needed: every call here returns
before its first CUDA call)."""
import ctypes
import os
import re

import pytest

import kimi_delta_attention_25_b200 as kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "libkda.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(kda_[a-z0-9_]+)\s*\(", src, re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from kimi_delta_attention_25_b200 import build
    build.build()
    return kda.load()


def test_header_declares_the_entry_points():
    assert declared_functions() == sorted(kda.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    nm = os.popen("nm -D --defined-only %s" % kda.library_path).read()
    for name in declared_functions():
        assert re.search(r"\bT %s\b" % name, nm), name


def test_status_strings_and_version(lib):
    assert kda.status_string(kda.KDA_OK) == "ok"
    assert "invalid" in kda.status_string(kda.KDA_ERR_INVALID_ARG)
    assert lib.kda_version() >= 100


def test_workspace_size(lib):
    assert kda.chunk_fwd_workspace_size(1, 8192, 16, 1) >= 256
    assert kda.chunk_fwd_workspace_size(1, 8192, 16, 1, dk=64) == 0
    assert kda.chunk_fwd_workspace_size(-1, 8192, 16, 1) == 0


FAKE = 0x10000  # 16-byte aligned, never dereferenced: each call below fails a host check first


def _chunk(lib, **kw):
    P = ctypes.c_void_p
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S0=None, cu=None, out=FAKE, Sf=None,
             B=1, T=64, H=2, N=1, dk=128, dv=128, dtype=1, odt=0, ws=FAKE, wsb=256)
    a.update(kw)
    return lib.kda_chunk_fwd(P(a["q"]), P(a["k"]), P(a["v"]), P(a["la"]), P(a["beta"]), P(a["S0"]),
                             P(a["cu"]), P(a["out"]), P(a["Sf"]), a["B"], a["T"], a["H"], a["N"],
                             a["dk"], a["dv"], a["dtype"], a["odt"], P(a["ws"]), a["wsb"], None)


def test_chunk_fwd_host_checks(lib):
    assert _chunk(lib, dk=64) == kda.KDA_ERR_UNSUPPORTED
    assert _chunk(lib, dv=256) == kda.KDA_ERR_UNSUPPORTED
    assert _chunk(lib, q=None) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, q=FAKE + 2) == kda.KDA_ERR_INVALID_ARG            # misaligned
    assert _chunk(lib, S0=FAKE + 8) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, N=2) == kda.KDA_ERR_INVALID_ARG                    # N != B without cu_seqlens
    assert _chunk(lib, B=2, cu=FAKE) == kda.KDA_ERR_INVALID_ARG           # packed needs B == 1
    assert _chunk(lib, cu=FAKE + 2) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, ws=None) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, wsb=16) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, dtype=7) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, odt=5) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, H=0) == kda.KDA_ERR_INVALID_ARG
    assert _chunk(lib, T=-1) == kda.KDA_ERR_INVALID_ARG


def _decode(lib, **kw):
    P = ctypes.c_void_p
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S=FAKE, out=FAKE, N=4, H=2, dk=128,
             dv=128, dtype=1, odt=0)
    a.update(kw)
    return lib.kda_decode_step(P(a["q"]), P(a["k"]), P(a["v"]), P(a["la"]), P(a["beta"]), P(a["S"]),
                               P(a["out"]), a["N"], a["H"], a["dk"], a["dv"], a["dtype"], a["odt"],
                               None)


def test_decode_host_checks(lib):
    assert _decode(lib, N=0) == kda.KDA_OK                                # nothing to do
    assert _decode(lib, dk=96) == kda.KDA_ERR_UNSUPPORTED
    assert _decode(lib, S=None) == kda.KDA_ERR_INVALID_ARG
    assert _decode(lib, S=FAKE + 4) == kda.KDA_ERR_INVALID_ARG
    assert _decode(lib, beta=FAKE + 2) == kda.KDA_ERR_INVALID_ARG
    assert _decode(lib, H=-1) == kda.KDA_ERR_INVALID_ARG
    assert _decode(lib, dtype=3) == kda.KDA_ERR_INVALID_ARG
    assert _decode(lib, odt=2) == kda.KDA_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 64, 2, 128)
    with pytest.raises(ValueError):
        kda.chunk_fwd(x, x, x, x, torch.zeros(1, 64, 2))


def _prep(lib, **kw):
    P = ctypes.c_void_p
    a = dict(q=FAKE, k=FAKE, la=FAKE, beta=FAKE, cu=None, B=1, T=64, H=2, N=1, dk=128, dv=128,
             ws=FAKE, wsb=256)
    a.update(kw)
    return lib.kda_chunk_prep(P(a["q"]), P(a["k"]), P(a["la"]), P(a["beta"]), P(a["cu"]), a["B"], a["T"],
                              a["H"], a["N"], a["dk"], a["dv"], P(a["ws"]), a["wsb"], None)


def _scan(lib, **kw):
    P = ctypes.c_void_p
    a = dict(v=FAKE, S0=None, cu=None, out=FAKE, Sf=None, B=1, T=64, H=2, N=1, dk=128, dv=128, odt=1,
             ws=FAKE, wsb=256)
    a.update(kw)
    return lib.kda_chunk_scan(P(a["v"]), P(a["S0"]), P(a["cu"]), P(a["out"]), P(a["Sf"]), a["B"], a["T"],
                              a["H"], a["N"], a["dk"], a["dv"], a["odt"], P(a["ws"]), a["wsb"], None)


def test_two_pass_host_checks(lib):
    need = kda.chunk_fwd_workspace_size(1, 64, 2, 1)
    assert need > 256
    # the first failing check decides; none of these reaches a CUDA call
    assert _prep(lib, dk=64) == kda.KDA_ERR_UNSUPPORTED
    assert _prep(lib, q=None) == kda.KDA_ERR_INVALID_ARG
    assert _prep(lib, la=FAKE + 4) == kda.KDA_ERR_INVALID_ARG
    assert _prep(lib, N=3) == kda.KDA_ERR_INVALID_ARG
    assert _prep(lib) == kda.KDA_ERR_INVALID_ARG                          # workspace too small
    assert _scan(lib, dv=64) == kda.KDA_ERR_UNSUPPORTED
    assert _scan(lib, v=None) == kda.KDA_ERR_INVALID_ARG
    assert _scan(lib, out=FAKE + 2) == kda.KDA_ERR_INVALID_ARG
    assert _scan(lib, Sf=FAKE + 8) == kda.KDA_ERR_INVALID_ARG
    assert _scan(lib, odt=9) == kda.KDA_ERR_INVALID_ARG
    assert _scan(lib, B=2, cu=FAKE) == kda.KDA_ERR_INVALID_ARG
    assert _scan(lib) == kda.KDA_ERR_INVALID_ARG                          # workspace too small


def test_selftest_host_checks(lib):
    P = ctypes.c_void_p
    f = lib.kda_selftest_wait_timeout
    assert f(None, 256, 1000, None) == kda.KDA_ERR_INVALID_ARG
    assert f(P(FAKE), 128, 1000, None) == kda.KDA_ERR_INVALID_ARG          # smaller than the status header
    assert f(P(FAKE + 8), 256, 1000, None) == kda.KDA_ERR_INVALID_ARG      # misaligned
    assert f(P(FAKE), 256, 0, None) == kda.KDA_ERR_INVALID_ARG
    assert f(P(FAKE), 256, 2000000001, None) == kda.KDA_ERR_INVALID_ARG


def _bwd(lib, **kw):
    P = ctypes.c_void_p
    a = dict(q=FAKE, k=FAKE, v=FAKE, la=FAKE, beta=FAKE, S0=None, cu=None, do=FAKE, dSf=None,
             dq=FAKE, dk_=FAKE, dv_=FAKE, dla=FAKE, dbe=FAKE, dS0=None,
             B=1, T=64, H=2, N=1, dk=128, dv=128, dtype=1, ws=FAKE, wsb=256)
    a.update(kw)
    return lib.kda_chunk_bwd(*[P(a[x]) for x in ("q", "k", "v", "la", "beta", "S0", "cu", "do", "dSf", "dq",
                                                 "dk_", "dv_", "dla", "dbe", "dS0")],
                             a["B"], a["T"], a["H"], a["N"], a["dk"], a["dv"], a["dtype"], P(a["ws"]), a["wsb"],
                             None)


def test_backward_host_checks(lib):
    need = kda.chunk_bwd_workspace_size(1, 64, 2, 1)
    # 2 heads x (64 / 64 + 1 + 1) slots of fp32 records, after the status prefix
    # per (head, chunk slot): S, dS' (128 x 128); R, U, Y (64 x 128); the reverse scan's prepared
    # operands Kp, Bk, Y0 (64 x 128), G0 (128 x 128), gamma and beta (256)
    assert need == 256 + 2 * 3 * (3 * 128 * 128 + 6 * 64 * 128 + 256 + 64 * 64) * 4
    assert kda.chunk_bwd_workspace_size(1, 64, 2, 1, dk=64) == 0
    # the first failing check decides; none of these reaches a CUDA call
    assert _bwd(lib, dk=64) == kda.KDA_ERR_UNSUPPORTED
    assert _bwd(lib, dtype=7) == kda.KDA_ERR_INVALID_ARG
    assert _bwd(lib, do=None) == kda.KDA_ERR_INVALID_ARG
    assert _bwd(lib, dla=None) == kda.KDA_ERR_INVALID_ARG
    assert _bwd(lib, dq=FAKE + 4) == kda.KDA_ERR_INVALID_ARG
    assert _bwd(lib, dS0=FAKE + 8) == kda.KDA_ERR_INVALID_ARG
    assert _bwd(lib, N=2) == kda.KDA_ERR_INVALID_ARG
    assert _bwd(lib, B=2, N=2, cu=FAKE) == kda.KDA_ERR_INVALID_ARG
    assert _bwd(lib) == kda.KDA_ERR_INVALID_ARG                           # workspace too small
    assert _bwd(lib, ws=FAKE + 8, wsb=need) == kda.KDA_ERR_INVALID_ARG    # misaligned workspace


def test_backward_phase_host_checks(lib):
    P = ctypes.c_void_p
    f = lib.kda_chunk_bwd_phase
    args = [P(FAKE)] * 5 + [None, None, P(FAKE), None] + [P(FAKE)] * 5 + [None] + [1, 64, 2, 1, 128, 128, 1]
    assert f(3, *args, P(FAKE), 256, None) == kda.KDA_ERR_INVALID_ARG      # no such phase
    assert f(-1, *args, P(FAKE), 256, None) == kda.KDA_ERR_INVALID_ARG
    assert f(1, *args, P(FAKE), 256, None) == kda.KDA_ERR_INVALID_ARG      # workspace too small
    args[19] = 64                                                           # dk
    assert f(2, *args, P(FAKE), 1 << 30, None) == kda.KDA_ERR_UNSUPPORTED


def test_chunked_calls_refuse_more_heads_or_sequences_than_a_grid_dimension(lib):
    """Heads and sequences index launch-grid dimensions (at most 65535 each): more is refused on
    the host, before any launch."""
    assert _chunk(lib, H=65536) == kda.KDA_ERR_UNSUPPORTED
    assert _chunk(lib, B=65536, N=65536) == kda.KDA_ERR_UNSUPPORTED
    assert _chunk(lib, B=1, N=70000, cu=FAKE) == kda.KDA_ERR_UNSUPPORTED
    assert _prep(lib, H=70000) == kda.KDA_ERR_UNSUPPORTED
    assert _scan(lib, H=70000) == kda.KDA_ERR_UNSUPPORTED
    assert _bwd(lib, H=65536) == kda.KDA_ERR_UNSUPPORTED
    assert _bwd(lib, B=1, N=65536, cu=FAKE) == kda.KDA_ERR_UNSUPPORTED
    P = ctypes.c_void_p
    f = lib.kda_chunk_fwd_noalloc
    assert f(*[P(FAKE)] * 5, None, None, P(FAKE), None, 1, 64, 65536, 1, 128, 128, 1, 0, None) == \
        kda.KDA_ERR_UNSUPPORTED
    # the limit itself is accepted by the host checks (this call then stops at its workspace)
    assert _chunk(lib, H=65535) == kda.KDA_ERR_INVALID_ARG


def test_chunk_fwd_kernel_launches(lib):
    """The launch count of the prefill: a pipeline over token ranges (two kernels per range) with at
    most 64 (sequence, head) chains and at least 64 chunk slots, else the two passes once; one
    kernel for fp32 inputs."""
    bf, f32 = 1, 0
    assert lib.kda_chunk_fwd_kernel_launches(1, 131072, 32, 1, bf) == 32     # 16 ranges
    assert lib.kda_chunk_fwd_kernel_launches(1, 8192, 16, 1, bf) == 8        # 4 ranges
    assert lib.kda_chunk_fwd_kernel_launches(1, 262144, 32, 8, bf) == 2      # 256 chains
    assert lib.kda_chunk_fwd_kernel_launches(1, 2048, 4, 1, bf) == 2         # 34 slots
    assert lib.kda_chunk_fwd_kernel_launches(1, 100, 2, 1, f32) == 1
    assert lib.kda_chunk_fwd_kernel_launches(1, 100, 2, 0, bf) == 0
    assert lib.kda_chunk_fwd_kernel_launches(-1, 100, 2, 1, bf) == 0


def test_workspace_holds_the_pipeline_carry(lib):
    """A pipelined prefill carries the state between token ranges; without S_final it lives in the
    workspace, after the prepared blocks."""
    blocks = 256 + 32 * (131072 // 64 + 2) * 66048
    assert lib.kda_chunk_fwd_workspace_size(1, 131072, 32, 1, 128, 128, 1) == blocks + 32 * 128 * 128 * 4
    blocks = 256 + 32 * (262144 // 64 + 9) * 66048
    assert lib.kda_chunk_fwd_workspace_size(1, 262144, 32, 8, 128, 128, 1) == blocks
