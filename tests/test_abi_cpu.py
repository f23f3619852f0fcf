"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/gla.h declares, and rejects bad arguments before
enqueuing anything."""
import ctypes
import os
import re

import pytest

import chunkwise_linear_rnn_fwd_b200 as pkg
from chunkwise_linear_rnn_fwd_b200 import gla as G

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from chunkwise_linear_rnn_fwd_b200 import build
    build.build()
    return pkg.load()


def header_functions():
    src = open(os.path.join(ROOT, "include", "gla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gla_[a-z_0-9]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(G.EXPORTS) == names


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7, -8):
        assert G.status_string(code)
    assert "unknown" in G.status_string(12345)


def desc(**kw):
    base = dict(B=2, H=4, T=300, dk=128, dv=256, dtype=0, gate="vector")
    base.update(kw)
    return G.make_desc(base.pop("B"), base.pop("H"), base.pop("T"), base.pop("dk"), base.pop("dv"),
                       base.pop("dtype"), base.pop("gate"), **base)


def test_check_and_workspace(lib):
    d = desc()
    assert lib.gla_check(ctypes.byref(d), 64) == 0
    assert lib.gla_workspace_size(ctypes.byref(d), 64, 0) > 0
    assert lib.gla_workspace_size(ctypes.byref(d), 64, 1) >= lib.gla_workspace_size(ctypes.byref(d), 64, 0)
    assert lib.gla_check(ctypes.byref(d), 48) == -2            # chunk not supported
    assert lib.gla_check(ctypes.byref(desc(T=0)), 64) == -1
    assert lib.gla_check(ctypes.byref(desc(dtype=7)), 64) == -1
    assert lib.gla_check(ctypes.byref(desc(gate=5)), 64) == -1
    assert lib.gla_check(ctypes.byref(desc(dk=512)), 64) == -2
    assert lib.gla_check(ctypes.byref(desc(subchunk=24)), 64) == -2
    assert lib.gla_workspace_size(ctypes.byref(desc(T=0)), 64, 0) == 0
    assert lib.gla_check(None, 64) == -1
    assert lib.gla_check(ctypes.byref(desc(flags=1)), 64) == 0
    assert lib.gla_check(ctypes.byref(desc(flags=2)), 64) == 0
    assert lib.gla_check(ctypes.byref(desc(flags=3)), 64) == 0
    assert lib.gla_check(ctypes.byref(desc(flags=8)), 64) == -1               # unknown flag bit
    assert lib.gla_check(ctypes.byref(desc(flags=4)), 64) == 0                # GLA_FLAG_REUSE_SEGMENTS


def test_saved_state_workspace_layout(lib):
    """A forward that saves states needs the backward's workspace; the
    MATERIALIZED forward's fp32 states are appended after everything else."""
    fwd = lib.gla_workspace_size(ctypes.byref(desc()), 64, 0)
    bwd = lib.gla_workspace_size(ctypes.byref(desc()), 64, 1)
    assert 0 < fwd < bwd
    assert lib.gla_workspace_size(ctypes.byref(desc(flags=2)), 64, 1) == bwd
    mat = lib.gla_workspace_size(ctypes.byref(desc(flags=2, variant=2)), 64, 1)
    assert mat > bwd
    assert lib.gla_workspace_size(ctypes.byref(desc(variant=2)), 64, 1) == bwd


def test_bad_calls_enqueue_nothing(lib):
    """Every one of these returns an error from host validation alone (no GPU
    is touched: the status word is cleared only after validation passes)."""
    vp = ctypes.c_void_p
    a = vp(4096)           # aligned, never dereferenced
    mis = vp(4096 + 4)     # misaligned
    ws = vp(1 << 20)
    d = desc(T=64, dk=128, dv=128)
    d.workspace = 1 << 20
    d.workspace_bytes = 1 << 40
    f = lib.gla_fwd
    assert f(ctypes.byref(d), None, a, a, a, None, a, None, 64, None) == -1      # q NULL
    assert f(ctypes.byref(d), mis, a, a, a, None, a, None, 64, None) == -3       # q misaligned
    assert f(ctypes.byref(d), a, a, a, None, None, a, None, 64, None) == -1      # vector gate without log_alpha
    d.gate = 2
    assert f(ctypes.byref(d), a, a, a, a, None, a, None, 64, None) == -1         # none gate with log_alpha
    d.gate = 0
    d.workspace_bytes = 16
    assert f(ctypes.byref(d), a, a, a, a, None, a, None, 64, None) == -4         # workspace too small
    d.workspace_bytes = 1 << 40
    d.workspace = (1 << 20) + 8
    assert f(ctypes.byref(d), a, a, a, a, None, a, None, 64, None) == -3         # workspace misaligned
    d.workspace = 0
    assert f(ctypes.byref(d), a, a, a, a, None, a, None, 64, None) == -1         # no workspace
    d.workspace = 1 << 20
    b = lib.gla_bwd
    assert b(ctypes.byref(d), a, a, a, a, None, None, None, a, a, a, a, None, 64, None) == -1   # do NULL
    assert b(ctypes.byref(d), a, a, a, a, None, a, None, a, a, a, None, None, 64, None) == -1   # dlog_alpha NULL
    d.gate = 2
    assert b(ctypes.byref(d), a, a, a, None, None, a, None, a, a, a, a, None, 64, None) == -1   # none gate with dla


def test_decode_step_validation_enqueues_nothing(lib):
    """gla_decode_step rejects bad descriptors and pointers before any launch."""
    vp = ctypes.c_void_p
    a = vp(4096)
    mis = vp(4096 + 4)
    d = desc(T=1, dk=128, dv=128)
    f = lib.gla_decode_step
    f.argtypes = [ctypes.POINTER(type(d)), vp, vp, vp, vp, vp, vp, vp]
    assert f(None, a, a, a, a, a, a, None) == -1                              # no descriptor
    d.T = 2
    assert f(ctypes.byref(d), a, a, a, a, a, a, None) == -1                   # T must be 1
    d.T = 1
    d.dv = 126
    assert f(ctypes.byref(d), a, a, a, a, a, a, None) == -2                   # d_v not a multiple of 4
    d.dv = 128
    d.dk = 5000
    assert f(ctypes.byref(d), a, a, a, a, a, a, None) == -2                   # d_k too large
    d.dk = 128
    assert f(ctypes.byref(d), a, a, a, None, a, a, None) == -1                # vector gate without log_alpha
    assert f(ctypes.byref(d), a, a, a, a, None, a, None) == -1                # state NULL
    assert f(ctypes.byref(d), a, a, a, a, mis, a, None) == -3                 # state misaligned
    assert f(ctypes.byref(d), a, a, mis, a, a, a, None) == -3                 # v misaligned
    d.gate = 2
    assert f(ctypes.byref(d), a, a, a, a, a, a, None) == -1                   # none gate with log_alpha


def test_epilogue_validation_enqueues_nothing(lib):
    """gla_epilogue_fwd / _bwd reject bad descriptors, pointers and workspaces before
    any launch (every call below fails validation: none reaches a kernel)."""
    vp = ctypes.c_void_p
    a = vp(4096)
    mis = vp(4096 + 4)
    d = desc(T=10, dv=512)
    f, b = lib.gla_epilogue_fwd, lib.gla_epilogue_bwd
    d.dv = 12
    assert f(ctypes.byref(d), a, a, None, None, 1e-5, a, None) == -2          # d_v not a multiple of 8
    d.dv = 2048
    assert f(ctypes.byref(d), a, a, None, None, 1e-5, a, None) == -2          # d_v too large
    d.dv = 512
    assert f(ctypes.byref(d), a, a, None, None, 0.0, a, None) == -1           # eps must be positive
    assert f(ctypes.byref(d), None, a, None, None, 1e-5, a, None) == -1       # o NULL
    assert f(ctypes.byref(d), a, mis, None, None, 1e-5, a, None) == -3        # r misaligned
    assert f(ctypes.byref(d), a, a, mis, None, 1e-5, a, None) == -3          # w misaligned
    assert f(ctypes.byref(d), a, a, None, None, 1e-5, a, None) == -1         # no workspace (status word)
    d.workspace = (1 << 20) + 8
    d.workspace_bytes = 1 << 30
    assert f(ctypes.byref(d), a, a, None, None, 1e-5, a, None) == -3         # workspace misaligned
    d.workspace = 1 << 20
    d.workspace_bytes = 255
    assert f(ctypes.byref(d), a, a, None, None, 1e-5, a, None) == -4         # smaller than the status word
    assert b(ctypes.byref(d), a, a, None, None, 1e-5, a, a, a, None, None, None) == -4  # same, without dw/db
    d.workspace = None
    d.workspace_bytes = 0
    assert b(ctypes.byref(d), a, a, None, None, 1e-5, a, a, a, a, a, None) == -1   # dw asked, no workspace
    d.workspace = (1 << 20) + 8
    d.workspace_bytes = 1 << 30
    assert b(ctypes.byref(d), a, a, None, None, 1e-5, a, a, a, a, a, None) == -3   # workspace misaligned
    d.workspace = 1 << 20
    d.workspace_bytes = 16
    assert b(ctypes.byref(d), a, a, None, None, 1e-5, a, a, a, a, a, None) == -4   # workspace too small
    assert lib.gla_epilogue_workspace_size(ctypes.byref(d)) > 16
    # status word + per-CTA partial sums of dw, db (at most 1024 CTAs of 8 rows)
    assert lib.gla_epilogue_workspace_size(ctypes.byref(d)) == 256 + 10 * 2 * 512 * 4  # 80 rows, 10 CTAs
    big = desc(T=1 << 20, dv=512)
    assert lib.gla_epilogue_workspace_size(ctypes.byref(big)) == 256 + 1024 * 2 * 512 * 4
    assert b(ctypes.byref(d), a, a, None, None, 1e-5, None, a, a, a, a, None) == -1  # dy NULL


def test_oracle_not_imported_by_product():
    """The product package never imports, loads or links the oracle."""
    pkg_dir = os.path.join(ROOT, "chunkwise_linear_rnn_fwd_b200")
    pat = re.compile(r"^\s*(from\s+oracle|import\s+oracle)|libgla_oracle|gla_oracle", re.M)
    for root, _, files in os.walk(pkg_dir):
        for f in files:
            if f.endswith((".py", ".cu", ".h", ".cuh")):
                assert not pat.search(open(os.path.join(root, f)).read()), f


def test_sequence_state_validation_enqueues_nothing(lib):
    """gla_fwd_state / gla_bwd_state / gla_state_scan reject bad arguments before any
    launch (every call below fails validation: none reaches a kernel)."""
    vp = ctypes.c_void_p
    a, mis = vp(4096), vp(4096 + 4)
    d = desc(T=300, dk=256, dv=512)
    fs, bs, sc = lib.gla_fwd_state, lib.gla_bwd_state, lib.gla_state_scan
    d32 = desc(T=300, dk=256, dv=512, dtype=1)
    assert fs(ctypes.byref(d32), a, a, a, a, None, a, a, 64, None) == -2      # fp32: bf16 path only
    assert bs(ctypes.byref(d32), a, a, a, a, None, a, a, 64, None) == -2
    assert fs(ctypes.byref(d), None, a, a, a, None, a, a, 64, None) == -1     # q NULL
    assert fs(ctypes.byref(d), a, a, a, a, None, None, a, 64, None) == -1     # delta NULL
    assert fs(ctypes.byref(d), a, a, a, a, None, a, None, 64, None) == -1     # gamma NULL
    assert fs(ctypes.byref(d), a, a, a, a, mis, a, a, 64, None) == -3         # h0 misaligned
    assert fs(ctypes.byref(d), a, a, a, a, None, a, a, 64, None) == -1        # no workspace
    assert bs(ctypes.byref(d), a, a, a, None, None, a, None, 64, None) == -1  # do NULL
    assert bs(ctypes.byref(d), a, a, a, a, None, None, None, 64, None) == -1  # ddelta NULL
    assert bs(ctypes.byref(d), a, a, None, a, None, a, None, 64, None) == -1  # vector gate without log_alpha
    assert bs(ctypes.byref(d), a, a, a, a, None, a, None, 64, None) == -1     # no workspace
    d.workspace = 1 << 20
    d.workspace_bytes = 16
    assert fs(ctypes.byref(d), a, a, a, a, None, a, a, 64, None) == -4        # workspace too small
    assert bs(ctypes.byref(d), a, a, a, a, None, a, None, 64, None) == -4
    assert sc(ctypes.byref(d), 0, 0, 0, a, a, None, a, None) == -1            # no pieces
    assert sc(ctypes.byref(d), 3, 3, 0, a, a, None, a, None) == -1            # seg out of range
    assert sc(ctypes.byref(d), 3, -1, 0, a, a, None, a, None) == -1
    assert sc(ctypes.byref(d), 3, 1, 2, a, a, None, a, None) == -1            # reverse not 0/1
    assert sc(ctypes.byref(d), 3, 1, 0, None, a, None, a, None) == -1         # gammas NULL with a piece to fold
    assert sc(ctypes.byref(d), 3, 1, 1, a, None, None, a, None) == -1         # deltas NULL
    assert sc(ctypes.byref(d), 3, 1, 0, a, a, None, None, None) == -1         # out NULL
    assert sc(ctypes.byref(d), 3, 1, 0, a, a, mis, a, None) == -3             # init misaligned
    d.dv = 510
    assert sc(ctypes.byref(d), 3, 1, 0, a, a, None, a, None) == -2            # d_v not a multiple of 4


def test_general_gate_validation_enqueues_nothing(lib):
    """gla_fwd_general / gla_bwd_general reject bad arguments before any launch
    (every call below fails validation: none reaches a kernel)."""
    vp = ctypes.c_void_p
    a, mis = vp(4096), vp(4096 + 4)
    d = desc(T=100, dk=64, dv=64)
    f, b = lib.gla_fwd_general, lib.gla_bwd_general
    assert lib.gla_general_workspace_size(ctypes.byref(d), 64, 1) > lib.gla_general_workspace_size(ctypes.byref(d), 64, 0)
    assert f(ctypes.byref(d), a, a, a, a, None, None, a, None, 64, None) == -1      # log_beta NULL
    assert f(ctypes.byref(d), a, a, a, a, mis, None, a, None, 64, None) == -3       # log_beta misaligned
    assert f(ctypes.byref(d), a, a, a, None, a, None, a, None, 64, None) == -1      # vector gate without log_alpha
    assert f(ctypes.byref(d), a, a, a, a, a, None, a, None, 64, None) == -1         # no workspace
    assert b(ctypes.byref(d), a, a, a, a, a, None, a, None, a, a, a, a, None, None, 64, None) == -1  # dlog_beta NULL
    assert b(ctypes.byref(d), a, a, a, a, a, None, a, None, a, a, a, None, a, None, 64, None) == -1  # dlog_alpha NULL
    d.workspace = 1 << 20
    d.workspace_bytes = 16
    assert f(ctypes.byref(d), a, a, a, a, a, None, a, None, 64, None) == -4         # workspace too small
    assert b(ctypes.byref(d), a, a, a, a, a, None, a, None, a, a, a, a, a, None, 64, None) == -4


def test_saved_state_summary_needs_backward_workspace(lib):
    """gla_fwd_state with GLA_FLAG_SAVE_STATES lays out the backward's workspace; a
    workspace of the forward's size is refused before anything is enqueued."""
    vp = ctypes.c_void_p
    a = vp(4096)
    d = desc(T=4096, dk=256, dv=512, flags=2)
    fwd = lib.gla_workspace_size(ctypes.byref(d), 64, 0)
    bwd = lib.gla_workspace_size(ctypes.byref(d), 64, 1)
    assert 0 < fwd < bwd
    d.workspace = 1 << 20
    d.workspace_bytes = fwd
    assert lib.gla_fwd_state(ctypes.byref(d), a, a, a, a, None, a, a, 64, None) == -4
    d.workspace_bytes = bwd - 1
    assert lib.gla_fwd_state(ctypes.byref(d), a, a, a, a, None, a, a, 64, None) == -4


def test_noalloc_rejects_reuse_flags(lib):
    """The no-allocation forward's scratch holds nothing a later call may reuse: the
    reuse flags are refused before anything is enqueued (no GPU is touched)."""
    vp = ctypes.c_void_p
    a = vp(4096)
    for flags in (1, 4, 5, 3):
        d = desc(T=64, dk=128, dv=128, flags=flags)
        assert lib.gla_fwd_noalloc(ctypes.byref(d), a, a, a, a, None, a, None, 64, None) == -1
    assert lib.gla_fwd_noalloc(None, a, a, a, a, None, a, None, 64, None) == -1


def test_fused_epilogue_validation_enqueues_nothing(lib):
    """gla_fwd_epilogue checks the forward's and the epilogue's arguments before any
    launch (every call below fails validation: none reaches a kernel)."""
    vp = ctypes.c_void_p
    a = vp(4096)
    mis = vp(4096 + 4)
    f = lib.gla_fwd_epilogue
    d = desc(T=64, dk=128, dv=256)
    d.workspace = 1 << 20
    d.workspace_bytes = 1 << 40

    def call(q=a, r=a, w=None, b=None, eps=1e-5, o=a, y=a, dd=d):
        return f(ctypes.byref(dd), q, a, a, a, None, r, w, b, eps, o, y, None, 64, None)

    assert call(q=None) == -1                      # q NULL
    assert call(r=None) == -1                      # gate input r NULL
    assert call(y=None) == -1                      # y NULL
    assert call(y=mis) == -3                       # y misaligned
    assert call(w=mis) == -3                       # LayerNorm weight misaligned
    assert call(eps=0.0) == -1                     # eps must be positive
    assert call(eps=1.5) == -1
    d.flags = G.FLAG_REUSE_SEGMENTS
    assert call() == -1                            # segment contributions are not reused
    d.flags = 0
    d.workspace_bytes = 16
    assert call() == -4                            # workspace too small
    d.workspace_bytes = 1 << 40
    # shapes the fused walk does not take run two passes, so the epilogue's own
    # limits apply: fp32 with d_v = 12 (not a multiple of 8)
    e = desc(T=64, dk=64, dv=12, dtype=1)
    e.workspace = 1 << 20
    e.workspace_bytes = 1 << 40
    assert call(dd=e) == -2


def test_bf16_shapes_outside_the_tensor_core_path(lib):
    """bf16 descriptors the tensor-core path does not take (chunk 16, 32, 128; d_k 64;
    d_v not a multiple of 64) are valid and sized for the CUDA-core path; the
    sequence summaries, which exist on the tensor-core path only, refuse them."""
    vp = ctypes.c_void_p
    a = vp(4096)
    for kw, chunk in ((dict(), 16), (dict(), 32), (dict(), 128), (dict(dk=64), 64), (dict(dv=200), 64)):
        d = desc(**kw)
        assert lib.gla_check(ctypes.byref(d), chunk) == 0, (kw, chunk)
        assert lib.gla_workspace_size(ctypes.byref(d), chunk, 1) > 0
        d.workspace = 1 << 20
        d.workspace_bytes = 1 << 40
        assert lib.gla_fwd_state(ctypes.byref(d), a, a, a, a, None, a, a, chunk, None) == -2
    # the same bf16 shape sizes its workspace by the path that runs it
    d64, d128 = desc(), desc()
    assert lib.gla_workspace_size(ctypes.byref(d64), 64, 0) != lib.gla_workspace_size(ctypes.byref(d128), 128, 0)
