"""C ABI checks that need no GPU: the library loads, exports every function the
header declares, sizes workspaces and rejects bad arguments before any CUDA call."""

import ctypes
import os
import re

import pytest

from attention_pass_rope_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ttt_attn.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return _lib.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ttt_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "ttt_attn_fwd" in names and "ttt_attn_bwd" in names
    for n in names:
        assert hasattr(L, n), n


def desc(**kw):
    d = _lib.TTTDesc()
    d.layout, d.P, d.B, d.S, d.H, d.Hkv, d.D = 0, 3, 2, 4096, 32, 8, 128
    d.rope_theta, d.softmax_scale = 1e6, 0.0
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_workspace_size_dense(L):
    d = desc()
    fwd = L.ttt_attn_workspace_size(ctypes.byref(d), 0)
    bwd = L.ttt_attn_workspace_size(ctypes.byref(d), 1)
    P, T, H, Hkv, D = 3, 8192, 32, 8, 128
    assert fwd >= P * T * H * D * 2 + P * T * Hkv * D * 2
    assert bwd >= P * T * H * D * 2 + P * T * Hkv * D * 2 + P * H * T * 4 + P * T * H * D * 4
    offs = (ctypes.c_size_t * 8)()
    n = L.ttt_attn_workspace_layout(ctypes.byref(d), 1, offs)
    assert n == 6
    assert all(offs[i] % 1024 == 0 for i in range(1, n))
    assert list(offs[:n]) == sorted(offs[:n])


@pytest.mark.parametrize("field,value,status", [
    ("D", 96, _lib.TTT_ERR_UNSUPPORTED),
    ("D", 0, _lib.TTT_ERR_INVALID_ARG),
    ("H", 30, _lib.TTT_ERR_INVALID_ARG),      # not a multiple of Hkv
    ("P", 0, _lib.TTT_ERR_INVALID_ARG),
    ("P", 17, _lib.TTT_ERR_UNSUPPORTED),
    ("rope_theta", 0.0, _lib.TTT_ERR_INVALID_ARG),
    ("rope_theta", -1.0, _lib.TTT_ERR_INVALID_ARG),
    ("softmax_scale", -0.5, _lib.TTT_ERR_INVALID_ARG),
    ("layout", 7, _lib.TTT_ERR_INVALID_ARG),
    ("B", -1, _lib.TTT_ERR_INVALID_ARG),
    ("flags", 4, _lib.TTT_ERR_INVALID_ARG),     # unknown flag bit
    ("flags", -1, _lib.TTT_ERR_INVALID_ARG),
])
def test_invalid_descriptor(L, field, value, status):
    d = desc(**{field: value})
    assert L.ttt_attn_workspace_size(ctypes.byref(d), 0) == 0
    fake = ctypes.c_void_p(1 << 20)
    st = L.ttt_attn_fwd(ctypes.byref(d), fake, fake, fake, fake, fake, fake, 1 << 40, None)
    assert st == status


@pytest.mark.parametrize("field", ["pass_stride_q", "pass_stride_kv"])
def test_pass_stride_validation(L, field):
    """A non-zero pass stride must be a multiple of 8 elements and no shorter than a packed
    pass; it does not change the workspace (the rotated copies are packed); with P = 1 it
    is ignored."""
    packed = 8192 * (32 if field == "pass_stride_q" else 8) * 128
    base = L.ttt_attn_workspace_size(ctypes.byref(desc()), 1)
    for value, ok in ((packed, True), (packed + 8, True), (3 * packed, True), (packed - 8, False),
                      (packed + 4, False), (-8, False)):
        d = desc(**{field: value})
        assert (L.ttt_attn_workspace_size(ctypes.byref(d), 1) == base) == ok, value
        if not ok:
            fake = ctypes.c_void_p(1 << 20)
            st = L.ttt_attn_fwd(ctypes.byref(d), fake, fake, fake, fake, fake, fake, 1 << 40, None)
            assert st == _lib.TTT_ERR_INVALID_ARG
    d = desc(P=1, **{field: 5})
    assert L.ttt_attn_workspace_size(ctypes.byref(d), 0) > 0


def test_known_flags_accepted(L):
    for f in (_lib.TTT_FLAG_ROTATED_IN_WORKSPACE, _lib.TTT_FLAG_DETERMINISTIC_DQ,
              _lib.TTT_FLAG_ROTATED_IN_WORKSPACE | _lib.TTT_FLAG_DETERMINISTIC_DQ):
        d = desc(flags=f)
        assert L.ttt_attn_workspace_size(ctypes.byref(d), 1) == L.ttt_attn_workspace_size(ctypes.byref(desc()), 1) > 0


def test_null_descriptor(L):
    assert L.ttt_attn_fwd(None, None, None, None, None, None, None, 0, None) == _lib.TTT_ERR_INVALID_ARG
    assert L.ttt_attn_workspace_size(None, 0) == 0


def test_null_tensor_pointers(L):
    d = desc()
    fake = ctypes.c_void_p(1 << 20)
    st = L.ttt_attn_fwd(ctypes.byref(d), None, fake, fake, fake, fake, fake, 1 << 40, None)
    assert st == _lib.TTT_ERR_INVALID_ARG
    st = L.ttt_attn_bwd(ctypes.byref(d), fake, fake, fake, fake, fake, None, fake, fake, fake, fake, 1 << 40, None)
    assert st == _lib.TTT_ERR_INVALID_ARG


def test_misaligned_tensor(L):
    d = desc()
    fake = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 2)
    st = L.ttt_attn_fwd(ctypes.byref(d), odd, fake, fake, fake, fake, fake, 1 << 40, None)
    assert st == _lib.TTT_ERR_INVALID_ARG


def test_workspace_errors(L):
    d = desc()
    fake = ctypes.c_void_p(1 << 20)
    need = L.ttt_attn_workspace_size(ctypes.byref(d), 0)
    st = L.ttt_attn_fwd(ctypes.byref(d), fake, fake, fake, fake, fake, fake, need - 1, None)
    assert st == _lib.TTT_ERR_WORKSPACE
    st = L.ttt_attn_fwd(ctypes.byref(d), fake, fake, fake, fake, fake, None, need, None)
    assert st == _lib.TTT_ERR_WORKSPACE
    st = L.ttt_attn_fwd(ctypes.byref(d), fake, fake, fake, fake, fake, ctypes.c_void_p((1 << 20) + 64), need, None)
    assert st == _lib.TTT_ERR_WORKSPACE


def test_packed_layout_validation(L):
    d = desc(layout=1, nseq=2, total_tokens=100, max_seqlen=60)
    assert L.ttt_attn_workspace_size(ctypes.byref(d), 0) == 0       # cu_seqlens missing
    d.cu_seqlens = 1 << 20
    assert L.ttt_attn_workspace_size(ctypes.byref(d), 0) > 0
    d.max_seqlen = 101                                               # longer than the batch
    assert L.ttt_attn_workspace_size(ctypes.byref(d), 0) == 0


def test_empty_batch_is_a_no_op(L):
    d = desc(B=0)
    assert L.ttt_attn_fwd(ctypes.byref(d), None, None, None, None, None, None, 0, None) == _lib.TTT_OK
    d = desc(layout=1, nseq=0, total_tokens=0, max_seqlen=0)
    assert L.ttt_attn_bwd(ctypes.byref(d), None, None, None, None, None, None, None, None, None, None, 0,
                          None) == _lib.TTT_OK


def test_status_strings(L):
    for s in range(6):
        assert L.ttt_status_string(s)
    assert L.ttt_attn_version().decode().count(".") == 2


def test_one_version_string(L):
    """The library, the Python package and the header's example name the same version."""
    import attention_pass_rope_b200 as pkg
    v = L.ttt_attn_version().decode()
    assert pkg.__version__ == v
    assert f'"{v}"' in open(HEADER).read()


@pytest.mark.parametrize("kw", [dict(), dict(P=1, H=4, Hkv=4, D=64), dict(P=16, B=1, S=130),
                                dict(layout=1, nseq=3, total_tokens=200, max_seqlen=129, cu_seqlens=1 << 20)])
def test_forward_layout_is_a_prefix_of_backward(L, kw):
    """TTT_FLAG_ROTATED_IN_WORKSPACE relies on it: the rotated q~ / k~ sit at the same
    offsets in the forward's and the backward's workspace, and the backward's is larger."""
    d = desc(**kw)
    f = (ctypes.c_size_t * 8)()
    b = (ctypes.c_size_t * 8)()
    nf = L.ttt_attn_workspace_layout(ctypes.byref(d), 0, f)
    nb = L.ttt_attn_workspace_layout(ctypes.byref(d), 1, b)
    assert nf == 3 and nb == 6
    assert list(f[:nf]) == list(b[:nf])
    assert L.ttt_attn_workspace_size(ctypes.byref(d), 1) >= L.ttt_attn_workspace_size(ctypes.byref(d), 0) > 0


def block_desc(**kw):
    d = _lib.TTTBlockDesc()
    d.layout, d.B, d.S, d.nblk, d.H, d.Hkv, d.D, d.Bs = 0, 2, 4096, 256, 32, 8, 128, 16
    d.rope_theta, d.softmax_scale = 1e6, 0.0
    d.anchors = 0x1000  # only checked for NULL by the sizing call, never read on the host
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_block_window_validation(L):
    """Sliding-window block layers: window >= 0 (0 = the whole trunk) sizes the same
    workspace; a negative window is rejected before any CUDA call."""
    L.ttt_block_workspace_size.restype = ctypes.c_size_t
    L.ttt_block_workspace_size.argtypes = [ctypes.POINTER(_lib.TTTBlockDesc), ctypes.c_int]
    full = L.ttt_block_workspace_size(ctypes.byref(block_desc()), 1)
    assert full > 0
    for w in (1, 1024, 10 ** 6):
        assert L.ttt_block_workspace_size(ctypes.byref(block_desc(window=w)), 1) == full
    assert L.ttt_block_workspace_size(ctypes.byref(block_desc(window=-1)), 1) == 0
    assert ctypes.sizeof(_lib.TTTBlockDesc) % 8 == 0


def softce_desc(**kw):
    d = _lib.TTTSoftceDesc()
    d.P, d.T, d.d, d.V = 3, 8192, 4096, 151936
    d.nseq = 1
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_softce_workspace_sizes(L):
    """Forward: status block, teacher rows, counts, then 5 floats per (row, 256-column
    vocabulary tile); backward: rows, counts, coefficients and one chunk of bf16 dz
    (4096 rows by default) at a row stride of V rounded up to 64."""
    d = softce_desc()
    R, ntn = 3 * 8192, (151936 + 255) // 256
    fwd = L.ttt_softce_workspace_size(ctypes.byref(d), 0)
    bwd = L.ttt_softce_workspace_size(ctypes.byref(d), 1)
    assert fwd >= ntn * 5 * R * 4 and fwd - ntn * 5 * R * 4 < R * 4 + 4096
    assert bwd >= 4096 * 151936 * 2 and bwd - 4096 * 151936 * 2 < 2 * R * 4 + 4096
    d2 = softce_desc(token_chunk_size=100)
    assert L.ttt_softce_workspace_size(ctypes.byref(d2), 1) < bwd
    # fused: statistics, coefficients, one chunk of fp32 logits and one of bf16 dz
    fused = L.ttt_softce_workspace_size(ctypes.byref(d), 2)
    assert fused >= ntn * 5 * R * 4 + 4096 * 151936 * 6
    assert fused - (ntn * 5 * R * 4 + 4096 * 151936 * 6) < 2 * R * 4 + 8192
    assert L.ttt_softce_workspace_size(ctypes.byref(d), 3) == 0


def test_softce_rejects_bad_arguments(L):
    """Every rejection happens before any CUDA call (this machine has no GPU)."""
    ok = softce_desc()
    assert L.ttt_softce_workspace_size(None, 0) == 0
    for bad in (dict(P=0), dict(T=-1), dict(d=4), dict(V=0), dict(token_chunk_size=-1), dict(nseq=-1)):
        assert L.ttt_softce_workspace_size(ctypes.byref(softce_desc(**bad)), 0) == 0, bad
    # d or V not a multiple of 8, or smaller than one TMA box: unsupported
    for bad in (dict(d=4100), dict(V=151937), dict(d=32), dict(V=128)):
        assert L.ttt_softce_workspace_size(ctypes.byref(softce_desc(**bad)), 1) == 0, bad
    fake = ctypes.c_void_p(1 << 20)
    vp = ctypes.c_void_p
    # missing loss pointer, missing inputs, unaligned input, missing workspace
    assert L.ttt_softce_fwd(ctypes.byref(ok), fake, fake, fake, fake, fake, None, fake, 1 << 40, None) == \
        _lib.TTT_ERR_INVALID_ARG
    assert L.ttt_softce_fwd(ctypes.byref(ok), None, fake, fake, fake, fake, fake, fake, 1 << 40, None) == \
        _lib.TTT_ERR_INVALID_ARG
    assert L.ttt_softce_fwd(ctypes.byref(ok), vp((1 << 20) + 2), fake, fake, fake, fake, fake, fake, 1 << 40,
                            None) == _lib.TTT_ERR_INVALID_ARG
    assert L.ttt_softce_fwd(ctypes.byref(ok), fake, fake, fake, fake, fake, fake, None, 1 << 40, None) == \
        _lib.TTT_ERR_WORKSPACE
    assert L.ttt_softce_fwd(ctypes.byref(ok), fake, fake, fake, fake, fake, fake, fake, 1024, None) == \
        _lib.TTT_ERR_WORKSPACE
    assert L.ttt_softce_bwd(ctypes.byref(ok), fake, fake, fake, fake, ctypes.c_float(float("nan")), fake, None,
                            fake, 1 << 40, None) == _lib.TTT_ERR_INVALID_ARG
    assert L.ttt_softce_bwd(ctypes.byref(ok), fake, fake, fake, None, ctypes.c_float(1.0), fake, None, fake,
                            1 << 40, None) == _lib.TTT_ERR_INVALID_ARG
    assert L.ttt_softce_fwd_bwd(ctypes.byref(ok), fake, fake, fake, ctypes.c_float(1.0), fake, fake, None, fake,
                                None, fake, 1 << 40, None) == _lib.TTT_ERR_INVALID_ARG
    assert L.ttt_softce_fwd_bwd(ctypes.byref(ok), fake, fake, fake, ctypes.c_float(1.0), fake, fake, fake, fake,
                                None, fake, 1024, None) == _lib.TTT_ERR_WORKSPACE
    # general form: groups >= 1, and several groups need the group array
    d_g = softce_desc(row_teacher=fake.value, ngroups=0, teacher_rows=10)
    assert L.ttt_softce_workspace_size(ctypes.byref(d_g), 0) == 0
    d_g = softce_desc(row_teacher=fake.value, ngroups=4, teacher_rows=10)
    assert L.ttt_softce_workspace_size(ctypes.byref(d_g), 0) == 0
    d_g = softce_desc(row_teacher=fake.value, row_group=fake.value, ngroups=4, teacher_rows=10)
    assert L.ttt_softce_workspace_size(ctypes.byref(d_g), 0) > 0
    d_g = softce_desc(row_teacher=fake.value, ngroups=1, teacher_rows=-1)
    assert L.ttt_softce_workspace_size(ctypes.byref(d_g), 0) == 0
    # a dense descriptor whose T is not a multiple of nseq
    assert L.ttt_softce_workspace_size(ctypes.byref(softce_desc(nseq=3, T=8192)), 0) == 0
