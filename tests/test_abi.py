"""The C ABI library loads, exports every symbol include/kda.h declares, and rejects bad
arguments on the host before any launch (no GPU needed for these)."""
import ctypes
import os
import re

import pytest

from linear_attention_sequence_mshortconv_b200 import build as B
from linear_attention_sequence_mshortconv_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    src = open(os.path.join(ROOT, "include", "kda.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(",
                                 src, flags=re.M)) - {"defined"})


@pytest.fixture(scope="module")
def lib():
    B.build()
    return kda.load_library()


def test_header_declares_the_boundary():
    fns = _header_functions()
    assert set(kda.EXPORTED) == set(fns), fns


def test_library_exports_every_declared_symbol(lib):
    for fn in _header_functions():
        assert hasattr(lib, fn), fn


def test_status_strings(lib):
    for code, name in kda.STATUS.items():
        assert lib.kda_status_string(code).decode() == name


def test_host_rejects_bad_arguments(lib):
    P = None
    # unsupported head width, before touching the device
    assert lib.kda_forward(P, P, P, P, P, P, P, P, 1, 8, 1, 48, 48, 1, 1, 0, P, 0, P) == 2
    # negative batch
    assert lib.kda_forward(P, P, P, P, P, P, P, P, -1, 8, 1, 32, 32, 1, 1, 0, P, 0, P) == 1
    # null tensors with work to do
    assert lib.kda_forward(P, P, P, P, P, P, P, P, 1, 8, 1, 32, 32, 1, 1, 0, P, 0, P) == 1
    # chunk not in {16, 32, 64, 128}
    assert lib.kda_forward(P, P, P, P, P, P, P, P, 1, 8, 1, 32, 32, 1, 1, 24, P, 0, P) == 2
    assert lib.kda_forward(P, P, P, P, P, P, P, P, 1, 8, 1, 32, 32, 1, 1, 256, P, 0, P) == 2
    # bad dtype / output dtype
    assert lib.kda_forward(P, P, P, P, P, P, P, P, 1, 8, 1, 32, 32, 7, 1, 0, P, 0, P) == 1
    assert lib.kda_forward(P, P, P, P, P, P, P, P, 1, 8, 1, 32, 32, 1, 9, 0, P, 0, P) == 1
    # empty problem is a no-op
    assert lib.kda_forward(P, P, P, P, P, P, P, P, 0, 8, 1, 32, 32, 1, 1, 0, P, 0, P) == 0


def test_gated_forward_rejects_bad_arguments(lib):
    P = None
    d = ctypes.c_void_p(256)   # never dereferenced: validation fails first
    args = lambda gate, eps, Dk=32: (d, d, d, d, d, P, gate, P, eps, d, P, 1, 8, 1, Dk, Dk, 1, 1, 0, P, 0, P)
    assert lib.kda_forward_gated(*args(P, 1e-6)) == 1                    # no gate with work to do
    assert lib.kda_forward_gated(*args(d, -1.0)) == 1                    # eps < 0
    assert lib.kda_forward_gated(*args(d, float("nan"))) == 1            # eps NaN
    assert lib.kda_forward_gated(*args(d, float("inf"))) == 1            # eps not finite
    assert lib.kda_forward_gated(*args(d, 1e-6, Dk=48)) == 2             # unsupported head width
    # empty batch is a no-op
    assert lib.kda_forward_gated(d, d, d, d, d, P, P, P, 1e-6, d, P, 0, 8, 1, 32, 32, 1, 1, 0, P, 0, P) == 0


def test_sequence_parallel_calls_reject_bad_arguments(lib):
    P = None
    d = ctypes.c_void_p(256)   # never dereferenced: validation fails first
    # transition: unsupported head width, null MN with work to do, no workspace, empty batch
    assert lib.kda_sp_transition(d, d, d, d, d, d, 1, 8, 1, 48, 1, 0, P, 0, P) == 2
    assert lib.kda_sp_transition(d, d, d, d, d, P, 1, 8, 1, 32, 1, 0, P, 0, P) == 1
    assert lib.kda_sp_transition(d, d, d, d, d, d, 1, 8, 1, 32, 1, 0, P, 0, P) == 5
    assert lib.kda_sp_transition(d, d, d, d, d, d, 0, 8, 1, 32, 1, 0, P, 0, P) == 0
    # prefix: rank outside [0, R), null output, unsupported head width
    assert lib.kda_sp_prefix(d, 2, 2, P, d, 1, 1, 32, P) == 1
    assert lib.kda_sp_prefix(d, 2, -1, P, d, 1, 1, 32, P) == 1
    assert lib.kda_sp_prefix(d, 2, 1, P, P, 1, 1, 32, P) == 1
    assert lib.kda_sp_prefix(d, 2, 1, P, d, 1, 1, 48, P) == 2
    # output: bad output dtype, chunk not in {16, 32, 64, 128}
    assert lib.kda_sp_output(d, d, d, d, d, P, d, P, 1, 8, 1, 32, 1, 9, 0, P, 0, P) == 1
    assert lib.kda_sp_output(d, d, d, d, d, P, d, P, 1, 8, 1, 32, 1, 1, 24, P, 0, P) == 2
    assert lib.kda_sp_workspace_size(1, 8, 1, 48, 1, 0) == 0


def test_backward_rejects_bad_arguments(lib):
    P = None
    d = ctypes.c_void_p(256)   # never dereferenced: validation fails first
    full = lambda **kw: tuple(kw.get(n, d) for n in ("q", "k", "v", "g", "beta")) + (P, d, P) + \
        tuple(kw.get(n, d) for n in ("dq", "dk", "dv", "dg", "dbeta")) + (P,)
    sizes = lambda Dk=32, Dv=32, B=1, T=8, dt=1, dodt=1: (B, T, 1, Dk, Dv, dt, dodt, P, 0, P)
    assert lib.kda_backward(*full(), *sizes(Dk=48)) == 2            # unsupported head width
    assert lib.kda_backward(*full(), *sizes(Dv=96)) == 2
    assert lib.kda_backward(*full(dg=P), *sizes()) == 1             # missing gradient buffer
    assert lib.kda_backward(*full(q=P), *sizes()) == 1              # missing input
    assert lib.kda_backward(*full(), *sizes(dt=4)) == 1             # bad dtype
    assert lib.kda_backward(*full(), *sizes(dodt=4)) == 1           # bad d_o dtype
    assert lib.kda_backward(*full(), *sizes(B=-1)) == 1
    assert lib.kda_backward(*full(), *sizes(B=0)) == 0              # empty batch: no-op
    # per (b, h) and 32-token chunk: the Dk x Dv entry state and, per 16 value columns, T and Kd
    assert lib.kda_backward_workspace_size(1, 64, 2, 32, 64) == 2 * 2 * (32 * 64 + (64 // 16) * 2 * 32 * 32) * 4
    assert lib.kda_backward_workspace_size(1, 64, 2, 48, 64) == 0


def test_conv_backward_rejects_bad_arguments(lib):
    segs, n = kda.make_segments([(kda.MSC_TEXT, 0, 1, 1, 10, 0)])
    d = ctypes.c_void_p(256)   # never dereferenced: validation fails first
    sp = ctypes.cast(segs, ctypes.c_void_p)
    P = None
    # no dx with work to do; dw wanted without x; Kt outside 1..8; C not a multiple of 8
    assert lib.mshortconv_backward(d, d, P, 1, 10, 16, 1, sp, n, 4, d, 1, P, 0, P, 0, P, P, P, P) == 1
    assert lib.mshortconv_backward(P, d, d, 1, 10, 16, 1, sp, n, 4, d, 1, P, 0, P, 0, d, P, P, P) == 1
    assert lib.mshortconv_backward(d, d, d, 1, 10, 16, 1, sp, n, 9, d, 1, P, 0, P, 0, P, P, P, P) == 2
    assert lib.mshortconv_backward(d, d, d, 1, 10, 12, 1, sp, n, 4, d, 1, P, 0, P, 0, P, P, P, P) == 1


def test_conv_rejects_bad_segment_tables(lib):
    segs, n = kda.make_segments([(kda.MSC_TEXT, 0, 1, 1, 10, 0)])
    dummy = ctypes.c_void_p(16)   # never dereferenced: validation fails first
    sp = ctypes.cast(segs, ctypes.c_void_p)
    # segment runs past T
    assert lib.mshortconv_forward(dummy, ctypes.c_void_p(32), 1, 8, 16, 1, sp, n, 4,
                                  dummy, 1, None, 0, None, 0, None) == 1
    # C not a multiple of 8
    assert lib.mshortconv_forward(dummy, ctypes.c_void_p(32), 1, 10, 12, 1, sp, n, 4,
                                  dummy, 1, None, 0, None, 0, None) == 1
    # text segment without text weights
    assert lib.mshortconv_forward(dummy, ctypes.c_void_p(32), 1, 10, 16, 1, sp, n, 4,
                                  None, 0, None, 0, None, 0, None) == 1
    # weight_set out of range
    segs2, n2 = kda.make_segments([(kda.MSC_TEXT, 0, 1, 1, 10, 3)])
    assert lib.mshortconv_forward(dummy, ctypes.c_void_p(32), 1, 10, 16, 1,
                                  ctypes.cast(segs2, ctypes.c_void_p), n2, 4,
                                  dummy, 1, None, 0, None, 0, None) == 1
    # overlapping segments
    segs3, n3 = kda.make_segments([(kda.MSC_TEXT, 0, 1, 1, 6, 0), (kda.MSC_TEXT, 4, 1, 1, 4, 0)])
    assert lib.mshortconv_forward(dummy, ctypes.c_void_p(32), 1, 10, 16, 1,
                                  ctypes.cast(segs3, ctypes.c_void_p), n3, 4,
                                  dummy, 1, None, 0, None, 0, None) == 1
    # Kt out of range
    assert lib.mshortconv_forward(dummy, ctypes.c_void_p(32), 1, 10, 16, 1, sp, n, 9,
                                  dummy, 1, None, 0, None, 0, None) == 2


def test_segment_record_layout_matches_header():
    assert ctypes.sizeof(kda.MscSegment) == 32
    assert kda.MscSegment.start.offset == 8 and kda.MscSegment.weight_set.offset == 28


def test_binding_refuses_cpu_tensors(lib):
    import torch
    z = torch.zeros(1, 4, 1, 32)
    with pytest.raises(TypeError):
        kda.forward(z, z, z, z, torch.zeros(1, 4, 1))
