"""Host-side checks of libegnn.so: it loads, exports every function include/egnn.h
declares, and its host logic (sizes, argument checks) answers without a GPU."""
import ctypes
import os
import re

import pytest

from equivariant_gnn_electronic_b200 import egnn


def _declared(root):
    txt = open(os.path.join(root, "include", "egnn.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(egnn_[a-z_]+)\s*\(", txt)))


def test_every_declared_function_is_exported(root):
    names = _declared(root)
    assert len(names) >= 7
    for n in names:
        assert hasattr(egnn.lib, n), n
    assert set(names) == set(egnn.EXPORTED) | set(n for n in names if n not in egnn.EXPORTED)


def test_wigner_floats_closed_form():
    for lmax in range(7):
        for mmax in range(min(lmax, 2) + 1):
            ref = sum((2 * min(l, mmax) + 1) * (2 * l + 1) for l in range(lmax + 1))
            assert egnn.wigner_floats(lmax, mmax) == ref
    assert egnn.wigner_floats(4, 2) == 115 and egnn.wigner_floats(6, 2) == 235


def test_status_strings():
    for c in range(6):
        assert isinstance(egnn.status_string(c), str) and egnn.status_string(c)


def test_workspace_sizes_grow_with_atoms():
    d = egnn.make_desc(4, 2, 128, 8, 32, 10.0, "bf16")
    a = egnn.workspace_bytes(egnn.EGNN_WS_BUILD_GRAPH, None, 100, 0)
    b = egnn.workspace_bytes(egnn.EGNN_WS_BUILD_GRAPH, None, 10000, 0)
    assert 0 < a < b
    assert egnn.workspace_bytes(egnn.EGNN_WS_HAMILTONIAN, d, 100, 1000) > 0


def test_argument_checks_return_before_any_launch():
    lib = egnn.lib
    g = egnn.GraphStruct()
    box = (ctypes.c_double * 3)(10.0, 10.0, 10.0)
    # null positions
    assert lib.egnn_build_graph(None, None, 10, box, 5.0, 4, 2, ctypes.byref(g), None, 0, None) == \
        egnn.EGNN_ERR_INVALID_ARG
    # unsupported degree
    fake = ctypes.c_void_p(16)
    g.row_ptr = g.status = 16
    assert lib.egnn_build_graph(fake, fake, 10, box, 5.0, 9, 2, ctypes.byref(g), fake, 1 << 20, None) == \
        egnn.EGNN_ERR_UNSUPPORTED
    # null descriptor / unsupported descriptor
    assert lib.egnn_layer_forward(ctypes.byref(g), None, fake, fake, fake, None, 0, None) == \
        egnn.EGNN_ERR_INVALID_ARG
    d = egnn.make_desc(7, 2, 128, 8, 32, 8.0, "bf16")
    assert lib.egnn_layer_forward(ctypes.byref(g), ctypes.byref(d), fake, fake, fake, None, 0, None) == \
        egnn.EGNN_ERR_UNSUPPORTED
    d = egnn.make_desc(4, 2, 100, 8, 32, 8.0, "bf16")          # 100 channels not divisible by 8 heads
    assert lib.egnn_layer_forward(ctypes.byref(g), ctypes.byref(d), fake, fake, fake, None, 0, None) == \
        egnn.EGNN_ERR_UNSUPPORTED
    # graph built for another degree
    d = egnn.make_desc(4, 2, 128, 8, 32, 8.0, "bf16")
    g.n_atoms, g.lmax, g.mmax = 10, 2, 2
    assert lib.egnn_layer_forward(ctypes.byref(g), ctypes.byref(d), fake, fake, fake, None, 0, None) == \
        egnn.EGNN_ERR_INVALID_ARG
    # head: template needing a larger lmax than the layer has
    g.lmax, g.mmax = 2, 2
    d = egnn.make_desc(2, 2, 16, 1, 16, 6.0, "fp32")
    sh = (ctypes.c_int32 * 2)(1, 2)
    ws = 1 << 20
    assert lib.egnn_hamiltonian_blocks(ctypes.byref(g), ctypes.byref(d), fake, sh, 2, fake, fake, fake, ws,
                                       None) == egnn.EGNN_ERR_UNSUPPORTED


def test_profile_record_starts_empty_and_checks_outputs():
    egnn.profile(True)
    egnn.profile(False)
    assert egnn.profile_read() == (0.0, 0, 0)
    assert egnn.lib.egnn_profile_read(None, None, None) == egnn.EGNN_ERR_INVALID_ARG


def test_layer_workspace_stores_no_per_edge_message():
    # fused tensor-core layer: per 128-edge tile two partial-softmax records of
    # L^2 C + 32 floats, and a 4-byte destination index per edge; nothing else grows
    # with the edges once a range of tiles is full
    L, C, H = 5, 128, 8
    d = egnn.make_desc(4, 2, C, H, 32, 8.0, "bf16")
    e1, e2 = 4096 * 128 * 4, 4096 * 128 * 8          # both beyond one full range of tiles
    w1 = egnn.workspace_bytes(egnn.EGNN_WS_LAYER, d, 1000, e1)
    w2 = egnn.workspace_bytes(egnn.EGNN_WS_LAYER, d, 1000, e2)
    per_edge = (w2 - w1) / (e2 - e1)
    assert abs(per_edge - (2 * 4 * (L * L * C + 32) / 128 + 4)) < 0.01
    # per atom: one fp32 accumulator of L^2 C values
    a1 = egnn.workspace_bytes(egnn.EGNN_WS_LAYER, d, 10_000, e1)
    a2 = egnn.workspace_bytes(egnn.EGNN_WS_LAYER, d, 20_000, e1)
    assert abs((a2 - a1) / 10_000 - 4 * L * L * C) < 1.0


def test_head_workspace_grows_by_the_message_record_per_edge():
    # tensor-core head: per edge only the y record (y0 fp32, |m| > 0 bf16)
    L, C, H = 5, 128, 8
    d = egnn.make_desc(4, 2, C, H, 32, 8.0, "bf16")
    rec = 4 * L * C + 4 * C * ((L - 1) + (L - 2))
    e1, e2 = 4096 * 128 * 4, 4096 * 128 * 8
    w1 = egnn.workspace_bytes(egnn.EGNN_WS_HAMILTONIAN, d, 1000, e1)
    w2 = egnn.workspace_bytes(egnn.EGNN_WS_HAMILTONIAN, d, 1000, e2)
    per_edge = (w2 - w1) / (e2 - e1)
    assert abs(per_edge - rec) < 1.0
