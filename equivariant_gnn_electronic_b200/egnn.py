"""Thin ctypes binding of libegnn.so (include/egnn.h).

Argument marshalling only: torch tensors supply device memory and the CUDA
stream; every step of the computation runs in the library's kernels.  If the
shared library is missing the import fails loudly -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libegnn.so")

EGNN_OK, EGNN_ERR_INVALID_ARG, EGNN_ERR_CAPACITY, EGNN_ERR_UNSUPPORTED, EGNN_ERR_CUDA, \
    EGNN_ERR_DEVICE_CHECK = range(6)
EGNN_FP32, EGNN_BF16 = 0, 1
EGNN_WS_BUILD_GRAPH, EGNN_WS_LAYER, EGNN_WS_HAMILTONIAN, EGNN_WS_LABELS, EGNN_WS_ASSEMBLY = 0, 1, 2, 3, 4

EXPORTED = (
    "egnn_wigner_floats", "egnn_workspace_bytes", "egnn_build_graph", "egnn_layer_forward",
    "egnn_hamiltonian_blocks", "egnn_read_status", "egnn_status_string", "egnn_build_graph_noalloc",
    "egnn_profile", "egnn_profile_read", "egnn_edge_geometry", "egnn_check_bounded_wait",
    "egnn_label_count", "egnn_blocks_to_labels", "egnn_labels_to_blocks", "egnn_assemble_hamiltonian",
)
EGNN_DEV_BAD_POSITION, EGNN_DEV_SEGMENT_TOO_LARGE, EGNN_DEV_INDEX_RANGE, EGNN_DEV_COUNT_MISMATCH, \
    EGNN_DEV_EDGE_OVERFLOW, EGNN_DEV_WAIT_TIMEOUT, EGNN_DEV_BAD_GRAPH = range(1, 8)


class LayerDesc(ctypes.Structure):
    _fields_ = [("lmax", ctypes.c_int32), ("mmax", ctypes.c_int32), ("channels", ctypes.c_int32),
                ("heads", ctypes.c_int32), ("n_rbf", ctypes.c_int32), ("rcut", ctypes.c_float),
                ("dtype", ctypes.c_int32)]


class GraphStruct(ctypes.Structure):
    _fields_ = [("n_atoms", ctypes.c_int32), ("lmax", ctypes.c_int32), ("mmax", ctypes.c_int32),
                ("capacity", ctypes.c_int64), ("n_edges", ctypes.c_int64),
                ("row_ptr", ctypes.c_void_p), ("src", ctypes.c_void_p), ("shift", ctypes.c_void_p),
                ("dist", ctypes.c_void_p), ("wigner", ctypes.c_void_p), ("status", ctypes.c_void_p)]


class EgnnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {status_string(code)} (code {code})")
        self.code = code


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libegnn.so not built at {_LIB_PATH}; run __graft_entry__.build()")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    lib.egnn_wigner_floats.argtypes = [i32, i32]
    lib.egnn_wigner_floats.restype = i32
    lib.egnn_workspace_bytes.argtypes = [i32, ctypes.POINTER(LayerDesc), i32, i64]
    lib.egnn_workspace_bytes.restype = sz
    lib.egnn_build_graph.argtypes = [vp, vp, i32, ctypes.POINTER(ctypes.c_double), ctypes.c_double,
                                     i32, i32, ctypes.POINTER(GraphStruct), vp, sz, vp]
    lib.egnn_build_graph.restype = i32
    lib.egnn_build_graph_noalloc.argtypes = [vp, vp, i32, ctypes.POINTER(ctypes.c_double), ctypes.c_double,
                                             i32, i32, ctypes.POINTER(GraphStruct), vp]
    lib.egnn_build_graph_noalloc.restype = i32
    lib.egnn_layer_forward.argtypes = [ctypes.POINTER(GraphStruct), ctypes.POINTER(LayerDesc), vp, vp,
                                       vp, vp, sz, vp]
    lib.egnn_layer_forward.restype = i32
    lib.egnn_hamiltonian_blocks.argtypes = [ctypes.POINTER(GraphStruct), ctypes.POINTER(LayerDesc), vp,
                                            ctypes.POINTER(i32), i32, vp, vp, vp, sz, vp]
    lib.egnn_hamiltonian_blocks.restype = i32
    lib.egnn_read_status.argtypes = [ctypes.POINTER(GraphStruct), ctypes.POINTER(i32), vp]
    lib.egnn_read_status.restype = i32
    lib.egnn_status_string.argtypes = [i32]
    lib.egnn_status_string.restype = ctypes.c_char_p
    lib.egnn_edge_geometry.argtypes = [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(GraphStruct), vp]
    lib.egnn_edge_geometry.restype = i32
    lib.egnn_check_bounded_wait.argtypes = [ctypes.POINTER(GraphStruct), ctypes.c_uint32, vp]
    lib.egnn_check_bounded_wait.restype = i32
    lib.egnn_label_count.argtypes = [ctypes.POINTER(i32), i32]
    lib.egnn_label_count.restype = i32
    for name in ("egnn_blocks_to_labels", "egnn_labels_to_blocks"):
        getattr(lib, name).argtypes = [vp, i64, ctypes.POINTER(i32), i32, vp, vp, sz, vp]
        getattr(lib, name).restype = i32
    lib.egnn_assemble_hamiltonian.argtypes = [ctypes.POINTER(GraphStruct), vp, vp, i32, vp, vp, vp, i64, vp, sz, vp]
    lib.egnn_assemble_hamiltonian.restype = i32
    lib.egnn_profile.argtypes = [i32]
    lib.egnn_profile.restype = i32
    lib.egnn_profile_read.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64), ctypes.POINTER(i64)]
    lib.egnn_profile_read.restype = i32
    return lib


lib = _load()


def status_string(code: int) -> str:
    return lib.egnn_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != EGNN_OK:
        raise EgnnError(code, where)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def profile(enable: bool) -> None:
    """Start (clearing the record) or stop timing the fused-kernel launches of layer calls."""
    _check(lib.egnn_profile(1 if enable else 0), "egnn_profile")


def profile_read() -> tuple[float, int, int]:
    """(summed fused-kernel launch milliseconds, launches, edges processed) of the record."""
    ms, n, e = ctypes.c_double(0.0), ctypes.c_int64(0), ctypes.c_int64(0)
    _check(lib.egnn_profile_read(ctypes.byref(ms), ctypes.byref(n), ctypes.byref(e)), "egnn_profile_read")
    return ms.value, n.value, e.value


def wigner_floats(lmax: int, mmax: int) -> int:
    return int(lib.egnn_wigner_floats(lmax, mmax))


def make_desc(lmax, mmax, channels, heads, n_rbf, rcut, dtype) -> LayerDesc:
    dt = dtype if isinstance(dtype, int) else (EGNN_BF16 if dtype in ("bf16", torch.bfloat16) else EGNN_FP32)
    return LayerDesc(lmax, mmax, channels, heads, n_rbf, float(rcut), dt)


def desc_for(w) -> LayerDesc:
    """LayerDesc of a synth.Workload-like object."""
    return make_desc(w.lmax, w.mmax, w.channels, w.heads, w.n_rbf, w.rcut, w.dtype)


def torch_dtype(desc: LayerDesc):
    return torch.bfloat16 if desc.dtype == EGNN_BF16 else torch.float32


def workspace_bytes(which: int, desc: Optional[LayerDesc], n_atoms: int, n_edges: int) -> int:
    return int(lib.egnn_workspace_bytes(which, ctypes.byref(desc) if desc is not None else None,
                                        n_atoms, n_edges))


class Graph:
    """Device-resident destination-CSR graph (owns its torch tensors)."""

    def __init__(self, n_atoms: int, capacity: int, lmax: int, mmax: int, device):
        self.device = torch.device(device)
        self.lmax, self.mmax = lmax, mmax
        self.row_ptr = torch.zeros(n_atoms + 1, dtype=torch.int32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self._alloc(capacity)
        self.s = GraphStruct()
        self.s.n_atoms = n_atoms
        self.s.lmax, self.s.mmax = lmax, mmax
        self._sync_struct()

    def _alloc(self, capacity: int):
        cap = max(int(capacity), 1)
        dev = self.device
        self.capacity = cap
        self.src = torch.zeros(cap, dtype=torch.int32, device=dev)
        self.shift = torch.zeros(cap, 3, dtype=torch.int8, device=dev)
        self.dist = torch.zeros(cap, dtype=torch.float32, device=dev)
        self.wigner = torch.zeros(cap, wigner_floats(self.lmax, self.mmax), dtype=torch.float32, device=dev)

    def _sync_struct(self):
        s = self.s
        s.capacity = self.capacity
        s.row_ptr, s.src, s.shift = self.row_ptr.data_ptr(), self.src.data_ptr(), self.shift.data_ptr()
        s.dist, s.wigner, s.status = self.dist.data_ptr(), self.wigner.data_ptr(), self.status.data_ptr()

    @property
    def n_atoms(self) -> int:
        return int(self.s.n_atoms)

    @property
    def n_edges(self) -> int:
        return int(self.s.n_edges)

    def read_status(self, stream=None) -> int:
        code = ctypes.c_int32(0)
        lib.egnn_read_status(ctypes.byref(self.s), ctypes.byref(code), _stream(stream))
        return int(code.value)


def build_graph(pos: torch.Tensor, species: torch.Tensor, box: Sequence[float], rcut: float,
                lmax: int, mmax: int, capacity: Optional[int] = None, workspace: Optional[torch.Tensor] = None,
                graph: Optional[Graph] = None, stream=None) -> Graph:
    """Neighbour list + Wigner rows.  Grows the edge arrays and retries on EGNN_ERR_CAPACITY."""
    assert pos.dtype == torch.float64 and pos.is_cuda and pos.is_contiguous()
    assert species.dtype == torch.int32 and species.is_cuda
    n = pos.shape[0]
    if graph is None:
        cap = capacity if capacity is not None else 64 * n
        graph = Graph(n, cap, lmax, mmax, pos.device)
    need = workspace_bytes(EGNN_WS_BUILD_GRAPH, None, n, 0)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=pos.device)
    boxarr = (ctypes.c_double * 3)(*[float(b) for b in box])
    for _ in range(2):
        code = lib.egnn_build_graph(_ptr(pos), _ptr(species), n, boxarr, float(rcut), lmax, mmax,
                                    ctypes.byref(graph.s), _ptr(workspace), workspace.numel(),
                                    _stream(stream))
        if code == EGNN_ERR_CAPACITY:
            graph._alloc(int(graph.s.n_edges))
            graph._sync_struct()
            continue
        _check(code, "egnn_build_graph")
        return graph
    raise EgnnError(EGNN_ERR_CAPACITY, "egnn_build_graph")


def build_graph_noalloc(pos: torch.Tensor, species: torch.Tensor, box: Sequence[float], rcut: float,
                        lmax: int, mmax: int, graph: Graph, stream=None) -> int:
    """egnn_build_graph_noalloc into an existing Graph (no workspace); returns the status code."""
    assert pos.dtype == torch.float64 and pos.is_cuda and pos.is_contiguous()
    boxarr = (ctypes.c_double * 3)(*[float(b) for b in box])
    return int(lib.egnn_build_graph_noalloc(_ptr(pos), _ptr(species), pos.shape[0], boxarr, float(rcut),
                                            lmax, mmax, ctypes.byref(graph.s), _stream(stream)))


def edge_geometry(pos: torch.Tensor, box: Sequence[float], graph: Graph, stream=None) -> Graph:
    """Distances and Wigner rows of graph's edges for new positions (same neighbour list)."""
    assert pos.dtype == torch.float64 and pos.is_cuda and pos.is_contiguous()
    boxarr = (ctypes.c_double * 3)(*[float(b) for b in box])
    _check(lib.egnn_edge_geometry(_ptr(pos), boxarr, ctypes.byref(graph.s), _stream(stream)), "egnn_edge_geometry")
    return graph


def check_bounded_wait(graph: Graph, limit_us: int, stream=None) -> None:
    """Run the pipelined kernels' bounded wait on an mbarrier nothing arrives on."""
    _check(lib.egnn_check_bounded_wait(ctypes.byref(graph.s), int(limit_us), _stream(stream)),
           "egnn_check_bounded_wait")


def label_count(shells: Sequence[int]) -> int:
    sh = (ctypes.c_int32 * len(shells))(*shells)
    return int(lib.egnn_label_count(sh, len(shells)))


def _template_call(name, x: torch.Tensor, n: int, shells: Sequence[int], out: torch.Tensor, stream):
    ws = torch.empty(workspace_bytes(EGNN_WS_LABELS, None, 0, 0), dtype=torch.uint8, device=x.device)
    sh = (ctypes.c_int32 * len(shells))(*shells)
    _check(getattr(lib, name)(_ptr(x), n, sh, len(shells), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), name)
    return out


def blocks_to_labels(blocks: torch.Tensor, shells: Sequence[int], stream=None) -> torch.Tensor:
    """Matrix -> Label: [n, n_orb, n_orb] fp32 -> [n, n_lab] fp32."""
    assert blocks.dtype == torch.float32 and blocks.is_contiguous()
    out = torch.empty(blocks.shape[0], label_count(shells), dtype=torch.float32, device=blocks.device)
    return _template_call("egnn_blocks_to_labels", blocks, blocks.shape[0], shells, out, stream)


def labels_to_blocks(labels: torch.Tensor, shells: Sequence[int], stream=None) -> torch.Tensor:
    """Label -> Matrix: [n, n_lab] fp32 -> [n, n_orb, n_orb] fp32."""
    assert labels.dtype == torch.float32 and labels.is_contiguous()
    n_orb = sum(2 * l + 1 for l in shells)
    out = torch.empty(labels.shape[0], n_orb, n_orb, dtype=torch.float32, device=labels.device)
    return _template_call("egnn_labels_to_blocks", labels, labels.shape[0], shells, out, stream)


def assemble_hamiltonian(graph: Graph, onsite: torch.Tensor, edge_blocks: torch.Tensor, stream=None):
    """k = 0 Hamiltonian as block-sparse rows: (bsr_row_ptr [N+1], bsr_col [nnzb],
    bsr_val [nnzb, n_orb, n_orb]) with the arrays sized for N + E blocks (trim by
    bsr_row_ptr[N])."""
    n, n_orb = graph.n_atoms, onsite.shape[1]
    cap = n + graph.n_edges
    dev = onsite.device
    row_ptr = torch.empty(n + 1, dtype=torch.int32, device=dev)
    col = torch.empty(cap, dtype=torch.int32, device=dev)
    val = torch.empty(cap, n_orb, n_orb, dtype=torch.float32, device=dev)
    ws = torch.empty(workspace_bytes(EGNN_WS_ASSEMBLY, None, n, 0), dtype=torch.uint8, device=dev)
    _check(lib.egnn_assemble_hamiltonian(ctypes.byref(graph.s), _ptr(onsite), _ptr(edge_blocks), n_orb,
                                         _ptr(row_ptr), _ptr(col), _ptr(val), cap, _ptr(ws), ws.numel(),
                                         _stream(stream)), "egnn_assemble_hamiltonian")
    return row_ptr, col, val


def layer_forward(graph: Graph, desc: LayerDesc, weights: torch.Tensor, node_in: torch.Tensor,
                  node_out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  stream=None) -> torch.Tensor:
    if node_out is None:
        node_out = torch.empty_like(node_in)
    assert node_in.is_contiguous() and node_out.is_contiguous() and weights.is_contiguous()
    assert node_in.dtype == torch_dtype(desc) and weights.dtype == torch_dtype(desc)
    need = workspace_bytes(EGNN_WS_LAYER, desc, graph.n_atoms, graph.n_edges)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=node_in.device)
    code = lib.egnn_layer_forward(ctypes.byref(graph.s), ctypes.byref(desc), _ptr(weights), _ptr(node_in),
                                  _ptr(node_out), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(code, "egnn_layer_forward")
    return node_out


def hamiltonian_blocks(graph: Graph, desc: LayerDesc, head_weights: torch.Tensor, shells: Sequence[int],
                       node_emb: torch.Tensor, blocks: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    n_orb = sum(2 * l + 1 for l in shells)
    if blocks is None:
        blocks = torch.empty(graph.n_edges, n_orb, n_orb, dtype=torch.float32, device=node_emb.device)
    need = workspace_bytes(EGNN_WS_HAMILTONIAN, desc, graph.n_atoms, graph.n_edges)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=node_emb.device)
    sh = (ctypes.c_int32 * len(shells))(*shells)
    code = lib.egnn_hamiltonian_blocks(ctypes.byref(graph.s), ctypes.byref(desc), _ptr(head_weights), sh,
                                       len(shells), _ptr(node_emb), _ptr(blocks), _ptr(workspace),
                                       workspace.numel(), _stream(stream))
    _check(code, "egnn_hamiltonian_blocks")
    return blocks


# ---- weight packing (order of egnn.h; marshalling only) ----

def layer_weight_keys(mmax: int, attention: bool = True):
    keys = ["W1", "b1", "W2", "b2", "W0"]
    for m in range(1, mmax + 1):
        keys += [f"W{m}_1", f"W{m}_2"]
    if attention:
        keys += ["A", "bA"]
    return keys


def pack_weights(W: Dict[str, np.ndarray], desc: LayerDesc, attention: bool = True,
                 device="cuda") -> torch.Tensor:
    keys = layer_weight_keys(desc.mmax, attention)
    if not attention:
        keys += [f"U{L}" for L in range(desc.lmax + 1) if f"U{L}" in W]
    flat = np.concatenate([np.asarray(W[k], dtype=np.float64).ravel() for k in keys])
    t = torch.from_numpy(flat.astype(np.float32))
    return t.to(torch_dtype(desc)).to(device).contiguous()
