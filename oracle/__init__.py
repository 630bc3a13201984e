"""CPU oracle for CommunityKV decode and the prefill top-kappa graph.

TEST INFRASTRUCTURE ONLY.  This package wraps the plain single-threaded C
oracle in ``ckv_oracle.c`` (built with gcc, no FMA contraction).  Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import it; the CUDA library never does and shares no code with it.

Source: "CommunityKV: Efficient Long-Context Decoding via Graph
Partitioning" -- abstract, Figure 1 caption steps (1)-(3), Table 1.  The C
source states, per function, the passage it follows and the reading taken
where the pages are silent.

Parity pins: every oracle function is checked in tests/test_oracle_*.py
against brute force on tiny inputs, closed forms, library routines
(torch softmax/SDPA, numpy sorts and means) or hand-derived fixtures in
tests/golden/.  No function here is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ckv_oracle.c")
_SRC2 = os.path.join(_HERE, "leiden_oracle.c")
_HDR = os.path.join(_HERE, "ckv_oracle.h")
_LIB = os.path.join(_HERE, "libckv_oracle.so")

F32, BF16 = 0, 1
KMAX = 64


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/libckv_oracle.so (gcc, -O2, no FMA)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_SRC2), os.path.getmtime(_HDR))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
            "-fPIC", "-shared", "-Wall", "-Wextra", "-o", tmp, _SRC, _SRC2, "-lm",
        ])
        os.replace(tmp, _LIB)
    return _LIB


class StepInfo(ctypes.Structure):
    _fields_ = [
        ("C", ctypes.c_int32),
        ("T", ctypes.c_int32),
        ("cut_gap_lo", ctypes.c_float),
        ("cut_gap_hi", ctypes.c_float),
        ("n_edges", ctypes.c_int32),
        ("edge_col", ctypes.c_int32 * KMAX),
        ("edge_w", ctypes.c_float * KMAX),
        ("edge_comm", ctypes.c_int32 * KMAX),
        ("edge_gap", ctypes.c_float),
        ("assigned", ctypes.c_int32),
        ("vote_gap", ctypes.c_double),
        ("m", ctypes.c_double * KMAX),
        ("l", ctypes.c_double * KMAX),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int, ctypes.c_int64
        L.ckvo_graph_new.restype = P
        L.ckvo_graph_new.argtypes = [i32, i32, i32]
        L.ckvo_graph_free.argtypes = [P]
        L.ckvo_graph_ntok.argtypes = [P]
        L.ckvo_init.argtypes = [P, i32, i32, P, P, i32]
        L.ckvo_get_centroids.argtypes = [P, P]
        L.ckvo_get_sizes.argtypes = [P, P]
        L.ckvo_get_members.argtypes = [P, P]
        L.ckvo_set_state.argtypes = [P, i32, P, P, P]
        L.ckvo_score.argtypes = [P, i32, P, i32, P]
        L.ckvo_select.argtypes = [i32, P, P, i32, P, P, P]
        L.ckvo_attend.argtypes = [i32, i32, P, i32, P, P, i32, P, i32, P, P, P, P]
        L.ckvo_topk.argtypes = [i32, P, P, i32, P, P]
        L.ckvo_vote.argtypes = [i32, P, P, P]
        L.ckvo_update.argtypes = [P, i32, i32, P, i32]
        L.ckvo_decode_step.argtypes = [P, i32, i32, i32, i32, i32, P, P, P, i32, P, P,
                                       ctypes.POINTER(StepInfo)]
        L.ckvo_row_ptr.restype = i64
        L.ckvo_row_ptr.argtypes = [i64, i32, i32]
        L.ckvo_prefill_rows_grouped.argtypes = [i32, i32, i32, i32, i32, P, P, i32, P, i32, P, P, P, P]
        L.ckvo_leiden.restype = i32
        L.ckvo_leiden.argtypes = [i32, P, P, P, ctypes.c_double, i32, P]
        L.ckvo_modularity.restype = ctypes.c_double
        L.ckvo_modularity.argtypes = [i32, P, P, P, P, ctypes.c_double]
        L.ckvo_dense_stats.argtypes = [i32, i32, P, i32, P, i32, i32, P, P]
        L.ckvo_prefill_rows.argtypes = [i32, i32, i32, i32, P, P, i32, P, i32, P, P, P, P]
        _lib = L
    return _lib


def _p(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16          # bfloat16 stored as its raw 16 bits
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"oracle takes float32 or bfloat16-as-uint16, got {a.dtype}")


# ---------------------------------------------------------------- pieces
def score(graph: "Graph", q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q)
    s = np.empty(graph.n_comm, np.float32)
    lib().ckvo_score(graph.h, q.shape[0], _p(q), _dtype_code(q), _p(s))
    return s


def select(s: np.ndarray, size: np.ndarray, budget: int):
    s = np.ascontiguousarray(s, np.float32)
    size = np.ascontiguousarray(size, np.int32)
    sel = np.empty(max(1, len(s)), np.int32)
    lo, hi = ctypes.c_float(), ctypes.c_float()
    C = lib().ckvo_select(len(s), _p(s), _p(size), budget, _p(sel),
                          ctypes.byref(lo), ctypes.byref(hi))
    return sel[:C].copy(), lo.value, hi.value


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, rows: np.ndarray):
    """Exact attention of q [H][D] over rows of K, V ([n][D]).  Returns
    (out [H][D] float32, p [H][R] float64, m [H], l [H])."""
    q = np.ascontiguousarray(q)
    rows = np.ascontiguousarray(rows, np.int32)
    H, D = q.shape
    R = len(rows)
    out = np.empty((H, D), np.float32)
    p = np.empty((H, max(R, 1)), np.float64)
    m = np.empty(H, np.float64)
    l = np.empty(H, np.float64)
    lib().ckvo_attend(H, D, _p(q), _dtype_code(q), _p(K), _p(V), _dtype_code(K),
                      _p(rows), R, _p(out), _p(p), _p(m), _p(l))
    return out, p[:, :R], m, l


def topk(w: np.ndarray, tok: np.ndarray, kappa: int):
    w = np.ascontiguousarray(w, np.float32)
    tok = np.ascontiguousarray(tok, np.int32)
    idx = np.empty(max(kappa, 1), np.int32)
    gap = ctypes.c_float()
    E = lib().ckvo_topk(len(w), _p(w), _p(tok), kappa, _p(idx), ctypes.byref(gap))
    return idx[:E].copy(), gap.value


def vote(edge_comm, edge_w):
    edge_comm = np.ascontiguousarray(edge_comm, np.int32)
    edge_w = np.ascontiguousarray(edge_w, np.float32)
    gap = ctypes.c_double()
    c = lib().ckvo_vote(len(edge_comm), _p(edge_comm), _p(edge_w), ctypes.byref(gap))
    return c, gap.value


def row_ptr(i: int, n_sinks: int, kappa: int) -> int:
    return lib().ckvo_row_ptr(i, n_sinks, kappa)


def prefill_rows(Q: np.ndarray, K: np.ndarray, rows, n_sinks: int, kappa: int):
    """Prefill top-kappa edges for the listed rows of one head (Q, K [n][D]).
    Returns (col [R][kappa], w [R][kappa], deg [R], gap [R])."""
    Q = np.ascontiguousarray(Q)
    K = np.ascontiguousarray(K)
    rows = np.ascontiguousarray(rows, np.int32)
    n, D = Q.shape
    R = len(rows)
    col = np.full((R, kappa), -1, np.int32)
    w = np.zeros((R, kappa), np.float32)
    deg = np.empty(R, np.int32)
    gap = np.empty(R, np.float32)
    lib().ckvo_prefill_rows(n, D, n_sinks, kappa, _p(Q), _p(K), _dtype_code(Q),
                            _p(rows), R, _p(col), _p(w), _p(deg), _p(gap))
    return col, w, deg, gap


def prefill_rows_grouped(Q: np.ndarray, K: np.ndarray, rows, n_sinks: int, kappa: int):
    """Query-group aggregated prefill rows: Q [nh][n][D] (the group's heads),
    K [n][D].  Returns (col [R][kappa], w [R][kappa], deg [R], gap [R])."""
    Q = np.ascontiguousarray(Q)
    K = np.ascontiguousarray(K)
    rows = np.ascontiguousarray(rows, np.int32)
    nh, n, D = Q.shape
    R = len(rows)
    col = np.full((R, kappa), -1, np.int32)
    w = np.zeros((R, kappa), np.float32)
    deg = np.empty(R, np.int32)
    gap = np.empty(R, np.float32)
    lib().ckvo_prefill_rows_grouped(n, D, n_sinks, kappa, nh, _p(Q), _p(K), _dtype_code(Q),
                                    _p(rows), R, _p(col), _p(w), _p(deg), _p(gap))
    return col, w, deg, gap


def leiden(row_ptr, col, w, n: int, gamma: float = 1.0, max_levels: int = 64):
    """Leiden partition (deterministic variant of leiden_oracle.c) of the
    directed top-kappa CSR read as an undirected graph: (labels [n], C)."""
    row_ptr = np.ascontiguousarray(row_ptr, np.int64)
    col = np.ascontiguousarray(col, np.int32)
    w = np.ascontiguousarray(w, np.float32)
    labels = np.empty(max(n, 1), np.int32)
    C = lib().ckvo_leiden(n, _p(row_ptr), _p(col), _p(w), float(gamma), max_levels, _p(labels))
    return labels[:n].copy(), C


def modularity(row_ptr, col, w, labels, gamma: float = 1.0) -> float:
    row_ptr = np.ascontiguousarray(row_ptr, np.int64)
    col = np.ascontiguousarray(col, np.int32)
    w = np.ascontiguousarray(w, np.float32)
    labels = np.ascontiguousarray(labels, np.int32)
    return lib().ckvo_modularity(len(row_ptr) - 1, _p(row_ptr), _p(col), _p(w), _p(labels), float(gamma))


# ---------------------------------------------------------------- state
class Graph:
    """One graph's community state (centroids, sizes, ascending members)."""

    def __init__(self, n_comm: int, head_dim: int, n_max: int):
        self.n_comm, self.D, self.n_max = n_comm, head_dim, n_max
        self.h = lib().ckvo_graph_new(n_comm, head_dim, n_max)
        if not self.h:
            raise ValueError("bad oracle graph dimensions")

    def __del__(self):
        h = getattr(self, "h", None)
        if h and _lib is not None:
            _lib.ckvo_graph_free(h)
            self.h = None

    @property
    def ntok(self) -> int:
        return lib().ckvo_graph_ntok(self.h)

    def init(self, n: int, n_sinks: int, labels: np.ndarray, K: np.ndarray):
        labels = np.ascontiguousarray(labels, np.int32)
        rc = lib().ckvo_init(self.h, n, n_sinks, _p(labels), _p(K), _dtype_code(K))
        if rc != 0:
            raise ValueError("oracle init rejected the labels or n")

    def centroids(self) -> np.ndarray:
        mu = np.empty((self.n_comm, self.D), np.float32)
        lib().ckvo_get_centroids(self.h, _p(mu))
        return mu

    def sizes(self) -> np.ndarray:
        s = np.empty(self.n_comm, np.int32)
        lib().ckvo_get_sizes(self.h, _p(s))
        return s

    def members(self) -> np.ndarray:
        out = np.empty(max(1, self.n_max), np.int32)
        k = lib().ckvo_get_members(self.h, _p(out))
        return out[:k].copy()

    def set_state(self, n_tok: int, mu: np.ndarray, size: np.ndarray, members: np.ndarray):
        mu = np.ascontiguousarray(mu, np.float32)
        size = np.ascontiguousarray(size, np.int32)
        members = np.ascontiguousarray(members, np.int32)
        if lib().ckvo_set_state(self.h, n_tok, _p(mu), _p(size), _p(members)) != 0:
            raise ValueError("bad oracle state")

    def update(self, c: int, t: int, k_t: np.ndarray):
        k_t = np.ascontiguousarray(k_t)
        if lib().ckvo_update(self.h, c, t, _p(k_t), _dtype_code(k_t)) != 0:
            raise ValueError("bad community id")


def dense_stats(q: np.ndarray, K: np.ndarray, n: int):
    """Dense softmax statistics of q [H][D] over rows [0, n) of K: (m [H], l [H])."""
    q = np.ascontiguousarray(q)
    H, D = q.shape
    m = np.empty(H, np.float64)
    l = np.empty(H, np.float64)
    lib().ckvo_dense_stats(H, D, _p(q), _dtype_code(q), _p(np.ascontiguousarray(K)), _dtype_code(K), n,
                           _p(m), _p(l))
    return m, l


def recall(m_sel, l_sel, m_den, l_den):
    """Attention-mass recall per head: the dense softmax mass of the attended
    rows, l_sel * exp(m_sel - m_den) / l_den (Figure 3 right, reading in
    ckv_oracle.c)."""
    m_sel, l_sel, m_den, l_den = (np.asarray(x, np.float64) for x in (m_sel, l_sel, m_den, l_den))
    return l_sel * np.exp(m_sel - m_den) / l_den


@dataclass
class StepResult:
    out: np.ndarray          # [H][D] float32
    sel: np.ndarray          # selected community ids, selection order
    C: int
    T: int
    cut_gap_lo: float
    cut_gap_hi: float
    edge_col: np.ndarray
    edge_w: np.ndarray
    edge_comm: np.ndarray
    edge_gap: float
    assigned: int
    vote_gap: float
    m: np.ndarray
    l: np.ndarray


def decode_step(graph: Graph, q: np.ndarray, K: np.ndarray, V: np.ndarray, n: int,
                n_sinks: int, kappa: int, budget: int) -> StepResult:
    """One decode step of one graph (q [H][D]; K, V [>=n][D] of its KV head)."""
    q = np.ascontiguousarray(q)
    H, D = q.shape
    out = np.empty((H, D), np.float32)
    sel = np.empty(max(1, graph.n_comm), np.int32)
    info = StepInfo()
    rc = lib().ckvo_decode_step(graph.h, H, n_sinks, kappa, budget, n, _p(q), _p(K), _p(V),
                                _dtype_code(K), _p(out), _p(sel), ctypes.byref(info))
    if rc != 0:
        raise ValueError(f"oracle decode_step rejected n={n} (ntok={graph.ntok})")
    E = info.n_edges
    return StepResult(
        out=out, sel=sel[:info.C].copy(), C=info.C, T=info.T,
        cut_gap_lo=info.cut_gap_lo, cut_gap_hi=info.cut_gap_hi,
        edge_col=np.array(info.edge_col[:E], np.int32),
        edge_w=np.array(info.edge_w[:E], np.float32),
        edge_comm=np.array(info.edge_comm[:E], np.int32),
        edge_gap=info.edge_gap, assigned=info.assigned, vote_gap=info.vote_gap,
        m=np.array(info.m[:H]), l=np.array(info.l[:H]))
