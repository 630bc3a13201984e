"""Python binding of libckv: CommunityKV community-retrieval sparse decode
attention for B200 (sm_100a).

Argument marshalling only: every function below calls the C entry point of
the same name in libckv.so (declared in include/ckv.h), passing device
pointers of torch tensors and the raw CUDA stream.  A device argument must be
a CUDA tensor (or a raw int address) and a host argument a numpy array or CPU
tensor; the wrong kind raises TypeError before the call.  No step of the
method runs in Python.  If the compiled library is missing, the first call raises
``RuntimeError`` -- there is no fallback.

Method: "CommunityKV: Efficient Long-Context Decoding via Graph
Partitioning" (Figure 1: graph construction, initial partitioning,
incremental update).
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
# CKV_DEBUG_BOUNDS=1 in the environment selects the range-checked build
DEBUG_BOUNDS = os.environ.get("CKV_DEBUG_BOUNDS") == "1"
LIB_PATH = os.path.join(HERE, "libckv_debug.so" if DEBUG_BOUNDS else "libckv.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "ckv.h")
HEADER_DEBUG = os.path.join(os.path.dirname(HERE), "include", "ckv_debug.h")

CKV_OK, CKV_ERR_INVALID_ARG, CKV_ERR_CAPACITY, CKV_ERR_OOM = 0, 1, 2, 3
CKV_ERR_CUDA, CKV_ERR_TIMEOUT, CKV_ERR_STATE = 4, 5, 6
CKV_F32, CKV_BF16 = 0, 1
CKV_PER_HEAD, CKV_QUERY_GROUP = 0, 1


class ckv_config(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int) for name in (
        "batch", "n_q_heads", "n_kv_heads", "head_dim", "n_max", "max_communities",
        "n_sinks", "kappa", "budget", "slack", "kv_dtype", "mode", "device", "pool_capacity")]


class CkvError(RuntimeError):
    def __init__(self, call: str, status: int):
        self.status = status
        super().__init__(f"{call} failed: {status_string(status)} ({status})")


_lib = None


def declared_functions(header: str = HEADER):
    """Names of every function declared in a header (default include/ckv.h)."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ckv_[a-z_0-9]+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{os.path.basename(LIB_PATH)} is not built ({LIB_PATH}); run __graft_entry__.build()")
    L = ctypes.CDLL(LIB_PATH)
    P, I, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_int
    sz = ctypes.c_size_t
    L.ckv_graph_count.restype = I
    L.ckv_graph_count.argtypes = [ctypes.POINTER(ckv_config)]
    L.ckv_create.restype = st
    L.ckv_create.argtypes = [ctypes.POINTER(ckv_config), ctypes.POINTER(P)]
    L.ckv_destroy.restype = None
    L.ckv_destroy.argtypes = [P]
    L.ckv_build_graph.restype = st
    L.ckv_build_graph.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P]
    L.ckv_init_communities.restype = st
    L.ckv_init_communities.argtypes = [P, P, I, I, P, I, P]
    L.ckv_decode_step.restype = st
    L.ckv_decode_step.argtypes = [P, P, P, P, I, P, P]
    L.ckv_assign_update.restype = st
    L.ckv_assign_update.argtypes = [P, P, I, P]
    L.ckv_decode_host.restype = st
    L.ckv_decode_host.argtypes = [P, P, P, P, P, P, I, P, P]
    L.ckv_last_error.restype = st
    L.ckv_last_error.argtypes = [P]
    L.ckv_step_launches.restype = I
    L.ckv_step_launches.argtypes = [P]
    L.ckv_set_wait_limit.restype = st
    L.ckv_set_wait_limit.argtypes = [P, ctypes.c_uint]
    L.ckv_get_step_debug.restype = st
    L.ckv_get_step_debug.argtypes = [P, P, P, P, P, P, P, P]
    L.ckv_profile_begin.restype = st
    L.ckv_profile_begin.argtypes = [P]
    L.ckv_profile_end.restype = st
    L.ckv_profile_end.argtypes = [P, P, ctypes.POINTER(ctypes.c_int)]
    L.ckv_export_state.restype = st
    L.ckv_export_state.argtypes = [P, P, ctypes.POINTER(sz)]
    L.ckv_import_state.restype = st
    L.ckv_import_state.argtypes = [P, P, sz]
    L.ckv_aux_bytes.restype = st
    L.ckv_aux_bytes.argtypes = [P, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.ckv_attend_rows_static.restype = st
    L.ckv_attend_rows_static.argtypes = [ctypes.POINTER(ckv_config), P, P, P, I, P, P, I, P, P]
    L.ckv_build_graph_grouped_workspace.restype = sz
    L.ckv_build_graph_grouped_workspace.argtypes = [I, I, I]
    L.ckv_build_graph_grouped.restype = st
    L.ckv_build_graph_grouped.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P, P, P]
    L.ckv_leiden.restype = st
    L.ckv_leiden.argtypes = [I, P, P, P, ctypes.c_double, P, ctypes.POINTER(ctypes.c_int)]
    L.ckv_modularity_workspace.restype = sz
    L.ckv_modularity_workspace.argtypes = [I]
    L.ckv_modularity.restype = st
    L.ckv_modularity.argtypes = [I, P, P, P, P, I, ctypes.c_double, P, ctypes.POINTER(ctypes.c_double), P]
    L.ckv_set_token_graph.restype = st
    L.ckv_set_token_graph.argtypes = [P, P, P, P, I]
    L.ckv_refresh.restype = st
    L.ckv_refresh.argtypes = [P, P, ctypes.c_double, P, P]
    L.ckv_graph_modularity.restype = st
    L.ckv_graph_modularity.argtypes = [P, ctypes.c_double, P, P]
    L.ckv_step_recall.restype = st
    L.ckv_step_recall.argtypes = [P, P, P, I, P, P]
    L.ckv_dense_decode.restype = st
    L.ckv_dense_decode.argtypes = [P, P, P, P, I, P, P, P]
    L.ckv_status_string.restype = ctypes.c_char_p
    L.ckv_status_string.argtypes = [I]
    _lib = L
    return L


def _dev(x) -> int | None:
    """Address of a device-memory argument: a CUDA torch tensor, a raw int
    address (taken as device memory) or None.  Host memory is refused here,
    before the call, since a kernel cannot dereference it."""
    if x is None or isinstance(x, int):
        return x
    if hasattr(x, "is_cuda"):
        if not x.is_cuda:
            raise TypeError("expected device memory (a CUDA tensor), got a CPU tensor")
        return x.data_ptr()
    raise TypeError(f"expected device memory (a CUDA tensor), got {type(x).__name__}")


def _hostp(x) -> int | None:
    """Address of a host-memory argument: a numpy array, a CPU torch tensor,
    a raw int address (taken as host memory) or None.  A CUDA tensor is
    refused."""
    if x is None or isinstance(x, int):
        return x
    if hasattr(x, "is_cuda"):
        if x.is_cuda:
            raise TypeError("expected host memory, got a CUDA tensor")
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    raise TypeError(f"expected host memory (a numpy array or CPU tensor), got {type(x).__name__}")


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(call: str, status: int):
    if status != CKV_OK:
        raise CkvError(call, status)


# ------------------------------------------------------------ entry points
def status_string(status: int) -> str:
    return lib().ckv_status_string(status).decode()


def ckv_status_string(status: int) -> str:
    return status_string(status)


def ckv_graph_count(cfg: ckv_config) -> int:
    return lib().ckv_graph_count(ctypes.byref(cfg))


def ckv_create(cfg: ckv_config) -> int:
    h = ctypes.c_void_p()
    _check("ckv_create", lib().ckv_create(ctypes.byref(cfg), ctypes.byref(h)))
    return h.value


def ckv_destroy(ctx: int) -> None:
    lib().ckv_destroy(ctx)


def ckv_build_graph(n_heads, n, head_dim, n_sinks, kappa, dtype, Q, K, row_ptr, col, w, stream=None):
    _check("ckv_build_graph", lib().ckv_build_graph(
        n_heads, n, head_dim, n_sinks, kappa, dtype, _dev(Q), _dev(K), _dev(row_ptr), _dev(col),
        _dev(w), _stream(stream)))


def ckv_build_graph_grouped_workspace(n_kv_heads, group, n) -> int:
    return lib().ckv_build_graph_grouped_workspace(n_kv_heads, group, n)


def ckv_build_graph_grouped(n_kv_heads, group, n, head_dim, n_sinks, kappa, dtype, Q, K, workspace, row_ptr, col, w,
                            stream=None):
    _check("ckv_build_graph_grouped", lib().ckv_build_graph_grouped(
        n_kv_heads, group, n, head_dim, n_sinks, kappa, dtype, _dev(Q), _dev(K), _dev(workspace), _dev(row_ptr),
        _dev(col), _dev(w), _stream(stream)))


def _host_in(a, dtype):
    """A host array for an input argument: C-contiguous, of exactly `dtype`."""
    import numpy as np
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected a {np.dtype(dtype).name} array, got {a.dtype}")
    return np.ascontiguousarray(a)


def _host_out(a, dtype):
    """A host array the library writes: C-contiguous, writable, exactly `dtype`."""
    import numpy as np
    if not isinstance(a, np.ndarray) or a.dtype != dtype or not a.flags["C_CONTIGUOUS"] or not a.flags["WRITEABLE"]:
        raise TypeError(f"expected a writable C-contiguous {np.dtype(dtype).name} numpy array")
    return a


def ckv_leiden(n, row_ptr_host, col_host, w_host, gamma, labels_host) -> int:
    """Leiden partition on the host (numpy arrays); returns the community count."""
    import numpy as np
    row_ptr_host = _host_in(row_ptr_host, np.int64)
    col_host = _host_in(col_host, np.int32)
    w_host = _host_in(w_host, np.float32)
    labels_host = _host_out(labels_host, np.int32)
    if len(row_ptr_host) < n + 1 or len(labels_host) < n or len(col_host) < row_ptr_host[n] or \
            len(w_host) < row_ptr_host[n]:
        raise ValueError("array shorter than the graph")
    c = ctypes.c_int(0)
    _check("ckv_leiden", lib().ckv_leiden(n, _hostp(row_ptr_host), _hostp(col_host), _hostp(w_host), float(gamma),
                                          _hostp(labels_host), ctypes.byref(c)))
    return c.value


def ckv_modularity_workspace(n_communities) -> int:
    return lib().ckv_modularity_workspace(n_communities)


def ckv_modularity(n, row_ptr, col, w, labels, n_communities, gamma, workspace, stream=None) -> float:
    q = ctypes.c_double(0.0)
    _check("ckv_modularity", lib().ckv_modularity(n, _dev(row_ptr), _dev(col), _dev(w), _dev(labels), n_communities,
                                                  float(gamma), _dev(workspace), ctypes.byref(q), _stream(stream)))
    return q.value


def ckv_set_token_graph(ctx, row_ptr_host, col_host, w_host, n):
    import numpy as np
    row_ptr_host = _host_in(row_ptr_host, np.int64)
    col_host = _host_in(col_host, np.int32)
    w_host = _host_in(w_host, np.float32)
    _check("ckv_set_token_graph", lib().ckv_set_token_graph(ctx, _hostp(row_ptr_host), _hostp(col_host), _hostp(w_host),
                                                            n))


def ckv_refresh(ctx, K, gamma, n_communities_host=None, stream=None):
    import numpy as np
    if n_communities_host is not None:
        n_communities_host = _host_out(n_communities_host, np.int32)
    _check("ckv_refresh", lib().ckv_refresh(ctx, _dev(K), float(gamma), _hostp(n_communities_host), _stream(stream)))


def ckv_graph_modularity(ctx, gamma, q_host, stream=None):
    import numpy as np
    q_host = _host_out(q_host, np.float64)
    _check("ckv_graph_modularity", lib().ckv_graph_modularity(ctx, float(gamma), _hostp(q_host), _stream(stream)))


def ckv_init_communities(ctx, labels, labels_on_device, n_communities, K, n, stream=None):
    _check("ckv_init_communities", lib().ckv_init_communities(
        ctx, (_dev(labels) if labels_on_device else _hostp(labels)), int(labels_on_device), n_communities, _dev(K), n, _stream(stream)))


def ckv_decode_step(ctx, q, K, V, n, out, stream=None):
    _check("ckv_decode_step", lib().ckv_decode_step(ctx, _dev(q), _dev(K), _dev(V), n, _dev(out),
                                                    _stream(stream)))


def ckv_assign_update(ctx, K, n, stream=None):
    _check("ckv_assign_update", lib().ckv_assign_update(ctx, _dev(K), n, _stream(stream)))


def ckv_decode_host(ctx, q_host, k_new_host, v_new_host, K, V, n, out_host, stream=None):
    _check("ckv_decode_host", lib().ckv_decode_host(
        ctx, _hostp(q_host), _hostp(k_new_host), _hostp(v_new_host), _dev(K), _dev(V), n, _hostp(out_host),
        _stream(stream)))


def ckv_last_error(ctx) -> int:
    return lib().ckv_last_error(ctx)


def ckv_step_launches(ctx) -> int:
    return lib().ckv_step_launches(ctx)


def ckv_set_wait_limit(ctx, polls: int):
    _check("ckv_set_wait_limit", lib().ckv_set_wait_limit(ctx, int(polls)))


def ckv_get_step_debug(ctx, n_sel=None, sel=None, n_tok_sel=None, n_edges=None, edges=None,
                       edge_w=None, assigned=None):
    _check("ckv_get_step_debug", lib().ckv_get_step_debug(
        ctx, _hostp(n_sel), _hostp(sel), _hostp(n_tok_sel), _hostp(n_edges), _hostp(edges), _hostp(edge_w),
        _hostp(assigned)))


def ckv_profile_begin(ctx) -> None:
    _check("ckv_profile_begin", lib().ckv_profile_begin(ctx))


def ckv_profile_end(ctx):
    """Summed device milliseconds of (score, select, attend, assign) and the
    number of profiled steps."""
    ms = (ctypes.c_float * 4)()
    steps = ctypes.c_int(0)
    _check("ckv_profile_end", lib().ckv_profile_end(ctx, ms, ctypes.byref(steps)))
    return list(ms), steps.value


def ckv_export_state(ctx) -> bytes:
    n = ctypes.c_size_t(0)
    _check("ckv_export_state", lib().ckv_export_state(ctx, None, ctypes.byref(n)))
    buf = ctypes.create_string_buffer(n.value)
    _check("ckv_export_state", lib().ckv_export_state(ctx, buf, ctypes.byref(n)))
    return buf.raw[:n.value]


def ckv_import_state(ctx, blob: bytes) -> None:
    _check("ckv_import_state", lib().ckv_import_state(ctx, blob, len(blob)))


def ckv_attend_rows_static(cfg, q, K, V, n, rows_host, n_rows_host, max_rows, out, stream=None):
    """Attention over caller-chosen rows with no device allocation (scratch
    in the library's static device array); rows_host / n_rows_host are host
    arrays."""
    _check("ckv_attend_rows_static", lib().ckv_attend_rows_static(
        ctypes.byref(cfg), _dev(q), _dev(K), _dev(V), n, _hostp(rows_host), _hostp(n_rows_host), max_rows,
        _dev(out), _stream(stream)))


def ckv_step_recall(ctx, q, K, n, recall, stream=None):
    """Attention-mass recall [B][H_q] of the last decode step (n), per query head."""
    _check("ckv_step_recall", lib().ckv_step_recall(ctx, _dev(q), _dev(K), n, _dev(recall), _stream(stream)))


def ckv_dense_decode(ctx, q, K, V, n, out, lse=None, stream=None):
    """Dense decode attention over [0, n): out [B][H_q][D], lse [B][H_q] (optional)."""
    _check("ckv_dense_decode", lib().ckv_dense_decode(ctx, _dev(q), _dev(K), _dev(V), n, _dev(out), _dev(lse),
                                                      _stream(stream)))


def ckv_debug_poke(ctx, what: int, g: int, c: int, r: int, value: int):
    """Overwrite one int32 of the device community state (range-checked
    build only): what 0 = member r of community c, 1 = community c's segment
    offset."""
    L = lib()
    if not hasattr(L, "ckv_debug_poke"):
        raise RuntimeError("ckv_debug_poke needs the range-checked build (CKV_DEBUG_BOUNDS=1)")
    fn = L.ckv_debug_poke
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int32]
    _check("ckv_debug_poke", fn(ctx, int(what), int(g), int(c), int(r), int(value)))


def ckv_aux_bytes(ctx):
    a, k = ctypes.c_size_t(), ctypes.c_size_t()
    _check("ckv_aux_bytes", lib().ckv_aux_bytes(ctx, ctypes.byref(a), ctypes.byref(k)))
    return a.value, k.value
