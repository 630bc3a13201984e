"""The C-ABI library builds, loads without a GPU, exports every symbol that
include/ckv.h declares, and rejects bad configurations on the host."""
import ctypes
import os

import numpy as np
import pytest

import long_context_decode_ckv_b200 as ckv
from long_context_decode_ckv_b200 import build as ckv_build
from long_context_decode_ckv_b200 import state as ckv_state


@pytest.fixture(scope="module")
def L():
    ckv_build.build()
    return ckv.lib()


def test_exports_every_declared_symbol(L):
    names = ckv.declared_functions()
    assert len(names) >= 14
    raw = ctypes.CDLL(ckv.LIB_PATH)
    for name in names:
        assert hasattr(raw, name), f"libckv.so does not export {name}"


def _exports(path):
    out = os.popen(f"nm -D --defined-only {path}").read().split("\n")
    return {ln.split()[-1] for ln in out if " T ckv_" in ln}


def test_exports_nothing_undeclared(L):
    assert _exports(ckv_build.LIB) == set(ckv.declared_functions())


def test_range_checked_build_exports_both_headers():
    # libckv_debug.so: every ckv.h entry point plus the fault injection of
    # ckv_debug.h, which the release library does not export
    ckv_build.build(debug=True)
    dbg = set(ckv.declared_functions(ckv.HEADER_DEBUG)) - set(ckv.declared_functions())
    assert dbg == {"ckv_debug_poke"}
    assert _exports(ckv_build.LIB_DEBUG) == set(ckv.declared_functions()) | dbg
    assert not (_exports(ckv_build.LIB) & dbg)
    raw = ctypes.CDLL(ckv_build.LIB_DEBUG)
    assert hasattr(raw, "ckv_debug_poke")


def good_config():
    c = ckv.ckv_config()
    c.batch, c.n_q_heads, c.n_kv_heads, c.head_dim = 4, 32, 8, 128
    c.n_max, c.max_communities, c.n_sinks = 131200, 8192, 4
    c.kappa, c.budget, c.slack = 8, 4096, 16
    c.kv_dtype, c.mode, c.device, c.pool_capacity = ckv.CKV_BF16, ckv.CKV_QUERY_GROUP, 0, 0
    return c


def test_graph_count_and_status_strings(L):
    c = good_config()
    assert ckv.ckv_graph_count(c) == 32
    c.mode = ckv.CKV_PER_HEAD
    assert ckv.ckv_graph_count(c) == 128
    c.mode = 7
    assert ckv.ckv_graph_count(c) == -1
    for s in range(7):
        assert ckv.status_string(s) and ckv.status_string(s) != "unknown status"
    assert ckv.status_string(99) == "unknown status"


@pytest.mark.parametrize("field,value", [
    ("batch", 0), ("n_q_heads", 0), ("n_kv_heads", 3), ("head_dim", 64), ("n_max", 0),
    ("max_communities", 0), ("n_sinks", -1), ("n_sinks", 131200), ("kappa", 0), ("kappa", 33),
    ("budget", 0), ("slack", -1), ("kv_dtype", 5), ("mode", 2), ("device", -1),
    ("pool_capacity", -1),
])
def test_bad_config_rejected_on_host(L, field, value):
    c = good_config()
    setattr(c, field, value)
    h = ctypes.c_void_p()
    assert L.ckv_create(ctypes.byref(c), ctypes.byref(h)) == ckv.CKV_ERR_INVALID_ARG
    assert h.value is None


def test_group_size_must_be_supported(L):
    c = good_config()
    c.n_q_heads, c.n_kv_heads = 48, 8          # group of 6
    h = ctypes.c_void_p()
    assert L.ckv_create(ctypes.byref(c), ctypes.byref(h)) == ckv.CKV_ERR_INVALID_ARG


def test_null_arguments_rejected(L):
    assert L.ckv_create(None, None) == ckv.CKV_ERR_INVALID_ARG
    assert L.ckv_decode_step(None, None, None, None, 1, None, None) == ckv.CKV_ERR_INVALID_ARG
    assert L.ckv_assign_update(None, None, 1, None) == ckv.CKV_ERR_INVALID_ARG
    assert L.ckv_last_error(None) == ckv.CKV_ERR_INVALID_ARG
    assert L.ckv_import_state(None, None, 0) == ckv.CKV_ERR_INVALID_ARG
    assert L.ckv_build_graph(8, 64, 128, 4, 8, ckv.CKV_BF16, None, None, None, None, None, None) \
        == ckv.CKV_ERR_INVALID_ARG
    # prefill takes bf16 only, head_dim 128, kappa 1..32
    p = ctypes.c_void_p(16)
    assert L.ckv_build_graph(8, 64, 128, 4, 8, ckv.CKV_F32, p, p, p, p, p, None) == ckv.CKV_ERR_INVALID_ARG
    assert L.ckv_build_graph(8, 64, 64, 4, 8, ckv.CKV_BF16, p, p, p, p, p, None) == ckv.CKV_ERR_INVALID_ARG
    assert L.ckv_build_graph(8, 64, 128, 4, 40, ckv.CKV_BF16, p, p, p, p, p, None) == ckv.CKV_ERR_INVALID_ARG
    ckv.ckv_destroy(None)   # ignored


def test_newer_entry_points_check_arguments_on_host(L):
    # every check below runs before any device call
    p = ctypes.c_void_p(16)
    q = ctypes.c_double(0.0)
    one = ctypes.c_double(1.0)
    bad = ckv.CKV_ERR_INVALID_ARG
    # query-group prefill graph: pointers, group (1, 2, 4 or 8 heads), kappa, bf16 only
    assert L.ckv_build_graph_grouped(2, 4, 64, 128, 4, 8, ckv.CKV_BF16, None, None, None, None, None, None, None) == bad
    assert L.ckv_build_graph_grouped(2, 3, 64, 128, 4, 8, ckv.CKV_BF16, p, p, p, p, p, p, None) == bad
    assert L.ckv_build_graph_grouped(2, 4, 64, 128, 4, 0, ckv.CKV_BF16, p, p, p, p, p, p, None) == bad
    assert L.ckv_build_graph_grouped(2, 4, 64, 128, 4, 8, ckv.CKV_F32, p, p, p, p, p, p, None) == bad
    assert L.ckv_build_graph_grouped_workspace(0, 4, 64) == 0
    # modularity: n, pointers, resolution
    assert L.ckv_modularity(0, p, p, p, p, 1, one, p, ctypes.byref(q), None) == bad
    assert L.ckv_modularity(4, None, p, p, p, 1, one, p, ctypes.byref(q), None) == bad
    assert L.ckv_modularity(4, p, p, p, p, 1, ctypes.c_double(0.0), p, ctypes.byref(q), None) == bad
    assert L.ckv_modularity(4, p, p, p, p, 1, ctypes.c_double(float("inf")), p, ctypes.byref(q), None) == bad
    assert L.ckv_modularity_workspace(0) == 0
    # calls on a context refuse a null one
    assert L.ckv_step_recall(None, p, p, 1, p, None) == bad
    assert L.ckv_dense_decode(None, p, p, p, 1, p, None, None) == bad
    assert L.ckv_set_token_graph(None, p, p, p, 4) == bad
    assert L.ckv_refresh(None, p, one, None, None) == bad
    assert L.ckv_graph_modularity(None, one, ctypes.byref(q), None) == bad
    assert L.ckv_init_communities(None, None, 0, 1, None, 4, None) == bad
    assert L.ckv_decode_host(None, None, None, None, None, None, 1, None, None) == bad
    assert L.ckv_get_step_debug(None, None, None, None, None, None, None, None) == bad
    assert L.ckv_export_state(None, None, None) == bad
    assert L.ckv_profile_begin(None) == bad
    assert L.ckv_aux_bytes(None, None, None) == bad
    assert L.ckv_attend_rows_static(None, p, p, p, 5, p, p, 4, p, None) == bad


def test_checkpoint_record_roundtrip():
    rng = np.random.default_rng(0)
    G, Nc, D, S, kap, n_init, n_tok = 3, 5, 128, 4, 8, 40, 43
    sizes = np.zeros((G, Nc), np.int32)
    for g in range(G):
        sizes[g] = np.bincount(rng.integers(0, Nc, n_tok - S), minlength=Nc)
    s = ckv_state.State(G, Nc, D, n_tok, S, kap, n_init,
                        rng.standard_normal((G, Nc, D)).astype(np.float32), sizes,
                        np.tile(np.arange(S, n_tok, dtype=np.int32), (G, 1)),
                        rng.integers(0, kap + 1, (G, n_tok - n_init)).astype(np.int32),
                        rng.integers(0, n_tok, (G, n_tok - n_init, kap)).astype(np.int32),
                        rng.random((G, n_tok - n_init, kap)).astype(np.float32))
    blob = ckv_state.pack(s)
    assert len(blob) == 36 + 4 * (G * Nc * D + G * Nc + G * (n_tok - S) + G * (n_tok - n_init) * (1 + 2 * kap))
    t = ckv_state.parse(blob)
    for f in ("centroids", "sizes", "members", "deg", "col", "w"):
        np.testing.assert_array_equal(getattr(t, f), getattr(s, f))
    with pytest.raises(ValueError):
        ckv_state.parse(b"\0" * 64)


class _FakeCudaTensor:
    """Stands in for a CUDA tensor on a machine without one (never dereferenced)."""
    is_cuda = True

    def data_ptr(self):
        return 0x1000


def test_binding_refuses_the_wrong_memory_kind():
    # device arguments take CUDA tensors only, host arguments never a CUDA
    # tensor: both are refused before the C call, so no kernel is handed a
    # host address
    import torch
    dev = _FakeCudaTensor()
    host = np.zeros(4, np.float32)
    calls = [
        lambda: ckv.ckv_decode_step(None, host, dev, dev, 1, dev),                 # numpy for q
        lambda: ckv.ckv_decode_step(None, dev, torch.zeros(4), dev, 1, dev),       # CPU tensor for K
        lambda: ckv.ckv_assign_update(None, host, 1),
        lambda: ckv.ckv_decode_host(None, dev, host, host, dev, dev, 1, host),     # CUDA tensor for q_host
        lambda: ckv.ckv_decode_host(None, host, host, host, host, dev, 1, host),   # numpy for K
        lambda: ckv.ckv_get_step_debug(None, n_sel=dev),
        lambda: ckv.ckv_init_communities(None, host, 1, 1, dev, 4),                # host labels said on device
        lambda: ckv.ckv_init_communities(None, dev, 0, 1, dev, 4),                 # device labels said on host
        lambda: ckv.ckv_build_graph(1, 8, 128, 4, 8, ckv.CKV_BF16, host, dev, dev, dev, dev),
        lambda: ckv.ckv_modularity(4, dev, dev, dev, host, 1, 1.0, dev),
        lambda: ckv.ckv_step_recall(None, dev, dev, 1, host),
        lambda: ckv.ckv_dense_decode(None, dev, dev, dev, 1, dev, host),
        lambda: ckv.ckv_refresh(None, host, 1.0),
        lambda: ckv.ckv_graph_modularity(None, 1.0, dev),
    ]
    for fn in calls:
        with pytest.raises(TypeError):
            fn()
    # the right kinds reach the C entry point, which rejects the null context
    with pytest.raises(ckv.CkvError) as e:
        ckv.ckv_decode_step(None, dev, dev, dev, 1, dev)
    assert e.value.status == ckv.CKV_ERR_INVALID_ARG
