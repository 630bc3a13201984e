"""Host-side reader/writer of the library's checkpoint record (the layout-free
format of ckv_export_state / ckv_import_state in include/ckv.h).

Pure data-format code: it moves arrays in and out of the byte record and
holds none of the method's arithmetic.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

MAGIC = 0x31564B43


@dataclass
class State:
    n_graphs: int
    n_comm: int
    head_dim: int
    n_tok: int
    n_sinks: int
    kappa: int
    n_init: int
    centroids: np.ndarray   # [G][Nc][D] float32
    sizes: np.ndarray       # [G][Nc] int32
    members: np.ndarray     # [G][n_tok - S] int32, community-major, ascending
    deg: np.ndarray         # [G][n_tok - n_init] int32
    col: np.ndarray         # [G][n_tok - n_init][kappa] int32
    w: np.ndarray           # [G][n_tok - n_init][kappa] float32

    def community_members(self, g: int, c: int) -> np.ndarray:
        starts = np.concatenate([[0], np.cumsum(self.sizes[g])])
        return self.members[g, starts[c]:starts[c + 1]]


def parse(blob: bytes) -> State:
    hdr = np.frombuffer(blob, np.int32, 9)
    if int(hdr[0]) & 0xFFFFFFFF != MAGIC or hdr[1] != 1:
        raise ValueError("not a CKV1 record")
    G, Nc, D, n_tok, S, kap, n_init = (int(v) for v in hdr[2:9])
    off = 36

    def take(dtype, shape):
        nonlocal off
        cnt = int(np.prod(shape))
        a = np.frombuffer(blob, dtype, cnt, off).reshape(shape).copy()
        off += cnt * 4
        return a

    mu = take(np.float32, (G, Nc, D))
    sizes = take(np.int32, (G, Nc))
    members = take(np.int32, (G, n_tok - S))
    rows = n_tok - n_init
    deg = take(np.int32, (G, rows))
    col = take(np.int32, (G, rows, kap))
    w = take(np.float32, (G, rows, kap))
    return State(G, Nc, D, n_tok, S, kap, n_init, mu, sizes, members, deg, col, w)


def pack(s: State) -> bytes:
    hdr = np.array([MAGIC, 1, s.n_graphs, s.n_comm, s.head_dim, s.n_tok, s.n_sinks, s.kappa,
                    s.n_init], np.uint32).view(np.int32)
    parts = [hdr, s.centroids.astype(np.float32), s.sizes.astype(np.int32),
             s.members.astype(np.int32), s.deg.astype(np.int32), s.col.astype(np.int32),
             s.w.astype(np.float32)]
    return b"".join(np.ascontiguousarray(p).tobytes() for p in parts)
