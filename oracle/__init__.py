"""ctypes wrapper of the plain C CPU oracle (``oracle/moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline leg are the only users.  The product path (the CUDA
library and its Python binding) never imports this package, and this package
never imports the product.

Every function mirrors one function of the C file, which states the
definitions it follows (block formats, routing, SwiGLU, combine, LRU rules).
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

Q4_0 = 2
Q4_1 = 3
Q5_0 = 6
Q5_1 = 7
Q8_0 = 8
Q4_K = 12
Q6_K = 14
QTYPE = {"q4_0": Q4_0, "q4_1": Q4_1, "q5_0": Q5_0, "q5_1": Q5_1, "q8_0": Q8_0,
         "q4_k": Q4_K, "q6_k": Q6_K}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP on) into oracle/liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _declare(_lib)
    return _lib


_p = C.c_void_p
_i = C.c_int


def _declare(L):
    L.orc_half_to_double.restype = C.c_double
    L.orc_half_to_double.argtypes = [C.c_uint16]
    L.orc_block_bytes.restype = _i
    L.orc_block_bytes.argtypes = [_i]
    L.orc_block_weights.restype = _i
    L.orc_block_weights.argtypes = [_i]
    L.orc_dequant_row.restype = _i
    L.orc_dequant_row.argtypes = [_p, _i, _i, _p]
    L.orc_router_logits.restype = None
    L.orc_router_logits.argtypes = [_p, _p, _p, _i, _i, _i, _p]
    L.orc_select.restype = None
    L.orc_select.argtypes = [_p, _i, _i, _i, _i, _p, _p]
    L.orc_permute.restype = _i
    L.orc_permute.argtypes = [_p, _i, _i, _i, _p, _p, _p, _p]
    L.orc_layer.restype = _i
    L.orc_layer.argtypes = [_p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p,
                            _p, _p, _p, _i, _i, _p, _i, _i, _i, _p]
    L.orc_expert_rows.restype = _i
    L.orc_expert_rows.argtypes = [_p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p,
                                  _p, _i, _i, _p]
    L.orc_quantize_act8.restype = None
    L.orc_quantize_act8.argtypes = [_p, _i, _p, _p]
    L.orc_layer_a8.restype = _i
    L.orc_layer_a8.argtypes = [_p, _i, _i, _i, _i, _i, _i, _p, _p, _p, _p, _p,
                               _p, _p, _p, _i, _i, _p, _i, _i, C.c_double, _p, _p]
    L.orc_lru_new.restype = _p
    L.orc_lru_new.argtypes = [_i, _i]
    L.orc_lru_free.restype = None
    L.orc_lru_free.argtypes = [_p]
    L.orc_lru_request.restype = _i
    L.orc_lru_request.argtypes = [_p, _p, _i, _p, _p, _p]
    L.orc_glru_new.restype = _p
    L.orc_glru_new.argtypes = [_i, _i, _i, _i]
    L.orc_glru_free.restype = None
    L.orc_glru_free.argtypes = [_p]
    L.orc_glru_request.restype = _i
    L.orc_glru_request.argtypes = [_p, _i, _p, _i, _p, _p, _p]
    L.orc_glru_resize.restype = _i
    L.orc_glru_resize.argtypes = [_p, _i, _p, _p, _p, _p]


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _qt(q):
    return QTYPE[q] if isinstance(q, str) else int(q)


# --------------------------------------------------------------------------
def half_to_double(h: int) -> float:
    return lib().orc_half_to_double(int(h))


def block_bytes(qtype) -> int:
    return lib().orc_block_bytes(_qt(qtype))


def block_weights(qtype) -> int:
    return lib().orc_block_weights(_qt(qtype))


def dequant_row(row_bytes: np.ndarray, qtype, ncols: int) -> np.ndarray:
    row = _c(row_bytes, np.uint8)
    out = np.empty(ncols, np.float64)
    rc = lib().orc_dequant_row(_ptr(row), _qt(qtype), ncols, _ptr(out))
    if rc != 0:
        raise ValueError("bad qtype or ncols")
    return out


def dequant_matrix(mat_bytes: np.ndarray, qtype, ncols: int) -> np.ndarray:
    mat = _c(mat_bytes, np.uint8)
    return np.stack([dequant_row(r, qtype, ncols) for r in mat])


def router_logits(x, w_r, bias=None) -> np.ndarray:
    x = _c(x, np.float32)
    w_r = _c(w_r, np.float32)
    bias = _c(bias, np.float32)
    T, D = x.shape
    E = w_r.shape[1]
    out = np.empty((T, E), np.float32)
    lib().orc_router_logits(_ptr(x), _ptr(w_r), _ptr(bias), T, D, E, _ptr(out))
    return out


def select(logits, k: int, renorm: bool = True):
    L = _c(logits, np.float32)
    T, E = L.shape
    ids = np.empty((T, k), np.int32)
    g = np.empty((T, k), np.float64)
    lib().orc_select(_ptr(L), T, E, k, int(renorm), _ptr(ids), _ptr(g))
    return ids, g


def permute(ids, E: int):
    ids = _c(ids, np.int32)
    T, k = ids.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    rc = lib().orc_permute(_ptr(ids), T, k, E, _ptr(counts), _ptr(offsets),
                           _ptr(perm), _ptr(inv))
    if rc != 0:
        raise ValueError("expert id out of range")
    return counts, offsets, perm, inv


def layer(x, ids, gates, gate, up, down, qtype, F: int, shared=None,
          tokens=None, dense: bool = False, threads: int = 0,
          shared_qtype="q8_0") -> np.ndarray:
    """y [n_tok, D] (float64) of the routed layer for the listed tokens.

    ``gate/up/down``: pools [E, rows, bytes]; ``shared``: optional
    (gate, up, down) of one expert in ``shared_qtype`` with its own F.
    """
    x = _c(x, np.float32)
    T, D = x.shape
    ids = _c(ids, np.int32)
    k = ids.shape[1]
    gates = _c(gates, np.float64)
    gate, up, down = (_c(a, np.uint8) for a in (gate, up, down))
    E = gate.shape[0]
    sg = su = sd = None
    sF = 0
    if shared is not None:
        sg, su, sd = (_c(a, np.uint8) for a in shared)
        sF = sg.shape[1]
    tl = _c(tokens, np.int32)
    n = T if tl is None else len(tl)
    y = np.empty((n, D), np.float64)
    rc = lib().orc_layer(_ptr(x), T, D, F, E, k, _qt(qtype), _ptr(gate), _ptr(up),
                         _ptr(down), _ptr(ids), _ptr(gates), _ptr(sg), _ptr(su),
                         _ptr(sd), sF, _qt(shared_qtype), _ptr(tl), n, int(dense), threads, _ptr(y))
    if rc != 0:
        raise ValueError("oracle layer: bad arguments")
    return y


def quantize_act8(v):
    """8-bit activation blocks of the rows of v [.., n] (n % 32 == 0):
    (q int8 [.., n], d float32 [.., n/32])."""
    v = _c(v, np.float32)
    n = v.shape[-1]
    flat = v.reshape(-1, n)
    q = np.empty(flat.shape, np.int8)
    d = np.empty((flat.shape[0], n // 32), np.float32)
    for r in range(flat.shape[0]):
        qr, dr = q[r], d[r]
        lib().orc_quantize_act8(_ptr(np.ascontiguousarray(flat[r])), n, _ptr(qr), _ptr(dr))
    return q.reshape(v.shape), d.reshape(v.shape[:-1] + (n // 32,))


def layer_a8(x, ids, gates, gate, up, down, qtype, F: int, shared=None, tokens=None,
             threads: int = 0, shared_qtype="q8_0", eps: float = 0.0, want_bound=False):
    """y [n_tok, D] (float64) of the layer with 8-bit activations into every
    expert matmul; with want_bound, also the per-output room that h codes
    within eps of a rounding boundary leave (see the C function)."""
    x = _c(x, np.float32)
    T, D = x.shape
    ids = _c(ids, np.int32)
    k = ids.shape[1]
    gates = _c(gates, np.float64)
    gate, up, down = (_c(a, np.uint8) for a in (gate, up, down))
    E = gate.shape[0]
    sg = su = sd = None
    sF = 0
    if shared is not None:
        sg, su, sd = (_c(a, np.uint8) for a in shared)
        sF = sg.shape[1]
    tl = _c(tokens, np.int32)
    n = T if tl is None else len(tl)
    y = np.empty((n, D), np.float64)
    b = np.empty((n, D), np.float64) if want_bound else None
    rc = lib().orc_layer_a8(_ptr(x), T, D, F, E, k, _qt(qtype), _ptr(gate), _ptr(up),
                            _ptr(down), _ptr(ids), _ptr(gates), _ptr(sg), _ptr(su), _ptr(sd),
                            sF, _qt(shared_qtype), _ptr(tl), n, threads, float(eps), _ptr(y),
                            _ptr(b))
    if rc != 0:
        raise ValueError("oracle layer_a8: bad arguments")
    return (y, b) if want_bound else y


def expert_rows(x, perm, offsets, k: int, gate, up, down, qtype, F: int,
                positions=None, threads: int = 0) -> np.ndarray:
    """Y [n_pos, D] (float64): un-gated expert outputs at permuted positions."""
    x = _c(x, np.float32)
    T, D = x.shape
    perm = _c(perm, np.int32)
    offsets = _c(offsets, np.int32)
    gate, up, down = (_c(a, np.uint8) for a in (gate, up, down))
    E = gate.shape[0]
    pl = _c(positions, np.int32)
    n = T * k if pl is None else len(pl)
    Y = np.empty((n, D), np.float64)
    rc = lib().orc_expert_rows(_ptr(x), T, D, F, E, k, _qt(qtype), _ptr(gate),
                               _ptr(up), _ptr(down), _ptr(perm), _ptr(offsets),
                               _ptr(pl), n, threads, _ptr(Y))
    if rc != 0:
        raise ValueError("oracle expert_rows: bad arguments")
    return Y


def route(x, w_r, bias, k: int, renorm: bool = True, logits=None):
    """Logits (fp32), ids and gates of one layer call."""
    if logits is None:
        logits = router_logits(x, w_r, bias)
    ids, g = select(logits, k, renorm)
    return logits, ids, g


class LRU:
    """Per-layer expert-cache LRU simulation (rules in moe_oracle.c)."""

    def __init__(self, E: int, n_slots: int):
        self._h = lib().orc_lru_new(E, n_slots)
        self.E, self.n_slots = E, n_slots

    def request(self, ids):
        ids = _c(ids, np.int32)
        n = len(ids)
        slot = np.empty(n, np.int32)
        miss = np.empty(n, np.int32)
        ev = np.empty(n, np.int32)
        rc = lib().orc_lru_request(self._h, _ptr(ids), n, _ptr(slot), _ptr(miss), _ptr(ev))
        if rc == -2:
            raise OverflowError("more ids than slots")
        if rc < 0:
            raise ValueError("bad or duplicate expert id")
        return slot, miss.astype(bool), ev

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            lib().orc_lru_free(h)
            self._h = None


class GlobalLRU:
    """Expert-cache LRU simulation shared by all layers, with run-time resize
    (rules in moe_oracle.c, orc_glru_request / orc_glru_resize).  Entries are
    keyed layer * E + expert."""

    def __init__(self, n_layers: int, E: int, max_slots: int, cap: int):
        self._h = lib().orc_glru_new(n_layers, E, max_slots, cap)
        if not self._h:
            raise ValueError("bad global LRU shape")
        self.n_layers, self.E, self.max_slots = n_layers, E, max_slots

    def request(self, layer: int, ids):
        ids = _c(ids, np.int32)
        n = len(ids)
        slot = np.empty(n, np.int32)
        miss = np.empty(n, np.int32)
        ev = np.empty(n, np.int32)
        rc = lib().orc_glru_request(self._h, layer, _ptr(ids), n, _ptr(slot), _ptr(miss),
                                    _ptr(ev))
        if rc == -2:
            raise OverflowError("more ids than the capacity")
        if rc < 0:
            raise ValueError("bad layer, or bad or duplicate expert id")
        return slot, miss.astype(bool), ev

    def resize(self, cap: int):
        """-> (evicted keys, moves as an [n, 2] array of (from, to) slots)."""
        ev = np.empty(self.max_slots, np.int32)
        mv = np.empty(2 * self.max_slots, np.int32)
        ne, nm = C.c_int(0), C.c_int(0)
        rc = lib().orc_glru_resize(self._h, cap, _ptr(ev), C.byref(ne), _ptr(mv), C.byref(nm))
        if rc < 0:
            raise ValueError("capacity out of range")
        return ev[: ne.value].copy(), mv[: 2 * nm.value].reshape(-1, 2).copy()

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            lib().orc_glru_free(h)
            self._h = None


def near_tie_tokens(logits, k: int, eps: float = 1e-5) -> np.ndarray:
    """Tokens whose selection or order is decided by a logit gap below eps:
    the gap between the k-th and (k+1)-th largest logits, or between two
    adjacent logits inside the top k."""
    L = np.sort(np.asarray(logits, np.float64), axis=1)[:, ::-1]
    kk = min(k + 1, L.shape[1])
    gaps = L[:, : kk - 1] - L[:, 1:kk]
    return np.nonzero((gaps < eps).any(axis=1))[0]
