"""Python binding of libmoe (include/moe.h): argument marshalling only.

Every step of the layer runs in the CUDA library; this module turns torch
tensors into device pointers and streams, allocates the caller-owned
buffers the C calls write into, and raises on a non-OK status.  There is no
fallback: if ``libmoe.so`` is missing the first call raises.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

# enums of include/moe.h
MOE_OK = 0
Q4_0, Q4_1, Q5_0, Q5_1, Q8_0, Q4_K, Q6_K = 2, 3, 6, 7, 8, 12, 14
F32, BF16, F16 = 0, 1, 2
QTYPES = {"q4_0": Q4_0, "q4_1": Q4_1, "q5_0": Q5_0, "q5_1": Q5_1, "q8_0": Q8_0,
          "q4_k": Q4_K, "q6_k": Q6_K}
BLOCK_BYTES = {Q4_0: 18, Q4_1: 20, Q5_0: 22, Q5_1: 24, Q8_0: 34, Q4_K: 144, Q6_K: 210}
BLOCK_WEIGHTS = {q: (256 if q in (Q4_K, Q6_K) else 32) for q in BLOCK_BYTES}
_DT = {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16}
STATUS = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_QTYPE",
          3: "MOE_ERR_SHAPE", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_CAPACITY",
          6: "MOE_ERR_TIMEOUT", 7: "MOE_ERR_WORKSPACE"}
# device status word codes (moe_device_status)
DEV_OK, DEV_TIMEOUT_FULL, DEV_TIMEOUT_EMPTY, DEV_TIMEOUT_DRAIN, DEV_BAD_SLOT, DEV_TIMEOUT_MMA = range(6)
# moe_layer_forward phases
PHASE_ROUTE, PHASE_FFN, PHASE_SHARED, PHASE_COMBINE = 1, 2, 4, 8
PHASE_ALL = 15


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class Pool(C.Structure):
    _fields_ = [("qtype", C.c_int32), ("n_slots", C.c_int32), ("gate", C.c_void_p),
                ("up", C.c_void_p), ("down", C.c_void_p), ("slot_of_expert", C.c_void_p)]


TRACE_MAX = 24
KERNEL_KINDS = {1: "route", 2: "route_logits", 3: "route_select", 4: "permute", 5: "gateup",
                6: "down", 7: "combine", 8: "shared_gateup", 9: "shared_down", 10: "convert",
                11: "zero", 12: "ffn_decode"}


class Trace(C.Structure):
    _fields_ = [("events", C.POINTER(C.c_void_p)), ("capacity", C.c_int32),
                ("count", C.c_int32), ("kinds", C.c_int32 * TRACE_MAX)]


class LayerArgs(C.Structure):
    _fields_ = [("T", C.c_int32), ("D", C.c_int32), ("E", C.c_int32), ("k", C.c_int32),
                ("F", C.c_int32), ("shared_F", C.c_int32), ("renorm", C.c_int32),
                ("x_dtype", C.c_int32), ("y_dtype", C.c_int32), ("phases", C.c_int32),
                ("x", C.c_void_p), ("w_router", C.c_void_p), ("bias", C.c_void_p),
                ("logits_in", C.c_void_p), ("pool", C.POINTER(Pool)),
                ("shared", C.POINTER(Pool)), ("y", C.c_void_p), ("ids_out", C.c_void_p),
                ("gates_out", C.c_void_p), ("logits_out", C.c_void_p),
                ("trace", C.POINTER(Trace)), ("expert_mask", C.c_void_p),
                ("counts_out", C.c_void_p), ("offsets_out", C.c_void_p),
                ("perm_out", C.c_void_p), ("inv_out", C.c_void_p), ("act_bits", C.c_int32)]


class CacheDesc(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("E", C.c_int32), ("n_slots", C.c_int32),
                ("qtype", C.c_int32), ("bytes_gate", C.c_size_t), ("bytes_up", C.c_size_t),
                ("bytes_down", C.c_size_t), ("host_gate", C.POINTER(C.c_void_p)),
                ("host_up", C.POINTER(C.c_void_p)), ("host_down", C.POINTER(C.c_void_p)),
                ("dev_gate", C.c_void_p), ("dev_up", C.c_void_p), ("dev_down", C.c_void_p),
                ("dev_slot_map", C.c_void_p), ("copy_stream", C.c_void_p),
                ("dev_masks", C.c_void_p), ("global_", C.c_int32), ("max_slots", C.c_int32)]


class StreamerDesc(C.Structure):
    _fields_ = [("n_layers", C.c_int32), ("E", C.c_int32), ("qtype", C.c_int32),
                ("reserved", C.c_int32), ("bytes_gate", C.c_size_t), ("bytes_up", C.c_size_t),
                ("bytes_down", C.c_size_t), ("host_gate", C.POINTER(C.c_void_p)),
                ("host_up", C.POINTER(C.c_void_p)), ("host_down", C.POINTER(C.c_void_p)),
                ("dev_gate", C.c_void_p * 2), ("dev_up", C.c_void_p * 2),
                ("dev_down", C.c_void_p * 2), ("copy_stream", C.c_void_p)]


_lib = None
_v, _i, _sz = C.c_void_p, C.c_int, C.c_size_t


def lib():
    """The loaded libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmoe.so is not built ({LIB_PATH}); run "
                               "`python -m quantized_routed_expert_top_b200.build`")
        L = C.CDLL(LIB_PATH)
        L.moe_last_error.restype = C.c_char_p
        L.moe_version.restype = C.c_char_p
        L.moe_block_bytes.argtypes = [C.c_int32]
        L.moe_workspace_status.argtypes = [_v, C.POINTER(C.c_int32), _i, _v]
        L.moe_selftest_wait_timeout.argtypes = [_v, _sz, C.c_int64, _v]
        L.moe_block_weights.argtypes = [C.c_int32]
        L.moe_route_workspace_size.restype = _sz
        L.moe_route_workspace_size.argtypes = [_i, _i, _i, _i]
        L.moe_route.argtypes = [_v, C.c_int32, _v, _v, _i, _i, _i, _i, _i, _v, _v, _v, _v, _sz, _v]
        L.moe_permute.argtypes = [_v, _i, _i, _i, _v, _v, _v, _v, _v]
        L.moe_expert_ffn_workspace_size.restype = _sz
        L.moe_expert_ffn_workspace_size.argtypes = [_i, _i, _i, _i]
        L.moe_expert_ffn.argtypes = [_v, C.c_int32, _i, _i, _i, _i, _i, _v, _v, C.POINTER(Pool),
                                     _v, _v, _v, _sz, _v]
        L.moe_combine.argtypes = [_v, _v, _v, _i, _i, _i, _v, _v, C.c_int32, _v]
        L.moe_layer_workspace_size.restype = _sz
        L.moe_layer_workspace_size.argtypes = [C.POINTER(LayerArgs)]
        L.moe_layer_forward.argtypes = [C.POINTER(LayerArgs), _v, _sz, _v]
        L.moe_cache_init.argtypes = [C.POINTER(CacheDesc), C.POINTER(_v)]
        L.moe_cache_destroy.argtypes = [_v]
        L.moe_cache_destroy.restype = None
        L.moe_cache_request.argtypes = [_v, _i, _v, _i, _v, _v, _v, C.POINTER(_i), _v]
        L.moe_cache_sync.argtypes = [_v, _i, _v]
        L.moe_cache_release.argtypes = [_v, _i, _v]
        L.moe_cache_layer_pool.argtypes = [_v, _i, C.POINTER(Pool)]
        L.moe_cache_layer_masks.argtypes = [_v, _i, C.POINTER(_v), C.POINTER(_v)]
        L.moe_cache_resize.argtypes = [_v, _i, C.POINTER(_i), C.POINTER(_i), _v]
        L.moe_cache_stats.argtypes = [_v, C.POINTER(C.c_int64), C.POINTER(C.c_int64),
                                      C.POINTER(C.c_int64), C.POINTER(C.c_int64)]
        L.moe_route_noalloc.argtypes = [_v, C.c_int32, _v, _v, _i, _i, _i, _i, _i, _v, _v, _v,
                                        _v]
        L.moe_streamer_init.argtypes = [C.POINTER(StreamerDesc), C.POINTER(_v)]
        L.moe_streamer_destroy.argtypes = [_v]
        L.moe_streamer_destroy.restype = None
        L.moe_streamer_prefetch.argtypes = [_v, _i]
        L.moe_streamer_acquire.argtypes = [_v, _i, _v, C.POINTER(Pool)]
        L.moe_streamer_release.argtypes = [_v, _i, _v]
        L.moe_streamer_stats.argtypes = [_v, C.POINTER(C.c_int64), C.POINTER(C.c_int64)]
        L.moe_cache_debug_fail_copy.argtypes = [_v, _i]
        L.moe_cache_debug_fail_copy.restype = None
        _lib = L
    return _lib


def _check(status: int):
    if status != MOE_OK:
        raise MoeError(status, lib().moe_last_error().decode())


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _dev(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensor must live on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensor must be contiguous")


def _qt(q):
    return QTYPES[q] if isinstance(q, str) else int(q)


def _zeros_ws(nbytes, device):
    return torch.zeros(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def workspace_status(ws, clear: bool = True, stream=None):
    """moe_workspace_status: (status, code) of a workspace's device status
    word; waits for the stream.  status is MOE_OK when code == DEV_OK."""
    code = C.c_int32(0)
    st = lib().moe_workspace_status(_p(ws), C.byref(code), int(clear), _stream(stream))
    return st, code.value


def selftest_wait_timeout(ws, budget_cycles: int, stream=None):
    """moe_selftest_wait_timeout: one warp waits, with the kernels' bounded
    wait, on a barrier nothing arrives at; the status word of ``ws`` then
    reads DEV_TIMEOUT_FULL (see workspace_status)."""
    _check(lib().moe_selftest_wait_timeout(_p(ws), ws.numel() * ws.element_size(),
                                           int(budget_cycles), _stream(stream)))


# ----------------------------------------------------------------- pools
class ExpertPool:
    """Device expert pool: gate/up [S, F, D/32*bs], down [S, D, F/32*bs] uint8."""

    def __init__(self, gate, up, down, qtype, slot_of_expert=None):
        _dev(gate, up, down, slot_of_expert)
        for t in (gate, up, down):
            if t.dtype != torch.uint8:
                raise ValueError("pool tensors must be uint8 block bytes")
        self.gate, self.up, self.down = gate, up, down
        self.qtype = _qt(qtype)
        self.slot_of_expert = slot_of_expert
        self.c = Pool(self.qtype, gate.shape[0], gate.data_ptr(), up.data_ptr(), down.data_ptr(),
                      None if slot_of_expert is None else slot_of_expert.data_ptr())

    @classmethod
    def from_numpy(cls, gate, up, down, qtype, device="cuda"):
        t = lambda a: torch.from_numpy(a).to(device)
        return cls(t(gate), t(up), t(down), qtype)


# ----------------------------------------------------- step-by-step calls
def route(x, w_router, bias, k: int, renorm: bool = True, want_logits: bool = False,
          stream=None):
    """moe_route.  x [T, D] (f32/bf16), or the logits [T, E] when w_router is None."""
    _dev(x, w_router, bias)
    T = x.shape[0]
    if w_router is None:
        D, E = 32, x.shape[1]
    else:
        D, E = x.shape[1], w_router.shape[1]
    dev = x.device
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    logits = torch.empty((T, E), dtype=torch.float32, device=dev) if want_logits else None
    nbytes = lib().moe_route_workspace_size(T, D, E, k)
    ws = _zeros_ws(nbytes, dev)
    _check(lib().moe_route(_p(x), _DT[x.dtype], _p(w_router), _p(bias), T, D, E, k, int(renorm),
                           _p(ids), _p(gates), _p(logits), _p(ws), ws.numel(), _stream(stream)))
    return (ids, gates, logits) if want_logits else (ids, gates)


def permute(ids, E: int, stream=None):
    """moe_permute -> counts [E], offsets [E+1], perm [T*k], inv [T*k] (int32)."""
    _dev(ids)
    T, k = ids.shape
    dev = ids.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)[: T * k]
    inv = torch.empty(max(T * k, 1), dtype=torch.int32, device=dev)[: T * k]
    _check(lib().moe_permute(_p(ids), T, k, E, _p(counts), _p(offsets), _p(perm), _p(inv),
                             _stream(stream)))
    return counts, offsets, perm, inv


def expert_ffn(x, perm, offsets, pool: ExpertPool, k: int, F: int, mask=None, out=None,
               stream=None, ws=None):
    """moe_expert_ffn -> out_rows [T*k, D] fp32 in permuted order.  ``ws``:
    an optional caller workspace (zero-filled uint8 tensor of at least
    expert_ffn_workspace_size bytes), e.g. to read its status word after."""
    _dev(x, perm, offsets, mask, out, ws)
    T, D = x.shape
    E = offsets.numel() - 1
    if out is None:
        out = torch.empty((T * k, D), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = _zeros_ws(expert_ffn_workspace_size(T, k, D, F), x.device)
    _check(lib().moe_expert_ffn(_p(x), _DT[x.dtype], T, D, F, E, k, _p(perm), _p(offsets),
                                C.byref(pool.c), _p(mask), _p(out), _p(ws), ws.numel(),
                                _stream(stream)))
    return out


def expert_ffn_workspace_size(T: int, k: int, D: int, F: int) -> int:
    return int(lib().moe_expert_ffn_workspace_size(T, k, D, F))


def combine(rows, inv, gates, shared_rows=None, y_dtype=torch.bfloat16, out=None, stream=None):
    """moe_combine -> y [T, D]."""
    _dev(rows, inv, gates, shared_rows, out)
    T, k = gates.shape
    D = rows.shape[1]
    if out is None:
        out = torch.empty((T, D), dtype=y_dtype, device=rows.device)
    _check(lib().moe_combine(_p(rows), _p(inv), _p(gates), T, k, D, _p(shared_rows), _p(out),
                             _DT[out.dtype], _stream(stream)))
    return out


# ------------------------------------------------------------ fused layer
class Layer:
    """One prepared moe_layer_forward call: weights, shapes and a workspace.

    ``forward(x)`` (or ``forward(None, logits)`` when routing from given
    logits) runs the fused layer and returns y; ids/gates of the last call
    are kept in ``self.ids`` / ``self.gates``.
    """

    def __init__(self, pool: ExpertPool, D: int, F: int, E: int, k: int, T_max: int,
                 w_router=None, bias=None, shared: ExpertPool | None = None, shared_F: int = 0,
                 renorm: bool = True, x_dtype=torch.bfloat16, y_dtype=torch.bfloat16,
                 device="cuda", act_bits: int = 16):
        """act_bits=8: 8-bit activation blocks into every expert matmul (the
        W4A8 / W8A8 mode; decode shapes with Q4_0 / Q8_0 experts)."""
        _dev(w_router, bias)
        self.act_bits = int(act_bits)
        self.pool, self.shared = pool, shared
        self.D, self.F, self.E, self.k, self.shared_F = D, F, E, k, shared_F
        self.w_router, self.bias = w_router, bias
        self.renorm, self.x_dtype, self.y_dtype = renorm, x_dtype, y_dtype
        self.device = torch.device(device)
        self.T_max = T_max
        self.ids = torch.empty((T_max, k), dtype=torch.int32, device=self.device)
        self.gates = torch.empty((T_max, k), dtype=torch.float32, device=self.device)
        self.ws = _zeros_ws(self.workspace_size(T_max), self.device)

    def _args(self, T, x, logits, y, logits_out=None, trace=None, phases=0, mask=None,
              routing_out=None):
        a = LayerArgs()
        a.T, a.D, a.E, a.k, a.F = T, self.D, self.E, self.k, self.F
        a.shared_F = self.shared_F if self.shared is not None else 0
        a.renorm = int(self.renorm)
        a.x_dtype = _DT[self.x_dtype]
        a.y_dtype = _DT[self.y_dtype if y is None else y.dtype]
        a.x = None if x is None else x.data_ptr()
        a.w_router = None if self.w_router is None else self.w_router.data_ptr()
        a.bias = None if self.bias is None else self.bias.data_ptr()
        a.logits_in = None if logits is None else logits.data_ptr()
        a.pool = C.pointer(self.pool.c)
        a.shared = C.pointer(self.shared.c) if self.shared is not None else None
        a.y = None if y is None else y.data_ptr()
        a.ids_out = self.ids.data_ptr()
        a.gates_out = self.gates.data_ptr()
        a.logits_out = None if logits_out is None else logits_out.data_ptr()
        a.trace = C.pointer(trace) if trace is not None else None
        a.phases = int(phases)
        a.act_bits = self.act_bits
        a.expert_mask = None if mask is None else mask.data_ptr()
        if routing_out is not None:
            a.counts_out, a.offsets_out, a.perm_out, a.inv_out = (t.data_ptr() for t in routing_out)
        return a

    def workspace_size(self, T):
        a = self._args(T, None, None, None)
        a.x = 1  # non-null placeholders: the size depends on shapes only
        return lib().moe_layer_workspace_size(C.byref(a))

    def routing_buffers(self, T=None):
        """Device int32 (counts [E], offsets [E+1], perm [T*k], inv [T*k]) for
        ``forward(routing_out=...)``."""
        T = self.T_max if T is None else T
        n = max(T * self.k, 1)
        mk = lambda m: torch.empty(m, dtype=torch.int32, device=self.device)
        return (mk(self.E), mk(self.E + 1), mk(n)[: T * self.k], mk(n)[: T * self.k])

    def forward(self, x, logits=None, out=None, logits_out=None, stream=None, trace=None,
                phases=0, mask=None, routing_out=None):
        """Run the layer (or the parts ``phases`` names, PHASE_* bits; 0 =
        all); ``mask``: device uint8 [E] restricting the FFN part;
        ``routing_out``: a routing_buffers() tuple that receives the
        permutation; ``trace`` is an optional KernelTrace."""
        _dev(x, logits, out, logits_out, mask)
        T = (x if x is not None else logits).shape[0]
        if T > self.T_max:
            raise ValueError(f"T={T} exceeds T_max={self.T_max}")
        if x is not None and x.dtype != self.x_dtype:
            raise ValueError(f"x dtype {x.dtype} != {self.x_dtype}")
        if out is None:
            out = torch.empty((T, self.D), dtype=self.y_dtype, device=self.device)
        a = self._args(T, x, logits, out, logits_out, trace.c if trace is not None else None,
                       phases, mask, routing_out)
        _check(lib().moe_layer_forward(C.byref(a), _p(self.ws), self.ws.numel(), _stream(stream)))
        if trace is not None:
            trace.record()
        return out


class KernelTrace:
    """Caller-owned CUDA events for moe_trace; collects per-kernel times.

    Each traced forward appends (kind, start_event, end_event) triples;
    ``durations()`` (after a synchronize) returns {kind: [ms, ...]}.
    """

    def __init__(self, n_calls: int, per_call: int = 16):
        self.pool = [torch.cuda.Event(enable_timing=True) for _ in range(n_calls * per_call)]
        for e in self.pool:          # torch creates events lazily: force the handles
            e.record()
        torch.cuda.synchronize()
        self.per_call = per_call
        self.calls = []
        self._next = 0
        self.c = None
        self._arm()

    def _arm(self):
        evs = self.pool[self._next:self._next + self.per_call]
        if len(evs) < self.per_call:
            raise RuntimeError("KernelTrace: out of events")
        self._evs = evs
        self._arr = (C.c_void_p * self.per_call)(*[e.cuda_event for e in evs])
        self.c = Trace(C.cast(self._arr, C.POINTER(C.c_void_p)), self.per_call, 0)

    def record(self):
        n = self.c.count
        kinds = [self.c.kinds[i] for i in range(n)]
        self.calls.append([(KERNEL_KINDS.get(kinds[i], str(kinds[i])), self._evs[i], self._evs[i + 1])
                           for i in range(n - 1)])
        self._next += self.per_call
        if self._next + self.per_call <= len(self.pool):
            self._arm()

    def durations(self):
        out = {}
        for call in self.calls:
            for kind, a, b in call:
                out.setdefault(kind, []).append(a.elapsed_time(b))
        return out


# ----------------------------------------------------------- expert cache
class ExpertCache:
    """moe_cache over pinned host pools of n_layers layers (see moe.h).

    ``global_slots=0``: per-layer mode, ``n_slots`` slots per layer.
    ``global_slots=M``: global mode, one pool of M slots shared by every
    layer with ``n_slots`` of them in use (``resize`` changes that)."""

    def __init__(self, host_gate, host_up, host_down, qtype, n_slots: int, copy_stream,
                 device="cuda", global_slots: int = 0):
        # host_* : lists (one per layer) of pinned uint8 tensors [E, rows, bytes]
        self.n_layers = len(host_gate)
        self.E = host_gate[0].shape[0]
        self.n_slots = n_slots
        self.qtype = _qt(qtype)
        self.host = (host_gate, host_up, host_down)
        for lst in self.host:
            for t in lst:
                if t.is_cuda or not t.is_pinned():
                    raise ValueError("host pools must be pinned host tensors")
        bg, bu, bd = (lst[0][0].numel() for lst in self.host)
        self.bytes = (bg, bu, bd)
        dev = torch.device(device)
        self.global_slots = int(global_slots)
        lead = (self.global_slots,) if self.global_slots else (self.n_layers, n_slots)
        self.dev_gate = torch.empty(lead + tuple(host_gate[0].shape[1:]), dtype=torch.uint8, device=dev)
        self.dev_up = torch.empty(lead + tuple(host_up[0].shape[1:]), dtype=torch.uint8, device=dev)
        self.dev_down = torch.empty(lead + tuple(host_down[0].shape[1:]), dtype=torch.uint8, device=dev)
        self.slot_map = torch.full((self.n_layers, self.E), -1, dtype=torch.int32, device=dev)
        # per layer: [hit mask, miss mask] of the last request
        self.masks = torch.zeros((self.n_layers, 2, self.E), dtype=torch.uint8, device=dev)
        self.copy_stream = copy_stream
        arr = lambda lst: (C.c_void_p * self.n_layers)(*[t.data_ptr() for t in lst])
        self._ptrs = [arr(l) for l in self.host]
        d = CacheDesc()
        d.n_layers, d.E, d.n_slots, d.qtype = self.n_layers, self.E, n_slots, self.qtype
        d.bytes_gate, d.bytes_up, d.bytes_down = bg, bu, bd
        d.host_gate = C.cast(self._ptrs[0], C.POINTER(C.c_void_p))
        d.host_up = C.cast(self._ptrs[1], C.POINTER(C.c_void_p))
        d.host_down = C.cast(self._ptrs[2], C.POINTER(C.c_void_p))
        d.dev_gate, d.dev_up, d.dev_down = (self.dev_gate.data_ptr(), self.dev_up.data_ptr(),
                                            self.dev_down.data_ptr())
        d.dev_slot_map = self.slot_map.data_ptr()
        d.copy_stream = copy_stream.cuda_stream
        d.dev_masks = self.masks.data_ptr()
        d.global_ = 1 if self.global_slots else 0
        d.max_slots = self.global_slots
        self._desc = d
        h = C.c_void_p()
        _check(lib().moe_cache_init(C.byref(d), C.byref(h)))
        self._h = h
        self.pools = []
        for l in range(self.n_layers):
            p = Pool()
            _check(lib().moe_cache_layer_pool(self._h, l, C.byref(p)))
            ep = ExpertPool.__new__(ExpertPool)
            if self.global_slots:
                ep.gate, ep.up, ep.down = self.dev_gate, self.dev_up, self.dev_down
            else:
                ep.gate, ep.up, ep.down = self.dev_gate[l], self.dev_up[l], self.dev_down[l]
            ep.qtype, ep.slot_of_expert, ep.c = self.qtype, self.slot_map[l], p
            self.pools.append(ep)

    def request(self, layer: int, ids, stream=None):
        """ids: host int sequence.  Returns (slots, miss, evicted) numpy arrays."""
        import numpy as np
        ids = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
        n = len(ids)
        slots = np.empty(n, np.int32)
        miss = np.empty(n, np.int32)
        ev = np.empty(n, np.int32)
        nm = C.c_int(0)
        f = lambda a: a.ctypes.data_as(C.c_void_p)
        _check(lib().moe_cache_request(self._h, layer, f(ids), n, f(slots), f(miss), f(ev),
                                       C.byref(nm), _stream(stream)))
        return slots, miss.astype(bool), ev

    def resize(self, n_slots: int, stream=None):
        """Global mode: change the capacity at run time -> (evicted, moved)."""
        ne, nm = C.c_int(0), C.c_int(0)
        _check(lib().moe_cache_resize(self._h, int(n_slots), C.byref(ne), C.byref(nm), _stream(stream)))
        return ne.value, nm.value

    def hit_mask(self, layer: int):
        """Device uint8 [E]: experts of the layer's last request already resident."""
        return self.masks[layer, 0]

    def miss_mask(self, layer: int):
        """Device uint8 [E]: experts the layer's last request copied."""
        return self.masks[layer, 1]

    def sync(self, layer: int, stream=None):
        _check(lib().moe_cache_sync(self._h, layer, _stream(stream)))

    def release(self, layer: int, stream=None):
        """Every kernel reading the layer's slots for its last request is enqueued."""
        _check(lib().moe_cache_release(self._h, layer, _stream(stream)))

    def stats(self):
        """(hits, misses, bytes copied)."""
        h, m, b = C.c_int64(), C.c_int64(), C.c_int64()
        _check(lib().moe_cache_stats(self._h, C.byref(h), C.byref(m), C.byref(b), None))
        return h.value, m.value, b.value

    def exposed_ns(self):
        """Time the compute stream has waited in sync() for copies (ns);
        waits for the compute stream to pass its pending sync points."""
        e = C.c_int64()
        _check(lib().moe_cache_stats(self._h, None, None, None, C.byref(e)))
        return e.value

    def inject_copy_failure(self, nth: int):
        lib().moe_cache_debug_fail_copy(self._h, nth)

    def close(self):
        if getattr(self, "_h", None):
            lib().moe_cache_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# -------------------------------------------------- prefill layer streaming
class LayerStreamer:
    """moe_streamer: whole layers of experts double-buffered from pinned host
    memory (see moe.h).  host_* are lists (one per layer) of pinned uint8
    tensors [E, rows, bytes]; two device buffers of one layer each are
    allocated here."""

    def __init__(self, host_gate, host_up, host_down, qtype, copy_stream, device="cuda"):
        self.n_layers = len(host_gate)
        self.E = host_gate[0].shape[0]
        self.qtype = _qt(qtype)
        self.host = (host_gate, host_up, host_down)
        for lst in self.host:
            for t in lst:
                if t.is_cuda or not t.is_pinned():
                    raise ValueError("host pools must be pinned host tensors")
        dev = torch.device(device)
        self.bufs = [[torch.empty(lst[0].shape, dtype=torch.uint8, device=dev) for lst in self.host]
                     for _ in range(2)]
        arr = lambda lst: (C.c_void_p * self.n_layers)(*[t.data_ptr() for t in lst])
        self._ptrs = [arr(l) for l in self.host]
        d = StreamerDesc()
        d.n_layers, d.E, d.qtype = self.n_layers, self.E, self.qtype
        d.bytes_gate, d.bytes_up, d.bytes_down = (lst[0][0].numel() for lst in self.host)
        d.host_gate = C.cast(self._ptrs[0], C.POINTER(C.c_void_p))
        d.host_up = C.cast(self._ptrs[1], C.POINTER(C.c_void_p))
        d.host_down = C.cast(self._ptrs[2], C.POINTER(C.c_void_p))
        for b in range(2):
            d.dev_gate[b], d.dev_up[b], d.dev_down[b] = (t.data_ptr() for t in self.bufs[b])
        d.copy_stream = copy_stream.cuda_stream
        self.copy_stream = copy_stream
        self._desc = d
        h = C.c_void_p()
        _check(lib().moe_streamer_init(C.byref(d), C.byref(h)))
        self._h = h
        self._pools = [None, None]

    def prefetch(self, layer: int):
        _check(lib().moe_streamer_prefetch(self._h, layer))

    def acquire(self, layer: int, stream=None) -> ExpertPool:
        """The layer's pool view (valid for work enqueued on ``stream`` after this)."""
        p = Pool()
        _check(lib().moe_streamer_acquire(self._h, layer, _stream(stream), C.byref(p)))
        ep = ExpertPool.__new__(ExpertPool)
        b = self.bufs[layer & 1]
        ep.gate, ep.up, ep.down = b
        ep.qtype, ep.slot_of_expert, ep.c = self.qtype, None, p
        return ep

    def release(self, layer: int, stream=None):
        _check(lib().moe_streamer_release(self._h, layer, _stream(stream)))

    def stats(self):
        """(bytes copied, exposed ns)."""
        b, e = C.c_int64(), C.c_int64()
        _check(lib().moe_streamer_stats(self._h, C.byref(b), C.byref(e)))
        return b.value, e.value

    def close(self):
        if getattr(self, "_h", None):
            lib().moe_streamer_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
