"""The C-ABI boundary on the host: the library loads, exports every symbol
that include/moe.h declares, its tables match the header, and bad arguments
come back as status codes before any kernel is enqueued (no GPU needed)."""
import ctypes as C
import os
import re

import pytest

import synthetic as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def _header_defines():
    out = {}
    for m in re.finditer(r"#define\s+(MOE_\w+)\s+(\d+)", open(HEADER).read()):
        out[m.group(1)] = int(m.group(2))
    return out


def test_every_declared_symbol_is_exported(moe):
    names = _declared_functions()
    assert len(names) >= 17
    L = C.CDLL(moe.LIB_PATH)
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_block_tables_agree_with_header(moe, orc):
    h = _header_defines()
    assert h["MOE_QK"] == S.QK == 32
    assert h["MOE_QK_K"] == S.QK_K == 256
    for q in S.QTYPES:
        qid = moe.QTYPES[q]
        assert qid == S.GGML_TYPE_ID[q]
        assert h[f"MOE_{q.upper()}_BLOCK_BYTES"] == S.BLOCK_BYTES[q] == moe.BLOCK_BYTES[qid]
        assert moe.lib().moe_block_bytes(qid) == S.BLOCK_BYTES[q] == orc.block_bytes(q)
        assert moe.lib().moe_block_weights(qid) == S.BLOCK_WEIGHTS[q] == orc.block_weights(q) \
            == moe.BLOCK_WEIGHTS[qid]
    for unknown in (0, 1, 4, 5, 9, 10, 11, 13, 15, -1):    # unknown type -> 0, never garbage
        assert moe.lib().moe_block_bytes(unknown) == 0
        assert moe.lib().moe_block_weights(unknown) == 0
    assert set(moe.QTYPES) == set(S.QTYPES)


def _err(L):
    return L.moe_last_error().decode()


P = C.c_void_p
FAKE = C.c_void_p(0x1000)      # never dereferenced: every call below fails its checks first


def test_route_argument_errors(moe):
    L = moe.lib()
    ws, n = FAKE, 1 << 20
    # k > E
    assert L.moe_route(FAKE, moe.BF16, FAKE, None, 4, 256, 8, 9, 1, FAKE, FAKE, None, ws, n, None) == 3
    assert "k" in _err(L)
    # D not a multiple of 32
    assert L.moe_route(FAKE, moe.BF16, FAKE, None, 4, 100, 8, 2, 1, FAKE, FAKE, None, ws, n, None) == 3
    # bad dtype, bad renorm flag
    assert L.moe_route(FAKE, 7, FAKE, None, 4, 256, 8, 2, 1, FAKE, FAKE, None, ws, n, None) == 1
    assert L.moe_route(FAKE, moe.BF16, FAKE, None, 4, 256, 8, 2, 2, FAKE, FAKE, None, ws, n, None) == 1
    # given logits must be F32
    assert L.moe_route(FAKE, moe.BF16, None, None, 4, 0, 8, 2, 1, FAKE, FAKE, None, ws, n, None) == 1
    # NULL outputs
    assert L.moe_route(FAKE, moe.BF16, FAKE, None, 4, 256, 8, 2, 1, None, FAKE, None, ws, n, None) == 1
    # workspace too small
    assert L.moe_route(FAKE, moe.BF16, FAKE, None, 4, 256, 8, 2, 1, FAKE, FAKE, None, ws, 1, None) == 7
    # too many experts
    assert L.moe_route(FAKE, moe.BF16, FAKE, None, 4, 256, 2048, 2, 1, FAKE, FAKE, None, ws, n, None) == 3
    # T == 0 is a successful no-op
    assert L.moe_route(None, moe.BF16, FAKE, None, 0, 256, 8, 2, 1, None, None, None, None, 0, None) == 0


def test_expert_ffn_rejects_unknown_and_missing_pools(moe):
    L = moe.lib()
    bad = moe.Pool(9, 8, 0x1000, 0x1000, 0x1000, None)       # type 9 (Q8_1) is not supported
    assert L.moe_expert_ffn(FAKE, moe.BF16, 4, 256, 512, 8, 2, FAKE, FAKE, C.byref(bad), None,
                            FAKE, FAKE, 1 << 30, None) == 2
    assert "quant type" in _err(L)
    nul = moe.Pool(moe.Q8_0, 8, 0x1000, 0, 0x1000, None)
    assert L.moe_expert_ffn(FAKE, moe.BF16, 4, 256, 512, 8, 2, FAKE, FAKE, C.byref(nul), None,
                            FAKE, FAKE, 1 << 30, None) == 1
    # K-quant blocks hold 256 weights: D or F not a multiple of 256 is a shape error
    for qk in (moe.Q4_K, moe.Q6_K):
        kp = moe.Pool(qk, 8, 0x1000, 0x1000, 0x1000, None)
        for D, F in ((256, 384), (384, 256), (96, 512)):
            assert L.moe_expert_ffn(FAKE, moe.BF16, 4, D, F, 8, 2, FAKE, FAKE, C.byref(kp), None,
                                    FAKE, FAKE, 1 << 30, None) == 3
            assert "multiples of 256" in _err(L)
    ok = moe.Pool(moe.Q8_0, 8, 0x1000, 0x1000, 0x1000, None)
    # F not a multiple of 32
    assert L.moe_expert_ffn(FAKE, moe.BF16, 4, 256, 500, 8, 2, FAKE, FAKE, C.byref(ok), None,
                            FAKE, FAKE, 1 << 30, None) == 3
    # workspace too small
    assert L.moe_expert_ffn(FAKE, moe.BF16, 4, 256, 512, 8, 2, FAKE, FAKE, C.byref(ok), None,
                            FAKE, FAKE, 16, None) == 7
    # scratch for the hidden activations: fp16 rows on the small-batch path,
    # fp32 rows on the general one (D=96 has no small-batch kernel)
    assert L.moe_expert_ffn_workspace_size(4, 2, 256, 512) >= 4 * 2 * 512 * 2
    assert L.moe_expert_ffn_workspace_size(4, 2, 96, 512) >= 4 * 2 * 512 * 4


def test_combine_and_permute_errors(moe):
    L = moe.lib()
    assert L.moe_combine(FAKE, FAKE, FAKE, 4, 2, 256, None, FAKE, 9, None) == 1
    assert L.moe_combine(None, FAKE, FAKE, 4, 2, 256, None, FAKE, moe.F32, None) == 1
    assert L.moe_permute(FAKE, 4, 3, 2, FAKE, FAKE, FAKE, FAKE, None) == 3     # k > E
    assert L.moe_permute(FAKE, 4, 2, 8, None, FAKE, FAKE, FAKE, None) == 1


def test_layer_forward_errors(moe):
    L = moe.lib()
    pool = moe.Pool(moe.Q4_0, 8, 0x1000, 0x1000, 0x1000, None)
    a = moe.LayerArgs()
    a.T, a.D, a.E, a.k, a.F, a.renorm = 4, 256, 8, 2, 512, 1
    a.x_dtype, a.y_dtype = moe.BF16, moe.BF16
    a.x, a.y, a.w_router = 0x1000, 0x1000, 0x1000
    a.pool = C.pointer(pool)
    need = L.moe_layer_workspace_size(C.byref(a))
    assert need > 0
    assert L.moe_layer_forward(C.byref(a), FAKE, need - 1, None) == 7
    a.y_dtype = moe.F16
    assert L.moe_layer_forward(C.byref(a), FAKE, need, None) == 1
    a.y_dtype = moe.BF16
    sh = moe.Pool(moe.Q8_0, 1, 0x1000, 0x1000, 0x1000, None)
    a.shared = C.pointer(sh)
    a.shared_F = 100
    assert L.moe_layer_forward(C.byref(a), FAKE, 1 << 40, None) == 3
    a.shared_F = 512
    badpool = moe.Pool(5, 8, 0x1000, 0x1000, 0x1000, None)
    a.pool = C.pointer(badpool)
    assert L.moe_layer_forward(C.byref(a), FAKE, 1 << 40, None) == 2
    assert L.moe_layer_forward(None, FAKE, 0, None) == 1


def test_cache_init_argument_errors(moe):
    L = moe.lib()
    h = C.c_void_p()
    assert L.moe_cache_init(None, C.byref(h)) == 1
    d = moe.CacheDesc()
    d.n_layers, d.E, d.n_slots, d.qtype = 2, 8, 9, moe.Q8_0      # more slots than experts
    assert L.moe_cache_init(C.byref(d), C.byref(h)) == 3
    d.n_slots, d.qtype = 4, 9
    assert L.moe_cache_init(C.byref(d), C.byref(h)) == 2
    d.qtype = moe.Q8_0
    assert L.moe_cache_init(C.byref(d), C.byref(h)) == 1          # NULL pools
    assert not h.value


def test_error_message_is_per_call(moe):
    L = moe.lib()
    L.moe_permute(FAKE, 4, 3, 2, FAKE, FAKE, FAKE, FAKE, None)
    assert _err(L)
    assert L.moe_route(None, moe.BF16, FAKE, None, 0, 256, 8, 2, 1, None, None, None, None, 0, None) == 0
    assert _err(L) == ""


def test_workspace_status_and_phase_errors(moe):
    L = moe.lib()
    code = C.c_int32(-1)
    assert L.moe_workspace_status(None, C.byref(code), 1, None) == 1
    assert L.moe_workspace_status(FAKE, None, 1, None) == 1
    pool = moe.Pool(moe.Q4_0, 8, 0x1000, 0x1000, 0x1000, None)
    a = moe.LayerArgs()
    a.T, a.D, a.E, a.k, a.F, a.renorm = 4, 256, 8, 2, 512, 1
    a.x_dtype, a.y_dtype = moe.BF16, moe.BF16
    a.x, a.y, a.w_router = 0x1000, 0x1000, 0x1000
    a.pool = C.pointer(pool)
    a.phases = 16                       # no such phase bit
    assert L.moe_layer_forward(C.byref(a), FAKE, 1 << 40, None) == 1
    assert "phases" in _err(L)
    a.phases = moe.PHASE_COMBINE        # combining needs y
    a.y = None
    assert L.moe_layer_forward(C.byref(a), FAKE, 1 << 40, None) == 1
    a.phases, a.y = moe.PHASE_ROUTE, None   # routing alone writes no y
    a.w_router = None                       # ... but needs a router or logits
    assert L.moe_layer_forward(C.byref(a), FAKE, 1 << 40, None) == 1


def test_cache_stats_rejects_null_cache(moe):
    L = moe.lib()
    assert L.moe_cache_stats(None, None, None, None, None) == 1


def test_device_status_codes_agree_with_header(moe):
    src = open(HEADER).read()
    names = ["MOE_DEV_OK", "MOE_DEV_TIMEOUT_FULL", "MOE_DEV_TIMEOUT_EMPTY", "MOE_DEV_TIMEOUT_DRAIN",
             "MOE_DEV_BAD_SLOT", "MOE_DEV_TIMEOUT_MMA"]
    vals = [int(re.search(n + r"\s*=\s*(\d+)", src).group(1)) for n in names]
    assert vals == [moe.DEV_OK, moe.DEV_TIMEOUT_FULL, moe.DEV_TIMEOUT_EMPTY, moe.DEV_TIMEOUT_DRAIN,
                    moe.DEV_BAD_SLOT, moe.DEV_TIMEOUT_MMA]
    ph = {n: int(v, 0) for n, v in re.findall(r"#define\s+(MOE_PHASE_\w+)\s+(\w+?)u", src)}
    assert ph == {"MOE_PHASE_ROUTE": moe.PHASE_ROUTE, "MOE_PHASE_FFN": moe.PHASE_FFN,
                  "MOE_PHASE_SHARED": moe.PHASE_SHARED, "MOE_PHASE_COMBINE": moe.PHASE_COMBINE,
                  "MOE_PHASE_ALL": moe.PHASE_ALL}


def test_global_cache_arguments(moe):
    L = moe.lib()
    h = C.c_void_p()
    d = moe.CacheDesc()
    d.n_layers, d.E, d.n_slots, d.qtype = 2, 8, 6, moe.Q8_0
    d.global_, d.max_slots = 1, 4                     # capacity above the pool
    assert L.moe_cache_init(C.byref(d), C.byref(h)) == 3
    d.max_slots = 17                                  # more than n_layers * E
    assert L.moe_cache_init(C.byref(d), C.byref(h)) == 3
    d.global_ = 2
    assert L.moe_cache_init(C.byref(d), C.byref(h)) == 1
    assert not h.value
    ne, nm = C.c_int(-1), C.c_int(-1)
    assert L.moe_cache_resize(None, 4, C.byref(ne), C.byref(nm), None) == 1
    assert ne.value == 0 and nm.value == 0


def test_streamer_arguments(moe):
    L = moe.lib()
    h = C.c_void_p()
    assert L.moe_streamer_init(None, C.byref(h)) == 1
    d = moe.StreamerDesc()
    d.n_layers, d.E, d.qtype = 2, 8, 9                 # unknown quant type
    assert L.moe_streamer_init(C.byref(d), C.byref(h)) == 2
    d.qtype = moe.Q8_0
    assert L.moe_streamer_init(C.byref(d), C.byref(h)) == 1   # NULL pools
    d.n_layers = 0
    assert L.moe_streamer_init(C.byref(d), C.byref(h)) == 3
    assert not h.value
    assert L.moe_streamer_prefetch(None, 0) == 1
    assert L.moe_streamer_stats(None, None, None) == 1


def test_layer_forward_act_bits_errors(moe):
    # 8-bit activations: a bad act_bits, a type other than Q4_0/Q8_0, and a
    # shape outside the decode kernels are refused before any kernel runs
    L = moe.lib()

    def args(qtype, T=4, act_bits=8):
        pool = moe.Pool(qtype, 8, 0x1000, 0x1000, 0x1000, None)
        a = moe.LayerArgs()
        a.T, a.D, a.E, a.k, a.F, a.renorm = T, 256, 8, 2, 512, 1
        a.x_dtype, a.y_dtype = moe.BF16, moe.BF16
        a.x, a.y, a.w_router = 0x1000, 0x1000, 0x1000
        a.pool = C.pointer(pool)
        a.act_bits = act_bits
        return a, pool

    a, _p = args(moe.Q4_0, act_bits=5)
    assert L.moe_layer_forward(C.byref(a), FAKE, 1 << 40, None) == 1
    assert "act_bits" in _err(L)
    for q in (moe.Q5_0, moe.Q4_1, moe.Q4_K):
        a, _p = args(q)
        assert L.moe_layer_forward(C.byref(a), FAKE, 1 << 40, None) == 2
        assert "8-bit activations" in _err(L)
    a, _p = args(moe.Q8_0, T=32)
    assert L.moe_layer_forward(C.byref(a), FAKE, 1 << 40, None) == 3
    assert "decode shapes" in _err(L)
    # a valid 8-bit call sizes its own workspace (h codes instead of fp16 rows)
    a8, _p = args(moe.Q8_0)
    a16, _p2 = args(moe.Q8_0, act_bits=0)
    assert L.moe_layer_workspace_size(C.byref(a8)) != L.moe_layer_workspace_size(C.byref(a16))


def test_selftest_wait_timeout_argument_errors(moe):
    L = moe.lib()
    # 7 = MOE_ERR_WORKSPACE, 1 = MOE_ERR_INVALID_ARG; nothing is launched
    assert L.moe_selftest_wait_timeout(None, 64, 1000, None) == 7
    assert L.moe_selftest_wait_timeout(FAKE, 16, 1000, None) == 7
    assert L.moe_selftest_wait_timeout(FAKE, 64, 0, None) == 1
    assert L.moe_selftest_wait_timeout(FAKE, 64, 5_000_000_000, None) == 1
    assert "budget" in _err(L)
