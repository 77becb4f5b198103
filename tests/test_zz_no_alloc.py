"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Such callers (code inside an allocator's callbacks, serving loops that freeze
their memory after start-up, embedders whose runtime owns all device memory)
get the small-batch router with its scratch in a fixed array inside the
library.  This file is collected last on purpose.  It checks, through the
C ABI, that two consecutive calls of the allocation-free entry point select
the oracle's experts (a selection decided by a logit gap under 1e-5 is
logged, as in every routing test), agree with moe_route on every other
token, and give gates and logits within the tolerances the other routing
tests use; and that sizes over the array's limit are refused.  The two
entry points run different kernels (a split-K reduction here, a cluster
reduction in moe_route for T <= 16), so their fp32 logits may differ in
the last bits and a near tie may go either way.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import synthetic as S
from helpers import GATE_TOL, TIE_EPS, check_ids, dev, dev_x, oracle_route

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(moe):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return moe.lib()


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _route_both(moe, lib, name, T):
    Li = S.make_layer(S.CONFIGS[name], T=T, experts=False)
    cfg = Li.cfg
    x, w, b = dev_x(Li), dev(Li.w_router), dev(Li.bias)
    D, E, k = cfg.D, cfg.E, cfg.k
    xdt = moe.BF16 if cfg.x_dtype == "bf16" else moe.F32
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    # the existing entry point, with its caller-owned workspace
    ref_ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    ref_g = torch.empty((T, k), dtype=torch.float32, device="cuda")
    ref_l = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ws = torch.zeros(lib.moe_route_workspace_size(T, D, E, k), dtype=torch.uint8, device="cuda")
    assert lib.moe_route(_p(x), xdt, _p(w), _p(b), T, D, E, k, 1, _p(ref_ids), _p(ref_g),
                         _p(ref_l), _p(ws), ws.numel(), stream) == 0
    outs = []
    for _ in range(2):     # two calls in a row: the second sees the first's leftovers
        ids = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
        g = torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda")
        lg = torch.full((T, E), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.moe_route_noalloc(_p(x), xdt, _p(w), _p(b), T, D, E, k, 1, _p(ids), _p(g),
                                   _p(lg), stream)
        assert st == 0, lib.moe_last_error().decode()
        outs.append((ids, g, lg))
    torch.cuda.synchronize()
    orc_logits, orc_ids, _ = oracle_route(Li)
    ties = set(oracle.near_tie_tokens(orc_logits, k, TIE_EPS).tolist())
    ref_ids_h, ref_g_h = ref_ids.cpu().numpy(), ref_g.cpu().numpy()
    for ids, g, lg in outs:
        ids_h, g_h, lg_h = ids.cpu().numpy(), g.cpu().numpy(), lg.cpu().numpy()
        check_ids(ids_h, orc_ids, orc_logits, k, log=print)
        same = np.array([t not in ties for t in range(T)])
        np.testing.assert_array_equal(ids_h[same], ref_ids_h[same])
        assert np.abs(g_h[same] - ref_g_h[same]).max(initial=0.0) <= GATE_TOL
        scale = 1.0 + np.abs(orc_logits)
        assert np.all(np.abs(lg_h - orc_logits) <= 2e-5 * scale)
        assert np.abs(lg_h - ref_l.cpu().numpy()).max() <= 1e-5


@pytest.mark.parametrize("name,T", [("tiny", 4), ("decode", 1), ("decode", 16)])
def test_noalloc_route_matches_route(moe, L, name, T):
    _route_both(moe, L, name, T)


def test_noalloc_route_refuses_sizes_over_its_limit(moe, L):
    x = torch.zeros((17, 2048), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((2048, 128), dtype=torch.float32, device="cuda")
    ids = torch.empty((17, 8), dtype=torch.int32, device="cuda")
    g = torch.empty((17, 8), dtype=torch.float32, device="cuda")
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    # T above 16
    assert L.moe_route_noalloc(_p(x), moe.BF16, _p(w), None, 17, 2048, 128, 8, 1, _p(ids), _p(g),
                               None, s) == 3
    assert "T <= 16" in L.moe_last_error().decode()
    # scratch: ceil(8192/32) * 16 * 256 floats > 524288
    x2 = torch.zeros((16, 8192), dtype=torch.bfloat16, device="cuda")
    w2 = torch.zeros((8192, 256), dtype=torch.float32, device="cuda")
    assert L.moe_route_noalloc(_p(x2), moe.BF16, _p(w2), None, 16, 8192, 256, 8, 1, _p(ids),
                               _p(g), None, s) == 3
    assert "scratch" in L.moe_last_error().decode()
