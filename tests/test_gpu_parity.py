"""CUDA path vs the CPU oracle, element by element, on seeded inputs.

Routing indices and the permutation must be bit-exact (a selection decided
by a logit gap under 1e-5 is logged instead); gates within 1e-6; layer
outputs within max|gpu-oracle|/max|oracle| <= 2e-3.  Full-size configs are
compared on sampled tokens/rows the oracle computes one by one, in the same
launch configuration the bench times (moe_layer_forward).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from helpers import (GATE_TOL, REL_TOL, check_ids, dev, dev_pool, dev_shared, dev_x,
                     gates_at, oracle_route, rel_err)

pytestmark = pytest.mark.gpu

_cache = {}


def layer_inputs(name, T=None, seed=None):
    key = (name, T, seed)
    if key not in _cache:
        _cache[key] = S.make_layer(S.CONFIGS[name], T=T, seed=seed)
    return _cache[key]


@pytest.fixture(scope="module", autouse=True)
def _cuda(moe):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    _cache.clear()


def _route_gpu(moe, L):
    if L.logits is not None:
        return moe.route(dev(L.logits), None, dev(L.bias), L.cfg.k, L.cfg.renorm, want_logits=True)
    return moe.route(dev_x(L), dev(L.w_router), dev(L.bias), L.cfg.k, L.cfg.renorm,
                     want_logits=True)


ROUTE_CASES = [("tiny", None), ("decode", 1), ("decode", 4), ("decode", 16), ("decode", 17),
               ("decode", 37), ("prefill", 8192), ("wide", 1), ("wide", 2048)]


@pytest.mark.parametrize("name,T", ROUTE_CASES)
def test_route_parity(moe, name, T):
    L = layer_inputs(name, T)
    ids, gates, logits = _route_gpu(moe, L)
    torch.cuda.synchronize()
    ref_logits, ref_ids, ref_g = oracle_route(L)
    ids, gates, logits = ids.cpu().numpy(), gates.cpu().numpy(), logits.cpu().numpy()
    scale = 1.0 + np.abs(ref_logits)
    assert np.all(np.abs(logits - ref_logits) <= 2e-5 * scale)
    check_ids(ids, ref_ids, ref_logits, L.cfg.k, log=print)
    # (a) the gate arithmetic: softmax/renormalisation of the GPU's own fp32
    # logits at the GPU's selection, to 1e-6
    assert np.abs(gates - gates_at(logits, ids, L.cfg.renorm)).max() <= GATE_TOL
    # (b) end to end against the oracle's logits: 1e-6 plus the propagated
    # fp32 logit error (|dg_j| <= g_j * 2 max_i |dL_i| <= 2 max_i |dL_i|)
    dL = np.abs(logits.astype(np.float64) - ref_logits).max(axis=1, keepdims=True)
    g_ref = gates_at(ref_logits, ids, L.cfg.renorm)
    assert np.all(np.abs(gates - g_ref) <= GATE_TOL + 2 * dL)
    assert np.all(np.abs(gates.sum(axis=1) - 1) <= 1e-5)


def test_route_ties_and_extremes(moe):
    # exact ties in the logits go to the lower expert id; E=1024, k=32
    rng = np.random.default_rng(3)
    E, k, T = 1024, 32, 5
    Lg = rng.standard_normal((T, E)).astype(np.float32)
    Lg[0, :] = 0.0                         # all equal -> ids 0..k-1
    Lg[1, 100:140] = 5.0                   # a block of equal maxima
    ids, gates = moe.route(dev(Lg), None, None, k)
    torch.cuda.synchronize()
    ref_ids, ref_g = oracle.select(Lg, k)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    assert np.abs(gates.cpu().numpy() - ref_g).max() <= GATE_TOL
    # k = E
    ids2, g2 = moe.route(dev(Lg[:, :8].copy()), None, None, 8)
    r2, rg2 = oracle.select(Lg[:, :8], 8)
    np.testing.assert_array_equal(ids2.cpu().numpy(), r2)
    assert np.abs(g2.cpu().numpy() - rg2).max() <= GATE_TOL


def test_route_without_renorm(moe):
    L = layer_inputs("tiny")
    ids, gates = moe.route(dev_x(L), dev(L.w_router), None, L.cfg.k, renorm=False)
    logits, ref_ids, _ = oracle.route(L.x, L.w_router, None, L.cfg.k)
    ref_ids2, ref_g = oracle.select(logits, L.cfg.k, renorm=False)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids2)
    assert np.abs(gates.cpu().numpy() - ref_g).max() <= GATE_TOL


@pytest.mark.parametrize("T,k,E", [(1, 8, 128), (16, 8, 128), (37, 2, 8), (8192, 8, 128),
                                   (2048, 10, 512), (3, 32, 1024), (1000, 1, 1)])
def test_permute_parity(moe, T, k, E):
    rng = np.random.default_rng(T * 31 + k)
    if E == 128 and T == 8192:       # skewed, like the prefill routing
        p = (np.arange(1, E + 1) ** -1.1)
        p /= p.sum()
        ids = np.stack([rng.choice(E, k, replace=False, p=p) for _ in range(T)])
    else:
        ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    ids = ids.astype(np.int32)
    counts, offsets, perm, inv = moe.permute(dev(ids), E)
    torch.cuda.synchronize()
    rc, ro, rp, ri = oracle.permute(ids, E)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(offsets.cpu().numpy(), ro)
    np.testing.assert_array_equal(perm.cpu().numpy(), rp)
    np.testing.assert_array_equal(inv.cpu().numpy(), ri)


def _sample(n, m, seed):
    if n <= m:
        return np.arange(n, dtype=np.int32)
    rng = np.random.default_rng(seed)
    s = np.sort(rng.choice(n, m, replace=False)).astype(np.int32)
    s[0], s[-1] = 0, n - 1                 # both ends of the range
    return np.unique(s)


@pytest.mark.parametrize("name,T,n_rows", [("tiny", None, 999), ("decode", 16, 999),
                                           ("decode", 5, 999), ("prefill", 8192, 40),
                                           ("wide", 2048, 40)])
def test_expert_ffn_and_combine_parity(moe, name, T, n_rows):
    L = layer_inputs(name, T)
    cfg = L.cfg
    ids_d, gates_d = _route_gpu(moe, L)[:2]
    counts, offsets, perm, inv = moe.permute(ids_d, cfg.E)
    pool = dev_pool(moe, L)
    rows = moe.expert_ffn(dev_x(L), perm, offsets, pool, cfg.k, cfg.F)
    y = moe.combine(rows, inv, gates_d, y_dtype=torch.float32)
    torch.cuda.synchronize()
    Tn = L.x.shape[0]
    pos = _sample(Tn * cfg.k, n_rows, 11)
    ref = oracle.expert_rows(L.x, perm.cpu().numpy(), offsets.cpu().numpy(), cfg.k, L.gate,
                             L.up, L.down, cfg.qtype, cfg.F, positions=pos)
    got = rows.cpu().numpy()[pos]
    assert rel_err(got, ref) <= REL_TOL
    # combine of the GPU rows, recomputed in double from the same rows
    toks = _sample(Tn, 64, 12)
    rows_h, inv_h, g_h = rows.cpu().numpy().astype(np.float64), inv.cpu().numpy(), gates_d.cpu().numpy()
    yref = np.stack([sum(g_h[t, j] * rows_h[inv_h[t * cfg.k + j]] for j in range(cfg.k)) for t in toks])
    assert np.abs(y.cpu().numpy()[toks] - yref).max() <= 1e-5 * np.abs(yref).max()


def _layer(moe, L, T_max=None):
    cfg = L.cfg
    T = L.x.shape[0]
    shared = dev_shared(moe, L)
    xdt = torch.bfloat16 if cfg.x_dtype == "bf16" else torch.float32
    ydt = torch.bfloat16 if cfg.y_dtype == "bf16" else torch.float32
    return moe.Layer(dev_pool(moe, L), cfg.D, cfg.F, cfg.E, cfg.k, T_max or T,
                     w_router=dev(L.w_router), bias=dev(L.bias), shared=shared,
                     shared_F=cfg.shared_F, renorm=cfg.renorm, x_dtype=xdt, y_dtype=ydt)


def _check_layer(moe, L, y_gpu, ids_gpu, n_tok, log=print, extra=None):
    """Parity of an fp32 layer output with the oracle on sampled tokens
    (plus the tokens listed in ``extra``)."""
    cfg = L.cfg
    T = L.x.shape[0]
    ref_logits, ref_ids, ref_g = oracle_route(L)
    ids_gpu = ids_gpu.cpu().numpy()[:T]
    tied = check_ids(ids_gpu, ref_ids, ref_logits, cfg.k, log=log)
    toks = _sample(T, n_tok, 13)
    if extra is not None and len(extra):
        toks = np.unique(np.concatenate([toks, np.asarray(extra, np.int32)]))
    # tokens whose selection differs (near ties) are checked against the
    # oracle run on the GPU's selection
    use_ids = ref_ids.copy()
    use_g = ref_g.copy()
    if tied:
        use_ids[tied] = ids_gpu[tied]
        use_g[tied] = gates_at(ref_logits[tied], ids_gpu[tied], cfg.renorm)
    ref = oracle.layer(L.x, use_ids, use_g, L.gate, L.up, L.down, cfg.qtype, cfg.F,
                       shared=L.shared, tokens=toks, shared_qtype=cfg.shared_qtype)
    got = y_gpu.float().cpu().numpy()[toks]
    err = rel_err(got, ref)
    assert err <= REL_TOL, err
    return err


LAYER_CASES = [("tiny", None, 99), ("decode", 1, 99), ("decode", 4, 99), ("decode", 16, 99),
               ("decode", 37, 99), ("prefill", 8192, 48), ("wide", 1, 99), ("wide", 2048, 40),
               ("cache", 1, 99), ("cache", 4, 99), ("cache", 16, 99)]


def _small_expert_tokens(ids, E, T, limit=10, max_tokens=64):
    """Tokens routed to an expert that receives fewer than ``limit`` entries
    (single, partial row tiles on the tensor-core path), at most max_tokens."""
    counts = np.bincount(ids[:T].ravel(), minlength=E)
    small = np.nonzero((counts > 0) & (counts < limit))[0]
    toks = np.unique(np.nonzero(np.isin(ids[:T], small).any(axis=1))[0])
    return toks[:max_tokens].astype(np.int32)


@pytest.mark.parametrize("name,T,n_tok", LAYER_CASES)
def test_layer_forward_parity(moe, name, T, n_tok):
    # the 2e-3 bar applies to the fp32-accumulated result (fp32 output); the
    # configured output type (bf16 for most configs) must then be exactly the
    # round-to-nearest-even of that fp32 result
    L = layer_inputs(name, T)
    lay = _layer(moe, L)
    Tn = L.x.shape[0]
    logits = None if L.logits is None else dev(L.logits)
    y32 = torch.empty((Tn, L.cfg.D), dtype=torch.float32, device="cuda")
    lay.forward(dev_x(L), logits=logits, out=y32)
    y = lay.forward(dev_x(L), logits=logits)
    torch.cuda.synchronize()
    extra = None
    if Tn > 16:   # aim at the experts with few tokens (partial row tiles)
        extra = _small_expert_tokens(lay.ids.cpu().numpy(), L.cfg.E, Tn)
    print(f"rel err {_check_layer(moe, L, y32, lay.ids, n_tok, extra=extra):.3e}")
    assert torch.equal(y, y32.to(y.dtype))
    assert moe.workspace_status(lay.ws) == (0, moe.DEV_OK)   # no bounded wait ran out


def test_layer_forward_repeated_calls_are_identical(moe):
    # the workspace carries state between calls (the router's ticket); a
    # second call must reproduce the first bit for bit
    L = layer_inputs("decode", 4)
    lay = _layer(moe, L)
    x = dev_x(L)
    y1 = lay.forward(x).clone()
    y2 = lay.forward(x).clone()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_layer_zero_tokens_is_noop(moe):
    L = layer_inputs("tiny")
    lay = _layer(moe, L, T_max=4)
    y = lay.forward(dev_x(L)[:0])
    torch.cuda.synchronize()
    assert y.shape == (0, L.cfg.D)


@pytest.mark.parametrize("qtype", ["q4_0", "q8_0"])
def test_layer_odd_shapes(moe, qtype):
    # D, F multiples of 32 but not of 256; E = k; ragged T
    cfg = S.LayerConfig("odd", T=7, D=96, E=3, k=3, F=160, qtype=qtype, x_dtype="bf16",
                        y_dtype="f32", router_std=0.1, seed=77)
    L = S.make_layer(cfg)
    lay = _layer(moe, L)
    y = lay.forward(dev_x(L))
    torch.cuda.synchronize()
    _check_layer(moe, L, y, lay.ids, 99)


def test_single_expert_layer(moe):
    cfg = S.LayerConfig("one", T=9, D=256, E=1, k=1, F=256, qtype="q8_0", x_dtype="f32",
                        y_dtype="f32", seed=78)
    L = S.make_layer(cfg)
    lay = _layer(moe, L)
    y = lay.forward(dev_x(L))
    torch.cuda.synchronize()
    _check_layer(moe, L, y, lay.ids, 99)
    assert np.all(lay.gates.cpu().numpy() == 1.0)


def test_layer_crowded_experts_with_shared(moe):
    # T=16 over 4 experts with a skewed router bias: experts with more than
    # 8 tokens (several MMA column groups) plus a shared expert over all 16
    cfg = S.LayerConfig("crowd", T=16, D=512, E=4, k=2, F=256, qtype="q4_0", x_dtype="bf16",
                        y_dtype="f32", router_std=0.05, zipf_s=1.5, shared_F=256, seed=79)
    L = S.make_layer(cfg)
    lay = _layer(moe, L)
    y = lay.forward(dev_x(L))
    torch.cuda.synchronize()
    counts = np.bincount(lay.ids.cpu().numpy()[:16].ravel(), minlength=4)
    assert counts.max() > 8, counts
    _check_layer(moe, L, y, lay.ids, 16)
    assert int(lay.ws[:4].view(torch.int32)[0]) == 0


def test_masked_two_phase_rows_are_bit_identical(moe):
    L = layer_inputs("decode", 16)
    cfg = L.cfg
    ids_d, gates_d = _route_gpu(moe, L)[:2]
    counts, offsets, perm, inv = moe.permute(ids_d, cfg.E)
    pool = dev_pool(moe, L)
    x = dev_x(L)
    full = moe.expert_ffn(x, perm, offsets, pool, cfg.k, cfg.F)
    rng = np.random.default_rng(4)
    m = torch.from_numpy(rng.integers(0, 2, cfg.E).astype(np.uint8)).cuda()
    two = torch.full_like(full, float("nan"))
    moe.expert_ffn(x, perm, offsets, pool, cfg.k, cfg.F, mask=m, out=two)
    moe.expert_ffn(x, perm, offsets, pool, cfg.k, cfg.F, mask=1 - m, out=two)
    torch.cuda.synchronize()
    assert torch.equal(full, two)


@pytest.mark.parametrize("name,T", [("decode", 1), ("decode", 16), ("wide", 1)])
def test_graph_replay_matches_eager(moe, name, T):
    # the bench replays captured CUDA graphs: the replayed layer must give the
    # eager call's output bit for bit (same kernels, same order)
    L = layer_inputs(name, T)
    lay = _layer(moe, L)
    x = dev_x(L)
    lg = None if L.logits is None else dev(L.logits)
    y_eager = lay.forward(x, logits=lg).clone()
    out = torch.empty_like(y_eager)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        lay.forward(x, logits=lg, out=out)
    out.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, y_eager)


# ------------------------------------------------ permutations the layer runs
# The fused layer permutes inside its routing kernels (the router cluster's
# CTA 0 for T <= 16 with a router; the select+permute kernel for given logits
# up to T = 64; the stand-alone kernel otherwise).  Layer outputs cannot see
# the order inside a segment, so each of them is compared with the oracle's
# stable counting sort directly.
PERM_CASES = [("tiny", None), ("decode", 1), ("decode", 4), ("decode", 16), ("wide", 1),
              ("cache", 1), ("cache", 16), ("wide", 64), ("decode", 37), ("prefill", 8192),
              ("wide", 2048)]


@pytest.mark.parametrize("name,T", PERM_CASES)
def test_layer_permutation_is_the_oracles(moe, name, T):
    L = layer_inputs(name, T)
    lay = _layer(moe, L)
    Tn = L.x.shape[0]
    bufs = lay.routing_buffers(Tn)
    logits = None if L.logits is None else dev(L.logits)
    lay.forward(dev_x(L), logits=logits, routing_out=bufs)
    torch.cuda.synchronize()
    ref_logits, ref_ids, _ = oracle_route(L)
    ids = lay.ids.cpu().numpy()[:Tn]
    check_ids(ids, ref_ids, ref_logits, L.cfg.k, log=print)
    # exact: the permutation of the ids the GPU selected
    want = oracle.permute(ids, L.cfg.E)
    for got, w, what in zip(bufs, want, ("counts", "offsets", "perm", "inv")):
        np.testing.assert_array_equal(got.cpu().numpy(), w, err_msg=what)


# ------------------------------------ tensor-core rows at the tile boundaries
def _aimed_positions(offsets, cap_small=10, seed=21, n_random=48):
    """Permuted positions where a tile-boundary slip would show: every row of
    each expert with fewer than cap_small rows, the first and last row of
    every segment, the first row of each segment's last 128-row tile, and a
    few random rows."""
    off = np.asarray(offsets, np.int64)
    pos = []
    for e in range(len(off) - 1):
        a, b = int(off[e]), int(off[e + 1])
        n = b - a
        if n == 0:
            continue
        if n < cap_small:
            pos.extend(range(a, b))
        pos.extend([a, b - 1, a + (n - 1) // 128 * 128])
    rng = np.random.default_rng(seed)
    pos.extend(rng.integers(0, int(off[-1]), n_random).tolist())
    return np.unique(np.asarray(pos, np.int32))


@pytest.mark.parametrize("name,T", [("prefill", 8192), ("wide", 2048), ("decode", 300)])
def test_tensor_core_rows_at_tile_edges(moe, name, T):
    # moe_expert_ffn at T > 16 runs the tcgen05 grouped GEMM (the fused
    # layer's kernels); its un-gated rows are compared with the oracle's at
    # the positions above
    L = layer_inputs(name, T)
    cfg = L.cfg
    ids_d = _route_gpu(moe, L)[0]
    counts, offsets, perm, inv = moe.permute(ids_d, cfg.E)
    rows = moe.expert_ffn(dev_x(L), perm, offsets, dev_pool(moe, L), cfg.k, cfg.F)
    torch.cuda.synchronize()
    off_h = offsets.cpu().numpy()
    pos = _aimed_positions(off_h)
    ref = oracle.expert_rows(L.x, perm.cpu().numpy(), off_h, cfg.k, L.gate, L.up, L.down,
                             cfg.qtype, cfg.F, positions=pos)
    got = rows.cpu().numpy()[pos]
    err = rel_err(got, ref)
    print(f"{len(pos)} rows, rel err {err:.3e}")
    assert err <= REL_TOL
    # row by row as well: a wrong row in a small expert must not hide behind
    # the global maximum
    per_row = np.abs(got - ref).max(axis=1) / np.abs(ref).max()
    assert per_row.max() <= REL_TOL


def test_tensor_core_masked_two_phase_rows_are_bit_identical(moe):
    L = layer_inputs("prefill", 8192)
    cfg = L.cfg
    ids_d = _route_gpu(moe, L)[0]
    counts, offsets, perm, inv = moe.permute(ids_d, cfg.E)
    pool = dev_pool(moe, L)
    x = dev_x(L)
    full = moe.expert_ffn(x, perm, offsets, pool, cfg.k, cfg.F)
    m = torch.from_numpy(np.random.default_rng(5).integers(0, 2, cfg.E).astype(np.uint8)).cuda()
    two = torch.full_like(full, float("nan"))
    moe.expert_ffn(x, perm, offsets, pool, cfg.k, cfg.F, mask=m, out=two)
    moe.expert_ffn(x, perm, offsets, pool, cfg.k, cfg.F, mask=1 - m, out=two)
    torch.cuda.synchronize()
    assert torch.equal(full, two)


# ------------------------------------------------------- split layer calls
@pytest.mark.parametrize("name,T", [("decode", 4), ("tiny", None), ("wide", 1), ("wide", 2048),
                                    ("prefill", 8192)])
def test_layer_phases_are_bit_identical(moe, name, T):
    # route + resident FFN (+ shared), then the rest of the experts + combine,
    # with a random expert split: the same bits as one call
    L = layer_inputs(name, T)
    cfg = L.cfg
    lay = _layer(moe, L)
    x = dev_x(L)
    lg = None if L.logits is None else dev(L.logits)
    y1 = lay.forward(x, logits=lg).clone()
    m = torch.from_numpy(np.random.default_rng(6).integers(0, 2, cfg.E).astype(np.uint8)).cuda()
    y2 = torch.full_like(y1, float("nan"))
    lay.forward(x, logits=lg, out=y2, mask=m,
                phases=moe.PHASE_ROUTE | moe.PHASE_FFN | moe.PHASE_SHARED)
    lay.forward(x, logits=lg, out=y2, mask=1 - m, phases=moe.PHASE_FFN | moe.PHASE_COMBINE)
    # route alone, then everything else (ids read back on the host between)
    y3 = torch.full_like(y1, float("nan"))
    lay.forward(x, logits=lg, out=y3, phases=moe.PHASE_ROUTE)
    torch.cuda.synchronize()
    lay.forward(x, logits=lg, out=y3, phases=moe.PHASE_FFN | moe.PHASE_SHARED | moe.PHASE_COMBINE)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert torch.equal(y1, y3)
    assert moe.workspace_status(lay.ws) == (0, moe.DEV_OK)


# ---------------------------------------------------- slots out of range
ODD = S.LayerConfig("odd", T=7, D=96, E=4, k=2, F=160, qtype="q8_0", x_dtype="bf16",
                    y_dtype="f32", router_std=0.1, seed=80)


@pytest.mark.parametrize("name,T", [("decode", 4), ("decode", 300), ("tiny", None), ("odd", 7)])
def test_bad_slot_is_reported_and_skipped(moe, name, T):
    # a slot map that leaves one routed expert at -1 (not resident): the call
    # records MOE_DEV_BAD_SLOT, reads nothing through that slot, and every
    # other expert's rows are exact; the same for a slot past n_slots.  The
    # four cases reach the decode GEMV, the tensor-core GEMM and (D = 96)
    # the portable kernels.
    L = S.make_layer(ODD) if name == "odd" else layer_inputs(name, T)
    cfg = L.cfg
    ids_d = _route_gpu(moe, L)[0]
    counts, offsets, perm, inv = moe.permute(ids_d, cfg.E)
    x = dev_x(L)
    base = dev_pool(moe, L)
    ref = moe.expert_ffn(x, perm, offsets, base, cfg.k, cfg.F)
    cnt = counts.cpu().numpy()
    victim = int(np.nonzero(cnt)[0][len(np.nonzero(cnt)[0]) // 2])
    off = offsets.cpu().numpy()
    for bad in (-1, cfg.E):
        smap = torch.arange(cfg.E, dtype=torch.int32, device="cuda")
        smap[victim] = bad
        pool = moe.ExpertPool(base.gate, base.up, base.down, cfg.qtype, slot_of_expert=smap)
        ws = torch.zeros(moe.expert_ffn_workspace_size(x.shape[0], cfg.k, cfg.D, cfg.F),
                         dtype=torch.uint8, device="cuda")
        out = torch.full_like(ref, float("nan"))
        moe.expert_ffn(x, perm, offsets, pool, cfg.k, cfg.F, out=out, ws=ws)
        st, code = moe.workspace_status(ws)
        assert code == moe.DEV_BAD_SLOT and st != 0, (st, code)
        keep = np.ones(ref.shape[0], bool)
        keep[off[victim]:off[victim + 1]] = False
        assert torch.equal(out[torch.from_numpy(keep).cuda()], ref[torch.from_numpy(keep).cuda()])
        assert torch.isnan(out[off[victim]:off[victim + 1]]).all()   # skipped, untouched
        assert moe.workspace_status(ws) == (0, moe.DEV_OK)            # cleared by the read


def test_bad_slot_in_the_fused_layer(moe):
    L = layer_inputs("cache", 4)
    cfg = L.cfg
    lay0 = _layer(moe, L)
    x, lg = dev_x(L), dev(L.logits)
    y_ref = lay0.forward(x, logits=lg).clone()
    torch.cuda.synchronize()
    ids = lay0.ids.cpu().numpy()[:4]
    # the expert used by the fewest tokens (the locality trace repeats most)
    cnt = np.bincount(ids.ravel(), minlength=cfg.E)
    victim = int(np.argmin(np.where(cnt > 0, cnt, 1 << 30)))
    smap = torch.arange(cfg.E, dtype=torch.int32, device="cuda")
    smap[victim] = -1
    pool = moe.ExpertPool(lay0.pool.gate, lay0.pool.up, lay0.pool.down, cfg.qtype,
                          slot_of_expert=smap)
    lay = moe.Layer(pool, cfg.D, cfg.F, cfg.E, cfg.k, 4, y_dtype=torch.bfloat16)
    y = lay.forward(x, logits=lg)
    st, code = moe.workspace_status(lay.ws)
    assert code == moe.DEV_BAD_SLOT
    clean = ~np.isin(ids, [victim]).any(axis=1)
    assert clean.any()
    c = torch.from_numpy(clean).cuda()
    assert torch.equal(y[c], y_ref[c])
