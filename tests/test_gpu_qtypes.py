"""The rest of the Standard quant family (Q4_1, Q5_0, Q5_1) and the K-quants
(Q4_K, Q6_K) through every kernel family, against the CPU oracle on the same
seeded bytes.

Each type runs the decode GEMV (T <= 16, every compiled D geometry), the
tcgen05 grouped GEMM (T > 16, ragged row tiles, experts with a handful of
rows) and the portable kernel (D, F not multiples of 256, or F > 1024), as
a routed pool and as the shared expert beside a routed pool of another type.
Q6_K's 210-byte blocks give rows that are whole 16-byte units only at
D = 2048 (gate/up) or in 8-row groups (down): it runs the decode GEMV at
D = 2048 (down rows packed at a pitch that is 2 mod 4 when F / 256 is odd,
each warp taking rows of one parity), the portable kernel at other decode
shapes and through moe_expert_ffn at T > 16, and the tensor-core GEMM on
fp16 copies of its pool in the fused layer at T > 16.  The bar is the one of
the Q4_0 / Q8_0 parity tests: max|gpu - oracle| / max|oracle| <= 2e-3 on fp32
outputs, and bit-identical rows for a masked two-call split.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from helpers import REL_TOL, dev, dev_pool, dev_x, rel_err
from test_gpu_parity import (_aimed_positions, _check_layer, _layer, _route_gpu,
                             _small_expert_tokens)

pytestmark = pytest.mark.gpu

NEW = ["q4_1", "q5_0", "q5_1", "q4_k", "q6_k"]
STD = ["q4_1", "q5_0", "q5_1"]
_cache = {}


@pytest.fixture(scope="module", autouse=True)
def _cuda(moe):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    _cache.clear()


def _cfg(qtype, T, D=2048, E=32, k=8, F=768, shared_F=0, shared_qtype="q8_0", seed=500,
         zipf_s=None):
    return S.LayerConfig(f"{qtype}_{D}x{F}", T=T, D=D, E=E, k=k, F=F, qtype=qtype,
                         x_dtype="bf16", y_dtype="f32", router_std=0.05, zipf_s=zipf_s,
                         shared_F=shared_F, shared_qtype=shared_qtype, seed=seed)


def _inputs(cfg):
    key = (cfg, cfg.T)
    if key not in _cache:
        _cache[key] = S.make_layer(cfg)
    return _cache[key]


def _run_layer(moe, L, n_tok=99, extra_small=False):
    lay = _layer(moe, L)
    y = lay.forward(dev_x(L))
    torch.cuda.synchronize()
    extra = None
    if extra_small:
        extra = _small_expert_tokens(lay.ids.cpu().numpy(), L.cfg.E, L.x.shape[0])
    err = _check_layer(moe, L, y, lay.ids, n_tok, extra=extra)
    assert moe.workspace_status(lay.ws) == (0, moe.DEV_OK)
    return err


# ----------------------------------------------------------------- decode
@pytest.mark.parametrize("T", [1, 5, 16])
@pytest.mark.parametrize("qtype", NEW)
def test_decode_layer(moe, qtype, T):
    err = _run_layer(moe, _inputs(_cfg(qtype, T)))
    print(f"{qtype} T={T}: rel err {err:.3e}")


@pytest.mark.parametrize("D,F", [(256, 256), (512, 512), (768, 256), (1024, 1024)])
@pytest.mark.parametrize("qtype", NEW[:4])
def test_decode_geometries(moe, qtype, D, F):
    # every compiled K-slice geometry of the gate/up kernel, F up to the
    # down kernel's one-box limit
    _run_layer(moe, _inputs(_cfg(qtype, 4, D=D, F=F, E=16, k=4, seed=501)))


def test_decode_full_size_rows(moe):
    # the 30B-A3B-shaped decode layer (E=128, k=8, D=2048, F=768) per type
    for i, qtype in enumerate(NEW):
        _run_layer(moe, _inputs(_cfg(qtype, 16, E=128, seed=510 + i)))


# ---------------------------------------------------------------- prefill
@pytest.mark.parametrize("qtype", NEW)
def test_prefill_rows_at_tile_edges(moe, qtype):
    # T > 16: the tcgen05 grouped GEMM; a skewed router leaves some experts a
    # handful of rows (partial 128-row tiles) and others several tiles
    L = _inputs(_cfg(qtype, 300, zipf_s=1.2, seed=520))
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
    print(f"{qtype}: {len(pos)} rows, rel err {err:.3e}")
    assert err <= REL_TOL
    per_row = np.abs(got - ref).max(axis=1) / np.abs(ref).max()
    assert per_row.max() <= REL_TOL


@pytest.mark.parametrize("qtype", NEW)
def test_prefill_layer(moe, qtype):
    _run_layer(moe, _inputs(_cfg(qtype, 700, D=1024, F=512, E=16, k=4, seed=530)), n_tok=48,
               extra_small=True)


# ------------------------------------------------ shared expert of another type
@pytest.mark.parametrize("routed,shared", [("q5_0", "q4_1"), ("q4_1", "q5_1"),
                                           ("q5_1", "q8_0"), ("q4_0", "q5_0"),
                                           ("q8_0", "q5_1")])
@pytest.mark.parametrize("T", [3, 200])
def test_mixed_routed_and_shared_types(moe, routed, shared, T):
    F = 512
    L = _inputs(_cfg(routed, T, D=1024, F=F, E=16, k=4, shared_F=F, shared_qtype=shared,
                     seed=540))
    _run_layer(moe, L, n_tok=40)


@pytest.mark.parametrize("routed,shared", [("q4_k", "q8_0"), ("q5_0", "q4_k"), ("q4_k", "q6_k")])
@pytest.mark.parametrize("T", [3, 200])
def test_mixed_k_quant_shared(moe, routed, shared, T):
    F = 512
    L = _inputs(_cfg(routed, T, D=1024, F=F, E=16, k=4, shared_F=F, shared_qtype=shared,
                     seed=545))
    _run_layer(moe, L, n_tok=40)


# ---------------------------------------------------------------- generic
@pytest.mark.parametrize("qtype", ["q4_k", "q6_k"])
@pytest.mark.parametrize("T", [4, 40])
def test_generic_wide_f(moe, qtype, T):
    # F = 1280 is past the decode kernel's one-box limit: the portable kernel
    _run_layer(moe, _inputs(_cfg(qtype, T, D=512, F=1280, E=8, k=2, seed=570)), n_tok=40)


@pytest.mark.parametrize("qtype", STD)
def test_generic_odd_shapes(moe, qtype):
    # D, F multiples of 32 but not of 256: the portable kernel; E = k
    cfg = S.LayerConfig("odd", T=7, D=96, E=3, k=3, F=160, qtype=qtype, x_dtype="bf16",
                        y_dtype="f32", router_std=0.1, shared_F=64, shared_qtype=qtype, seed=77)
    _run_layer(moe, S.make_layer(cfg))


# --------------------------------------------------------- two-call splits
@pytest.mark.parametrize("T", [4, 300])
@pytest.mark.parametrize("qtype", NEW)
def test_masked_two_phase_rows_are_bit_identical(moe, qtype, T):
    L = _inputs(_cfg(qtype, T, seed=550))
    cfg = L.cfg
    ids_d = _route_gpu(moe, L)[0]
    counts, offsets, perm, inv = moe.permute(ids_d, cfg.E)
    pool = dev_pool(moe, L)
    x = dev_x(L)
    full = moe.expert_ffn(x, perm, offsets, pool, cfg.k, cfg.F)
    m = torch.from_numpy(np.random.default_rng(7).integers(0, 2, cfg.E).astype(np.uint8)).cuda()
    two = torch.full_like(full, float("nan"))
    moe.expert_ffn(x, perm, offsets, pool, cfg.k, cfg.F, mask=m, out=two)
    moe.expert_ffn(x, perm, offsets, pool, cfg.k, cfg.F, mask=1 - m, out=two)
    torch.cuda.synchronize()
    assert torch.equal(full, two)


def test_q6k_prefill_layer_phases_are_bit_identical(moe):
    # Q6_K at T > 16 runs the tensor-core GEMM on fp16 copies of the pool made
    # in the layer's workspace; a masked two-call split gives the same bits
    L = _inputs(_cfg("q6_k", 300, D=1024, F=512, E=16, k=4, shared_F=512, shared_qtype="q6_k",
                     seed=580))
    lay = _layer(moe, L)
    x = dev_x(L)
    y1 = lay.forward(x).clone()
    m = torch.from_numpy(np.random.default_rng(9).integers(0, 2, L.cfg.E).astype(np.uint8)).cuda()
    y2 = torch.full_like(y1, float("nan"))
    lay.forward(x, out=y2, mask=m, phases=moe.PHASE_ROUTE | moe.PHASE_FFN | moe.PHASE_SHARED)
    lay.forward(x, out=y2, mask=1 - m, phases=moe.PHASE_FFN | moe.PHASE_COMBINE)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    _check_layer(moe, L, y1, lay.ids, 40)
    assert moe.workspace_status(lay.ws) == (0, moe.DEV_OK)


# ------------------------------------------------------------- Q6_K decode
def _kinds(moe, L):
    lay = _layer(moe, L)
    tr = moe.KernelTrace(n_calls=1)
    y = lay.forward(dev_x(L), trace=tr)
    torch.cuda.synchronize()
    return lay, y, {k for call in tr.calls for k, _, _ in call}


@pytest.mark.parametrize("F", [256, 512, 768, 1024])
@pytest.mark.parametrize("T", [1, 16])
def test_q6k_decode_kernels(moe, T, F):
    # D = 2048: the decode GEMV, not the portable kernel; F / 256 odd packs
    # the down rows at a pitch of 2 mod 4
    L = _inputs(_cfg("q6_k", T, D=2048, F=F, E=16, k=4, seed=590))
    lay, y, kinds = _kinds(moe, L)
    assert "ffn_decode" in kinds and "gateup" not in kinds, kinds
    err = _check_layer(moe, L, y, lay.ids, 99)
    assert moe.workspace_status(lay.ws) == (0, moe.DEV_OK)
    print(f"q6_k T={T} F={F}: rel err {err:.3e}")


@pytest.mark.parametrize("routed,shared", [("q6_k", "q4_0"), ("q4_0", "q6_k"), ("q6_k", "q6_k"),
                                           ("q5_1", "q6_k")])
@pytest.mark.parametrize("T", [2, 16])
def test_q6k_decode_with_shared_expert(moe, routed, shared, T):
    L = _inputs(_cfg(routed, T, D=2048, F=768, E=16, k=4, shared_F=512, shared_qtype=shared,
                     seed=591))
    lay, y, kinds = _kinds(moe, L)
    assert "ffn_decode" in kinds, kinds
    _check_layer(moe, L, y, lay.ids, 99)
    assert moe.workspace_status(lay.ws) == (0, moe.DEV_OK)


def test_q6k_decode_at_other_d_takes_the_portable_kernel(moe):
    L = _inputs(_cfg("q6_k", 4, D=1024, F=768, E=16, k=4, seed=592))
    lay, y, kinds = _kinds(moe, L)
    assert "ffn_decode" not in kinds and "gateup" in kinds, kinds
    _check_layer(moe, L, y, lay.ids, 99)
