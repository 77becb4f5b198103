"""The 8-bit-activation layer (the W4A8 / W8A8 mode) against the oracle.

x and h are quantized per 32-value block on both sides with the same fp32
operations, so the x codes agree exactly; h is a float computed in different
orders (fp32 tensor-core sums on the GPU, double in the oracle), and an h
value within eps of a rounding boundary may take the neighbouring code.  The
oracle reports, per output, how far such codes can move it (the sum of one
code step times the down weights over those elements); the bar is
|gpu - oracle| <= 2e-3 * max|oracle| + that room, with eps = 2e-3 code units
(the fp32 error of h relative to its block maximum stays under 1e-5, i.e.
1.3e-3 code units).
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from helpers import REL_TOL, check_ids, dev, dev_x, gates_at, oracle_route, rel_err
from test_gpu_parity import _layer

pytestmark = pytest.mark.gpu

EPS = 2e-3
_cache = {}


@pytest.fixture(scope="module", autouse=True)
def _cuda(moe):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    _cache.clear()


def _cfg(qtype, T, D=2048, E=32, k=8, F=768, shared_F=0, shared_qtype="q8_0", seed=600):
    return S.LayerConfig(f"a8_{qtype}_{D}x{F}", T=T, D=D, E=E, k=k, F=F, qtype=qtype,
                         x_dtype="bf16", y_dtype="f32", router_std=0.05, shared_F=shared_F,
                         shared_qtype=shared_qtype, seed=seed)


def _inputs(cfg):
    if cfg not in _cache:
        _cache[cfg] = S.make_layer(cfg)
    return _cache[cfg]


def _a8_layer(moe, L):
    cfg = L.cfg
    lay = _layer(moe, L)
    return moe.Layer(lay.pool, cfg.D, cfg.F, cfg.E, cfg.k, L.x.shape[0], w_router=lay.w_router,
                     bias=lay.bias, shared=lay.shared, shared_F=cfg.shared_F, renorm=cfg.renorm,
                     x_dtype=torch.bfloat16, y_dtype=torch.float32, act_bits=8)


def _check_a8(moe, L, y, ids_gpu):
    cfg = L.cfg
    T = L.x.shape[0]
    ref_logits, ref_ids, ref_g = oracle_route(L)
    ids_gpu = ids_gpu.cpu().numpy()[:T]
    tied = check_ids(ids_gpu, ref_ids, ref_logits, cfg.k, log=print)
    use_ids, use_g = ref_ids.copy(), ref_g.copy()
    if tied:
        use_ids[tied] = ids_gpu[tied]
        use_g[tied] = gates_at(ref_logits[tied], ids_gpu[tied], cfg.renorm)
    ref, room = oracle.layer_a8(L.x, use_ids, use_g, L.gate, L.up, L.down, cfg.qtype, cfg.F,
                                shared=L.shared, shared_qtype=cfg.shared_qtype, eps=EPS,
                                want_bound=True)
    got = y.float().cpu().numpy()
    diff = np.abs(got - ref)
    bar = REL_TOL * np.abs(ref).max() + room
    assert np.all(diff <= bar), (diff - bar).max()
    # the 16-bit layer is a different function: the quantization is real
    ref16 = oracle.layer(L.x, use_ids, use_g, L.gate, L.up, L.down, cfg.qtype, cfg.F,
                         shared=L.shared, shared_qtype=cfg.shared_qtype)
    return rel_err(got, ref), rel_err(ref, ref16), float(room.max() / np.abs(ref).max())


@pytest.mark.parametrize("T", [1, 5, 16])
@pytest.mark.parametrize("qtype", ["q4_0", "q8_0"])
def test_a8_decode_layer(moe, qtype, T):
    L = _inputs(_cfg(qtype, T))
    lay = _a8_layer(moe, L)
    y = lay.forward(dev_x(L))
    torch.cuda.synchronize()
    e, e16, r = _check_a8(moe, L, y, lay.ids)
    print(f"{qtype} T={T}: rel err vs the 8-bit oracle {e:.2e}, 8-bit vs 16-bit {e16:.2e}, "
          f"boundary room {r:.2e}")
    assert e16 > 1e-4
    assert moe.workspace_status(lay.ws) == (0, moe.DEV_OK)


@pytest.mark.parametrize("D,F", [(256, 256), (512, 512), (768, 256), (1024, 1024)])
@pytest.mark.parametrize("qtype", ["q4_0", "q8_0"])
def test_a8_geometries(moe, qtype, D, F):
    L = _inputs(_cfg(qtype, 4, D=D, F=F, E=16, k=4, seed=601))
    lay = _a8_layer(moe, L)
    y = lay.forward(dev_x(L))
    torch.cuda.synchronize()
    _check_a8(moe, L, y, lay.ids)


@pytest.mark.parametrize("routed,shared", [("q4_0", "q8_0"), ("q8_0", "q4_0"), ("q4_0", "q4_0")])
@pytest.mark.parametrize("T", [1, 16])
def test_a8_with_shared_expert(moe, routed, shared, T):
    L = _inputs(_cfg(routed, T, D=1024, F=512, E=16, k=4, shared_F=512, shared_qtype=shared,
                     seed=602))
    lay = _a8_layer(moe, L)
    y = lay.forward(dev_x(L))
    torch.cuda.synchronize()
    _check_a8(moe, L, y, lay.ids)


def test_a8_full_size_decode_layer(moe):
    # the 30B-A3B-shaped decode layer with all 128 experts, T = 16
    cfg = S.CONFIGS["decode"]
    L = S.make_layer(cfg, T=16)
    lay = moe.Layer(moe.ExpertPool(dev(L.gate), dev(L.up), dev(L.down), cfg.qtype), cfg.D, cfg.F,
                    cfg.E, cfg.k, 16, w_router=dev(L.w_router), bias=dev(L.bias),
                    x_dtype=torch.bfloat16, y_dtype=torch.float32, act_bits=8)
    y = lay.forward(dev_x(L))
    torch.cuda.synchronize()
    _check_a8(moe, L, y, lay.ids)


@pytest.mark.parametrize("T", [4, 16])
def test_a8_phases_are_bit_identical(moe, T):
    L = _inputs(_cfg("q4_0", T, shared_F=768, seed=603))
    lay = _a8_layer(moe, L)
    x = dev_x(L)
    y1 = lay.forward(x).clone()
    m = torch.from_numpy(np.random.default_rng(8).integers(0, 2, L.cfg.E).astype(np.uint8)).cuda()
    y2 = torch.full_like(y1, float("nan"))
    lay.forward(x, out=y2, mask=m, phases=moe.PHASE_ROUTE | moe.PHASE_FFN | moe.PHASE_SHARED)
    lay.forward(x, out=y2, mask=1 - m, phases=moe.PHASE_FFN | moe.PHASE_COMBINE)
    y3 = lay.forward(x).clone()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert torch.equal(y1, y3)
