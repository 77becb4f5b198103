"""Full-layer double-buffered streaming of expert weights for prefill: a stack
of layers whose experts live in pinned host memory, each layer computed from
one of two device buffers while the next layer is copied into the other.
Every layer's output must equal the same layer run from resident weights
bit for bit (same kernels, same reduction order; only the weight addresses
differ), over two passes of the stack."""
import numpy as np
import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu

N_LAYERS = 5
CFG = S.LayerConfig("stream", T=300, D=512, E=16, k=4, F=256, qtype="q8_0", x_dtype="bf16",
                    y_dtype="f32", router_std=0.05, zipf_s=1.1, seed=930)


@pytest.fixture(scope="module")
def stack(moe):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    layers = [S.make_layer(CFG, seed=930 + l) for l in range(N_LAYERS)]
    return layers


def test_streamed_layers_are_bit_identical_to_resident(moe, stack):
    dev = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).cuda()
    pin = lambda a: torch.from_numpy(a).pin_memory()
    stream = torch.cuda.current_stream()
    st = moe.LayerStreamer([pin(L.gate) for L in stack], [pin(L.up) for L in stack],
                           [pin(L.down) for L in stack], CFG.qtype, torch.cuda.Stream())
    mk = lambda pool, L: moe.Layer(pool, CFG.D, CFG.F, CFG.E, CFG.k, CFG.T,
                                   w_router=dev(L.w_router), bias=dev(L.bias),
                                   y_dtype=torch.float32)
    resident = [mk(moe.ExpertPool.from_numpy(L.gate, L.up, L.down, CFG.qtype), L) for L in stack]
    xs = [torch.from_numpy(L.x_raw.view(np.int16)).cuda().view(torch.bfloat16) for L in stack]
    y_ref = [resident[l].forward(xs[l]).clone() for l in range(N_LAYERS)]
    torch.cuda.synchronize()
    for rep in range(2):
        ys = []
        st.prefetch(0)
        st.prefetch(1)
        for l in range(N_LAYERS):
            pool = st.acquire(l, stream=stream)
            lay = mk(pool, stack[l])
            ys.append(lay.forward(xs[l]))
            st.release(l, stream=stream)
            if l + 2 < N_LAYERS:
                st.prefetch(l + 2)
        torch.cuda.synchronize()
        for l in range(N_LAYERS):
            assert torch.equal(ys[l], y_ref[l]), (rep, l)
    nbytes, exposed = st.stats()
    per_layer = sum(a.nbytes for a in (stack[0].gate, stack[0].up, stack[0].down))
    assert nbytes == 2 * N_LAYERS * per_layer
    assert exposed >= 0
    st.close()
