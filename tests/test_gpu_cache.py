"""Expert cache on the GPU: the hit/miss/victim sequence against the oracle's
LRU simulation, layer outputs with the cache against the fully resident
pool (bit for bit: same kernels, same reduction order, only the slot
addresses differ), and an injected copy failure.

A small stack of layers (Q8_0, D=256, F=256, E=16, k=4, 6 slots per layer)
routed from per-layer locality traces, T=1 per step, as the cache workload
does at full size.
"""
import numpy as np
import pytest
import torch

import oracle
import synthetic as S
from helpers import check_ids

pytestmark = pytest.mark.gpu

N_LAYERS, E, K, D, F, SLOTS, STEPS = 3, 16, 4, 256, 256, 6, 30


@pytest.fixture(scope="module")
def stack(moe):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pools = [S.gen_expert_pool(900 + l, E, D, F, "q8_0", 0.02) for l in range(N_LAYERS)]
    traces = [S.locality_trace(np.random.default_rng([910, l]), STEPS, E, K)[0]
              for l in range(N_LAYERS)]
    x = S.make_layer(S.LayerConfig("cachex", T=STEPS, D=D, E=E, k=K, F=F, qtype="q8_0",
                                   x_dtype="bf16", y_dtype="f32", seed=920), experts=False)
    return pools, traces, x


def _cache(moe, pools, stream):
    pin = lambda a: torch.from_numpy(a).pin_memory()
    hg = [pin(p[0]) for p in pools]
    hu = [pin(p[1]) for p in pools]
    hd = [pin(p[2]) for p in pools]
    return moe.ExpertCache(hg, hu, hd, "q8_0", SLOTS, stream)


def _ids(logits_row):
    ids, _ = oracle.select(logits_row[None, :].astype(np.float64), K, True)
    return ids[0]


def test_cache_sequence_matches_lru_simulation(moe, stack):
    pools, traces, _ = stack
    cache = _cache(moe, pools, torch.cuda.Stream())
    sims = [oracle.LRU(E, SLOTS) for _ in range(N_LAYERS)]
    n_miss = 0
    for t in range(STEPS):
        for l in range(N_LAYERS):
            ids = _ids(traces[l][t])
            got = cache.request(l, ids)
            want = sims[l].request(ids)
            for g, w in zip(got, want):
                assert np.array_equal(np.asarray(g), np.asarray(w)), (t, l, got, want)
            n_miss += int(want[1].sum())
    torch.cuda.synchronize()
    hits, misses, nbytes = cache.stats()
    assert misses == n_miss and hits + misses == STEPS * N_LAYERS * K
    assert nbytes == n_miss * sum(p[0][0].nbytes + p[1][0].nbytes + p[2][0].nbytes
                                  for p in pools[:1])
    cache.close()


def test_cached_layers_are_bit_identical_to_resident(moe, stack):
    pools, traces, x = stack
    stream = torch.cuda.current_stream()
    cache = _cache(moe, pools, torch.cuda.Stream())
    xd = torch.from_numpy(x.x_raw.view(np.int16)).cuda().view(torch.bfloat16)
    resident = [moe.Layer(moe.ExpertPool.from_numpy(*p, "q8_0"), D, F, E, K, 1,
                          y_dtype=torch.float32) for p in pools]
    cached = [moe.Layer(cache.pools[l], D, F, E, K, 1, y_dtype=torch.float32)
              for l in range(N_LAYERS)]
    for t in range(STEPS):
        for l in range(N_LAYERS):
            lg = torch.from_numpy(traces[l][t:t + 1]).cuda()
            cache.request(l, _ids(traces[l][t]), stream=stream)
            cache.sync(l, stream=stream)
            y_c = cached[l].forward(xd[t:t + 1], logits=lg).clone()
            y_r = resident[l].forward(xd[t:t + 1], logits=lg).clone()
            torch.cuda.synchronize()
            assert torch.equal(y_c, y_r), (t, l)
            assert torch.equal(cached[l].ids[:1], resident[l].ids[:1])
    cache.close()


def test_injected_copy_failure_is_reported_and_recovered(moe, stack):
    # a failed miss copy raises; the experts of the failed request are not
    # left mapped to half-written slots, and a retry serves the layer exactly
    pools, traces, x = stack
    stream = torch.cuda.current_stream()
    cache = _cache(moe, pools, torch.cuda.Stream())
    xd = torch.from_numpy(x.x_raw.view(np.int16)).cuda().view(torch.bfloat16)
    first = _ids(traces[0][0])
    cache.request(0, first, stream=stream)
    cache.sync(0, stream=stream)
    torch.cuda.synchronize()
    ids, t_ids = None, None
    for t in range(1, STEPS):
        cand = _ids(traces[0][t])
        if not set(cand.tolist()) <= set(first.tolist()):
            ids, t_ids = cand, t
            break
    assert ids is not None
    missing = [e for e in ids.tolist() if e not in set(first.tolist())]
    cache.inject_copy_failure(0)
    with pytest.raises(moe.MoeError):
        cache.request(0, ids, stream=stream)
    torch.cuda.synchronize()
    smap = cache.slot_map[0].cpu().numpy()
    assert all(smap[e] == -1 for e in missing)
    # retry (no failure armed now) and compare the layer with the resident one
    cache.inject_copy_failure(-1)
    cache.request(0, ids, stream=stream)
    cache.sync(0, stream=stream)
    lg = torch.from_numpy(traces[0][t_ids:t_ids + 1]).cuda()
    lay_c = moe.Layer(cache.pools[0], D, F, E, K, 1, y_dtype=torch.float32)
    lay_r = moe.Layer(moe.ExpertPool.from_numpy(*pools[0], "q8_0"), D, F, E, K, 1,
                      y_dtype=torch.float32)
    y_c = lay_c.forward(xd[t_ids:t_ids + 1], logits=lg).clone()
    y_r = lay_r.forward(xd[t_ids:t_ids + 1], logits=lg).clone()
    torch.cuda.synchronize()
    assert torch.equal(y_c, y_r)
    cache.close()


def test_released_copies_overlap_and_stay_exact(moe, stack):
    # with a release point after every layer's FFN, a layer's miss copies wait
    # only for that layer's previous FFN: the host enqueues all steps of all
    # layers before synchronising once, and every output must still equal the
    # fully resident layers' bit for bit
    pools, traces, x = stack
    stream = torch.cuda.current_stream()
    cache = _cache(moe, pools, torch.cuda.Stream())
    xd = torch.from_numpy(x.x_raw.view(np.int16)).cuda().view(torch.bfloat16)
    resident = [moe.Layer(moe.ExpertPool.from_numpy(*p, "q8_0"), D, F, E, K, 1,
                          y_dtype=torch.float32) for p in pools]
    cached = [moe.Layer(cache.pools[l], D, F, E, K, 1, y_dtype=torch.float32)
              for l in range(N_LAYERS)]
    lg = [torch.from_numpy(traces[l]).cuda() for l in range(N_LAYERS)]
    y_c = torch.empty((STEPS, N_LAYERS, D), dtype=torch.float32, device="cuda")
    y_r = torch.empty_like(y_c)
    for t in range(STEPS):
        for l in range(N_LAYERS):
            cache.request(l, _ids(traces[l][t]), stream=stream)
            cache.sync(l, stream=stream)
            cached[l].forward(xd[t:t + 1], logits=lg[l][t:t + 1], out=y_c[t, l:l + 1])
            cache.release(l, stream=stream)
            resident[l].forward(xd[t:t + 1], logits=lg[l][t:t + 1], out=y_r[t, l:l + 1])
    torch.cuda.synchronize()
    assert torch.equal(y_c, y_r)
    hits, misses, _ = cache.stats()
    assert misses > 0 and hits > 0
    cache.close()


def _masks(E, ids, miss):
    """Device uint8 masks of the requested experts that were resident (hits)
    and of those whose copies were just enqueued (misses)."""
    hit = np.zeros(E, np.uint8)
    mis = np.zeros(E, np.uint8)
    ids = np.asarray(ids)
    hit[ids[~miss]] = 1
    mis[ids[miss]] = 1
    return torch.from_numpy(hit).cuda(), torch.from_numpy(mis).cuda()


def _two_phase(moe, cache, lay, l, ids, x, lg, out, stream, check_masks=False):
    """One cached layer step with the miss copies overlapping the FFN of the
    resident experts: route + resident FFN, wait for the copies, the copied
    experts' FFN + combine.  The masks are the ones the cache writes with
    the slot map (optionally checked against the host's request result)."""
    _, miss, _ = cache.request(l, ids, stream=stream)
    lay.forward(x, logits=lg, out=out, mask=cache.hit_mask(l),
                phases=moe.PHASE_ROUTE | moe.PHASE_FFN | moe.PHASE_SHARED)
    cache.sync(l, stream=stream)
    lay.forward(x, logits=lg, out=out, mask=cache.miss_mask(l),
                phases=moe.PHASE_FFN | moe.PHASE_COMBINE)
    if check_masks:
        m_hit, m_miss = _masks(lay.E, ids, miss)
        assert torch.equal(cache.hit_mask(l), m_hit) and torch.equal(cache.miss_mask(l), m_miss)
    return int(miss.sum())


def test_two_phase_cached_layers_are_bit_identical_to_resident(moe, stack):
    pools, traces, x = stack
    stream = torch.cuda.current_stream()
    cache = _cache(moe, pools, torch.cuda.Stream())
    xd = torch.from_numpy(x.x_raw.view(np.int16)).cuda().view(torch.bfloat16)
    resident = [moe.Layer(moe.ExpertPool.from_numpy(*p, "q8_0"), D, F, E, K, 1,
                          y_dtype=torch.float32) for p in pools]
    cached = [moe.Layer(cache.pools[l], D, F, E, K, 1, y_dtype=torch.float32)
              for l in range(N_LAYERS)]
    n_miss = 0
    for t in range(STEPS):
        for l in range(N_LAYERS):
            lg = torch.from_numpy(traces[l][t:t + 1]).cuda()
            y_c = torch.full((1, D), float("nan"), device="cuda")
            n_miss += _two_phase(moe, cache, cached[l], l, _ids(traces[l][t]), xd[t:t + 1], lg,
                                 y_c, stream, check_masks=(t % 7 == 0))
            cache.release(l, stream=stream)
            y_r = resident[l].forward(xd[t:t + 1], logits=lg).clone()
            torch.cuda.synchronize()
            assert torch.equal(y_c, y_r), (t, l)
            assert moe.workspace_status(cached[l].ws) == (0, moe.DEV_OK)
    assert n_miss > 0
    assert cache.exposed_ns() >= 0
    cache.close()


def test_exposed_copy_time_is_measured(moe, stack):
    # a copy the compute stream must wait for (the first, cold request of a
    # layer, synced at once) shows up as exposed time; requests that hit
    # add nothing
    pools, traces, _ = stack
    stream = torch.cuda.current_stream()
    cache = _cache(moe, pools, torch.cuda.Stream())
    assert cache.exposed_ns() == 0
    ids = _ids(traces[0][0])
    cache.request(0, ids, stream=stream)
    cache.sync(0, stream=stream)
    torch.cuda.synchronize()
    e1 = cache.exposed_ns()
    assert e1 > 0
    cache.request(0, ids, stream=stream)      # all hits: nothing to wait for
    cache.sync(0, stream=stream)
    torch.cuda.synchronize()
    assert cache.exposed_ns() == e1
    cache.close()


def test_cache_at_the_full_layer_shape_matches_the_oracle(moe):
    # the expert-cache layer at its real shape (Q8_0, D=2048, F=768, E=128,
    # top-8, 51 slots = 40%) for a few cold-start steps: each step's output
    # against the oracle, two-phase (resident experts, then the copied ones)
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cfg = S.CONFIGS["cache"]
    n_slots = int(np.floor(S.CACHE_FRACTION * cfg.E))
    pool = S.gen_expert_pool(cfg.seed, cfg.E, cfg.D, cfg.F, cfg.qtype, cfg.expert_std)
    steps = 6
    logits, sets = S.locality_trace(np.random.default_rng([cfg.seed, 0]), steps, cfg.E, cfg.k)
    xin = S.make_layer(S.with_T(cfg, steps), experts=False)
    pin = lambda a: torch.from_numpy(a).pin_memory()
    cache = moe.ExpertCache([pin(pool[0])], [pin(pool[1])], [pin(pool[2])], cfg.qtype, n_slots,
                            torch.cuda.Stream())
    lay = moe.Layer(cache.pools[0], cfg.D, cfg.F, cfg.E, cfg.k, 1, y_dtype=torch.float32)
    stream = torch.cuda.current_stream()
    xd = torch.from_numpy(xin.x_raw.view(np.int16)).cuda().view(torch.bfloat16)
    lgd = torch.from_numpy(logits).cuda()
    for t in range(steps):
        ids, g = oracle.select(logits[t:t + 1].astype(np.float64), cfg.k, cfg.renorm)
        y = torch.full((1, cfg.D), float("nan"), device="cuda")
        _two_phase(moe, cache, lay, 0, ids[0], xd[t:t + 1], lgd[t:t + 1], y, stream)
        torch.cuda.synchronize()
        check_ids(lay.ids.cpu().numpy()[:1], ids, logits[t:t + 1], cfg.k, log=print)
        ref = oracle.layer(xin.x[t:t + 1], ids, g, *pool, cfg.qtype, cfg.F)
        err = np.abs(y.cpu().numpy() - ref).max() / np.abs(ref).max()
        assert err <= 2e-3, (t, err)
    assert moe.workspace_status(lay.ws) == (0, moe.DEV_OK)
    cache.close()


# ------------------------------------------------- global LRU with resizing
def _global_cache(moe, pools, stream, cap, max_slots):
    pin = lambda a: torch.from_numpy(a).pin_memory()
    return moe.ExpertCache([pin(p[0]) for p in pools], [pin(p[1]) for p in pools],
                           [pin(p[2]) for p in pools], "q8_0", cap, stream,
                           global_slots=max_slots)


RESIZES = {9: 6, 19: 14, 27: 5}      # step -> new capacity (shrink, grow, shrink)


def test_global_cache_sequence_matches_simulation(moe, stack):
    # every request's (slot, miss, evicted key) and every resize's eviction
    # and move counts equal the oracle's global LRU simulation
    pools, traces, _ = stack
    cache = _global_cache(moe, pools, torch.cuda.Stream(), 10, 16)
    sim = oracle.GlobalLRU(N_LAYERS, E, 16, 10)
    cross = 0
    for t in range(STEPS):
        if t in RESIZES:
            ne, nm = cache.resize(RESIZES[t])
            ev, mv = sim.resize(RESIZES[t])
            assert (ne, nm) == (len(ev), len(mv)), t
        for l in range(N_LAYERS):
            ids = _ids(traces[l][t])
            got = cache.request(l, ids)
            want = sim.request(l, ids)
            for g, w in zip(got, want):
                assert np.array_equal(np.asarray(g), np.asarray(w)), (t, l, got, want)
            cross += int(np.sum((want[2] >= 0) & (want[2] // E != l)))
    torch.cuda.synchronize()
    assert cross > 0                  # some victims came from other layers
    cache.close()


def test_global_cached_layers_are_bit_identical_to_resident(moe, stack):
    # two-phase layer calls through the shared pool, with the capacity
    # shrunk (evictions and moves inside the pool) and grown on the way
    pools, traces, x = stack
    stream = torch.cuda.current_stream()
    cache = _global_cache(moe, pools, torch.cuda.Stream(), 10, 16)
    xd = torch.from_numpy(x.x_raw.view(np.int16)).cuda().view(torch.bfloat16)
    resident = [moe.Layer(moe.ExpertPool.from_numpy(*p, "q8_0"), D, F, E, K, 1,
                          y_dtype=torch.float32) for p in pools]
    cached = [moe.Layer(cache.pools[l], D, F, E, K, 1, y_dtype=torch.float32)
              for l in range(N_LAYERS)]
    moved = 0
    for t in range(STEPS):
        if t in RESIZES:
            moved += cache.resize(RESIZES[t], stream=stream)[1]
        for l in range(N_LAYERS):
            lg = torch.from_numpy(traces[l][t:t + 1]).cuda()
            y_c = torch.full((1, D), float("nan"), device="cuda")
            _two_phase(moe, cache, cached[l], l, _ids(traces[l][t]), xd[t:t + 1], lg, y_c, stream)
            cache.release(l, stream=stream)
            y_r = resident[l].forward(xd[t:t + 1], logits=lg).clone()
            torch.cuda.synchronize()
            assert torch.equal(y_c, y_r), (t, l)
            assert moe.workspace_status(cached[l].ws) == (0, moe.DEV_OK)
    assert moved > 0
    cache.close()
