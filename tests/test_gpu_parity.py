"""GPU parity: every CUDA kernel, called through the C ABI, against the CPU oracle.

Bit-exact: packed codes and scales, router indices, grouping (counts/offsets/perm/inv), slot
tables. Floating point: router weights to ROUTE_RTOL; FFN outputs to max-abs 2e-2 and
relative L2 5e-3 against the oracle on the same dequantised weights (the packed bytes the
oracle produced are uploaded unchanged). Sizes span several tiles and ragged tails; the
full-size workloads are checked on sampled tokens.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from gpu_util import (Layer, assert_ffn_close, bits_to_dev, dev_to_bits, bf16_dev_to_f32, ROUTE_RTOL)

pytestmark = pytest.mark.gpu

q = pytest.importorskip("quantized_mixture_experts_grouped_b200")

FFN_PATHS = ["simple", "decode", "grouped", "sequential"]


def _supported(path, T, k):
    """The fused decode path takes small batches only (T <= 16 and T*k <= 256)."""
    if path == "decode" and not (1 <= T <= 16 and T * k <= 256):
        pytest.skip("fused decode path is for small batches")


def _supported_h(path, H):
    if path == "decode" and H > 3072:
        pytest.skip("fused decode path stages the activations in shared memory: H <= 3072")
    if path == "grouped" and H % 256:
        pytest.skip("grouped GEMM pairs 128-row blocks of W2: H must be a multiple of 256")


def _ws(T, H, I, E, k):
    return q.alloc_workspace(T, H, I, E, k)


# ----------------------------------------------------------------------------- pack

def _pack_on_gpu(w_bits: np.ndarray):
    E, N, K = w_bits.shape
    w = bits_to_dev(w_bits)
    packed, scales = q.alloc_bank(E, N, K)
    q.moe_quantize_pack(w, packed, scales)
    torch.cuda.synchronize()
    return packed.cpu().numpy(), dev_to_bits(scales)


@pytest.mark.parametrize("dist", ["normal", "heavy_zero_groups", "ties"])
def test_pack_bit_exact_small(dist):
    g = np.random.default_rng(7)
    E, N, K = 3, 384, 512
    if dist == "normal":
        w = g.standard_normal((E, N, K)) * 0.02
    elif dist == "heavy_zero_groups":
        w = g.standard_t(2, (E, N, K)) * np.exp(g.uniform(-30, 3, (E, N, 1)))
        w[:, 5, 128:256] = 0.0
        w[1, 130:140, :] = 0.0
    else:   # quarter-integer multiples of a power of two: many w/s exactly on .5
        w = g.integers(-28, 29, (E, N, K)) * 0.125
        w[..., 0] = 3.5
    wb = mi.to_bf16_bits(w.astype(np.float32))
    packed, scales = _pack_on_gpu(wb)
    for e in range(E):
        ref_p, ref_s = oracle.pack(*oracle.quantize(wb[e]))
        np.testing.assert_array_equal(packed[e], ref_p)
        np.testing.assert_array_equal(scales[e], ref_s)


def test_pack_bit_exact_full_size_experts():
    """OLMoE gate/up (2048x2048) and down (2048x1024) of two experts, and the large-expert
    gate/up (28672x4096) of one expert."""
    wl = mi.WORKLOADS["olmoe_decode"]
    for e in (0, 63):
        a, b = mi.expert_weights(wl, 3, e)
        for m in (a, b):
            packed, scales = _pack_on_gpu(m[None])
            ref_p, ref_s = oracle.pack(*oracle.quantize(m))
            np.testing.assert_array_equal(packed[0], ref_p)
            np.testing.assert_array_equal(scales[0], ref_s)
    wl = mi.WORKLOADS["large_expert"]
    a, _ = mi.expert_weights(wl, 0, 5)
    packed, scales = _pack_on_gpu(a[None])
    ref_p, ref_s = oracle.pack(*oracle.quantize(a))
    np.testing.assert_array_equal(packed[0], ref_p)
    np.testing.assert_array_equal(scales[0], ref_s)


# ----------------------------------------------------------------------------- route

def _route_gpu(lb: np.ndarray, k: int):
    T, E = lb.shape
    logits = bits_to_dev(lb)
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    wts = torch.empty((T, k), dtype=torch.float32, device="cuda")
    q.moe_route_topk(logits, k, idx, wts)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), wts.cpu().numpy()


@pytest.mark.parametrize("T,E,k,kind", [(4, 8, 2, "normal"), (2048, 64, 8, "zipf"), (2048, 64, 8, "normal"),
                                        (17, 64, 64, "ties"), (33, 256, 8, "ties"), (512, 8, 2, "normal"),
                                        (5, 3, 1, "ties"), (1, 64, 8, "normal")])
def test_route_matches_oracle(T, E, k, kind):
    g = np.random.default_rng(T + E + k)
    if kind == "zipf":
        wl = mi.Workload("z", H=128, I=128, E=E, k=k, T=T, routing="zipf")
        lb = mi.router_logits(wl, 0, 0)
    else:
        l = g.standard_normal((T, E)).astype(np.float32)
        if kind == "ties":
            l = np.round(l * 2) / 2
            l[:, 1::5] = -0.0
            l[:, 2::5] = 0.0
        lb = mi.to_bf16_bits(l)
    idx, wts = _route_gpu(lb, k)
    ridx, rwts = oracle.route(lb, k)
    np.testing.assert_array_equal(idx, ridx)
    np.testing.assert_allclose(wts, rwts, rtol=ROUTE_RTOL, atol=0)


def test_route_empty_batch_is_noop():
    idx = torch.full((1, 2), -7, dtype=torch.int32, device="cuda")
    wts = torch.zeros((1, 2), device="cuda")
    assert q.lib.moe_route_topk(None, 0, 8, 2, None, None, None) == 0
    assert (idx == -7).all()


# ----------------------------------------------------------------------------- permute

@pytest.mark.parametrize("T,E,k", [(1, 64, 8), (16, 64, 8), (2048, 64, 8), (3000, 256, 8), (4, 8, 2)])
def test_permute_bit_exact(T, E, k):
    g = np.random.default_rng(T * 7 + E)
    if E == 64 and T == 2048:
        wl = mi.Workload("z", H=128, I=128, E=E, k=k, T=T, routing="zipf")
        idx, _ = oracle.route(mi.router_logits(wl), k)
    else:
        idx = np.stack([g.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    d_idx = torch.from_numpy(idx).cuda()
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    scratch = torch.empty(max(1, q.moe_permute_scratch_count(T, k, E)), dtype=torch.int32, device="cuda")
    q.moe_permute(d_idx, E, counts, offsets, perm, inv, scratch)
    torch.cuda.synchronize()
    rc, ro, rp, ri = oracle.permute(idx, E)
    np.testing.assert_array_equal(counts.cpu().numpy(), rc)
    np.testing.assert_array_equal(offsets.cpu().numpy(), ro)
    np.testing.assert_array_equal(perm.cpu().numpy(), rp)
    np.testing.assert_array_equal(inv.cpu().numpy(), ri)


# ----------------------------------------------------------------------------- FFN

def _run_ffn(layer: Layer, path: str, out=None, slot=None):
    _supported(path, layer.T, layer.wl.k)
    _supported_h(path, layer.wl.H)
    d = layer.to_device()
    wl = layer.wl
    ws = _ws(layer.T, wl.H, wl.I, wl.E, wl.k)
    out = torch.empty((layer.T, wl.H), dtype=torch.bfloat16, device="cuda") if out is None else out
    q.moe_w4a16_ffn(d["x"], d["idx"], d["wts"], d["w13"], d["s13"], d["w2"], d["s2"], wl.H, wl.I, wl.E, ws, out,
                    slot_of_expert=slot, flags=q.PATHS[path])
    torch.cuda.synchronize()
    assert q.moe_workspace_status(ws) == 0
    return out, ws


@pytest.mark.parametrize("path", FFN_PATHS)
@pytest.mark.parametrize("T", [4, 1, 16, 17, 64])
def test_ffn_tiny_shapes(path, T):
    layer = Layer(mi.WORKLOADS["tiny"], T=T)
    out, _ = _run_ffn(layer, path)
    assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"tiny T={T} {path}")


@pytest.mark.parametrize("path", FFN_PATHS)
def test_ffn_edge_cases(path):
    wl = mi.Workload("edge", H=512, I=384, E=8, k=3, T=37)
    g = np.random.default_rng(2)
    # one expert takes every token (its logit dominates), two experts get none
    l = g.standard_normal((wl.T, wl.E)).astype(np.float32)
    l[:, 5] += 100.0
    l[:, 0] -= 100.0
    l[:, 7] -= 100.0
    layer = Layer(wl, logits=mi.to_bf16_bits(l))
    # an all-zero weight group in one expert
    layer.w13[5][:8192] = 0x88      # code 8 = q 0 for a whole tile
    out, _ = _run_ffn(layer, path)
    assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"edge {path}")



@pytest.mark.parametrize("path", FFN_PATHS)
def test_ffn_k_equals_e(path):
    """k = E: every expert on every token."""
    wl2 = mi.Workload("kE", H=256, I=128, E=4, k=4, T=9)
    layer2 = Layer(wl2)
    out2, _ = _run_ffn(layer2, path)
    assert_ffn_close(bf16_dev_to_f32(out2), layer2.oracle_out(), f"k=E {path}")


@pytest.mark.parametrize("path", FFN_PATHS)
def test_ffn_edge_cases_small_batch(path):
    """Decode-sized batch: one expert takes every token, two get none, one all-zero group."""
    wl = mi.Workload("edge_small", H=512, I=384, E=8, k=3, T=13)
    g = np.random.default_rng(3)
    l = g.standard_normal((wl.T, wl.E)).astype(np.float32)
    l[:, 2] += 100.0
    l[:, 0] -= 100.0
    l[:, 7] -= 100.0
    layer = Layer(wl, logits=mi.to_bf16_bits(l))
    layer.w2[2][8192:16384] = 0x88
    out, _ = _run_ffn(layer, path)
    assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"edge small {path}")


@pytest.mark.parametrize("path", ["decode", "grouped"])
def test_ffn_experts_with_every_token_count_width(path):
    """16 tokens, top-3 of 8, routed so that five experts take 16, 10, 6, 3 and 13 tokens and
    three take none: on the batched decode kernel these are four, three, two, one and four MMA
    blocks of compact tokens per tile, in both phases."""
    wl = mi.Workload("widths", H=512, I=256, E=8, k=3, T=16)
    g = np.random.default_rng(12)
    l = g.standard_normal((wl.T, wl.E)).astype(np.float32)
    chosen = [(0, 1, 4)] * 10 + [(0, 2, 3)] * 3 + [(0, 2, 4)] * 3
    for t, es in enumerate(chosen):
        l[t, list(es)] += 100.0
    layer = Layer(wl, logits=mi.to_bf16_bits(l))
    counts = np.bincount(layer.idx.ravel(), minlength=wl.E)
    assert counts.tolist() == [16, 10, 6, 3, 13, 0, 0, 0]
    out, _ = _run_ffn(layer, path)
    assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"token-count widths {path}")


@pytest.mark.parametrize("path", ["auto", "decode", "simple", "grouped", "sequential"])
@pytest.mark.parametrize("T", [1, 5, 16, 300])
def test_layer_call_routes_and_runs(path, T):
    """moe_w4a16_layer: routing (in-kernel on the fused path) + FFN in one call."""
    _supported(path, T, 4)
    wl = mi.Workload("layer", H=512, I=256, E=16, k=4, T=T)
    layer = Layer(wl, layer=1, step=T)
    d = layer.to_device()
    ws = _ws(T, wl.H, wl.I, wl.E, wl.k)
    idx = torch.full((T, wl.k), -1, dtype=torch.int32, device="cuda")
    wts = torch.zeros((T, wl.k), dtype=torch.float32, device="cuda")
    out = torch.empty((T, wl.H), dtype=torch.bfloat16, device="cuda")
    for rep in range(2):
        q.moe_w4a16_layer(d["x"], d["logits"], wl.k, d["w13"], d["s13"], d["w2"], d["s2"], wl.H, wl.I, idx, wts,
                          ws, out, flags=q.PATHS[path])
        torch.cuda.synchronize()
        assert q.moe_workspace_status(ws) == 0
        np.testing.assert_array_equal(idx.cpu().numpy(), layer.idx)
        np.testing.assert_allclose(wts.cpu().numpy(), layer.wts, rtol=ROUTE_RTOL)
        assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"layer {path} T={T} rep={rep}")


@pytest.mark.parametrize("path", FFN_PATHS)
def test_ffn_olmoe_decode_and_batched(path):
    for name, T in (("olmoe_decode", 1), ("olmoe_slots", 16)):
        wl = mi.WORKLOADS[name]
        probe = Layer(mi.Workload("p", H=128, I=128, E=wl.E, k=wl.k, T=T, routing=wl.routing, seed=wl.seed),
                      layer=2, step=5, experts=[])
        routed = sorted(set(probe.idx.ravel().tolist()))
        layer = Layer(wl, layer=2, step=5, T=T, experts=routed, logits=probe.logits)
        out, _ = _run_ffn(layer, path)
        assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"{name} {path}")


_FULL = {}


def _full_layer(name):
    """The full-size layer and the oracle's output for every one of its tokens, computed once per
    process (tens of seconds of oracle on the host cores) and shared by the paths."""
    if name not in _FULL:
        layer = Layer(mi.WORKLOADS[name])
        _FULL[name] = (layer, layer.oracle_out())
    return _FULL[name]


@pytest.mark.parametrize("path", FFN_PATHS)
def test_ffn_prefill_full_size(path):
    """All 2048 tokens of the OLMoE prefill layer (Zipf routing: experts with one to fifteen
    128-token chunks, ragged tails, experts with few tokens) against the oracle."""
    _supported(path, 2048, 8)
    wl = mi.WORKLOADS["olmoe_prefill"]
    layer, ref = _full_layer("olmoe_prefill")
    counts = np.bincount(layer.idx.ravel(), minlength=wl.E)
    assert counts.max() > 1000 and counts.min() < 200      # Zipf skew reached the kernels
    assert np.any(counts % 128 != 0) and np.any(counts > 128)
    out, _ = _run_ffn(layer, path)
    got = bf16_dev_to_f32(out)
    assert_ffn_close(got, ref, f"full: prefill T=2048 {path}")
    # every token on its own as well: a local error cannot hide in the global norm
    for t in range(0, wl.T, 97):
        assert_ffn_close(got[t:t + 1], ref[t:t + 1], f"prefill token {t} {path}")


@pytest.mark.parametrize("path", FFN_PATHS)
def test_ffn_large_expert_full_size(path):
    """All 512 tokens of the large-expert layer (H=4096, I=14336, top-2 of 8)."""
    _supported(path, 512, 2)
    layer, ref = _full_layer("large_expert")
    out, _ = _run_ffn(layer, path)
    got = bf16_dev_to_f32(out)
    assert_ffn_close(got, ref, f"full: large_expert T=512 {path}")
    for t in range(0, 512, 61):
        assert_ffn_close(got[t:t + 1], ref[t:t + 1], f"large_expert token {t} {path}")


@pytest.mark.parametrize("path", FFN_PATHS)
def test_ffn_deterministic_and_slot_indirection(path):
    layer = Layer(mi.WORKLOADS["tiny"], T=15)
    _supported(path, layer.T, layer.wl.k)
    a, _ = _run_ffn(layer, path)
    b, _ = _run_ffn(layer, path)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # the same experts stored in permuted slots through the expert -> slot table
    d = layer.to_device()
    E = layer.wl.E
    perm = np.random.default_rng(0).permutation(E).astype(np.int32)     # expert e lives in slot perm[e]
    w13 = torch.empty_like(d["w13"]); s13 = torch.empty_like(d["s13"])
    w2 = torch.empty_like(d["w2"]); s2 = torch.empty_like(d["s2"])
    for e in range(E):
        w13[perm[e]] = d["w13"][e]; s13[perm[e]] = d["s13"][e]
        w2[perm[e]] = d["w2"][e]; s2[perm[e]] = d["s2"][e]
    table = torch.from_numpy(perm).cuda()
    ws = _ws(layer.T, layer.wl.H, layer.wl.I, E, layer.wl.k)
    c = torch.empty_like(a)
    q.moe_w4a16_ffn(d["x"], d["idx"], d["wts"], w13, s13, w2, s2, layer.wl.H, layer.wl.I, E, ws, c,
                    slot_of_expert=table, flags=q.PATHS[path])
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))


@pytest.mark.parametrize("path", FFN_PATHS)
def test_ffn_wave_accumulation(path):
    """Experts split into two waves (slot -1 skips), accumulated in fp32, equal one pass."""
    layer = Layer(mi.WORKLOADS["tiny"], T=11)
    _supported(path, layer.T, layer.wl.k)
    d = layer.to_device()
    wl = layer.wl
    ws = _ws(layer.T, wl.H, wl.I, wl.E, wl.k)
    t1 = torch.tensor([e if e < 4 else -1 for e in range(wl.E)], dtype=torch.int32, device="cuda")
    t2 = torch.tensor([e if e >= 4 else -1 for e in range(wl.E)], dtype=torch.int32, device="cuda")
    out = torch.empty((layer.T, wl.H), dtype=torch.bfloat16, device="cuda")
    args = (d["x"], d["idx"], d["wts"], d["w13"], d["s13"], d["w2"], d["s2"], wl.H, wl.I, wl.E, ws)
    q.moe_w4a16_ffn(*args, None, slot_of_expert=t1, flags=q.PATHS[path] | q.MOE_FLAG_ACCUMULATE)
    q.moe_w4a16_ffn(*args, out, slot_of_expert=t2, flags=q.PATHS[path] | q.MOE_FLAG_ACCUMULATE)
    torch.cuda.synchronize()
    assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"waves {path}")
    # the accumulator was cleared again: a plain call gives the same answer
    out2, _ = _run_ffn(layer, path)
    assert_ffn_close(bf16_dev_to_f32(out2), layer.oracle_out(), f"after waves {path}")


# ----------------------------------------------------------------------------- slot cache

def _make_cache(wl: mi.Workload, S: int, layer: Layer):
    E = wl.E
    bank = [torch.from_numpy(layer.w13).pin_memory(),
            torch.from_numpy(layer.s13.view(np.int16)).view(torch.bfloat16).pin_memory(),
            torch.from_numpy(layer.w2).pin_memory(),
            torch.from_numpy(layer.s2.view(np.int16)).view(torch.bfloat16).pin_memory()]
    pool = [torch.zeros((S,) + tuple(b.shape[1:]), dtype=b.dtype, device="cuda") for b in bank]
    return q.SlotCache(E, S, wl.H, wl.I, bank, pool)


def _replay_layer_waves(ref_state, needed, S):
    """The oracle's policy on the wave schedule of moe_slot_cache_layer for one step: with two or
    more slots, waves of at most S // 2 experts, each protecting the slots of the wave before it
    (its refills overlap that wave's FFN); with one slot, plain waves. Returns (waves, loads)."""
    cap = S // 2 if S >= 2 else S
    prot = np.zeros(S, np.uint8)
    waves = loads = 0
    while needed.any():
        table, ld = ref_state.wave(needed, cap=cap, protect=prot if S >= 2 else None)
        prot = np.zeros(S, np.uint8)
        prot[table[table >= 0]] = 1
        waves += 1
        loads += len(ld)
    return waves, loads

@pytest.mark.parametrize("path", FFN_PATHS)
def test_slot_cache_layer_matches_oracle(path):
    wl = mi.Workload("cache", H=256, I=128, E=8, k=3, T=3)
    base = Layer(wl)
    S = 3
    cache = _make_cache(wl, S, base)
    ref_state = oracle.SlotState(wl.E, S)
    copy_stream = torch.cuda.Stream()
    ws = _ws(wl.T, wl.H, wl.I, wl.E, wl.k)
    wave_tables = torch.empty(wl.E * (wl.E // S + 2), dtype=torch.int32, device="cuda")
    total_waves = 0
    for step in range(12):
        layer = Layer(wl, step=step, experts=[])
        layer.w13, layer.s13, layer.w2, layer.s2 = base.w13, base.s13, base.w2, base.s2
        d = layer.to_device()
        idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
        wts = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
        out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
        n_waves, n_loads = cache.layer(d["x"], d["logits"], wl.k, idx, wts, wave_tables, ws, out, path=q.PATHS[path],
                                       copy_stream=copy_stream)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(idx.cpu().numpy(), layer.idx)
        # replay the oracle's policy with the layer's wave schedule
        needed = np.zeros(wl.E, np.uint8)
        needed[np.unique(layer.idx)] = 1
        assert (n_waves, n_loads) == _replay_layer_waves(ref_state, needed, S)
        se, lu, clock = cache.state()
        np.testing.assert_array_equal(se, ref_state.slot_expert)
        np.testing.assert_array_equal(lu, ref_state.last_used)
        assert clock == ref_state.clock[0]
        assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"cache step {step}")
        total_waves += n_waves
    assert total_waves > 12          # some steps needed more than one wave (k*T > S)


@pytest.mark.parametrize("path", ["auto", "grouped"])
def test_slot_cache_olmoe_slots_full_size(path):
    """The batched-decode slot-cache workload at its own shapes: E=64 experts, 16 slots, 16 tokens
    per step, Zipf(1.1) routing (about 40 distinct experts per step, so five or six waves of at
    most 8), H=2048, I=1024, three consecutive steps of one layer. Waves, loads, LRU state and
    slot tables bit-exact against the oracle's policy; every step's output against the oracle's
    FFN."""
    wl = mi.WORKLOADS["olmoe_slots"]
    S = wl.slots
    base = Layer(wl, layer=4)
    cache = _make_cache(wl, S, base)
    ref_state = oracle.SlotState(wl.E, S)
    copy_stream = torch.cuda.Stream()
    ws = _ws(wl.T, wl.H, wl.I, wl.E, wl.k)
    wave_tables = torch.empty(wl.E * (wl.E // S + 2), dtype=torch.int32, device="cuda")
    seen_waves = 0
    for step in range(3):
        layer = Layer(wl, layer=4, step=step, experts=[])
        layer.w13, layer.s13, layer.w2, layer.s2 = base.w13, base.s13, base.w2, base.s2
        d = layer.to_device()
        idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
        wts = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
        out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
        n_waves, n_loads = cache.layer(d["x"], d["logits"], wl.k, idx, wts, wave_tables, ws, out,
                                       path=q.PATHS[path], copy_stream=copy_stream)
        torch.cuda.synchronize()
        assert q.moe_workspace_status(ws) == 0
        np.testing.assert_array_equal(idx.cpu().numpy(), layer.idx)
        np.testing.assert_allclose(wts.cpu().numpy(), layer.wts, rtol=ROUTE_RTOL)
        needed = np.zeros(wl.E, np.uint8)
        needed[np.unique(layer.idx)] = 1
        assert (n_waves, n_loads) == _replay_layer_waves(ref_state, needed, S)
        se, lu, clock = cache.state()
        np.testing.assert_array_equal(se, ref_state.slot_expert)
        np.testing.assert_array_equal(lu, ref_state.last_used)
        assert clock == ref_state.clock[0]
        assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"full: olmoe_slots step {step} {path}")
        seen_waves += n_waves
    assert seen_waves >= 6           # the routed set exceeded the 16 slots


def test_workspace_reused_across_sizes_and_paths():
    """One workspace sized for the largest call serves calls of other batch sizes and paths in
    turn (the counters that must start at zero sit at offsets that do not depend on T)."""
    wl = mi.Workload("reuse", H=512, I=256, E=16, k=4, T=64)
    layers = {T: Layer(wl, layer=1, step=T, T=T) for T in (1, 2, 4, 16, 64)}
    ws = _ws(64, wl.H, wl.I, wl.E, wl.k)
    seq = [(1, "auto"), (2, "auto"), (1, "decode"), (64, "grouped"), (16, "decode"), (4, "simple"),
           (1, "auto"), (16, "grouped"), (2, "decode"), (64, "auto"), (1, "decode")]
    for T, path in seq:
        layer = layers[T]
        d = layer.to_device()
        idx = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
        wts = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
        out = torch.empty((T, wl.H), dtype=torch.bfloat16, device="cuda")
        q.moe_w4a16_layer(d["x"], d["logits"], wl.k, d["w13"], d["s13"], d["w2"], d["s2"], wl.H, wl.I, idx, wts,
                          ws, out, flags=q.PATHS[path])
        torch.cuda.synchronize()
        assert q.moe_workspace_status(ws) == 0, (T, path)
        np.testing.assert_array_equal(idx.cpu().numpy(), layer.idx)
        assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"reused workspace T={T} {path}")


@pytest.mark.parametrize("path", ["decode", "grouped"])
def test_slot_cache_layer_after_a_failed_wave_is_clean(path):
    """A refill that fails in the second wave ends the layer call with MOE_ERR_CUDA after the
    first wave's FFN has written the workspace's fp32 accumulator. The next call on the same
    workspace starts its first wave by storing into the accumulator, not adding to it, so its
    output matches the oracle."""
    wl = mi.Workload("cachefail_layer", H=256, I=128, E=8, k=2, T=3)
    layer = Layer(wl, step=4)
    assert len(np.unique(layer.idx)) >= 3          # at least three waves of one expert (S = 2)
    S = 2
    cache = _make_cache(wl, S, layer)
    copy_stream = torch.cuda.Stream()
    ws = _ws(wl.T, wl.H, wl.I, wl.E, wl.k)
    wave_tables = torch.empty(wl.E * (wl.E // S + 2), dtype=torch.int32, device="cuda")
    d = layer.to_device()
    idx = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    wts = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    out = torch.empty((wl.T, wl.H), dtype=torch.bfloat16, device="cuda")
    cache.fail_copy_after(5)      # wave 1 (one expert, four copies) succeeds, wave 2's second copy fails
    with pytest.raises(q.MoeError) as ei:
        cache.layer(d["x"], d["logits"], wl.k, idx, wts, wave_tables, ws, out, path=q.PATHS[path],
                    copy_stream=copy_stream)
    assert ei.value.code == q.MOE_ERR_CUDA
    torch.cuda.synchronize()
    assert q.moe_workspace_status(ws) == 0
    out2 = torch.full((wl.T, wl.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    n_waves, _ = cache.layer(d["x"], d["logits"], wl.k, idx, wts, wave_tables, ws, out2, path=q.PATHS[path],
                             copy_stream=copy_stream)
    torch.cuda.synchronize()
    assert n_waves >= 2 and q.moe_workspace_status(ws) == 0
    assert_ffn_close(bf16_dev_to_f32(out2), layer.oracle_out(), f"slot cache after a failed wave {path}")


def test_slot_table_update_refill_failure_is_reported():
    wl = mi.Workload("cachefail", H=256, I=128, E=8, k=2, T=2)
    base = Layer(wl, experts=range(8))
    cache = _make_cache(wl, 2, base)
    copy_stream = torch.cuda.Stream()
    mask = np.array([0b00000110], dtype=np.uint64)         # experts 1 and 2
    table = np.zeros(wl.E, np.int32)
    misses = np.zeros(2, np.int32)
    cache.fail_copy_after(5)      # expert 1's four copies succeed, expert 2's second copy fails
    with pytest.raises(q.MoeError) as ei:
        cache.slot_table_update(mask, table, misses, copy_stream)
    assert ei.value.code == q.MOE_ERR_CUDA
    se, _, clock = cache.state()
    assert se.tolist() == [-1, -1] and clock == 0 and mask[0] == 0b110     # nothing committed
    # the next attempt succeeds and loads both
    n = cache.slot_table_update(mask, table, misses, copy_stream)
    torch.cuda.synchronize()
    assert n == 2 and misses.tolist() == [1, 2] and mask[0] == 0
    assert table.tolist() == [-1, 0, 1, -1, -1, -1, -1, -1]
    pool_w13 = cache.pool[0].cpu().numpy()
    np.testing.assert_array_equal(pool_w13[0], base.w13[1])
    np.testing.assert_array_equal(pool_w13[1], base.w13[2])
