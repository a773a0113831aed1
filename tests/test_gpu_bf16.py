"""GPU parity of the BF16 comparison layer (moe_bf16_ffn / moe_bf16_layer: the grouped scheduler
and tcgen05 GEMMs on unquantised bf16 experts) against the oracle's FFN on the same bf16 weights,
within the tolerance of the W4A16 layer (max-abs 2e-2, relative L2 5e-3). Covers ragged token
chunks, the down GEMM's K split (decode-sized batches, three K groups split 1 + 2), an expert
taking every token, experts with none, waves through the expert -> slot table, and the OLMoE
prefill layer on a stratified sample of its tokens."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
import oracle
from gpu_util import assert_ffn_close, bits_to_dev, bf16_dev_to_f32, ROUTE_RTOL

pytestmark = pytest.mark.gpu

q = pytest.importorskip("quantized_mixture_experts_grouped_b200")


class Bf16Layer:
    def __init__(self, wl, layer=0, step=0, T=None, experts=None, logits=None):
        self.wl = wl
        self.T = wl.T if T is None else T
        self.x = mi.activations(wl, layer, step, self.T)
        self.logits = mi.router_logits(wl, layer, step, self.T) if logits is None else logits
        self.idx, self.wts = oracle.route(self.logits, wl.k)
        need = range(wl.E) if experts is None else experts
        self.w13 = np.zeros((wl.E, 2 * wl.I, wl.H), np.uint16)
        self.w2 = np.zeros((wl.E, wl.H, wl.I), np.uint16)
        for e in need:
            self.w13[e], self.w2[e] = mi.expert_weights(wl, layer, e)

    def dev(self):
        return dict(x=bits_to_dev(self.x), logits=bits_to_dev(self.logits), w13=bits_to_dev(self.w13),
                    w2=bits_to_dev(self.w2), idx=torch.from_numpy(self.idx).cuda(),
                    wts=torch.from_numpy(self.wts).cuda())

    def oracle_out(self, tokens=None, active=None):
        return oracle.moe_ffn_bf16(self.x, self.idx, self.wts, self.w13, self.w2, self.wl.H, self.wl.I,
                                   tokens=tokens, active=active)


def _layer_call(layer, d, ws):
    wl, T = layer.wl, layer.T
    idx = torch.full((T, wl.k), -1, dtype=torch.int32, device="cuda")
    wts = torch.zeros((T, wl.k), dtype=torch.float32, device="cuda")
    out = torch.full((T, wl.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    q.moe_bf16_layer(d["x"], d["logits"], wl.k, d["w13"], d["w2"], wl.H, wl.I, idx, wts, ws, out)
    torch.cuda.synchronize()
    assert q.moe_workspace_status(ws) == 0
    np.testing.assert_array_equal(idx.cpu().numpy(), layer.idx)
    np.testing.assert_allclose(wts.cpu().numpy(), layer.wts, rtol=ROUTE_RTOL)
    return bf16_dev_to_f32(out)


@pytest.mark.parametrize("T", [1, 4, 17, 64])
def test_bf16_layer_tiny(T):
    wl = mi.WORKLOADS["tiny"]
    layer = Bf16Layer(wl, T=T, step=T)
    ws = q.alloc_workspace(T, wl.H, wl.I, wl.E, wl.k)
    got = _layer_call(layer, layer.dev(), ws)
    assert_ffn_close(got, layer.oracle_out(), f"bf16 tiny T={T}")


@pytest.mark.parametrize("T", [37, 5])
def test_bf16_edge_cases(T):
    """One expert takes every token, two get none; I = 384 (three K groups: the down GEMM's K
    split is uneven at the small batch)."""
    wl = mi.Workload("edge_bf16", H=512, I=384, E=8, k=3, T=T)
    g = np.random.default_rng(T)
    lg = g.standard_normal((T, wl.E)).astype(np.float32)
    lg[:, 5] += 100.0
    lg[:, 0] -= 100.0
    lg[:, 7] -= 100.0
    layer = Bf16Layer(wl, logits=mi.to_bf16_bits(lg))
    ws = q.alloc_workspace(T, wl.H, wl.I, wl.E, wl.k)
    got = _layer_call(layer, layer.dev(), ws)
    assert_ffn_close(got, layer.oracle_out(), f"bf16 edge T={T}")


@pytest.mark.parametrize("T", [1, 16])
def test_bf16_olmoe_decode_shapes(T):
    wl = mi.WORKLOADS["olmoe_decode"]
    probe = Bf16Layer(mi.Workload("p", H=128, I=128, E=wl.E, k=wl.k, T=T, seed=wl.seed), layer=2, step=5,
                      experts=[])
    routed = sorted(set(probe.idx.ravel().tolist()))
    layer = Bf16Layer(wl, layer=2, step=5, T=T, experts=routed, logits=probe.logits)
    ws = q.alloc_workspace(T, wl.H, wl.I, wl.E, wl.k)
    got = _layer_call(layer, layer.dev(), ws)
    assert_ffn_close(got, layer.oracle_out(), f"bf16 olmoe T={T}")


def test_bf16_waves_through_the_slot_table():
    """Experts split into two waves (slot -1 skips), accumulated in fp32, equal one pass."""
    wl = mi.WORKLOADS["tiny"]
    layer = Bf16Layer(wl, T=11, step=3)
    d = layer.dev()
    ws = q.alloc_workspace(11, wl.H, wl.I, wl.E, wl.k)
    t1 = torch.tensor([e if e < 4 else -1 for e in range(wl.E)], dtype=torch.int32, device="cuda")
    t2 = torch.tensor([e if e >= 4 else -1 for e in range(wl.E)], dtype=torch.int32, device="cuda")
    out = torch.empty((11, wl.H), dtype=torch.bfloat16, device="cuda")
    args = (d["x"], d["idx"], d["wts"], d["w13"], d["w2"], wl.H, wl.I, wl.E, ws)
    q.moe_bf16_ffn(*args, None, slot_of_expert=t1)
    q.moe_bf16_ffn(*args, out, slot_of_expert=t2, flags=q.MOE_FLAG_ACCUMULATE)
    torch.cuda.synchronize()
    assert q.moe_workspace_status(ws) == 0
    assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), "bf16 waves")


def test_bf16_prefill_full_size_sampled():
    """The OLMoE prefill layer (2048 tokens, Zipf routing) on bf16 weights; compared on 256 tokens
    that include, for every expert, its first and last token (first and last 128-token chunk)."""
    wl = mi.WORKLOADS["olmoe_prefill"]
    layer = Bf16Layer(wl)
    ws = q.alloc_workspace(wl.T, wl.H, wl.I, wl.E, wl.k)
    got = _layer_call(layer, layer.dev(), ws)
    assert np.all(np.isfinite(got))
    picks = set(range(0, wl.T, 16))
    for e in range(wl.E):
        toks = np.nonzero((layer.idx == e).any(axis=1))[0]
        if len(toks):
            picks.update((int(toks[0]), int(toks[-1])))
    tokens = sorted(picks)
    assert_ffn_close(got[tokens], layer.oracle_out(tokens=tokens), f"full: bf16 prefill ({len(tokens)} tokens)")


def test_bf16_rejects_paths_other_than_grouped():
    wl = mi.WORKLOADS["tiny"]
    layer = Bf16Layer(wl, T=4)
    d = layer.dev()
    ws = q.alloc_workspace(4, wl.H, wl.I, wl.E, wl.k)
    out = torch.empty((4, wl.H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(q.MoeError) as ei:
        q.moe_bf16_ffn(d["x"], d["idx"], d["wts"], d["w13"], d["w2"], wl.H, wl.I, wl.E, ws, out,
                       flags=q.MOE_PATH_DECODE)
    assert ei.value.code == q.MOE_ERR_ARG
