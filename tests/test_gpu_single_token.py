"""GPU parity of the single-token decode kernel (T = 1, the default decode path for one token):
slot-cache waves including waves with no resident expert, permuted slots, run-to-run identity,
k = E, other H / I, and the fallback to the batched decode kernel when k > 32. The oracle is the
reference throughout; tolerances as in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from gpu_util import Layer, assert_ffn_close, bf16_dev_to_f32

pytestmark = pytest.mark.gpu

q = pytest.importorskip("quantized_mixture_experts_grouped_b200")

PATHS = ["auto", "decode"]


def _call(layer: Layer, path: str, ws, out, slot=None, accumulate=False):
    d = layer.to_device()
    wl = layer.wl
    flags = q.PATHS[path] | (q.MOE_FLAG_ACCUMULATE if accumulate else 0)
    q.moe_w4a16_ffn(d["x"], d["idx"], d["wts"], d["w13"], d["s13"], d["w2"], d["s2"], wl.H, wl.I, wl.E, ws, out,
                    slot_of_expert=slot, flags=flags)


def _run(layer: Layer, path: str, slot=None):
    wl = layer.wl
    ws = q.alloc_workspace(1, wl.H, wl.I, wl.E, wl.k)
    out = torch.empty((1, wl.H), dtype=torch.bfloat16, device="cuda")
    _call(layer, path, ws, out, slot)
    torch.cuda.synchronize()
    assert q.moe_workspace_status(ws) == 0
    return out


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("shape", [(256, 128, 8, 2), (1024, 512, 32, 6), (2048, 1024, 64, 8), (512, 384, 4, 4)])
def test_single_token_shapes(path, shape):
    """Several H / I (K groups 2..16), k from 2 to E."""
    H, I, E, k = shape
    layer = Layer(mi.Workload("one", H=H, I=I, E=E, k=k, T=1), step=H + k)
    assert_ffn_close(bf16_dev_to_f32(_run(layer, path)), layer.oracle_out(), f"T=1 {shape} {path}")


@pytest.mark.parametrize("path", PATHS)
def test_single_token_waves(path):
    """Slot-cache waves at T = 1: a wave with no resident expert (accumulator only), two waves
    that split the routed experts, and a final wave with none resident that writes the output
    from the accumulator alone."""
    layer = Layer(mi.WORKLOADS["tiny"], T=1, step=5)
    wl = layer.wl
    E = wl.E
    ws = q.alloc_workspace(1, wl.H, wl.I, E, wl.k)
    none = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    t1 = torch.tensor([e if e < E // 2 else -1 for e in range(E)], dtype=torch.int32, device="cuda")
    t2 = torch.tensor([e if e >= E // 2 else -1 for e in range(E)], dtype=torch.int32, device="cuda")
    out = torch.empty((1, wl.H), dtype=torch.bfloat16, device="cuda")
    _call(layer, path, ws, None, slot=none, accumulate=True)
    _call(layer, path, ws, None, slot=t1, accumulate=True)
    _call(layer, path, ws, None, slot=t2, accumulate=True)
    _call(layer, path, ws, out, slot=none, accumulate=True)
    torch.cuda.synchronize()
    assert q.moe_workspace_status(ws) == 0
    assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"T=1 waves {path}")
    # the accumulator was cleared by the final wave: a plain call gives the same answer
    out2 = torch.empty_like(out)
    _call(layer, path, ws, out2)
    torch.cuda.synchronize()
    assert q.moe_workspace_status(ws) == 0
    assert_ffn_close(bf16_dev_to_f32(out2), layer.oracle_out(), f"T=1 after waves {path}")


@pytest.mark.parametrize("path", PATHS)
def test_single_token_slots_and_identity(path):
    """Bit-identical results run to run, and with the experts stored in permuted slots."""
    layer = Layer(mi.Workload("one_perm", H=512, I=256, E=16, k=4, T=1), step=9)
    a = _run(layer, path)
    b = _run(layer, path)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    d = layer.to_device()
    E = layer.wl.E
    perm = np.random.default_rng(7).permutation(E).astype(np.int32)
    banks = [torch.empty_like(d[n]) for n in ("w13", "s13", "w2", "s2")]
    for e in range(E):
        for bnk, n in zip(banks, ("w13", "s13", "w2", "s2")):
            bnk[perm[e]] = d[n][e]
    ws = q.alloc_workspace(1, layer.wl.H, layer.wl.I, E, layer.wl.k)
    c = torch.empty_like(a)
    q.moe_w4a16_ffn(d["x"], d["idx"], d["wts"], *banks, layer.wl.H, layer.wl.I, E, ws, c,
                    slot_of_expert=torch.from_numpy(perm).cuda(), flags=q.PATHS[path])
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), c.view(torch.int16))


@pytest.mark.parametrize("path", PATHS)
def test_single_token_many_choices_falls_back(path):
    """k > 32 is outside the single-token kernel; the batched decode kernel takes it."""
    layer = Layer(mi.Workload("one_wide", H=256, I=128, E=64, k=40, T=1), step=3)
    assert_ffn_close(bf16_dev_to_f32(_run(layer, path)), layer.oracle_out(), f"T=1 k=40 {path}")


def test_single_token_duplicate_routing_is_reported():
    """Given routing that names one expert twice for the token is reported in the status word."""
    layer = Layer(mi.WORKLOADS["tiny"], T=1, step=2)
    wl = layer.wl
    d = layer.to_device()
    idx = torch.tensor([[3, 3]], dtype=torch.int32, device="cuda")
    wts = torch.tensor([[0.5, 0.5]], dtype=torch.float32, device="cuda")
    ws = q.alloc_workspace(1, wl.H, wl.I, wl.E, wl.k)
    out = torch.empty((1, wl.H), dtype=torch.bfloat16, device="cuda")
    q.moe_w4a16_ffn(d["x"], idx, wts, d["w13"], d["s13"], d["w2"], d["s2"], wl.H, wl.I, wl.E, ws, out,
                    flags=q.MOE_PATH_DECODE)
    torch.cuda.synchronize()
    assert q.moe_workspace_status(ws) == q.MOE_ERR_ARG


def test_single_token_wait_timeout_is_reported_and_workspace_recovers():
    """Failure detection without a GPU fault: with a short wait limit (about 0.1 ms) and an
    exchange that waits for one arrival more than the kernel launches, the bounded wait runs out,
    the kernel records MOE_ERR_TIMEOUT in the workspace status word and exits. The next call on
    the same workspace, with the hook off, runs normally and matches the oracle."""
    wl = mi.WORKLOADS["olmoe_decode"]
    probe = Layer(mi.Workload("p", H=128, I=128, E=wl.E, k=wl.k, T=1, routing=wl.routing, seed=wl.seed),
                  layer=6, step=2, experts=[])
    routed = sorted(set(probe.idx.ravel().tolist()))
    layer = Layer(wl, layer=6, step=2, T=1, experts=routed, logits=probe.logits)
    ws = q.alloc_workspace(1, wl.H, wl.I, wl.E, wl.k)
    out = torch.empty((1, wl.H), dtype=torch.bfloat16, device="cuda")
    try:
        q.moe_debug_set_wait_limit(200_000, 1)
        _call(layer, "decode", ws, out)
        torch.cuda.synchronize()
    finally:
        q.moe_debug_set_wait_limit(0, 0)
    assert q.moe_workspace_status(ws) == q.MOE_ERR_TIMEOUT
    assert q.moe_workspace_status(ws) == 0          # read-and-clear
    for rep in range(2):
        out2 = torch.full((1, wl.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        _call(layer, "decode", ws, out2)
        torch.cuda.synchronize()
        assert q.moe_workspace_status(ws) == 0
        assert_ffn_close(bf16_dev_to_f32(out2), layer.oracle_out(), f"T=1 after a timeout, rep {rep}")
