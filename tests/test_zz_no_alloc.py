"""moe_w4a16_layer_noalloc: the layer call whose workspace is the library's static device array.

Collected last on purpose: it must also pass after every other test has run in the same
process (the array is shared by every call on a device and is cleared per call).
"""
import numpy as np
import pytest

import moe_inputs as mi

q = pytest.importorskip("quantized_mixture_experts_grouped_b200")


def test_noalloc_rejects_oversize_and_accumulate():
    """Host-side checks, before any device work: sizes whose workspace exceeds the 16 MiB array,
    and MOE_FLAG_ACCUMULATE (whose fp32 accumulator every call would share)."""
    rc = q.lib.moe_w4a16_layer_noalloc(None, None, 512, 4096, 14336, 8, 2, None, None, None, None, None,
                                       None, None, None, q.MOE_PATH_AUTO, None)
    assert rc == q.MOE_ERR_SHAPE
    assert b"static scratch" in q.lib.moe_last_error_string()
    rc = q.lib.moe_w4a16_layer_noalloc(None, None, 1, 2048, 1024, 64, 8, None, None, None, None, None,
                                       None, None, None, q.MOE_PATH_AUTO | q.MOE_FLAG_ACCUMULATE, None)
    assert rc == q.MOE_ERR_ARG


@pytest.mark.gpu
def test_noalloc_matches_layer_call_twice():
    """Two calls in a row of the no-allocation entry agree with moe_w4a16_layer (caller
    workspace) and with the oracle, on the one-token OLMoE decode layer and a small batch."""
    import torch
    from gpu_util import Layer, assert_ffn_close, bf16_dev_to_f32, ROUTE_RTOL

    cases = []
    wl = mi.WORKLOADS["olmoe_decode"]
    probe = Layer(mi.Workload("p", H=128, I=128, E=wl.E, k=wl.k, T=1, routing=wl.routing, seed=wl.seed),
                  layer=3, step=7, experts=[])
    routed = sorted(set(probe.idx.ravel().tolist()))
    cases.append(Layer(wl, layer=3, step=7, T=1, experts=routed, logits=probe.logits))
    cases.append(Layer(mi.Workload("small", H=512, I=256, E=16, k=4, T=6), layer=2, step=1))
    for layer in cases:
        w = layer.wl
        T = layer.x.shape[0]
        d = layer.to_device()
        ws = q.alloc_workspace(T, w.H, w.I, w.E, w.k)
        idx_ref = torch.full((T, w.k), -1, dtype=torch.int32, device="cuda")
        wts_ref = torch.zeros((T, w.k), dtype=torch.float32, device="cuda")
        out_ref = torch.empty((T, w.H), dtype=torch.bfloat16, device="cuda")
        q.moe_w4a16_layer(d["x"], d["logits"], w.k, d["w13"], d["s13"], d["w2"], d["s2"], w.H, w.I, idx_ref,
                          wts_ref, ws, out_ref)
        torch.cuda.synchronize()
        assert q.moe_workspace_status(ws) == 0
        ref = bf16_dev_to_f32(out_ref)
        oracle_out = layer.oracle_out()
        for rep in range(2):
            idx = torch.full((T, w.k), -1, dtype=torch.int32, device="cuda")
            wts = torch.zeros((T, w.k), dtype=torch.float32, device="cuda")
            out = torch.full((T, w.H), float("nan"), dtype=torch.bfloat16, device="cuda")
            q.moe_w4a16_layer_noalloc(d["x"], d["logits"], w.k, d["w13"], d["s13"], d["w2"], d["s2"], w.H, w.I,
                                      idx, wts, out)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(idx.cpu().numpy(), layer.idx)
            np.testing.assert_allclose(wts.cpu().numpy(), layer.wts, rtol=ROUTE_RTOL)
            assert q.moe_noalloc_status() == 0
            got = bf16_dev_to_f32(out)
            assert_ffn_close(got, ref, f"{w.name} no-alloc vs layer call, rep {rep}")
            assert_ffn_close(got, oracle_out, f"{w.name} no-alloc vs oracle, rep {rep}")


@pytest.mark.gpu
def test_noalloc_grouped_path_and_reuse_across_sizes():
    """Calls that the default path sends to the grouped GEMMs (64 tokens), and calls of other batch
    sizes in between, through the one static array: each against the oracle, status clean."""
    import torch
    from gpu_util import Layer, assert_ffn_close, bf16_dev_to_f32

    wl = mi.WORKLOADS["tiny"]
    for T in (64, 1, 16, 64, 3):
        layer = Layer(wl, T=T, step=T)
        d = layer.to_device()
        idx = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
        wts = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
        out = torch.full((T, wl.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        q.moe_w4a16_layer_noalloc(d["x"], d["logits"], wl.k, d["w13"], d["s13"], d["w2"], d["s2"], wl.H, wl.I,
                                  idx, wts, out)
        torch.cuda.synchronize()
        assert q.moe_noalloc_status() == 0
        np.testing.assert_array_equal(idx.cpu().numpy(), layer.idx)
        assert_ffn_close(bf16_dev_to_f32(out), layer.oracle_out(), f"no-alloc tiny T={T}")
