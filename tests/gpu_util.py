"""Helpers shared by the GPU parity tests: layer setup from seeded inputs, comparisons."""
import numpy as np
import torch

import moe_inputs as mi
import oracle

# FFN tolerance (fixed by the benchmark spec for the W4A16 layer): max-abs <= 2e-2 and
# relative L2 <= 5e-3 against the oracle on the same dequantised weights.
FFN_MAX_ABS = 2e-2
FFN_REL_L2 = 5e-3
# Router weights: fp32 softmax on the device vs fp64 in the oracle. The device error is a few
# ulp (expf <= 2 ulp, a k-term sum, two divisions), below 2e-6 relative.
ROUTE_RTOL = 2e-6


def bits_to_dev(a: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> bf16 device tensor (bit exact)."""
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def dev_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_dev_to_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


class Layer:
    """One MoE layer's inputs, packed on the host by the oracle and uploaded unchanged."""

    def __init__(self, wl: mi.Workload, layer: int = 0, step: int = 0, T: int | None = None,
                 experts=None, x=None, logits=None):
        self.wl = wl
        self.T = wl.T if T is None else T
        self.x = mi.activations(wl, layer, step, self.T) if x is None else x
        self.logits = mi.router_logits(wl, layer, step, self.T) if logits is None else logits
        E = wl.E
        self.idx, self.wts = oracle.route(self.logits, wl.k)
        need = set(range(E)) if experts is None else set(experts)
        self.w13 = np.zeros((E, oracle.packed_bytes(2 * wl.I, wl.H)), np.uint8)
        self.s13 = np.zeros((E, oracle.scale_count(2 * wl.I, wl.H)), np.uint16)
        self.w2 = np.zeros((E, oracle.packed_bytes(wl.H, wl.I)), np.uint8)
        self.s2 = np.zeros((E, oracle.scale_count(wl.H, wl.I)), np.uint16)
        for e in sorted(need):
            a, b = mi.expert_weights(wl, layer, e)
            self.w13[e], self.s13[e] = oracle.pack(*oracle.quantize(a))
            self.w2[e], self.s2[e] = oracle.pack(*oracle.quantize(b))
        self.dev = None

    def to_device(self):
        if self.dev is None:
            self.dev = dict(
                x=bits_to_dev(self.x), logits=bits_to_dev(self.logits),
                w13=torch.from_numpy(self.w13).cuda(), s13=bits_to_dev(self.s13),
                w2=torch.from_numpy(self.w2).cuda(), s2=bits_to_dev(self.s2),
                idx=torch.from_numpy(self.idx).cuda(), wts=torch.from_numpy(self.wts).cuda())
        return self.dev

    def oracle_out(self, tokens=None, active=None):
        return oracle.moe_ffn(self.x, self.idx, self.wts, self.w13, self.s13, self.w2, self.s2,
                              self.wl.H, self.wl.I, tokens=tokens, active=active)


# (case, max-abs error, relative L2 error) of every FFN comparison in this process, printed at
# the end of the run (tests/conftest.py) so that each case's margin against the tolerance shows.
FFN_RESULTS: list = []


def assert_ffn_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = got.astype(np.float64)
    ref = ref.astype(np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs = float(np.max(np.abs(got - ref))) if got.size else 0.0
    denom = float(np.linalg.norm(ref)) or 1.0
    rel = float(np.linalg.norm(got - ref)) / denom
    FFN_RESULTS.append((what, max_abs, rel))
    assert max_abs <= FFN_MAX_ABS and rel <= FFN_REL_L2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel
