"""Pins of the CPU oracle against what the method and mathematics fix (no GPU needed).

Each check compares the oracle with something other than itself: hand-worked fixtures under
tests/golden/, closed forms, brute force on tiny inputs, invariants, and library routines
(torch bf16 rounding, numpy sorting, scipy softmax, numpy matmul).
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import moe_inputs as mi
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(a):
    return mi.to_bf16_bits(np.asarray(a, np.float32))


def _f32(b):
    return mi.bf16_bits_to_f32(b)


# ----------------------------------------------------------------------------- quantiser

def _read_quant_golden():
    groups, cur = {}, None
    for line in open(os.path.join(GOLDEN, "quant_groups.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        tok = line.split()
        if tok[0] == "group":
            cur = tok[1]
            groups[cur] = {"scale": int(tok[3], 16), "entries": []}
        else:
            groups[cur]["entries"].append((int(tok[0]), int(tok[1], 16), int(tok[2])))
    return groups


def test_quantize_hand_worked_groups():
    groups = _read_quant_golden()
    names = sorted(groups)
    w = np.zeros((128, 128 * len(names)), np.uint16)
    for gi, name in enumerate(names):
        for k, wb, _ in groups[name]["entries"]:
            w[0, gi * 128 + k] = wb
    q, s = oracle.quantize(w)
    for gi, name in enumerate(names):
        assert s[0, gi] == groups[name]["scale"], name
        expect = np.zeros(128, np.int8)
        for k, _, qv in groups[name]["entries"]:
            expect[k] = qv
        np.testing.assert_array_equal(q[0, gi * 128:(gi + 1) * 128], expect, err_msg=name)
    # rows 1.. are all zero -> zero scale and zero codes
    assert not s[1:].any() and not q[1:].any()


@pytest.mark.parametrize("dist", ["normal", "heavy", "tiny", "mixed"])
def test_quantize_roundtrip_bound_and_scale(dist):
    """|w - q*s| <= s/2 for every element (up to the fp32 rounding of w/s), and the stored
    scale equals torch's bf16 rounding of fp32(max|w|)/7."""
    g = np.random.default_rng(11)
    N, K = 256, 512
    if dist == "normal":
        w = g.standard_normal((N, K)) * 0.02
    elif dist == "heavy":
        w = g.standard_t(2, (N, K)) * 0.05
    elif dist == "tiny":
        w = g.standard_normal((N, K)) * 1e-30
    else:
        w = g.standard_normal((N, K)) * np.exp(g.uniform(-20, 5, (N, 1)))
    wb = _bf16(w)
    q, s = oracle.quantize(wb)
    wf = _f32(wb).astype(np.float64).reshape(N, K // 128, 128)
    sf = _f32(s).astype(np.float64)
    err = np.abs(wf - q.reshape(N, K // 128, 128) * sf[..., None])
    slack = np.abs(wf) * 2.0 ** -23
    assert np.all(err <= sf[..., None] / 2 + slack)
    absmax = np.abs(_f32(wb)).reshape(N, K // 128, 128).max(-1).astype(np.float32)
    expect = (torch.from_numpy(absmax / np.float32(7.0)).to(torch.bfloat16)
              .view(torch.int16).numpy().view(np.uint16))
    np.testing.assert_array_equal(s, expect)
    # the symmetric codes never need -8: |w/s| <= 7*(1+2^-8) < 7.5
    assert q.min() >= -7 and q.max() <= 7


def test_quantize_exact_grid_is_lossless():
    """Weights on the grid w = s*m with max|m| = 7 in every group quantise with zero error."""
    g = np.random.default_rng(3)
    N, K = 128, 384
    # scales with at most 5 significant bits, so that every m*s (|m| <= 7) is bf16-exact
    s = ((16 + g.integers(0, 16, (N, K // 128))) / 16.0 * 2.0 ** g.integers(-12, 3, (N, K // 128))).astype(np.float32)
    m = g.integers(-7, 8, (N, K)).astype(np.float32)
    m[:, ::128] = 7.0
    w = (m.reshape(N, K // 128, 128) * s[..., None]).reshape(N, K)
    wb = _bf16(w)
    assert np.array_equal(_f32(wb), w), "grid values must be bf16-exact"
    q, sq = oracle.quantize(wb)
    np.testing.assert_array_equal(_f32(sq), s)
    np.testing.assert_array_equal(q, m.astype(np.int8))


def test_quantize_zero_group_and_library_rounding():
    g = np.random.default_rng(5)
    w = g.standard_normal((128, 256)).astype(np.float32) * 0.02
    w[7, 128:] = 0.0
    wb = _bf16(w)
    q, s = oracle.quantize(wb)
    assert s[7, 1] == 0 and not q[7, 128:].any()
    # the codes agree with torch's half-to-even rounding of the fp32 quotient
    wt = torch.from_numpy(_f32(wb)).reshape(128, 2, 128)
    st = torch.from_numpy(_f32(s)).reshape(128, 2, 1)
    qt = torch.where(st == 0, torch.zeros_like(wt), torch.clamp(torch.round(wt / st), -8, 7))
    np.testing.assert_array_equal(q, qt.reshape(128, 256).numpy().astype(np.int8))


# ----------------------------------------------------------------------------- packing

def _read_pack_golden():
    cases, cur = [], None
    for line in open(os.path.join(GOLDEN, "pack_bytes.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        tok = line.split()
        if tok[0] == "matrix":
            cur = {"N": int(tok[1]), "K": int(tok[2]), "q": [], "bytes": [], "scale": []}
            cases.append(cur)
        elif tok[0] == "q":
            cur["q"].append(tuple(int(t) for t in tok[1:]))
        elif tok[0] == "byte":
            cur["bytes"].append((int(tok[1]), int(tok[2], 16)))
        elif tok[0] == "scale":
            cur["scale"].append(tuple(int(t) for t in tok[1:]))
    return cases


def test_pack_hand_worked_bytes():
    for case in _read_pack_golden():
        N, K = case["N"], case["K"]
        q = np.full((N, K), -8, np.int8)
        for n, k, v in case["q"]:
            q[n, k] = v
        s = np.arange(N * (K // 128), dtype=np.uint16).reshape(N, K // 128)
        packed, st = oracle.pack(q, s)
        listed = dict(case["bytes"])
        for off, val in listed.items():
            assert packed[off] == val, (N, K, off)
        others = np.ones(len(packed), bool)
        others[list(listed)] = False
        assert not packed[others].any()
        for n, g, pos in case["scale"]:
            assert st[pos] == s[n, g]


def test_pack_unpack_roundtrip_all_codes():
    g = np.random.default_rng(9)
    for N, K in [(128, 128), (256, 384), (384, 256)]:
        q = g.integers(-8, 8, (N, K)).astype(np.int8)
        # every code in every nibble position of at least one word
        q[0, :128] = np.tile(np.arange(-8, 8), 8)
        q[1, :128] = np.repeat(np.arange(-8, 8), 8)
        s = g.integers(0, 1 << 16, (N, K // 128)).astype(np.uint16)
        packed, st = oracle.pack(q, s)
        q2, s2 = oracle.unpack(packed, st, N, K)
        np.testing.assert_array_equal(q, q2)
        np.testing.assert_array_equal(s, s2)
        # two codes per byte: the packed size is exactly N*K/2 bytes
        assert packed.nbytes == N * K // 2
        # dequant is q * s exactly
        sf = np.where(np.isfinite(_f32(s)), _f32(s), 0).astype(np.float32)
        s_fin = _bf16(sf)
        packed, st = oracle.pack(q, s_fin)
        deq = oracle.dequant(packed, st, N, K)
        # random scale bits include bf16 values near the fp32 maximum: q * s then overflows to
        # +-inf, in the oracle as here, and the two must still agree
        with np.errstate(over="ignore"):
            expect = (q.reshape(N, K // 128, 128) * _f32(s_fin)[..., None]).reshape(N, K)
        np.testing.assert_array_equal(deq, expect)


def test_pack_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.pack(np.zeros((100, 128), np.int8), np.zeros((100, 1), np.uint16))
    with pytest.raises(ValueError):
        oracle.quantize(np.zeros((128, 100), np.uint16))


# ----------------------------------------------------------------------------- router

def test_route_hand_worked_ties():
    for line in open(os.path.join(GOLDEN, "route_ties.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, lg, ids = line.split("|")
        _, E, k = head.split()
        E, k = int(E), int(k)
        logits = np.array([float(v) for v in lg.split()], np.float32)
        expect = [int(v) for v in ids.split()]
        idx, wts = oracle.route(_bf16(logits)[None, :], k)
        assert idx[0].tolist() == expect, line
        sel = logits[expect].astype(np.float64)
        closed = np.exp(sel) / np.exp(sel).sum()
        np.testing.assert_allclose(wts[0], closed, rtol=1e-6)


@pytest.mark.parametrize("T,E,k", [(64, 8, 2), (33, 64, 8), (17, 64, 64), (5, 3, 1)])
def test_route_matches_full_sort_and_softmax(T, E, k):
    g = np.random.default_rng(T * 100 + E)
    logits = g.standard_normal((T, E)).astype(np.float32)
    logits[:, ::3] = np.round(logits[:, ::3])          # many exact ties
    lb = _bf16(logits)
    idx, wts = oracle.route(lb, k)
    lf = _f32(lb)
    for t in range(T):
        order = np.argsort(-lf[t], kind="stable")      # library sort: ties keep the lower id
        assert idx[t].tolist() == order[:k].tolist()
        assert len(set(idx[t].tolist())) == k
        full = scipy.special.softmax(lf[t].astype(np.float64))
        renorm = full[idx[t]] / full[idx[t]].sum()
        np.testing.assert_allclose(wts[t], renorm, rtol=1e-6)
        assert abs(float(wts[t].astype(np.float64).sum()) - 1.0) <= 1e-6
        # the renormalised weights equal a softmax over the selected logits alone
        np.testing.assert_allclose(wts[t], scipy.special.softmax(lf[t][idx[t]].astype(np.float64)), rtol=1e-6)


def test_route_k_equals_e_is_plain_softmax():
    g = np.random.default_rng(1)
    lb = _bf16(g.standard_normal((4, 8)))
    idx, wts = oracle.route(lb, 8)
    for t in range(4):
        p = torch.softmax(torch.from_numpy(_f32(lb[t]).astype(np.float64)), 0).numpy()
        np.testing.assert_allclose(wts[t], p[idx[t]], rtol=1e-6)


# ----------------------------------------------------------------------------- permute

@pytest.mark.parametrize("T,E,k", [(1, 64, 8), (16, 64, 8), (300, 8, 2)])
def test_permute_matches_library_sort(T, E, k):
    g = np.random.default_rng(T)
    idx = np.stack([g.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = oracle.permute(idx, E)
    np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=E))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    np.testing.assert_array_equal(perm, np.argsort(idx.ravel(), kind="stable"))
    np.testing.assert_array_equal(inv, np.argsort(perm))


# ----------------------------------------------------------------------------- FFN

def _tiny_layer(H=256, I=128, E=8, k=2, T=6, seed=0, w_std=0.02):
    wl = mi.Workload("t", H=H, I=I, E=E, k=k, T=T, w_std=w_std, seed=seed)
    x = mi.activations(wl)
    logits = mi.router_logits(wl)
    w13b, w2b = mi.bank_weights(wl)
    w13, s13 = oracle.quantize_pack_bank(w13b)
    w2, s2 = oracle.quantize_pack_bank(w2b)
    return wl, x, logits, w13, s13, w2, s2


def _silu(z):
    return z / (1.0 + np.exp(-z))


def _dense_moe(wl, x, idx, wts, w13, s13, w2, s2):
    """Dense brute force: every expert on every token (numpy fp64 matmuls), masked by the
    routed weights."""
    H, I, E = wl.H, wl.I, wl.E
    xf = _f32(x).astype(np.float64)
    T = xf.shape[0]
    mask = np.zeros((T, E))
    for t in range(T):
        for j in range(idx.shape[1]):
            mask[t, idx[t, j]] += wts[t, j]
    out = np.zeros((T, H))
    for e in range(E):
        W13 = oracle.dequant(w13[e], s13[e], 2 * I, H).astype(np.float64)
        W2 = oracle.dequant(w2[e], s2[e], H, I).astype(np.float64)
        h = _silu(xf @ W13[:I].T) * (xf @ W13[I:].T)
        out += mask[:, e:e + 1] * (h @ W2.T)
    return out


def test_ffn_sparse_equals_dense_brute_force():
    wl, x, logits, w13, s13, w2, s2 = _tiny_layer()
    idx, wts = oracle.route(logits, wl.k)
    out = oracle.moe_ffn(x, idx, wts, w13, s13, w2, s2, wl.H, wl.I)
    dense = _dense_moe(wl, x, idx, wts, w13, s13, w2, s2)
    np.testing.assert_allclose(out, dense, rtol=1e-5, atol=1e-7)


def test_ffn_single_expert_is_swiglu():
    """k = E = 1: the layer is one SwiGLU MLP with weight 1."""
    wl, x, logits, w13, s13, w2, s2 = _tiny_layer(E=1, k=1, T=3)
    idx, wts = oracle.route(logits, 1)
    assert np.all(idx == 0) and np.all(wts == 1.0)
    out = oracle.moe_ffn(x, idx, wts, w13, s13, w2, s2, wl.H, wl.I)
    Wg = oracle.dequant(w13[0], s13[0], 2 * wl.I, wl.H)[: wl.I].astype(np.float64)
    Wu = oracle.dequant(w13[0], s13[0], 2 * wl.I, wl.H)[wl.I:].astype(np.float64)
    Wd = oracle.dequant(w2[0], s2[0], wl.H, wl.I).astype(np.float64)
    xf = _f32(x).astype(np.float64)
    ref = np.stack([Wd @ (_silu(Wg @ xt) * (Wu @ xt)) for xt in xf])
    np.testing.assert_allclose(out, ref, rtol=1e-5, atol=1e-7)


def test_ffn_one_hot_input_selects_columns():
    """x = e_c: gate and up are column c of the dequantised matrices (closed form)."""
    wl, _, logits, w13, s13, w2, s2 = _tiny_layer(T=2)
    c = 77
    x = np.zeros((2, wl.H), np.uint16)
    x[:, c] = _bf16([1.0])[0]
    idx, wts = oracle.route(logits, wl.k)
    out = oracle.moe_ffn(x, idx, wts, w13, s13, w2, s2, wl.H, wl.I)
    for t in range(2):
        ref = np.zeros(wl.H)
        for j in range(wl.k):
            e = idx[t, j]
            W13 = oracle.dequant(w13[e], s13[e], 2 * wl.I, wl.H).astype(np.float64)
            W2 = oracle.dequant(w2[e], s2[e], wl.H, wl.I).astype(np.float64)
            h = _silu(W13[: wl.I, c]) * W13[wl.I:, c]
            ref += wts[t, j] * (W2 @ h)
        np.testing.assert_allclose(out[t], ref, rtol=1e-5, atol=1e-8)


def test_ffn_token_subset_and_waves_compose():
    wl, x, logits, w13, s13, w2, s2 = _tiny_layer(T=5)
    idx, wts = oracle.route(logits, wl.k)
    full = oracle.moe_ffn(x, idx, wts, w13, s13, w2, s2, wl.H, wl.I)
    sub = oracle.moe_ffn(x, idx, wts, w13, s13, w2, s2, wl.H, wl.I, tokens=[4, 1])
    np.testing.assert_array_equal(sub, full[[4, 1]])
    a = np.zeros(wl.E, np.uint8)
    a[: wl.E // 2] = 1
    p1 = oracle.moe_ffn(x, idx, wts, w13, s13, w2, s2, wl.H, wl.I, active=a)
    p2 = oracle.moe_ffn(x, idx, wts, w13, s13, w2, s2, wl.H, wl.I, active=1 - a)
    np.testing.assert_allclose(p1.astype(np.float64) + p2, full, rtol=1e-5, atol=1e-7)


def test_ffn_pin_detects_planted_mistakes():
    """The dense brute force notices a dropped gate nonlinearity or a transposed operand."""
    wl, x, logits, w13, s13, w2, s2 = _tiny_layer()
    idx, wts = oracle.route(logits, wl.k)
    dense = _dense_moe(wl, x, idx, wts, w13, s13, w2, s2)
    xf = _f32(x).astype(np.float64)
    wrong = np.zeros_like(dense)
    for t in range(xf.shape[0]):
        for j in range(wl.k):
            e = idx[t, j]
            W13 = oracle.dequant(w13[e], s13[e], 2 * wl.I, wl.H).astype(np.float64)
            W2 = oracle.dequant(w2[e], s2[e], wl.H, wl.I).astype(np.float64)
            h = (W13[: wl.I] @ xf[t]) * (W13[wl.I:] @ xf[t])     # silu dropped
            wrong[t] += wts[t, j] * (W2 @ h)
    assert not np.allclose(wrong, dense, rtol=1e-3)


# ----------------------------------------------------------------------------- slot policy

def test_slot_lru_hand_worked_sequence():
    st = oracle.SlotState(6, 2)
    needed = np.zeros(6, np.uint8)
    for line in open(os.path.join(GOLDEN, "slot_lru.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, table, loads = line.split("|")
        want = [int(v) for v in head.split()[1:]]
        if not needed.any():
            needed[want] = 1
        else:
            assert sorted(np.flatnonzero(needed).tolist()) == want
        got_table, got_loads = st.wave(needed)
        assert got_table.tolist() == [int(v) for v in table.split()], line
        assert got_loads == [tuple(int(a) for a in l.split(":")) for l in loads.split()], line
    assert not needed.any()


def test_slot_waves_invariants_random():
    g = np.random.default_rng(4)
    E, S = 64, 16
    st = oracle.SlotState(E, S)
    for step in range(200):
        want = g.choice(E, g.integers(1, 50), replace=False)
        needed = np.zeros(E, np.uint8)
        needed[want] = 1
        seen = set()
        resident_before = set(st.slot_expert[st.slot_expert >= 0].tolist())
        while needed.any():
            before = set(st.slot_expert[st.slot_expert >= 0].tolist())
            table, loads = st.wave(needed)
            wave = set(np.flatnonzero(table >= 0).tolist())
            assert 0 < len(wave) <= S
            assert not (wave & seen)
            seen |= wave
            # a wave's experts sit in distinct slots that now hold them
            slots = table[table >= 0]
            assert len(set(slots.tolist())) == len(slots)
            for e in wave:
                assert st.slot_expert[table[e]] == e
            # loads are exactly the wave's experts that were not resident
            assert {e for e, _ in loads} == wave - before
        assert seen == set(want.tolist())
        # every expert resident at the start and needed this step is a hit (never reloaded)
        hits = resident_before & set(want.tolist())
        assert len(hits) <= S


def test_slot_capped_hand_worked_sequence():
    st = oracle.SlotState(6, 4)
    needed = np.zeros(6, np.uint8)
    for line in open(os.path.join(GOLDEN, "slot_lru_capped.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, table, loads = line.split("|")
        words = head.split()[1:]
        want = [int(v) for v in words[: words.index("p")]]
        prot = np.zeros(4, np.uint8)
        for v in words[words.index("p") + 1:]:
            if v != "-":
                prot[int(v)] = 1
        if not needed.any():
            needed[want] = 1
        else:
            assert sorted(np.flatnonzero(needed).tolist()) == want
        got_table, got_loads = st.wave(needed, cap=2, protect=prot)
        assert got_table.tolist() == [int(v) for v in table.split()], line
        assert got_loads == [tuple(int(a) for a in l.split(":")) for l in loads.split()], line
    assert not needed.any()


@pytest.mark.parametrize("E,S", [(64, 16), (9, 3), (40, 2)])
def test_slot_capped_waves_invariants_random(E, S):
    """Waves of at most S // 2 experts, each protecting the slots of the wave before it: every
    needed expert runs exactly once per step, no protected slot is written, an expert resident
    at the start of its step is never loaded again in it, and cap = S with nothing protected is
    the plain policy."""
    g = np.random.default_rng(E + S)
    cap = S // 2
    st = oracle.SlotState(E, S)
    plain, capped_as_plain = oracle.SlotState(E, S), oracle.SlotState(E, S)
    for step in range(150):
        want = g.choice(E, g.integers(1, min(E, 3 * S) + 1), replace=False)
        needed = np.zeros(E, np.uint8)
        needed[want] = 1
        resident_before = set(st.slot_expert[st.slot_expert >= 0].tolist())
        seen, loaded = set(), set()
        prot = np.zeros(S, np.uint8)
        while needed.any():
            before = st.slot_expert.copy()
            table, loads = st.wave(needed, cap=cap, protect=prot)
            wave = set(np.flatnonzero(table >= 0).tolist())
            assert 0 < len(wave) <= cap and not (wave & seen)
            seen |= wave
            for e, sl in loads:
                assert not prot[sl]                       # protected slots keep their expert
                assert e not in resident_before or e in loaded
                loaded.add(e)
            assert np.array_equal(st.slot_expert[prot == 1], before[prot == 1])
            for e in wave:
                assert st.slot_expert[table[e]] == e
            prot = np.zeros(S, np.uint8)
            prot[table[table >= 0]] = 1
        assert seen == set(want.tolist())
        assert not (loaded & resident_before)             # hits are never reloaded
        n1, n2 = needed.copy(), needed.copy()
        n1[want] = 1
        n2[want] = 1
        while n1.any():
            t1, l1 = plain.wave(n1)
            t2, l2 = capped_as_plain.wave(n2, cap=S, protect=np.zeros(S, np.uint8))
            assert t1.tolist() == t2.tolist() and l1 == l2


# ----------------------------------------------------------------------------- FFN on bf16 weights

def test_ffn_bf16_weights_equal_w4_on_exactly_representable_weights():
    """Weights q * 2^e (q in -8..7) are exact both as bf16 values and as packed codes with a
    power-of-two scale: the bf16-weight FFN and the packed-weight FFN then see the same numbers
    and sum them in the same order, so their outputs are identical."""
    g = np.random.default_rng(11)
    H, I, E, k, T = 256, 128, 4, 2, 5
    wl = mi.Workload("x", H=H, I=I, E=E, k=k, T=T)
    x = mi.activations(wl)
    idx, wts = oracle.route(mi.router_logits(wl), k)
    w13b = np.empty((E, 2 * I, H), np.uint16)
    w2b = np.empty((E, H, I), np.uint16)
    w13p, s13p, w2p, s2p = [], [], [], []
    for e in range(E):
        for (N, K, dst, lp, ls) in ((2 * I, H, w13b, w13p, s13p), (H, I, w2b, w2p, s2p)):
            q = g.integers(-8, 8, (N, K)).astype(np.int8)
            ex = g.integers(-12, -4, (N, K // 128))
            sc = np.ldexp(1.0, ex).astype(np.float32)
            w = q.astype(np.float32) * np.repeat(sc, 128, axis=1)
            dst[e] = mi.to_bf16_bits(w)
            assert np.array_equal(_f32(dst[e]), w)          # exact in bf16
            pk, st = oracle.pack(q, _bf16(sc))
            lp.append(pk)
            ls.append(st)
    a = oracle.moe_ffn(x, idx, wts, np.stack(w13p), np.stack(s13p), np.stack(w2p), np.stack(s2p), H, I)
    b = oracle.moe_ffn_bf16(x, idx, wts, w13b, w2b, H, I)
    assert np.array_equal(a, b)


def test_ffn_bf16_weights_equal_dense_brute_force():
    """Every expert on every token with numpy fp64 matmuls over the bf16 weights, masked by the
    routed weights; a planted transposed operand is caught."""
    wl = mi.Workload("b", H=256, I=128, E=6, k=3, T=7)
    x = mi.activations(wl)
    idx, wts = oracle.route(mi.router_logits(wl), wl.k)
    w13b, w2b = mi.bank_weights(wl)
    out = oracle.moe_ffn_bf16(x, idx, wts, w13b, w2b, wl.H, wl.I)
    xf = _f32(x).astype(np.float64)
    mask = np.zeros((wl.T, wl.E))
    for t in range(wl.T):
        for j in range(wl.k):
            mask[t, idx[t, j]] += wts[t, j]
    dense = np.zeros((wl.T, wl.H))
    wrong = np.zeros((wl.T, wl.H))
    for e in range(wl.E):
        W13 = _f32(w13b[e]).astype(np.float64)
        W2 = _f32(w2b[e]).astype(np.float64)
        h = _silu(xf @ W13[:wl.I].T) * (xf @ W13[wl.I:].T)
        dense += mask[:, e:e + 1] * (h @ W2.T)
        wrong += mask[:, e:e + 1] * (h @ W2.reshape(wl.I, wl.H))   # W2 read transposed
    np.testing.assert_allclose(out, dense, rtol=1e-5, atol=1e-7)
    assert not np.allclose(out, wrong, rtol=1e-3, atol=1e-5)
    # a token subset gives the same rows
    sub = oracle.moe_ffn_bf16(x, idx, wts, w13b, w2b, wl.H, wl.I, tokens=[6, 0, 3])
    np.testing.assert_array_equal(sub, out[[6, 0, 3]])
