"""Plain CPU oracle of the fused grouped W4A16 MoE FFN layer (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg
and reference arm (``bench.py --impl reference``) are the only callers. The product library never imports this package, and this package
imports nothing from the product package. The arithmetic lives in ``oracle.cpp`` (plain
C++17 loops); this module only compiles it with g++ and marshals numpy arrays.

Method: "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference", Abstract
(symmetric group-128 int4 routed experts, unchanged BF16 top-k router, every selected expert
executed through a GPU slot cache and fused grouped kernels).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp into liboracle.so (g++ -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-std=c++17", "-O2", "-fno-fast-math", "-ffp-contract=off",
                               "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        c = ctypes
        P = c.c_void_p
        L.orc_bf16_to_f32.argtypes = [c.c_uint16]
        L.orc_bf16_to_f32.restype = c.c_float
        L.orc_f32_to_bf16.argtypes = [c.c_float]
        L.orc_f32_to_bf16.restype = c.c_uint16
        L.orc_packed_bytes.argtypes = [c.c_int, c.c_int]
        L.orc_packed_bytes.restype = c.c_size_t
        L.orc_scale_count.argtypes = [c.c_int, c.c_int]
        L.orc_scale_count.restype = c.c_size_t
        L.orc_quantize.argtypes = [P, c.c_int, c.c_int, P, P]
        L.orc_pack.argtypes = [P, P, c.c_int, c.c_int, P, P]
        L.orc_unpack.argtypes = [P, P, c.c_int, c.c_int, P, P]
        L.orc_dequant.argtypes = [P, P, c.c_int, c.c_int, P]
        L.orc_route.argtypes = [P, c.c_int, c.c_int, c.c_int, P, P]
        L.orc_permute.argtypes = [P, c.c_int, c.c_int, c.c_int, P, P, P, P]
        L.orc_moe_ffn.argtypes = [P, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, P, P,
                                  P, P, P, P, P, c.c_int, P, P, c.c_int]
        L.orc_moe_ffn_bf16.argtypes = [P, c.c_int, c.c_int, c.c_int, c.c_int, c.c_int, P, P,
                                       P, P, P, c.c_int, P, P, c.c_int]
        L.orc_slot_wave.argtypes = [c.c_int, c.c_int, P, P, P, P, P, P, P, P]
        L.orc_slot_wave_capped.argtypes = [c.c_int, c.c_int, c.c_int, P, P, P, P, P, P, P, P, P]
        for f in ("orc_quantize", "orc_pack", "orc_unpack", "orc_dequant", "orc_route",
                  "orc_permute", "orc_moe_ffn", "orc_moe_ffn_bf16", "orc_slot_wave", "orc_slot_wave_capped"):
            getattr(L, f).restype = c.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (status {rc})")


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32 values (exact widening)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def packed_bytes(N: int, K: int) -> int:
    return int(lib().orc_packed_bytes(N, K))


def scale_count(N: int, K: int) -> int:
    return int(lib().orc_scale_count(N, K))


def quantize(w_bf16: np.ndarray):
    """w_bf16 uint16 [N][K] -> (q int8 [N][K], s uint16 bf16 bits [N][K/128])."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    N, K = w.shape
    q = np.zeros((N, K), np.int8)
    s = np.zeros((N, K // 128), np.uint16)
    _check(lib().orc_quantize(_p(w), N, K, _p(q), _p(s)), "quantize")
    return q, s


def pack(q: np.ndarray, s: np.ndarray):
    """q int8 [N][K], s uint16 [N][K/128] -> (packed uint8 [N*K/2], scales uint16 in the packed order [N*K/128])."""
    q = np.ascontiguousarray(q, dtype=np.int8)
    s = np.ascontiguousarray(s, dtype=np.uint16)
    N, K = q.shape
    packed = np.zeros(packed_bytes(N, K), np.uint8)
    st = np.zeros(scale_count(N, K), np.uint16)
    _check(lib().orc_pack(_p(q), _p(s), N, K, _p(packed), _p(st)), "pack")
    return packed, st


def unpack(packed: np.ndarray, scales_packed: np.ndarray, N: int, K: int):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    st = np.ascontiguousarray(scales_packed, dtype=np.uint16)
    q = np.zeros((N, K), np.int8)
    s = np.zeros((N, K // 128), np.uint16)
    _check(lib().orc_unpack(_p(packed), _p(st), N, K, _p(q), _p(s)), "unpack")
    return q, s


def dequant(packed: np.ndarray, scales_packed: np.ndarray, N: int, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    st = np.ascontiguousarray(scales_packed, dtype=np.uint16)
    out = np.zeros((N, K), np.float32)
    _check(lib().orc_dequant(_p(packed), _p(st), N, K, _p(out)), "dequant")
    return out


def quantize_pack_bank(w_bf16: np.ndarray):
    """w_bf16 uint16 [E][N][K] -> (packed uint8 [E][N*K/2], scales uint16 [E][N*K/128])."""
    E, N, K = w_bf16.shape
    packed = np.zeros((E, packed_bytes(N, K)), np.uint8)
    st = np.zeros((E, scale_count(N, K)), np.uint16)
    for e in range(E):
        q, s = quantize(w_bf16[e])
        packed[e], st[e] = pack(q, s)
    return packed, st


def route(logits_bf16: np.ndarray, k: int):
    """logits uint16 bf16 bits [T][E] -> (idx int32 [T][k], wts float32 [T][k])."""
    lg = np.ascontiguousarray(logits_bf16, dtype=np.uint16)
    T, E = lg.shape
    idx = np.zeros((T, k), np.int32)
    wts = np.zeros((T, k), np.float32)
    _check(lib().orc_route(_p(lg), T, E, k, _p(idx), _p(wts)), "route")
    return idx, wts


def permute(idx: np.ndarray, E: int):
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(T * k, np.int32)
    inv = np.zeros(T * k, np.int32)
    _check(lib().orc_permute(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm), _p(inv)), "permute")
    return counts, offsets, perm, inv


def moe_ffn(x_bf16, idx, wts, w13, s13, w2, s2, H: int, I: int, tokens=None, active=None,
            n_threads: int = 0) -> np.ndarray:
    """Layer output (fp32) for `tokens` (default: all), from packed banks indexed by expert."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    wts = np.ascontiguousarray(wts, dtype=np.float32)
    T, k = idx.shape
    E = w13.shape[0]
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    nt = T if tok is None else len(tok)
    act = None if active is None else np.ascontiguousarray(active, dtype=np.uint8)
    out = np.zeros((nt, H), np.float32)
    rc = lib().orc_moe_ffn(_p(x), T, H, I, E, k, _p(idx), _p(wts),
                           _p(np.ascontiguousarray(w13)), _p(np.ascontiguousarray(s13)),
                           _p(np.ascontiguousarray(w2)), _p(np.ascontiguousarray(s2)),
                           _p(tok), nt, _p(act), _p(out), int(n_threads))
    _check(rc, "moe_ffn")
    return out


def moe_ffn_bf16(x_bf16, idx, wts, w13_bf16, w2_bf16, H: int, I: int, tokens=None, active=None,
                 n_threads: int = 0) -> np.ndarray:
    """Layer output (fp32) for `tokens` (default: all) from unquantised bf16 banks
    w13 [E][2I][H], w2 [E][H][I] (uint16 bit patterns)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    wts = np.ascontiguousarray(wts, dtype=np.float32)
    T, k = idx.shape
    E = w13_bf16.shape[0]
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    nt = T if tok is None else len(tok)
    act = None if active is None else np.ascontiguousarray(active, dtype=np.uint8)
    out = np.zeros((nt, H), np.float32)
    rc = lib().orc_moe_ffn_bf16(_p(x), T, H, I, E, k, _p(idx), _p(wts),
                                _p(np.ascontiguousarray(w13_bf16, dtype=np.uint16)),
                                _p(np.ascontiguousarray(w2_bf16, dtype=np.uint16)),
                                _p(tok), nt, _p(act), _p(out), int(n_threads))
    _check(rc, "moe_ffn_bf16")
    return out


class SlotState:
    """LRU slot-cache state for one layer, advanced one wave at a time by the oracle."""

    def __init__(self, E: int, S: int):
        self.E, self.S = E, S
        self.slot_expert = np.full(S, -1, np.int32)
        self.last_used = np.zeros(S, np.int64)
        self.clock = np.zeros(1, np.int64)

    def wave(self, needed: np.ndarray, cap: int = None, protect: np.ndarray = None):
        """needed uint8 [E] (modified in place); cap: most experts in the wave (default S);
        protect: uint8 [S], nonzero = slot must not be overwritten. Returns (wave_table [E],
        loads [(expert, slot)])."""
        assert needed.dtype == np.uint8 and needed.flags["C_CONTIGUOUS"]
        table = np.zeros(self.E, np.int32)
        le = np.zeros(self.S, np.int32)
        ls = np.zeros(self.S, np.int32)
        n = np.zeros(1, np.int32)
        pr = None if protect is None else np.ascontiguousarray(protect, dtype=np.uint8)
        rc = lib().orc_slot_wave_capped(self.E, self.S, self.S if cap is None else int(cap), _p(pr),
                                        _p(self.slot_expert), _p(self.last_used), _p(self.clock), _p(needed),
                                        _p(table), _p(le), _p(ls), _p(n))
        _check(rc, "slot_wave")
        return table, list(zip(le[: n[0]].tolist(), ls[: n[0]].tolist()))
