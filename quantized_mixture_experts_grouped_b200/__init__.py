"""Python binding of libmoe_w4a16.so, the fused grouped W4A16 MoE FFN layer for sm_100a.

Argument marshalling only: every step of the layer runs in the library's CUDA kernels. The
functions carry the C ABI's names (include/moe_w4a16.h) and take torch tensors for device
memory and torch streams; torch provides memory, streams and nothing else. There is no CPU
fallback: importing this package without the built library raises.

Method: "Every Expert Counts: ExactMoE for Memory-Efficient W4A16 Inference", Abstract.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_w4a16.so")

MOE_OK, MOE_ERR_ARG, MOE_ERR_SHAPE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = 0, 1, 2, 3, 4
MOE_PATH_AUTO, MOE_PATH_SIMPLE, MOE_PATH_DECODE, MOE_PATH_GROUPED, MOE_PATH_SEQUENTIAL = 0, 1, 2, 3, 4
MOE_FLAG_ACCUMULATE = 0x100
PATHS = {"auto": MOE_PATH_AUTO, "simple": MOE_PATH_SIMPLE, "decode": MOE_PATH_DECODE,
         "grouped": MOE_PATH_GROUPED, "sequential": MOE_PATH_SEQUENTIAL}


class MoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python quantized_mixture_experts_grouped_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    c = ctypes
    P, I, Z = c.c_void_p, c.c_int, c.c_size_t
    sig = {
        "moe_abi_version": ([], I),
        "moe_packed_layout_version": ([], I),
        "moe_last_error_string": ([], c.c_char_p),
        "moe_launch_count": ([], c.c_ulonglong),
        "moe_debug_set_decode_trace": ([P], None),
        "moe_debug_set_wait_limit": ([c.c_ulonglong, I], None),
        "moe_packed_bytes": ([I, I], Z),
        "moe_scales_count": ([I, I], Z),
        "moe_quantize_pack": ([P, I, I, I, P, P, P], I),
        "moe_route_topk": ([P, I, I, I, P, P, P], I),
        "moe_permute_scratch_count": ([I, I, I], Z),
        "moe_permute": ([P, I, I, I, P, P, P, P, P, P], I),
        "moe_workspace_bytes": ([I, I, I, I, I, c.POINTER(Z)], I),
        "moe_workspace_init": ([P, Z, P], I),
        "moe_workspace_status": ([P, P, c.POINTER(I)], I),
        "moe_w4a16_ffn": ([P, I, I, I, I, I, P, P, P, P, P, P, P, P, Z, P, I, P], I),
        "moe_w4a16_layer": ([P, P, I, I, I, I, I, P, P, P, P, P, P, P, P, Z, P, I, P], I),
        "moe_w4a16_layer_noalloc": ([P, P, I, I, I, I, I, P, P, P, P, P, P, P, P, I, P], I),
        "moe_noalloc_status": ([P, c.POINTER(I)], I),
        "moe_bf16_ffn": ([P, I, I, I, I, I, P, P, P, P, P, P, Z, P, I, P], I),
        "moe_bf16_layer": ([P, P, I, I, I, I, I, P, P, P, P, P, P, Z, P, I, P], I),
        "moe_slot_cache_create": ([I, I, I, I, P, P, P, P, P, P, P, P, c.POINTER(P)], I),
        "moe_slot_cache_destroy": ([P], None),
        "moe_slot_cache_fail_copy_after": ([P, I], None),
        "moe_slot_cache_dry_run": ([P, I], None),
        "slot_table_update": ([P, P, P, P, c.POINTER(I), P, P, P], I),
        "slot_table_update_ex": ([P, P, P, P, c.POINTER(I), P, P, P, I, P], I),
        "moe_slot_cache_state": ([P, P, P], c.c_int64),
        "moe_slot_cache_layer": ([P, P, P, I, I, P, P, P, P, Z, P, I, P, P, c.POINTER(I), c.POINTER(I)], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    return L


lib = _load()


def _err(rc: int):
    if rc != MOE_OK:
        raise MoeError(rc, lib.moe_last_error_string().decode())


def _p(t):
    if t is None:
        return None
    if isinstance(t, int):
        return ctypes.c_void_p(t)
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def moe_abi_version() -> int:
    return lib.moe_abi_version()


def moe_launch_count() -> int:
    return lib.moe_launch_count()


def moe_debug_set_wait_limit(cycles: int, extra_arrivals: int = 0):
    """Testing aid: bounded-wait limit of the single-token decode kernel (0 = default) and extra
    arrivals its exchange waits for (> 0 makes that wait run out)."""
    lib.moe_debug_set_wait_limit(cycles, extra_arrivals)


def moe_packed_bytes(N: int, K: int) -> int:
    return lib.moe_packed_bytes(N, K)


def moe_scales_count(N: int, K: int) -> int:
    return lib.moe_scales_count(N, K)


def moe_quantize_pack(w_bf16: torch.Tensor, packed: torch.Tensor, scales: torch.Tensor, stream=None):
    """w_bf16 [E][N][K] bf16 -> packed uint8 [E][N*K/2], scales bf16 [E][N*K/128]."""
    E, N, K = w_bf16.shape
    _err(lib.moe_quantize_pack(_p(w_bf16), E, N, K, _p(packed), _p(scales), _s(stream)))


def moe_route_topk(logits: torch.Tensor, k: int, idx: torch.Tensor, wts: torch.Tensor, stream=None):
    T, E = logits.shape
    _err(lib.moe_route_topk(_p(logits), T, E, k, _p(idx), _p(wts), _s(stream)))


def moe_permute_scratch_count(T: int, k: int, E: int) -> int:
    return lib.moe_permute_scratch_count(T, k, E)


def moe_permute(idx, E: int, counts, offsets, perm, inv, scratch, stream=None):
    T, k = idx.shape
    _err(lib.moe_permute(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm), _p(inv), _p(scratch), _s(stream)))


def moe_workspace_bytes(T: int, H: int, I: int, E: int, k: int) -> int:
    out = ctypes.c_size_t(0)
    _err(lib.moe_workspace_bytes(T, H, I, E, k, ctypes.byref(out)))
    return out.value


def moe_workspace_init(ws: torch.Tensor, stream=None):
    _err(lib.moe_workspace_init(_p(ws), ws.numel() * ws.element_size(), _s(stream)))


def moe_workspace_status(ws: torch.Tensor, stream=None) -> int:
    st = ctypes.c_int(0)
    _err(lib.moe_workspace_status(_p(ws), _s(stream), ctypes.byref(st)))
    return st.value


def moe_w4a16_ffn(x, idx, wts, w13, s13, w2, s2, H: int, I: int, E: int, ws, out, slot_of_expert=None,
                  flags: int = MOE_PATH_AUTO, stream=None):
    T, k = idx.shape
    _err(lib.moe_w4a16_ffn(_p(x), T, H, I, E, k, _p(idx), _p(wts), _p(w13), _p(s13), _p(w2), _p(s2),
                           _p(slot_of_expert), _p(ws), ws.numel() * ws.element_size(), _p(out), flags, _s(stream)))


def moe_w4a16_layer(x, logits, k: int, w13, s13, w2, s2, H: int, I: int, idx, wts, ws, out,
                    slot_of_expert=None, flags: int = MOE_PATH_AUTO, stream=None):
    T, E = logits.shape
    _err(lib.moe_w4a16_layer(_p(x), _p(logits), T, H, I, E, k, _p(w13), _p(s13), _p(w2), _p(s2),
                             _p(slot_of_expert), _p(idx), _p(wts), _p(ws), ws.numel() * ws.element_size(),
                             _p(out), flags, _s(stream)))


def moe_w4a16_layer_noalloc(x, logits, k: int, w13, s13, w2, s2, H: int, I: int, idx, wts, out,
                            slot_of_expert=None, flags: int = MOE_PATH_AUTO, stream=None):
    """moe_w4a16_layer with the library's static device scratch as its workspace (no allocation)."""
    T, E = logits.shape
    _err(lib.moe_w4a16_layer_noalloc(_p(x), _p(logits), T, H, I, E, k, _p(w13), _p(s13), _p(w2), _p(s2),
                                     _p(slot_of_expert), _p(idx), _p(wts), _p(out), flags, _s(stream)))


def moe_bf16_ffn(x, idx, wts, w13, w2, H: int, I: int, E: int, ws, out, slot_of_expert=None,
                 flags: int = MOE_PATH_AUTO, stream=None):
    """The layer's FFN on unquantised bf16 experts: w13 [slots][2I][H], w2 [slots][H][I] (bf16)."""
    T, k = idx.shape
    _err(lib.moe_bf16_ffn(_p(x), T, H, I, E, k, _p(idx), _p(wts), _p(w13), _p(w2), _p(slot_of_expert),
                          _p(ws), ws.numel() * ws.element_size(), _p(out), flags, _s(stream)))


def moe_bf16_layer(x, logits, k: int, w13, w2, H: int, I: int, idx, wts, ws, out, slot_of_expert=None,
                   flags: int = MOE_PATH_AUTO, stream=None):
    T, E = logits.shape
    _err(lib.moe_bf16_layer(_p(x), _p(logits), T, H, I, E, k, _p(w13), _p(w2), _p(slot_of_expert), _p(idx),
                            _p(wts), _p(ws), ws.numel() * ws.element_size(), _p(out), flags, _s(stream)))


def moe_noalloc_status(stream=None) -> int:
    """Reads and clears the device status word of the static array of moe_w4a16_layer_noalloc."""
    st = ctypes.c_int(0)
    _err(lib.moe_noalloc_status(_s(stream), ctypes.byref(st)))
    return st.value


class SlotCache:
    """Owner of a moe_slot_cache handle (one layer's GPU slot pool over a pinned host bank)."""

    def __init__(self, E: int, S: int, H: int, I: int, bank, pool):
        self.E, self.S, self.H, self.I = E, S, H, I
        self.bank, self.pool = bank, pool          # keep the memory alive
        h = ctypes.c_void_p(0)
        _err(lib.moe_slot_cache_create(E, S, H, I, *(_p(t) for t in bank), *(_p(t) for t in pool),
                                       ctypes.byref(h)))
        self.handle = h

    def close(self):
        if self.handle:
            lib.moe_slot_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def fail_copy_after(self, n: int):
        lib.moe_slot_cache_fail_copy_after(self.handle, n)

    def dry_run(self, dry: bool = True):
        """Plan and commit refills without copying (testing the policy without a GPU)."""
        lib.moe_slot_cache_dry_run(self.handle, int(dry))

    def state(self):
        import numpy as np
        se = np.zeros(self.S, np.int32)
        lu = np.zeros(self.S, np.int64)
        clock = lib.moe_slot_cache_state(self.handle, se.ctypes.data_as(ctypes.c_void_p),
                                         lu.ctypes.data_as(ctypes.c_void_p))
        return se, lu, clock

    def slot_table_update(self, needed_mask, wave_table, misses, copy_stream, reuse_ok=None, loaded=None):
        """needed_mask: numpy uint64 [ceil(E/64)] (updated); wave_table: numpy int32 [E];
        misses: numpy int32 [S]. Returns the number of misses."""
        n = ctypes.c_int(0)
        ev = lambda e: None if e is None else ctypes.c_void_p(e.cuda_event)
        _err(lib.slot_table_update(self.handle, needed_mask.ctypes.data_as(ctypes.c_void_p),
                                   wave_table.ctypes.data_as(ctypes.c_void_p), misses.ctypes.data_as(ctypes.c_void_p),
                                   ctypes.byref(n), _s(copy_stream), ev(reuse_ok), ev(loaded)))
        return n.value

    def layer(self, x, logits, k: int, idx, wts, wave_tables, ws, out, path: int = MOE_PATH_AUTO,
              stream=None, copy_stream=None):
        T = logits.shape[0]
        nw, nl = ctypes.c_int(0), ctypes.c_int(0)
        _err(lib.moe_slot_cache_layer(self.handle, _p(x), _p(logits), T, k, _p(idx), _p(wts), _p(wave_tables),
                                      _p(ws), ws.numel() * ws.element_size(), _p(out), path, _s(stream),
                                      _s(copy_stream), ctypes.byref(nw), ctypes.byref(nl)))
        return nw.value, nl.value


def alloc_bank(E: int, N: int, K: int, device="cuda", pinned: bool = False):
    """Zeroed (packed uint8 [E][N*K/2], scales bf16 [E][N*K/128]) buffers for E matrices."""
    kw = dict(device=device) if not pinned else dict(device="cpu", pin_memory=True)
    packed = torch.zeros((E, moe_packed_bytes(N, K)), dtype=torch.uint8, **kw)
    scales = torch.zeros((E, moe_scales_count(N, K)), dtype=torch.bfloat16, **kw)
    return packed, scales


def alloc_workspace(T: int, H: int, I: int, E: int, k: int, device="cuda", stream=None) -> torch.Tensor:
    ws = torch.empty(moe_workspace_bytes(T, H, I, E, k), dtype=torch.uint8, device=device)
    moe_workspace_init(ws, stream)
    return ws
