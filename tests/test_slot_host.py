"""The slot cache's replacement policy (host C++ behind slot_table_update) against the oracle's,
on the CPU: the cache runs in dry-run mode (waves planned and committed, no copies issued), so
wave tables, load lists and the LRU state can be compared bit for bit without a GPU. The copies
themselves and the layer in waves are covered by the GPU tests."""
import ctypes

import numpy as np
import pytest
import torch

import oracle

q = pytest.importorskip("quantized_mixture_experts_grouped_b200")


def _update(cache, mask, table, misses):
    """slot_table_update with no copy stream and no events (nothing is copied in dry-run mode)."""
    n = ctypes.c_int(0)
    rc = q.lib.slot_table_update(cache.handle, mask.ctypes.data_as(ctypes.c_void_p),
                                 table.ctypes.data_as(ctypes.c_void_p),
                                 None if misses is None else misses.ctypes.data_as(ctypes.c_void_p),
                                 ctypes.byref(n), None, None, None)
    if rc:
        raise q.MoeError(rc, q.lib.moe_last_error_string().decode())
    return n.value


def _cache(E, S, H=256, I=128):
    # placeholders for the bank and pool: a dry-run cache never reads or writes them
    bank = [torch.zeros(1, dtype=torch.uint8) for _ in range(4)]
    pool = [torch.zeros(1, dtype=torch.uint8) for _ in range(4)]
    c = q.SlotCache(E, S, H, I, bank, pool)
    c.dry_run(True)
    return c


def _mask(needed: np.ndarray) -> np.ndarray:
    m = np.zeros((len(needed) + 63) // 64, np.uint64)
    for e in np.flatnonzero(needed):
        m[e >> 6] |= np.uint64(1) << np.uint64(e & 63)
    return m


def _unmask(m: np.ndarray, E: int) -> np.ndarray:
    return np.array([(int(m[e >> 6]) >> (e & 63)) & 1 for e in range(E)], np.uint8)


@pytest.mark.parametrize("E,S,steps,seed", [(8, 3, 60, 1), (64, 16, 150, 2), (200, 7, 40, 3)])
def test_policy_matches_the_oracle(E, S, steps, seed):
    g = np.random.default_rng(seed)
    cache = _cache(E, S)
    ref = oracle.SlotState(E, S)
    table = np.zeros(E, np.int32)
    misses = np.zeros(S, np.int32)
    total_waves = 0
    for _ in range(steps):
        want = g.choice(E, int(g.integers(1, min(E, 3 * S) + 1)), replace=False)
        needed = np.zeros(E, np.uint8)
        needed[want] = 1
        mask = _mask(needed)
        while needed.any():
            ref_table, ref_loads = ref.wave(needed)
            n = _update(cache, mask, table, misses)
            total_waves += 1
            np.testing.assert_array_equal(table, ref_table)
            assert [(int(misses[i]), int(table[misses[i]])) for i in range(n)] == ref_loads
            np.testing.assert_array_equal(_unmask(mask, E), needed)
            se, lu, clock = cache.state()
            np.testing.assert_array_equal(se, ref.slot_expert)
            np.testing.assert_array_equal(lu, ref.last_used)
            assert clock == ref.clock[0]
        assert not mask.any()
    assert total_waves > steps      # some steps needed more than one wave


def _update_ex(cache, mask, table, misses, cap, protect):
    n = ctypes.c_int(0)
    rc = q.lib.slot_table_update_ex(cache.handle, mask.ctypes.data_as(ctypes.c_void_p),
                                    table.ctypes.data_as(ctypes.c_void_p), misses.ctypes.data_as(ctypes.c_void_p),
                                    ctypes.byref(n), None, None, None, cap,
                                    None if protect is None else protect.ctypes.data_as(ctypes.c_void_p))
    if rc:
        raise q.MoeError(rc, q.lib.moe_last_error_string().decode())
    return n.value


@pytest.mark.parametrize("E,S,steps,seed", [(64, 16, 120, 5), (9, 3, 80, 6), (40, 2, 60, 7)])
def test_overlapped_waves_match_the_oracle(E, S, steps, seed):
    """The schedule of moe_slot_cache_layer with two or more slots: waves of at most S // 2
    experts, each protecting the slots of the wave before it in the step."""
    g = np.random.default_rng(seed)
    cache = _cache(E, S)
    ref = oracle.SlotState(E, S)
    table = np.zeros(E, np.int32)
    misses = np.zeros(S, np.int32)
    cap = S // 2
    for _ in range(steps):
        want = g.choice(E, int(g.integers(1, min(E, 3 * S) + 1)), replace=False)
        needed = np.zeros(E, np.uint8)
        needed[want] = 1
        mask = _mask(needed)
        prot = np.zeros(S, np.uint8)
        while needed.any():
            ref_table, ref_loads = ref.wave(needed, cap=cap, protect=prot)
            n = _update_ex(cache, mask, table, misses, cap, prot)
            np.testing.assert_array_equal(table, ref_table)
            assert [(int(misses[i]), int(table[misses[i]])) for i in range(n)] == ref_loads
            np.testing.assert_array_equal(_unmask(mask, E), needed)
            se, lu, clock = cache.state()
            np.testing.assert_array_equal(se, ref.slot_expert)
            np.testing.assert_array_equal(lu, ref.last_used)
            assert clock == ref.clock[0]
            prot = np.zeros(S, np.uint8)
            prot[table[table >= 0]] = 1


def test_update_ex_rejects_a_cap_above_the_slots():
    cache = _cache(8, 2)
    mask = np.array([0b110], np.uint64)
    with pytest.raises(q.MoeError) as ei:
        _update_ex(cache, mask, np.zeros(8, np.int32), np.zeros(2, np.int32), 3, None)
    assert ei.value.code == q.MOE_ERR_ARG
    assert mask[0] == 0b110


def test_failed_refill_commits_nothing():
    cache = _cache(8, 2)
    mask = np.array([0b00000110], np.uint64)        # experts 1 and 2
    table = np.full(8, 7, np.int32)
    misses = np.zeros(2, np.int32)
    cache.fail_copy_after(5)    # expert 1's four copies succeed, expert 2's second copy fails
    with pytest.raises(q.MoeError) as ei:
        _update(cache, mask, table, misses)
    assert ei.value.code == q.MOE_ERR_CUDA
    se, lu, clock = cache.state()
    assert se.tolist() == [-1, -1] and lu.tolist() == [0, 0] and clock == 0
    assert mask[0] == 0b110 and table.tolist() == [7] * 8          # nothing of the wave committed
    n = _update(cache, mask, table, misses)
    assert n == 2 and misses.tolist() == [1, 2] and mask[0] == 0
    assert table.tolist() == [-1, 0, 1, -1, -1, -1, -1, -1]
    # a failure after residents exist frees only the slots the failed wave had started to overwrite
    mask = np.array([0b00011000], np.uint64)        # experts 3 and 4: evict 1 (slot 0), 2 (slot 1)
    cache.fail_copy_after(4)    # expert 3's copies succeed into slot 0, expert 4's first copy fails
    with pytest.raises(q.MoeError):
        _update(cache, mask, table, misses)
    se, _, clock = cache.state()
    assert se.tolist() == [-1, -1] and clock == 1 and mask[0] == 0b11000


def test_cache_handle_errors():
    h = ctypes.c_void_p(0)
    p = ctypes.c_void_p(4096)
    assert q.lib.moe_slot_cache_create(0, 2, 256, 128, p, p, p, p, p, p, p, p, ctypes.byref(h)) == q.MOE_ERR_ARG
    assert q.lib.moe_slot_cache_create(8, 2, 200, 128, p, p, p, p, p, p, p, p, ctypes.byref(h)) == q.MOE_ERR_SHAPE
    assert not h.value
    cache = _cache(8, 2)
    with pytest.raises(q.MoeError) as ei:
        _update(cache, np.zeros(1, np.uint64), np.zeros(8, np.int32), None)
    assert ei.value.code == q.MOE_ERR_ARG
