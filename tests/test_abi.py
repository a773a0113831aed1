"""The C ABI library loads on a machine without a GPU and exports every declared symbol;
argument errors are reported before anything touches a device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_w4a16.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "while", "return")))


def test_header_declares_the_boundary_calls():
    names = _declared_functions()
    for required in ("moe_quantize_pack", "moe_route_topk", "moe_w4a16_ffn", "slot_table_update",
                     "moe_packed_bytes", "moe_workspace_bytes", "moe_slot_cache_create", "moe_slot_cache_destroy"):
        assert required in names


def test_library_exports_every_declared_symbol():
    import quantized_mixture_experts_grouped_b200 as q
    lib = ctypes.CDLL(q.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_host_side_calls_without_gpu():
    import quantized_mixture_experts_grouped_b200 as q
    assert q.moe_abi_version() == 1
    assert q.moe_packed_bytes(2048, 2048) == 2048 * 2048 // 2
    assert q.moe_scales_count(2048, 1024) == 2048 * 8
    assert q.moe_packed_bytes(100, 128) == 0
    # one OLMoE expert: 3,145,728 code bytes + 98,304 scale bytes
    per_expert = (q.moe_packed_bytes(2048, 2048) + q.moe_packed_bytes(2048, 1024)
                  + 2 * (q.moe_scales_count(2048, 2048) + q.moe_scales_count(2048, 1024)))
    assert per_expert == 3_244_032
    assert q.moe_workspace_bytes(1, 2048, 1024, 64, 8) > 0
    with pytest.raises(q.MoeError) as ei:
        q.moe_workspace_bytes(1, 2000, 1024, 64, 8)
    assert ei.value.code == q.MOE_ERR_SHAPE
    with pytest.raises(q.MoeError) as ei:
        q.moe_workspace_bytes(1, 2048, 1024, 4, 8)      # k > E
    assert ei.value.code == q.MOE_ERR_ARG


def test_argument_errors_before_launch():
    """Bad arguments come back as statuses without any CUDA call being made."""
    import quantized_mixture_experts_grouped_b200 as q
    L = q.lib
    assert L.moe_quantize_pack(None, 1, 128, 128, None, None, None) == q.MOE_ERR_ARG
    assert L.moe_quantize_pack(ctypes.c_void_p(256), 1, 100, 128, ctypes.c_void_p(256),
                               ctypes.c_void_p(256), None) == q.MOE_ERR_SHAPE
    assert L.moe_route_topk(ctypes.c_void_p(256), 4, 8, 9, ctypes.c_void_p(256), ctypes.c_void_p(256),
                            None) == q.MOE_ERR_ARG
    assert L.moe_route_topk(ctypes.c_void_p(256), 4, 300, 2, ctypes.c_void_p(256), ctypes.c_void_p(256),
                            None) == q.MOE_ERR_SHAPE
    p = ctypes.c_void_p(4096)
    # workspace too small
    rc = L.moe_w4a16_ffn(p, 4, 256, 128, 8, 2, p, p, p, p, p, p, None, p, 16, p, 0, None)
    assert rc == q.MOE_ERR_ARG and b"workspace" in L.moe_last_error_string()
    # H not a multiple of 128
    rc = L.moe_w4a16_ffn(p, 4, 200, 128, 8, 2, p, p, p, p, p, p, None, p, 1 << 30, p, 0, None)
    assert rc == q.MOE_ERR_SHAPE
    # unknown path
    rc = L.moe_w4a16_ffn(p, 4, 256, 128, 8, 2, p, p, p, p, p, p, None, p, 1 << 30, p, 77, None)
    assert rc == q.MOE_ERR_ARG
    # slot cache with null pools
    h = ctypes.c_void_p(0)
    rc = L.moe_slot_cache_create(8, 2, 256, 128, p, p, p, p, None, p, p, p, ctypes.byref(h))
    assert rc == q.MOE_ERR_ARG and not h.value


def test_binding_constants_match_the_header():
    """The Python binding's status, path and flag constants are the header's enum values."""
    import quantized_mixture_experts_grouped_b200 as q
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    values = {n: int(v, 0) for n, v in re.findall(r"\b(MOE_[A-Z0-9_]+)\s*=\s*(0x[0-9a-fA-F]+|\d+)", text)}
    for name in ("MOE_OK", "MOE_ERR_ARG", "MOE_ERR_SHAPE", "MOE_ERR_CUDA", "MOE_ERR_TIMEOUT",
                 "MOE_PATH_AUTO", "MOE_PATH_SIMPLE", "MOE_PATH_DECODE", "MOE_PATH_GROUPED",
                 "MOE_PATH_SEQUENTIAL", "MOE_FLAG_ACCUMULATE"):
        assert values[name] == getattr(q, name), name
    assert sorted(q.PATHS.values()) == sorted(values[n] for n in values if n.startswith("MOE_PATH_")
                                              and n != "MOE_PATH_MASK")
    assert q.lib.moe_packed_layout_version() == 2


def test_header_is_plain_c_and_links(tmp_path):
    """The header compiles as C99 and a C program linked against the library calls its host-side
    entry points (sizes, versions, argument errors: nothing that touches a device)."""
    import shutil
    import subprocess
    import quantized_mixture_experts_grouped_b200 as q
    if not shutil.which("gcc"):
        pytest.skip("gcc not available")
    src = tmp_path / "use_abi.c"
    src.write_text(r'''
#include <stdio.h>
#include "moe_w4a16.h"
int main(void) {
  size_t ws = 0;
  if (moe_abi_version() != 1 || moe_packed_layout_version() != 2) return 1;
  if (moe_packed_bytes(2048, 2048) != (size_t)2048 * 2048 / 2) return 2;
  if (moe_scales_count(2048, 1024) != (size_t)2048 * 8) return 3;
  if (moe_workspace_bytes(1, 2048, 1024, 64, 8, &ws) != MOE_OK || ws == 0) return 4;
  if (moe_workspace_bytes(1, 2000, 1024, 64, 8, &ws) != MOE_ERR_SHAPE) return 5;
  if (moe_quantize_pack(NULL, 1, 128, 128, NULL, NULL, NULL) != MOE_ERR_ARG) return 6;
  if (moe_last_error_string() == NULL) return 7;
  printf("ok %zu\n", ws);
  return 0;
}
''')
    exe = tmp_path / "use_abi"
    lib_dir = os.path.dirname(q.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe), "-L", lib_dir, "-l:libmoe_w4a16.so", f"-Wl,-rpath,{lib_dir}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stdout, out.stderr)
    assert out.stdout.startswith("ok ")
