"""C ABI checks that need no GPU: the library builds and loads, exports every
function include/moe.h declares, its structs match the binding's layout, and
argument errors are reported before any CUDA call."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")
SCRATCH = os.path.join(ROOT, "_build", "tests")   # compiled probes stay inside the repository


def _tmpdir():
    os.makedirs(SCRATCH, exist_ok=True)
    return tempfile.TemporaryDirectory(dir=SCRATCH)


@pytest.fixture(scope="module")
def M():
    from _lib import build_and_import
    return build_and_import()


def _declared_functions():
    src = open(HEADER).read()
    return re.findall(r"(?m)^(?:size_t|moe_status|const char\*|uint64_t)\s+(moe_\w+)\s*\(", src)


def test_header_declares_the_boundary():
    names = set(_declared_functions())
    for required in ("moe_router_topk", "moe_dispatch", "moe_grouped_ffn", "moe_combine",
                     "moe_layer_forward", "moe_expert_stats", "moe_workspace_size",
                     "moe_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(M):
    lib = ctypes.CDLL(M.LIB_PATH)
    declared = _declared_functions()
    assert declared
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(M.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True, text=True).stdout
    for name in declared:
        assert re.search(rf"\bT {name}\b", out), name


def test_struct_layout_matches_header(M):
    prog = r'''
#include <stdio.h>
#include <stddef.h>
#include "moe.h"
int main(void) {
  printf("%zu %zu %zu %zu\n", sizeof(moe_layer_desc), sizeof(moe_layer_weights),
         sizeof(moe_routing), sizeof(moe_stats));
  printf("%zu %zu %zu %zu %zu %zu\n", offsetof(moe_stats, capacity), offsetof(moe_stats, num_stragglers),
         offsetof(moe_stats, skew_ratio), offsetof(moe_stats, gini), offsetof(moe_stats, overflow_rate),
         offsetof(moe_stats, max_over_mean));
  printf("%zu %zu\n", offsetof(moe_layer_desc, dtype), offsetof(moe_routing, logits));
  return 0;
}
'''
    with _tmpdir() as d:
        c = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        open(c, "w").write(prog)
        subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), c, "-o", exe], check=True,
                       env=dict(os.environ, TMPDIR=d))
        got = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split()
    got = [int(v) for v in got]
    want = [ctypes.sizeof(M.MoELayerDesc), ctypes.sizeof(M.MoELayerWeights), ctypes.sizeof(M.MoERouting),
            ctypes.sizeof(M.MoEStats),
            M.MoEStats.capacity.offset, M.MoEStats.num_stragglers.offset, M.MoEStats.skew_ratio.offset,
            M.MoEStats.gini.offset, M.MoEStats.overflow_rate.offset, M.MoEStats.max_over_mean.offset,
            M.MoELayerDesc.dtype.offset, M.MoERouting.logits.offset]
    assert got == want


def test_header_compiles_as_c_and_cxx():
    with _tmpdir() as d:
        for lang, cc in (("c", "gcc"), ("cpp", "g++")):
            f = os.path.join(d, "inc." + lang)
            open(f, "w").write('#include "moe.h"\nint main(void){return (int)MOE_OK;}\n')
            subprocess.run([cc, "-Wall", "-Werror", "-I", os.path.dirname(HEADER), f, "-o", f + ".out"], check=True,
                           env=dict(os.environ, TMPDIR=d))


def test_workspace_size_rejects_bad_descriptors(M):
    good = M.make_desc(64, 256, 16, 2, 512, 0, M.MOE_F32)
    assert M.moe_workspace_size(good) > 0
    bad = [dict(K=17), dict(K=20, E=16), dict(E=513), dict(T=-1), dict(dtype=7), dict(H=0),
           dict(H=100, dtype=M.MOE_BF16), dict(D=1000, dtype=M.MOE_BF16), dict(H=258)]
    for kw in bad:
        args = dict(T=64, H=256, E=16, K=2, D=512, Ds=0, dtype=M.MOE_F32)
        args.update(kw)
        d = M.make_desc(**args)
        assert M.moe_workspace_size(d) == 0, kw


def test_workspace_size_grows_with_tokens(M):
    sizes = [M.moe_workspace_size(M.make_desc(T, 4096, 128, 8, 1024, 4096, M.MOE_BF16))
             for T in (0, 1, 16, 128, 16384)]
    assert sizes == sorted(sizes) and sizes[0] > 0


def _host_buffer(n):
    buf = ctypes.create_string_buffer(n + 256)
    addr = (ctypes.addressof(buf) + 255) & ~255
    return buf, ctypes.c_void_p(addr)


def test_argument_errors_are_reported_before_any_launch(M):
    lib = M._binding.lib
    d = M.make_desc(8, 256, 16, 2, 512, 0, M.MOE_F32)
    need = M.moe_workspace_size(d)
    keep, ws = _host_buffer(need)
    # no workspace / too small workspace
    assert lib.moe_router_topk(ctypes.byref(d), None, None, None, None, None, None, None, 0, None) == 3
    assert lib.moe_dispatch(ctypes.byref(d), None, None, None, None, None, ws, need - 1, None) == 3
    # missing tensors with a valid workspace
    assert lib.moe_router_topk(ctypes.byref(d), None, None, None, None, None, None, ws, need, None) == 1
    assert lib.moe_layer_forward(ctypes.byref(d), None, None, None, None, ws, need, None) == 1
    # misaligned pointer
    odd = ctypes.c_void_p(ws.value + 4)
    w = M.MoELayerWeights(ws.value, ws.value, ws.value, None, None, None)
    assert lib.moe_layer_forward(ctypes.byref(d), ctypes.byref(w), odd, ws, None, ws, need, None) == 1
    # K > E and unsupported shapes
    bad = M.make_desc(8, 256, 4, 5, 512, 0, M.MOE_F32)
    assert lib.moe_topk_from_logits(ctypes.byref(bad), ws, None, ws, ws, None) == 1
    uns = M.make_desc(8, 200, 16, 2, 512, 0, M.MOE_BF16)
    assert lib.moe_topk_from_logits(ctypes.byref(uns), ws, None, ws, ws, None) == 2
    # noisy routing: the noise tensor is required and aligned
    assert lib.moe_topk_from_logits_noisy(ctypes.byref(d), ws, None, None, ws, ws, None) == 1
    assert lib.moe_topk_from_logits_noisy(ctypes.byref(d), ws, None, odd, ws, ws, None) == 1
    assert lib.moe_layer_forward_noisy(ctypes.byref(d), ctypes.byref(w), ws, None, ws, None, ws,
                                       need, None) == 1
    # bias update: missing buffers, negative or non-finite step
    assert lib.moe_bias_update(ctypes.byref(d), None, ws, 0.1, None) == 1
    assert lib.moe_bias_update(ctypes.byref(d), ws, ws, -0.1, None) == 1
    assert lib.moe_bias_update(ctypes.byref(d), ws, ws, float("nan"), None) == 1
    assert lib.moe_bias_update(ctypes.byref(d), ws, ws, float("inf"), None) == 1
    # an empty batch is valid and launches nothing
    empty = M.make_desc(0, 256, 16, 2, 512, 0, M.MOE_F32)
    keep2, ws0 = _host_buffer(M.moe_workspace_size(empty))
    assert lib.moe_layer_forward(ctypes.byref(empty), ctypes.byref(w), None, None, None, ws0,
                                 M.moe_workspace_size(empty), None) == 0
    assert lib.moe_combine(ctypes.byref(empty), None, None, None, None, None, None) == 0
    assert lib.moe_check_status(None, 0, None) == 3


def test_status_strings(M):
    for code in range(6):
        s = M.status_string(code)
        assert s and s != "unknown status"
    assert M.status_string(99) == "unknown status"
