"""The C ABI without a GPU: the library builds and loads, exports every entry
point include/moe.h declares, and rejects bad arguments on the host before
anything is launched."""
import ctypes
import os
import re
import subprocess

import pytest

import mixture_experts_fp32_b200 as moe
from mixture_experts_fp32_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert set(names) == set(moe.EXPORTED)
    out = subprocess.check_output(["nm", "-D", "--defined-only", moe.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n)
    # nothing else with C linkage leaks out under the moe_ prefix
    assert {e for e in exported if e.startswith("moe_")} == set(names)


def test_library_is_built_for_sm100a(lib):
    # the build passes exactly one target, sm_100a (the tcgen05 and TMA
    # instructions the kernels use exist only there); the binary is not opened
    assert moe_build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert os.path.getmtime(moe.LIB_PATH) >= max(os.path.getmtime(f) for f in moe_build._inputs())


def cfg(**kw):
    base = dict(max_tokens=256, hidden=7168, num_experts=48, top_k_max=3, inter=5120,
                num_shared=1, shared_inter=5120, renormalize=1, wtype=moe.MOE_W_BF16)
    base.update(kw)
    return moe.moe_config(**base)


def test_plan_create_and_workspace_size(lib):
    plan, ws = moe.moe_plan_create(cfg())
    try:
        assert ws > 0 and ws % 256 == 0
        T, H, E, k, I, S = 256, 7168, 48, 3, 5120, 1
        R = T * (k + S)
        at_least = 2 * R * H * 2 + 2 * R * I + 4 * T * E
        assert ws >= at_least
        v = moe.moe_get_workspace_views(plan, 1 << 20)
        assert v.h_stride == I
        assert v.row_token is not None and v.row_token > (1 << 20)
    finally:
        moe.moe_plan_destroy(plan)


@pytest.mark.parametrize("bad,status", [
    (dict(max_tokens=0), moe.MOE_ERR_INVALID_ARG),
    (dict(hidden=7000), moe.MOE_ERR_UNSUPPORTED),
    (dict(inter=100), moe.MOE_ERR_UNSUPPORTED),
    (dict(num_experts=257, top_k_max=3), moe.MOE_ERR_UNSUPPORTED),
    (dict(top_k_max=9, num_experts=48), moe.MOE_ERR_UNSUPPORTED),
    (dict(top_k_max=5, num_experts=4), moe.MOE_ERR_INVALID_ARG),
    (dict(num_shared=2), moe.MOE_ERR_INVALID_ARG),
    (dict(num_shared=1, shared_inter=0), moe.MOE_ERR_INVALID_ARG),
    (dict(num_shared=1, shared_inter=200), moe.MOE_ERR_UNSUPPORTED),
    (dict(renormalize=2), moe.MOE_ERR_INVALID_ARG),
    (dict(wtype=7), moe.MOE_ERR_INVALID_ARG),
])
def test_plan_create_rejects(lib, bad, status):
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_plan_create(cfg(**bad))
    assert ei.value.status == status


def test_null_arguments(lib):
    plan = ctypes.c_void_p()
    ws = ctypes.c_size_t()
    assert lib.moe_plan_create(None, ctypes.byref(plan), ctypes.byref(ws)) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_plan_set_wait_limit(None, 0) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_forward(None, None, None, None, 1, 1, None, None, 0, None, None) == \
        moe.MOE_ERR_INVALID_ARG
    for s in (0, -1, -2, -3, -4, -5):
        assert moe.moe_status_string(s)


def test_forward_rejects_bad_arguments_before_launch(lib):
    # every case below must fail on the host: no CUDA device exists here
    plan, ws = moe.moe_plan_create(cfg())
    try:
        w = moe.make_weights(0x1000, None, 0x2000, 0x3000, ws_gate_up=0x4000, ws_down=0x5000)
        WS = 0x100000
        good = dict(hidden=0x6000, valid=None, T=16, k=3, out=0x7000, workspace=WS, ws_bytes=ws)

        def call(**kw):
            a = dict(good)
            a.update(kw)
            return lib.moe_forward(plan, ctypes.byref(w), a["hidden"], a["valid"], a["T"], a["k"],
                                   a["out"], a["workspace"], a["ws_bytes"], None, None)

        assert call(T=257) == moe.MOE_ERR_INVALID_ARG          # T > max_tokens
        assert call(T=-1) == moe.MOE_ERR_INVALID_ARG
        assert call(k=0) == moe.MOE_ERR_INVALID_ARG
        assert call(k=4) == moe.MOE_ERR_INVALID_ARG            # k > top_k_max
        assert call(ws_bytes=ws - 1) == moe.MOE_ERR_WORKSPACE
        assert call(workspace=WS + 16) == moe.MOE_ERR_INVALID_ARG   # not 256-byte aligned
        assert call(workspace=None) == moe.MOE_ERR_INVALID_ARG
        assert call(hidden=None) == moe.MOE_ERR_INVALID_ARG
        assert call(out=0x7008) == moe.MOE_ERR_INVALID_ARG     # not 16-byte aligned
        assert call(T=0) == moe.MOE_OK                          # nothing to do, nothing launched
        w_noshared = moe.make_weights(0x1000, None, 0x2000, 0x3000)
        assert lib.moe_forward(plan, ctypes.byref(w_noshared), 0x6000, None, 16, 3, 0x7000, WS,
                               ws, None, None) == moe.MOE_ERR_INVALID_ARG
        assert lib.moe_route_from_logits(plan, None, None, 4, 3, 0x10, 0x20, 0x30, 0x40, WS, ws,
                                         None) == moe.MOE_ERR_INVALID_ARG
    finally:
        moe.moe_plan_destroy(plan)


def test_pipeline_sizes_and_rejections_before_any_cuda_call(lib):
    plan, ws = moe.moe_plan_create(cfg())
    try:
        H = 7168
        a = lambda v: (v + 255) // 256 * 256                     # noqa: E731
        for rows, depth in ((256, 3), (1, 1), (100, 8)):
            stride = 2 * a(rows * H * 2) + a(rows)               # x, valid, out per slot
            assert moe.moe_pipeline_slot_bytes(plan, rows, depth) == depth * stride
        n = ctypes.c_size_t()
        for rows, depth in ((0, 3), (257, 3), (16, 0), (16, 9)):
            assert lib.moe_pipeline_slot_bytes(plan, rows, depth, ctypes.byref(n)) == \
                moe.MOE_ERR_INVALID_ARG
        w = moe.make_weights(0x1000, None, 0x2000, 0x3000, ws_gate_up=0x4000, ws_down=0x5000)
        need = moe.moe_pipeline_slot_bytes(plan, 16, 3)
        SL, WS = 0x200000, 0x100000
        good = dict(w=ctypes.byref(w), k=3, rows=16, depth=3, slots=SL, nslots=need,
                    workspace=WS, ws_bytes=ws)

        def create(**kw):
            g = dict(good)
            g.update(kw)
            h = ctypes.c_void_p(0x1234)
            st = lib.moe_pipeline_create(plan, g["w"], g["k"], g["rows"], g["depth"], 1,
                                         g["slots"], g["nslots"], g["workspace"], g["ws_bytes"],
                                         ctypes.byref(h))
            assert h.value is None                               # nothing created
            return st

        assert create(w=None) == moe.MOE_ERR_INVALID_ARG
        assert create(k=0) == moe.MOE_ERR_INVALID_ARG
        assert create(k=4) == moe.MOE_ERR_INVALID_ARG            # k > top_k_max
        assert create(rows=257) == moe.MOE_ERR_INVALID_ARG
        assert create(depth=9) == moe.MOE_ERR_INVALID_ARG
        assert create(slots=None) == moe.MOE_ERR_INVALID_ARG
        assert create(slots=SL + 16) == moe.MOE_ERR_INVALID_ARG  # not 256-byte aligned
        assert create(nslots=need - 1) == moe.MOE_ERR_WORKSPACE
        assert create(workspace=None) == moe.MOE_ERR_INVALID_ARG
        assert create(ws_bytes=ws - 1) == moe.MOE_ERR_WORKSPACE
        assert lib.moe_pipeline_submit(None, 0x10, None, 0x20) == moe.MOE_ERR_INVALID_ARG
        assert lib.moe_pipeline_synchronize(None) == moe.MOE_ERR_INVALID_ARG
        assert lib.moe_pipeline_streams(None, None, None, None) == moe.MOE_ERR_INVALID_ARG
        lib.moe_pipeline_destroy(None)
    finally:
        moe.moe_plan_destroy(plan)


def test_tensor_parallel_entry_points_reject_bad_arguments_before_launch(lib):
    plan, ws = moe.moe_plan_create(cfg())
    try:
        w = moe.make_weights(0x1000, None, 0x2000, 0x3000, ws_gate_up=0x4000, ws_down=0x5000)
        WS = 0x100000

        def scatter(dst, rpr, slot, T=16):
            arr = (ctypes.c_void_p * max(1, len(dst)))(*dst)
            return lib.moe_forward_scatter(plan, ctypes.byref(w), 0x6000, None, T, 3, arr,
                                           len(dst), rpr, slot, WS, ws, None, None)

        assert scatter([0x7000, 0x8000], 8, 0, T=17) == moe.MOE_ERR_INVALID_ARG   # n * rpr != T
        assert scatter([], 16, 0) == moe.MOE_ERR_INVALID_ARG                       # no owners
        assert scatter([0x7000] * 9, 2, 0, T=18) == moe.MOE_ERR_INVALID_ARG        # > 8 ranks
        assert scatter([0x7000, 0x8000], 8, 2) == moe.MOE_ERR_INVALID_ARG          # slot >= n
        assert scatter([0x7000, 0x8000], 8, -1) == moe.MOE_ERR_INVALID_ARG
        assert scatter([0x7000, 0x8008], 8, 0) == moe.MOE_ERR_INVALID_ARG          # unaligned
        assert scatter([0x7000, 0], 8, 0) == moe.MOE_ERR_INVALID_ARG               # null owner
        assert scatter([0x7000, 0x8000], 0, 0, T=0) == moe.MOE_ERR_INVALID_ARG     # rpr 0
        arr = (ctypes.c_void_p * 2)(0x7000, 0x8000)
        assert lib.moe_forward_scatter(plan, ctypes.byref(w), 0x6000, None, 16, 4, arr, 2, 8, 0,
                                       WS, ws, None, None) == moe.MOE_ERR_INVALID_ARG  # k > max
        red = lib.moe_reduce_partials
        assert red(None, 2, 4, 64, None, 0x9000, None) == moe.MOE_ERR_INVALID_ARG
        assert red(0x7000, 0, 4, 64, None, 0x9000, None) == moe.MOE_ERR_INVALID_ARG
        assert red(0x7000, 9, 4, 64, None, 0x9000, None) == moe.MOE_ERR_INVALID_ARG
        assert red(0x7000, 2, 4, 60, None, 0x9000, None) == moe.MOE_ERR_INVALID_ARG   # H % 8
        assert red(0x7004, 2, 4, 64, None, 0x9000, None) == moe.MOE_ERR_INVALID_ARG   # unaligned
        assert red(0x7000, 2, 0, 64, None, 0x9000, None) == moe.MOE_OK                 # no rows
    finally:
        moe.moe_plan_destroy(plan)


def test_plain_c_caller(lib, tmp_path):
    """The header compiles as C99 and a C program linked to the library gets the
    documented host-side behaviour (no GPU involved)."""
    exe = tmp_path / "host_only"
    libdir = os.path.dirname(moe.LIB_PATH)
    libname = os.path.basename(moe.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                           "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c", "host_only.c"),
                           "-o", str(exe), "-L", libdir, "-l:" + libname,
                           "-Wl,-rpath," + libdir])
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr + out.stdout
    assert "passed" in out.stdout


def test_ctypes_structures_match_the_header(tmp_path):
    """The binding's structures have the C header's sizes and field offsets (a
    mismatch would hand the library garbage pointers)."""
    structs = {"moe_config": moe.moe_config, "moe_weights": moe.moe_weights,
               "moe_debug": moe.moe_debug, "moe_workspace_views": moe.moe_workspace_views}
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "moe.h"', "int main(void) {"]
    for name, cls in structs.items():
        lines.append(f'  printf("{name} size %zu\\n", sizeof({name}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{name} {field} %zu\\n", offsetof({name}, {field}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe)])
    got = {}
    for line in subprocess.check_output([str(exe)], text=True).splitlines():
        parts = line.split()
        got[(parts[0], parts[1])] = int(parts[2])
    for name, cls in structs.items():
        assert got[(name, "size")] == ctypes.sizeof(cls), name
        for field, _ in cls._fields_:
            assert got[(name, field)] == getattr(cls, field).offset, (name, field)
