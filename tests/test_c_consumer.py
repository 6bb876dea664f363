"""The C ABI as a C program sees it (no GPU needed).

A C99 program compiled with gcc against include/sfc.h and linked to libsfc.so
prints the size and field offsets of every public struct and calls the
host-only entry points; the ctypes binding must agree with it on every
layout and every returned value. This checks the boundary from the side of
a C caller: the header compiles as plain C, the library links and resolves,
and the binding's struct layouts are the compiler's.
"""
import ctypes as C
import os
import subprocess

import pytest

from latency_self_synchronizing_b200 import _lib, api

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "latency_self_synchronizing_b200")

STRUCTS = {
    "sfc_config": (_lib.Config, ["ctas_per_rank", "timeout_us", "debug_checks", "protocol_mask", "device_epochs"]),
    "sfc_cost_entry": (_lib.CostEntry, ["alpha_us", "beta_us_per_byte", "table_us"]),
    "sfc_cost_model": (_lib.CostModel, ["c"]),
    "sfc_floor_result": (_lib.FloorResult, [f for f, _ in _lib.FloorResult._fields_]),
    "sfc_ll_view": (_lib.LLView, ["scratch", "slot_stride", "nranks", "status", "timeout_ns"]),
}
SIZES = [512, 2048, 16384, 131072, 1 << 20, 1 << 24, 1 << 26]


def _program():
    lines = ["#include <stddef.h>", "#include <stdio.h>", '#include "sfc.h"', "int main(void) {"]
    for name, (_, fields) in STRUCTS.items():
        lines.append(f'  printf("size {name} %zu\\n", sizeof({name}));')
        for f in fields:
            lines.append(f'  printf("offset {name}.{f} %zu\\n", offsetof({name}, {f}));')
    lines.append("  for (int s = 0; s <= 9; ++s) printf(\"status %d %s\\n\", s, sfc_status_string((sfc_status)s));")
    lines.append("  static sfc_cost_model m;")
    lines.append("  sfc_default_cost_model(&m);")
    sizes = ", ".join(f"{s}u" for s in SIZES)
    lines.append(f"  const size_t sizes[] = {{{sizes}}};")
    lines.append(f"  for (int i = 0; i < {len(SIZES)}; ++i)")
    lines.append("    for (int op = 0; op < 2; ++op)")
    lines.append("      for (int n = 2; n <= 8; ++n) {")
    lines.append("        printf(\"select %d %zu %d %d\\n\", op, sizes[i], n,"
                 " (int)sfc_select_protocol_model(&m, (sfc_op)op, sizes[i], n));")
    lines.append("        for (int p = 1; p < SFC_NUM_PROTOCOLS; ++p)")
    lines.append("          printf(\"bytes %d %d %zu %d %.17g\\n\", op, p, sizes[i] / 2, n,"
                 " sfc_algorithmic_bytes((sfc_op)op, (sfc_protocol)p, sizes[i] / 2, n));")
    lines.append("      }")
    lines.append('  printf("init_null %d\\n", (int)sfc_init(NULL, 4, 4096, NULL));')
    lines.append("  sfc_ctx* ctx = NULL;")
    lines.append('  printf("init_bad_ranks %d\\n", (int)sfc_init(&ctx, 1, 4096, NULL));')
    lines.append('  printf("destroy_null %d\\n", (int)sfc_destroy(NULL));')
    lines.append("  sfc_plan* plan = (sfc_plan*)1;")
    lines.append('  printf("plan_create_null %d\\n", (int)sfc_plan_create(NULL, SFC_OP_ALLREDUCE, NULL, NULL, 8, SFC_BF16,'
                 ' SFC_PROTO_LL, &plan));')
    lines.append('  printf("plan_cleared %d\\n", plan == NULL);')
    lines.append('  printf("plan_launch_null %d\\n", (int)sfc_plan_launch(NULL, NULL));')
    lines.append('  printf("plan_destroy_null %d\\n", (int)sfc_plan_destroy(NULL));')
    lines += ["  return 0;", "}"]
    return "\n".join(lines) + "\n"


@pytest.fixture(scope="module")
def c_output(tmp_path_factory):
    lib = _lib.LIB_PATH
    if not os.path.exists(lib):
        pytest.fail(f"{lib} is missing: build it first")
    d = tmp_path_factory.mktemp("c_consumer")
    src = d / "consumer.c"
    src.write_text(_program())
    exe = d / "consumer"
    subprocess.check_call(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", str(exe), lib, f"-Wl,-rpath,{os.path.dirname(lib)}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    return [line.split(" ", 1) for line in out.splitlines()]


def _records(c_output, kind):
    return [rest for k, rest in c_output if k == kind]


def test_struct_layouts_match_the_compiler(c_output):
    for rest in _records(c_output, "size"):
        name, size = rest.split()
        assert C.sizeof(STRUCTS[name][0]) == int(size), name
    for rest in _records(c_output, "offset"):
        path, off = rest.split()
        name, field = path.split(".")
        assert getattr(STRUCTS[name][0], field).offset == int(off), path


def test_status_strings_match(c_output):
    recs = _records(c_output, "status")
    assert len(recs) == 10
    for rest in recs:
        s, text = rest.split(" ", 1)
        assert api.status_string(int(s)) == text


def test_selector_and_bytes_agree_with_the_binding(c_output):
    m = api.default_cost_model()
    sel = _records(c_output, "select")
    assert len(sel) == len(SIZES) * 2 * 7
    for rest in sel:
        op, b, n, p = (int(v) for v in rest.split())
        assert int(api.select_protocol_model(m, op, b, n)) == p, (op, b, n)
    for rest in _records(c_output, "bytes"):
        op, p, count, n, v = rest.split()
        assert api.algorithmic_bytes(int(op), int(p), int(count), int(n)) == float(v)


def test_argument_checks_from_c(c_output):
    keys = ("init_null", "init_bad_ranks", "destroy_null", "plan_create_null", "plan_cleared", "plan_launch_null",
            "plan_destroy_null")
    vals = {k: int(v) for k, v in c_output if k in keys}
    assert vals == {"init_null": int(api.Status.INVALID), "init_bad_ranks": int(api.Status.INVALID),
                    "destroy_null": int(api.Status.INVALID), "plan_create_null": int(api.Status.INVALID),
                    "plan_cleared": 1, "plan_launch_null": int(api.Status.INVALID), "plan_destroy_null": 0}
