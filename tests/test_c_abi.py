"""The C ABI from plain C: a C99 program that includes include/ep.h, links
libep.so, takes the address of every entry point the header declares, and calls
the host-only ones (ep_status_str, ep_buffer_size, ep_shard_workspace_size, and a
refused ep_layout_static_scratch).  Its results must equal the Python binding's.
No GPU is needed: none of these calls reaches the device."""
import os
import re
import shutil
import subprocess

import pytest

from combine_ep_layout_12_b200 import _binding as abi
from combine_ep_layout_12_b200 import build as ep_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ep.h")

PROGRAM = r"""
#include <stdio.h>
#include "ep.h"

static void* const entry_points[] = {%(entries)s};

int main(void) {
    ep_config c = {1024, 7168, 8, 8, 128, 256, 0, 0, 0, 2, 1, 0};
    ep_buffer_sizes s;
    size_t ws = 0;
    int st;
    unsigned i;
    for (i = 0; i < sizeof(entry_points) / sizeof(entry_points[0]); ++i)
        if (!entry_points[i]) return 2;
    st = ep_buffer_size(&c, &s);
    printf("size %%d %%zu %%zu %%zu %%zu %%zu %%zu %%zu %%zu %%zu\n", st, s.expert_count, s.expert_offset,
           s.recv_count, s.dst_pos, s.recv_src, s.recv_x, s.recv_scale, s.token_scale, s.workspace);
    st = ep_shard_workspace_size(&c, &ws);
    printf("shard %%d %%zu\n", st, ws);
    c.B = 7;  /* not a multiple of P */
    printf("bad %%d\n", ep_buffer_size(&c, &s));
    c.B = 1024;
    printf("static %%d\n", ep_layout_static_scratch(&c, 0, 0, 0, 0, 0, 0, 0, 0));
    for (st = 0; st >= -4; --st) printf("status %%d %%s\n", st, ep_status_str(st));
    return 0;
}
"""


def declared_entry_points():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"EP_API\s+[^;]*?\b(ep_\w+)\s*\(", text, re.S)))


@pytest.fixture(scope="module")
def program(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    lib = ep_build.build()
    d = tmp_path_factory.mktemp("c_abi")
    src = d / "use_ep.c"
    names = declared_entry_points()
    src.write_text(PROGRAM % {"entries": ", ".join("(void*)%s" % n for n in names)})
    exe = d / "use_ep"
    libdir = os.path.dirname(lib)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-Wno-pedantic", "-I",
                    os.path.join(ROOT, "include"), str(src), "-o", str(exe), "-L", libdir, "-lep",
                    "-Wl,-rpath," + libdir], check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    return names, out.splitlines()


def test_every_declared_entry_point_links_from_c(program):
    names, _ = program
    assert "ep_shard_layout_dispatch" in names and "ep_combine" in names
    assert len(names) >= 16


def test_c_results_match_the_binding(program):
    _, lines = program
    fields = lines[0].split()
    assert fields[0] == "size" and int(fields[1]) == abi.EP_OK
    cfg = abi.make_config(1024, 7168, 8, 8, 128, 256, quant_mode=2, smooth_rows=1)
    s = abi.ep_buffer_size(cfg)
    want = [s.expert_count, s.expert_offset, s.recv_count, s.dst_pos, s.recv_src, s.recv_x, s.recv_scale,
            s.token_scale, s.workspace]
    assert [int(v) for v in fields[2:]] == want
    assert lines[1].split() == ["shard", str(abi.EP_OK), str(abi.ep_shard_workspace_size(cfg))]
    assert lines[2] == "bad %d" % abi.EP_ERR_INVALID_ARG
    assert lines[3] == "static %d" % abi.EP_ERR_INVALID_ARG
    for st, line in zip(range(0, -5, -1), lines[4:]):
        assert line == "status %d %s" % (st, abi.ep_status_str(st))
