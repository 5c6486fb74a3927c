"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
entry point include/ep.h declares, sizes its arrays as documented and rejects bad
configurations and pointers before touching CUDA."""
import ctypes
import os
import re

import pytest

from combine_ep_layout_12_b200 import _binding as abi
from combine_ep_layout_12_b200 import build as ep_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    ep_build.build()
    ep_build.build_checked()


def declared_entry_points():
    names = []
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^EP_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)
    return names


@pytest.mark.parametrize("path", [abi.LIB_PATH, abi.LIB_CHECKED_PATH])
def test_exports_every_declared_symbol(path):
    names = declared_entry_points()
    assert len(names) >= 8
    lib = ctypes.CDLL(path)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_has_same_names():
    import combine_ep_layout_12_b200 as pkg
    for n in declared_entry_points():
        assert hasattr(pkg, n), n


def cfg(**kw):
    base = dict(B=1024, d=7168, k=8, P=8, M=128, E=256, quant_mode=2)
    base.update(kw)
    return abi.make_config(**base)


def test_sizes_decode():
    s = abi.ep_buffer_size(cfg())
    rows = 256 * 8 * 128
    assert s.recv_x == rows * 7168
    assert s.recv_scale == 4 * rows
    assert s.token_scale == 4 * 1024
    assert s.dst_pos == 4 * 1024 * 8
    assert s.recv_src == 4 * rows
    assert s.recv_count == 4 * 256 * 8
    assert s.expert_count == 4 * 256 and s.expert_offset == 4 * 257
    assert s.workspace % 256 == 0 and s.workspace >= 256


def test_sizes_bf16_specials():
    s = abi.ep_buffer_size(cfg(quant_mode=0, n_zero=1, n_copy=1, n_const=1, B=8192, d=4096, E=64,
                               k=6, M=1024))
    rows = 64 * 8 * 1024
    assert s.recv_x == rows * 4096 * 2
    assert s.recv_scale == 0 and s.token_scale == 0
    assert s.expert_count == 4 * 67 and s.expert_offset == 4 * 68
    assert s.workspace >= 256 + 4 * 8 * 3


@pytest.mark.parametrize("kw,status", [
    (dict(E=250), abi.EP_ERR_INVALID_ARG),          # E % P != 0
    (dict(B=1001), abi.EP_ERR_INVALID_ARG),         # B % P != 0
    (dict(k=0), abi.EP_ERR_INVALID_ARG),
    (dict(k=17), abi.EP_ERR_INVALID_ARG),
    (dict(d=7160), abi.EP_ERR_INVALID_ARG),         # d % 16 != 0
    (dict(d=0), abi.EP_ERR_INVALID_ARG),
    (dict(d=65536), abi.EP_ERR_UNSUPPORTED),
    (dict(quant_mode=-1), abi.EP_ERR_INVALID_ARG),
    (dict(quant_mode=3), abi.EP_ERR_INVALID_ARG),
    (dict(M=64), abi.EP_ERR_CAPACITY),              # T = 128 > M
    (dict(E=4096, P=8), abi.EP_ERR_UNSUPPORTED),     # E above 2048
    (dict(M=2**20), abi.EP_ERR_CAPACITY),           # E*P*M >= 2^31
    (dict(n_zero=-1), abi.EP_ERR_INVALID_ARG),
    (dict(n_const=4096), abi.EP_ERR_UNSUPPORTED),
    (dict(layout=2), abi.EP_ERR_UNSUPPORTED),
    (dict(layout=1, E=2048, P=16, B=1024, M=64), abi.EP_ERR_UNSUPPORTED),   # E*P above the pack table
    (dict(smooth_rows=2), abi.EP_ERR_INVALID_ARG),
    (dict(smooth_rows=64, quant_mode=0), abi.EP_ERR_INVALID_ARG),  # per-expert scale needs int8
    (dict(P=0), abi.EP_ERR_INVALID_ARG),
])
def test_bad_configs(kw, status):
    with pytest.raises(abi.EPError) as ei:
        abi.ep_buffer_size(cfg(**kw))
    assert ei.value.status == status


def test_sizes_static_int8():
    """quant_mode 1 (static int8): an int8 payload and no scales."""
    s = abi.ep_buffer_size(cfg(quant_mode=1))
    rows = 256 * 8 * 128
    assert s.recv_x == rows * 7168
    assert s.recv_scale == 0 and s.token_scale == 0


def test_sizes_expert_smooth():
    """A per-expert smooth scale (smooth_rows = E) changes no buffer size."""
    assert abi.ep_buffer_size(cfg(smooth_rows=256)).recv_x == abi.ep_buffer_size(cfg()).recv_x


def test_sizes_packed():
    s = abi.ep_buffer_size(cfg(layout=1, M=0))       # M is not used by the packed layout
    rows = 1024 * 8
    assert s.recv_x == rows * 7168 and s.recv_src == 4 * rows and s.recv_scale == 4 * rows
    s0 = abi.ep_buffer_size(cfg(layout=1, quant_mode=0, M=0))
    assert s0.recv_x == rows * 7168 * 2 and s0.recv_scale == 0


def test_edge_configs_accepted():
    abi.ep_buffer_size(cfg(B=0))
    abi.ep_buffer_size(cfg(k=16))
    abi.ep_buffer_size(cfg(d=16))
    abi.ep_buffer_size(cfg(d=32768))
    abi.ep_buffer_size(cfg(E=2048, P=8, M=128))
    abi.ep_buffer_size(cfg(P=1, B=128, E=8, k=2, M=128, d=256))


def test_create_rejects_null_and_misaligned_pointers_before_cuda():
    c = cfg(B=16, d=256, k=2, P=2, M=8, E=4)
    s = abi.ep_buffer_size(c)
    fake = 1 << 40  # never dereferenced: validation fails first
    good = {n: (fake if getattr(s, n) else None) for n in abi.BUFFER_FIELDS}
    for victim in ("recv_x", "dst_pos", "workspace"):
        for bad in (None, fake + 8):
            ptrs = dict(good)
            ptrs[victim] = bad
            with pytest.raises(abi.EPError) as ei:
                abi.ep_buffer_create(c, abi.ep_buffer_ptrs(*[ptrs[n] for n in abi.BUFFER_FIELDS]))
            assert ei.value.status == abi.EP_ERR_INVALID_ARG


def test_calls_reject_null_handle():
    for f, args in ((abi.ep_layout, (None, 0)), (abi.ep_dispatch, (None, None, 0)),
                    (abi.ep_combine, (None,) * 8 + (0,))):
        with pytest.raises(abi.EPError) as ei:
            f(None, *args)
        assert ei.value.status == abi.EP_ERR_INVALID_ARG


def test_status_strings():
    for st in (0, -1, -2, -3, -4):
        assert abi.ep_status_str(st)
    assert abi.ep_status_str(12345) == "unknown status"


def test_product_path_has_no_oracle_import():
    """The library and binding never import or load the CPU oracle."""
    pkg = os.path.join(ROOT, "combine_ep_layout_12_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".cpp", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                bad = re.search(r"^\s*(import oracle|from oracle)|libep_oracle|orc_[a-z]+\(", text,
                                flags=re.M)
                assert not bad, os.path.join(dirpath, f)


def test_shard_workspace_size_and_unsupported_forms():
    # one rank's layout workspace (header + counts scratch), 256-byte granular
    n = abi.ep_shard_workspace_size(cfg())
    assert n % 256 == 0 and n >= 256 + 4 * (2 * 256 + 1)
    # above 256 tokens per rank the chunk counts of the rank's own tokens are added
    big = abi.ep_shard_workspace_size(cfg(B=8 * 1024, M=1024))
    assert big >= n + 4 * 4 * 256
    for kw, status in ((dict(layout=1), abi.EP_ERR_UNSUPPORTED),
                       (dict(smooth_rows=256), abi.EP_ERR_UNSUPPORTED),
                       (dict(P=128, E=256, B=128, M=1), abi.EP_ERR_UNSUPPORTED),
                       (dict(B=7), abi.EP_ERR_INVALID_ARG)):
        with pytest.raises(abi.EPError) as ei:
            abi.ep_shard_workspace_size(cfg(**kw))
        assert ei.value.status == status, kw


def test_shard_calls_reject_bad_arguments_before_cuda():
    c = cfg()
    fake = 1 << 40  # 16-byte aligned, never dereferenced: validation fails first
    good = abi.make_shard_table(0, [fake] * 8, [fake] * 8, [fake] * 8)
    # rank out of range
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_layout(c, 8, fake, None, fake, fake, fake)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    # a missing slab in the table
    holes = abi.make_shard_table(0, [fake] * 7 + [None], [fake] * 8, [fake] * 8)
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_dispatch(c, holes, fake, None, fake, None, fake, fake)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    # a misaligned slab
    odd = abi.make_shard_table(0, [fake + 8] + [fake] * 7, [fake] * 8, [fake] * 8)
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_dispatch(c, odd, fake, None, fake, None, fake, fake)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    # quant_mode 2 needs the scale slabs and token_scale
    no_scale = abi.make_shard_table(0, [fake] * 8, None, [fake] * 8)
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_dispatch(c, no_scale, fake, None, fake, None, fake, fake)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_dispatch(c, good, fake, None, fake, None, None, fake)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    # the count exchange: a misaligned owner recv_count or send_count
    odd_count = abi.make_shard_table(0, [fake] * 8, [fake] * 8, [fake] * 8, [fake] * 7 + [fake + 2])
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_dispatch(c, odd_count, fake, None, fake, fake, fake, fake)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_dispatch(c, good, fake, None, fake, fake + 2, fake, fake)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    # layout and dispatch as one call: send_count and the workspace are required
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_layout_dispatch(c, good, fake, None, fake, None, fake, None, fake, fake)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_layout_dispatch(c, good, fake, None, fake, None, fake, fake, fake, None)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_layout_dispatch(c, holes, fake, None, fake, None, fake, fake, fake, fake)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    # combine: y must be given and must not be ori_x
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_combine(c, good, fake, fake, None, fake, None, None, None, None, None, fake)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    # no workspace
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_layout(c, 0, fake, None, fake, fake, None)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
    with pytest.raises(abi.EPError) as ei:
        abi.ep_shard_check(None)
    assert ei.value.status == abi.EP_ERR_INVALID_ARG
