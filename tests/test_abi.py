"""The C-ABI library loads and exports every symbol include/gdpa.h declares;
host-side argument checks (no GPU needed: they return before any launch)."""
import ctypes
import os
import re

import pytest

from pffn_attention_b200 import gdpa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdpa.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDPA_API\s+[\w\s\*]+?\b(gdpa_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    return gdpa.load()


def test_header_declares_the_api():
    assert set(declared_symbols()) == set(gdpa.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_version_and_status_strings(lib):
    assert gdpa.gdpa_version() >= 100
    for code in range(7):
        assert gdpa.gdpa_status_string(code) not in ("", "unknown status")
    assert gdpa.gdpa_status_string(99) == "unknown status"


def _params(**kw):
    base = dict(B=2, H=2, D=64, total_q=10, total_kv=8, phi=0, scale=1.0)
    base.update(kw)
    B, H, D, tq, tk = (base.pop(x) for x in ("B", "H", "D", "total_q", "total_kv"))
    return gdpa.make_params(B, H, D, tq, tk, **base)


FAKE = 0x7f0000000000  # 16-byte aligned, never dereferenced: rejected first


@pytest.mark.parametrize("kw,expect", [
    (dict(D=48), 2), (dict(D=256), 2), (dict(phi=7), 2), (dict(bias_kind=5), 2),
    (dict(H=0), 1), (dict(B=-1), 1), (dict(total_q=-3), 1), (dict(window=(-2, 0)), 1),
    (dict(B=16385), 2), (dict(scale=float("nan")), 1),
])
def test_invalid_params_rejected(lib, kw, expect):
    p = _params(**kw)
    rc = gdpa.gdpa_forward(p, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, 1 << 20, None)
    assert rc == expect
    assert gdpa.gdpa_workspace_size(p, 0) == 0


def test_null_and_unaligned_pointers_rejected(lib):
    p = _params()
    assert gdpa.gdpa_forward(None if False else p, None, FAKE, FAKE, FAKE, FAKE, None, FAKE, None,
                             FAKE, 1 << 20, None) == 1
    assert gdpa.gdpa_forward(p, FAKE + 8, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, 1 << 20,
                             None) == 1
    assert gdpa.gdpa_forward(p, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, None, FAKE, 1 << 20,
                             None) == 1
    # bias pointer given without a bias kind, and a bias kind without a pointer
    assert gdpa.gdpa_forward(p, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 20,
                             None) == 1
    pb = _params(bias_kind=2)
    assert gdpa.gdpa_forward(pb, FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, 1 << 20,
                             None) == 1
    assert lib.gdpa_forward(None, None, None, None, None, None, None, None, None, None, 0,
                            None) == 1
    # a bias gradient without a bias, and an unaligned bias gradient
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert gdpa.gdpa_backward(p, *args, None, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert gdpa.gdpa_backward(pb, *args, FAKE, FAKE, FAKE, FAKE, FAKE + 2, FAKE, 1 << 20,
                              None) == 1


def test_workspace_size_grows_with_problem(lib):
    small = gdpa.gdpa_workspace_size(_params(), 0)
    big = gdpa.gdpa_workspace_size(_params(B=4000, total_q=4000), 0)
    assert 256 < small < big
    bwd = gdpa.gdpa_workspace_size(_params(phi=1, max_seqlen_q=10), 1)
    assert bwd > gdpa.gdpa_workspace_size(_params(phi=1), 0)


def test_tile_shape_query(lib):
    # 128 query rows; 64-key blocks when no sample has more than 64 keys
    rc, bm, bn = gdpa.gdpa_forward_tile_shape(_params(max_seqlen_kv=64))
    assert (rc, bm, bn) == (0, 128, 64)
    rc, bm, bn = gdpa.gdpa_forward_tile_shape(_params(max_seqlen_kv=65))
    assert (rc, bm, bn) == (0, 128, 128)


def test_head_phi_validation(lib):
    """A per-head activation vector: entries must be GDPA_PHI values and H <= 64;
    a softmax head anywhere makes the backward workspace hold delta."""
    assert gdpa.gdpa_workspace_size(_params(H=3, head_phi=[0, 1, 9]), 0) == 0
    assert gdpa.gdpa_workspace_size(_params(H=65, head_phi=[0] * 65), 0) == 0
    assert gdpa.gdpa_workspace_size(_params(H=65), 0) > 0
    plain = gdpa.gdpa_workspace_size(_params(H=3, phi=0), 1)
    mixed = gdpa.gdpa_workspace_size(_params(H=3, phi=0, head_phi=[0, 1, 3]), 1)
    assert mixed > plain > 0
    assert gdpa.gdpa_workspace_size(_params(H=3, phi=0, head_phi=[3, 2, 0]), 1) == plain


def test_grouped_forward_validation(lib):
    """Grouped calls are validated on the host before any launch: no problems,
    a problem with bad parameters or pointers, or an unaligned workspace."""
    def arr(*params):
        a = (gdpa.gdpa_forward_problem_t * len(params))()
        for i, p in enumerate(params):
            a[i].params = p
            for name in ("q", "k", "v", "q_offsets", "kv_offsets", "o"):
                setattr(a[i], name, FAKE)
        return a
    assert gdpa.gdpa_forward_grouped_workspace_size(None) == 0
    good = arr(_params(), _params(H=3, D=128, phi=1))
    assert gdpa.gdpa_forward_grouped_workspace_size(good) > 0
    assert gdpa.gdpa_forward_grouped_workspace_size(arr(_params(), _params(D=48))) == 0
    nobias = arr(_params(bias_kind=2))  # a gate without its tensor
    assert gdpa.gdpa_forward_grouped(nobias, FAKE, 1 << 20, None) == 1
    assert gdpa.gdpa_forward_grouped(None, FAKE, 1 << 20, None) == 1
    # tensor maps live in the workspace: it must be 64-byte aligned
    assert gdpa.gdpa_forward_grouped(good, FAKE + 16, 1 << 20, None) == 1


def test_grouped_backward_validation(lib):
    """The grouped backward checks every problem as gdpa_backward would before
    any launch; its workspace is the status block, the offsets table and one
    backward workspace per problem."""
    def arr(*params):
        a = (gdpa.gdpa_backward_problem_t * len(params))()
        for i, p in enumerate(params):
            a[i].params = p
            for name in ("q", "k", "v", "o", "dout", "lse", "q_offsets", "kv_offsets", "dq",
                         "dk", "dv"):
                setattr(a[i], name, FAKE)
        return a
    assert gdpa.gdpa_backward_grouped_workspace_size(None) == 0
    p1, p2 = _params(), _params(H=3, D=128, phi=1)
    good = arr(p1, p2)
    n = gdpa.gdpa_backward_grouped_workspace_size(good)
    each = gdpa.gdpa_workspace_size(p1, 1) + gdpa.gdpa_workspace_size(p2, 1)
    assert n >= each + 256 + 256
    assert gdpa.gdpa_backward_grouped_workspace_size(arr(_params(), _params(D=48))) == 0
    nobias = arr(_params(bias_kind=2))  # a gate without its tensor
    assert gdpa.gdpa_backward_grouped(nobias, FAKE, 1 << 30, None) == 1
    assert gdpa.gdpa_backward_grouped(None, FAKE, 1 << 30, None) == 1
    assert gdpa.gdpa_backward_grouped(good, FAKE + 8, 1 << 30, None) == 1  # unaligned
    assert gdpa.gdpa_backward_grouped(good, FAKE, n - 1, None) == 3        # workspace short


def test_rotary_validation(lib):
    """Rotary tables: D, time scale, jagged sizes and alignment are checked on
    the host; the tables must come as a pair; the streamed turn adds the
    turned copies to the workspace (single and grouped calls); the grouped
    call refuses the in-kernel turn."""
    def rp(D=64, scale=60.0):
        return gdpa.gdpa_rotary_params_t(D, scale, None, None)
    assert gdpa.gdpa_rotary_table_bytes(64, 10) == 10 * 32 * 4
    assert gdpa.gdpa_rotary_table_bytes(48, 10) == 0
    assert gdpa.gdpa_rotary_table(rp(D=48), 2, 10, FAKE, FAKE, FAKE, None) == 2
    assert gdpa.gdpa_rotary_table(rp(scale=0.0), 2, 10, FAKE, FAKE, FAKE, None) == 1
    assert gdpa.gdpa_rotary_table(rp(scale=float("inf")), 2, 10, FAKE, FAKE, FAKE, None) == 1
    assert gdpa.gdpa_rotary_table(rp(), 2, 10, FAKE, FAKE, FAKE + 4, None) == 1
    assert gdpa.gdpa_rotary_table(rp(), 2, 10, None, FAKE, FAKE, None) == 1
    assert gdpa.gdpa_rotary_table(rp(), 0, 0, None, None, None, None) == 0  # nothing to do
    bad_freq = (ctypes.c_float * 32)(*([1.0] * 31 + [float("nan")]))
    r = gdpa.gdpa_rotary_params_t(64, 60.0, ctypes.cast(bad_freq, ctypes.POINTER(ctypes.c_float)),
                                  None)
    assert gdpa.gdpa_rotary_table(r, 2, 10, FAKE, FAKE, FAKE, None) == 1
    p = _params()
    p.rope_q = FAKE
    assert gdpa.gdpa_workspace_size(p, 0) == 0  # one table without the other
    p.rope_kv = FAKE + 8
    assert gdpa.gdpa_workspace_size(p, 0) == 0  # unaligned
    p.rope_kv = FAKE
    assert gdpa.gdpa_workspace_size(p, 0) > 0
    # the turned copies of Q and K live in the workspace
    # (total_q = 10, total_kv = 8, H = 2, D = 64: 2560 + 2048 bytes, both 256-aligned)
    for backward in (0, 1):
        plain = gdpa.gdpa_workspace_size(_params(), backward)
        assert gdpa.gdpa_workspace_size(p, backward) == plain + 2560 + 2048
    p.debug_flags = 4  # turned inside the forward kernel: no copies
    assert gdpa.gdpa_workspace_size(p, 0) == gdpa.gdpa_workspace_size(_params(), 0)
    assert gdpa.gdpa_rotary_apply(10, 2, 48, FAKE, FAKE, FAKE, 0, None) == 2
    assert gdpa.gdpa_rotary_apply(10, 0, 64, FAKE, FAKE, FAKE, 0, None) == 1
    assert gdpa.gdpa_rotary_apply(10, 2, 64, FAKE + 2, FAKE, FAKE, 0, None) == 1
    assert gdpa.gdpa_rotary_apply(0, 2, 64, None, None, None, 0, None) == 0
    a = (gdpa.gdpa_forward_problem_t * 1)()
    a[0].params = p
    for name in ("q", "k", "v", "q_offsets", "kv_offsets", "o"):
        setattr(a[0], name, FAKE)
    assert gdpa.gdpa_forward_grouped_workspace_size(a) == 0  # bit 2 (in-kernel turn) set
    p.debug_flags = 0
    a[0].params = p
    plain = (gdpa.gdpa_forward_problem_t * 1)()
    plain[0].params = _params()
    for name in ("q", "k", "v", "q_offsets", "kv_offsets", "o"):
        setattr(plain[0], name, FAKE)
    # the grouped call keeps turned copies of the problem's Q and K
    assert gdpa.gdpa_forward_grouped_workspace_size(a) == \
        gdpa.gdpa_forward_grouped_workspace_size(plain) + 2560 + 2048


def test_struct_layouts_match_the_header(tmp_path):
    """The ctypes mirrors have the C structs' sizes and field offsets."""
    import subprocess
    structs = {"gdpa_params_t": gdpa.gdpa_params_t,
               "gdpa_forward_problem_t": gdpa.gdpa_forward_problem_t,
               "gdpa_rotary_params_t": gdpa.gdpa_rotary_params_t,
               "gdpa_sumkron_params_t": gdpa.gdpa_sumkron_params_t}
    lines = ['#include <stddef.h>', '#include <stdio.h>', '#include "gdpa.h"', 'int main(void) {']
    for name, cls in structs.items():
        lines.append(f'  printf("{name} %zu\\n", sizeof({name}));')
        for field, _ in cls._fields_:
            lines.append(f'  printf("{name}.{field} %zu\\n", offsetof({name}, {field}));')
    lines.append('  return 0; }')
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), str(src),
                           "-o", str(exe)])
    got = dict(line.rsplit(" ", 1) for line in subprocess.check_output([str(exe)]).decode().split("\n")
               if line)
    for name, cls in structs.items():
        assert int(got[name]) == ctypes.sizeof(cls), name
        for field, _ in cls._fields_:
            assert int(got[f"{name}.{field}"]) == getattr(cls, field).offset, (name, field)


def test_sumkron_validation(lib):
    """Shapes the fused kernel does not cover are refused before any launch."""
    def sp(**kw):
        base = dict(B=4, S=256, T=32, D=384, k=8, wait_timeout_us=0, debug_flags=0)
        base.update(kw)
        return gdpa.gdpa_sumkron_params_t(**base)
    assert gdpa.gdpa_sumkron_workspace_size(sp()) == 256
    for kw, expect in [(dict(T=16), 2), (dict(D=192), 2), (dict(S=100), 2), (dict(S=320), 2),
                       (dict(k=3), 2),
                       (dict(B=-1), 1), (dict(k=0), 1), (dict(S=0), 1)]:
        assert gdpa.gdpa_sumkron_workspace_size(sp(**kw)) == 0
        assert gdpa.gdpa_sumkron_forward(sp(**kw), FAKE, FAKE, FAKE, FAKE, FAKE, 256, None) == \
            expect, kw
    assert gdpa.gdpa_sumkron_forward(sp(), FAKE + 8, FAKE, FAKE, FAKE, FAKE, 256, None) == 1
    assert gdpa.gdpa_sumkron_forward(sp(), FAKE, FAKE, FAKE, FAKE, FAKE, 16, None) == 3
