"""The C ABI without a GPU: the library loads, exports every entry point that
include/ss_scan.h declares, and rejects invalid arguments on the host before any
CUDA call.  Pointers here are fake addresses that are never dereferenced: every
call below fails validation first."""
import ctypes
import os
import re

import pytest

from selective_state_space_18_b200 import build as ssbuild
from selective_state_space_18_b200 import ssscan

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ss_scan.h")


@pytest.fixture(scope="module")
def lib():
    ssbuild.build()
    return ssscan.load_library()


def _declared():
    text = open(HEADER).read()
    return re.findall(r"SS_API\s+[\w\s\*]*?\b(ss_\w+)\s*\(", text)


def _header_enum(name):
    text = open(HEADER).read()
    m = re.search(rf"\b{name}\s*=\s*(\d+)", text)
    return int(m.group(1))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert set(names) >= {"ss_scan_fwd", "ss_scan_workspace_bytes", "ss_scan_status",
                          "ss_state_update", "ss_status_string", "ss_abi_version"}
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(ssscan.EXPORTS)


def test_status_codes_match_header(lib):
    for code, name in ssscan.STATUS.items():
        assert _header_enum(name) == code
        assert lib.ss_status_string(code).decode().startswith(name)
    assert lib.ss_status_string(1234) == b"unknown status"
    assert lib.ss_abi_version() >> 16 == ssscan.ABI_MAJOR


# fake, well-aligned device addresses (never dereferenced)
P = [ctypes.c_void_p(0x7f0000000000 + i * 0x100000000) for i in range(12)]


def _scan(lib, **kw):
    a = dict(batch=2, channels=16, state_dim=16, seq=64, dtype=ssscan.SS_BF16, x=P[0], dt=P[1],
             A=P[2], B=P[3], C=P[4], D=None, z=None, dt_bias=None, reset=None, h0=None,
             flags=1, y=P[5], h_last=None, ws=None, ws_bytes=0, stream=None)
    a.update(kw)
    return lib.ss_scan_fwd(a["batch"], a["channels"], a["state_dim"], a["seq"], a["dtype"],
                           a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], a["z"], a["dt_bias"],
                           a["reset"], a["h0"], a["flags"], a["y"], a["h_last"], a["ws"],
                           a["ws_bytes"], a["stream"])


def _update(lib, **kw):
    a = dict(batch=4, channels=32, state_dim=16, dtype=ssscan.SS_F32, state=P[0], x=P[1], dt=P[2],
             A=P[3], B=P[4], C=P[5], D=None, z=None, dt_bias=None, flags=1, y=P[6], stream=None)
    a.update(kw)
    return lib.ss_state_update(a["batch"], a["channels"], a["state_dim"], a["dtype"], a["state"],
                               a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], a["z"],
                               a["dt_bias"], a["flags"], a["y"], a["stream"])


@pytest.mark.parametrize("field", ["x", "dt", "A", "B", "C", "y"])
def test_scan_null_pointer(lib, field):
    assert _scan(lib, **{field: None}) == 1


@pytest.mark.parametrize("field", ["batch", "channels", "state_dim", "seq"])
@pytest.mark.parametrize("value", [0, -3])
def test_scan_bad_size(lib, field, value):
    assert _scan(lib, **{field: value}) == 2


def test_scan_size_overflow(lib):
    assert _scan(lib, batch=1 << 40, channels=1 << 20, seq=1 << 10) == 2


def test_scan_bad_dtype(lib):
    assert _scan(lib, dtype=7) == 3


@pytest.mark.parametrize("n", [1, 2, 3, 5, 12, 32, 64])
def test_scan_unsupported_state_dim(lib, n):
    assert _scan(lib, state_dim=n) == 5


def test_scan_unknown_flag(lib):
    assert _scan(lib, flags=2) == 5


def test_scan_misaligned(lib):
    odd = ctypes.c_void_p(P[0].value + 1)
    assert _scan(lib, x=odd) == 4
    assert _scan(lib, dtype=ssscan.SS_F32, y=ctypes.c_void_p(P[5].value + 2)) == 4
    assert _scan(lib, A=ctypes.c_void_p(P[2].value + 2)) == 4


def test_scan_output_overlaps_input(lib):
    assert _scan(lib, y=ctypes.c_void_p(P[0].value + 64)) == 8
    assert _scan(lib, h_last=ctypes.c_void_p(P[1].value)) == 8
    assert _scan(lib, h_last=ctypes.c_void_p(P[5].value + 16)) == 8


def test_workspace_size_query(lib):
    # 2 x 16 channels at N = 16 -> 4 groups of 8 channels; the size grows with groups
    small = lib.ss_scan_workspace_bytes(2, 16, 16, 64)
    big = lib.ss_scan_workspace_bytes(2, 1600, 16, 64)
    assert 64 < small < big
    # with enough channel groups to fill the GPU (the chained schedule), independent of seq
    assert lib.ss_scan_workspace_bytes(2, 2400, 16, 1 << 20) == lib.ss_scan_workspace_bytes(2, 2400, 16, 64)
    # few groups and a long sequence: the two-level schedule's composites are included
    # (three floats per state element and segment)
    long_few = lib.ss_scan_workspace_bytes(1, 512, 16, 65536)
    assert long_few > lib.ss_scan_workspace_bytes(1, 512, 16, 64) + 3 * 4 * 512 * 16
    assert lib.ss_scan_workspace_bytes(2, 16, 5, 64) == 0
    assert lib.ss_scan_workspace_bytes(0, 16, 16, 64) == 0
    for n in (4, 8, 16):
        assert lib.ss_scan_workspace_bytes(3, 100, n, 10) > 64


def test_scan_workspace_checks(lib):
    need = lib.ss_scan_workspace_bytes(2, 16, 16, 64)
    ws = ctypes.c_void_p(P[8].value)
    assert _scan(lib, ws=ws, ws_bytes=need - 1) == 9
    assert _scan(lib, ws=ctypes.c_void_p(P[8].value + 8), ws_bytes=need) == 4
    assert _scan(lib, ws=ctypes.c_void_p(P[0].value + 32), ws_bytes=need) == 8
    assert _scan(lib, ws=ctypes.c_void_p(P[5].value), ws_bytes=need) == 8


def test_status_query_needs_output(lib):
    assert lib.ss_scan_status(None, None, None) == 1


@pytest.mark.parametrize("field", ["state", "x", "dt", "A", "B", "C", "y"])
def test_update_null_pointer(lib, field):
    assert _update(lib, **{field: None}) == 1


def test_update_bad_args(lib):
    assert _update(lib, batch=0) == 2
    assert _update(lib, dtype=2) == 3
    assert _update(lib, state_dim=6) == 5
    assert _update(lib, flags=4) == 5
    assert _update(lib, state=ctypes.c_void_p(P[0].value + 2)) == 4
    assert _update(lib, y=ctypes.c_void_p(P[0].value + 8)) == 8


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 8)
    with pytest.raises(ValueError):
        ssscan.ss_scan_fwd(x, x, torch.zeros(4, 4), torch.zeros(1, 4, 8), torch.zeros(1, 4, 8))
    with pytest.raises(ValueError):
        ssscan.ss_state_update(torch.zeros(1, 4, 4), x[:, :, 0], x[:, :, 0], torch.zeros(4, 4),
                               torch.zeros(1, 4), torch.zeros(1, 4))


def test_missing_library_is_an_error(tmp_path):
    saved = ssscan._lib
    try:
        ssscan._lib = None
        with pytest.raises(RuntimeError, match="not built"):
            ssscan.load_library(str(tmp_path / "nope.so"))
    finally:
        ssscan._lib = saved


def _scan_states(lib, h_all, **kw):
    a = dict(batch=2, channels=16, state_dim=16, seq=64, dtype=ssscan.SS_BF16, x=P[0], dt=P[1],
             A=P[2], B=P[3], C=P[4], D=None, z=None, dt_bias=None, reset=None, h0=None,
             flags=1, y=P[5], h_last=None, betas=None, ws=None, ws_bytes=0, stream=None)
    a.update(kw)
    return lib.ss_scan_fwd_states(a["batch"], a["channels"], a["state_dim"], a["seq"], a["dtype"],
                                  a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], a["z"], a["dt_bias"],
                                  a["reset"], a["h0"], a["flags"], a["y"], a["h_last"], h_all, a["betas"],
                                  a["ws"], a["ws_bytes"], a["stream"])


def test_scan_states_checks(lib):
    """ss_scan_fwd_states: at least one per-token output (states or step sizes), each
    4-byte aligned and overlapping nothing, the other arguments checked as for
    ss_scan_fwd."""
    assert ssscan.STATUS[_scan_states(lib, None)] == "SS_ERR_NULL"
    assert ssscan.STATUS[_scan_states(lib, None, betas=ctypes.c_void_p(P[10].value + 2))] == "SS_ERR_ALIGN"
    assert ssscan.STATUS[_scan_states(lib, None, betas=ctypes.c_void_p(P[1].value + 64))] == "SS_ERR_ALIAS"
    assert ssscan.STATUS[_scan_states(lib, P[9], betas=ctypes.c_void_p(P[9].value + 4096))] == "SS_ERR_ALIAS"
    assert ssscan.STATUS[_scan_states(lib, None, betas=ctypes.c_void_p(P[5].value + 8))] == "SS_ERR_ALIAS"
    assert ssscan.STATUS[_scan_states(lib, None, betas=P[10], state_dim=5)] == "SS_ERR_UNSUPPORTED"
    assert ssscan.STATUS[_scan_states(lib, ctypes.c_void_p(P[9].value + 2))] == "SS_ERR_ALIGN"
    assert ssscan.STATUS[_scan_states(lib, ctypes.c_void_p(P[0].value + 64))] == "SS_ERR_ALIAS"
    assert ssscan.STATUS[_scan_states(lib, ctypes.c_void_p(P[5].value))] == "SS_ERR_ALIAS"
    assert ssscan.STATUS[_scan_states(lib, P[9], state_dim=5)] == "SS_ERR_UNSUPPORTED"
    assert ssscan.STATUS[_scan_states(lib, P[9], x=None)] == "SS_ERR_NULL"


def test_gated_scan_checks(lib):
    def call(**kw):
        a = dict(batch=2, seq=16, dk=64, dv=32, dtype=ssscan.SS_BF16, q=P[0], k=P[1], v=P[2], gamma=P[3],
                 h0=None, y=P[4], fs=P[5])
        a.update(kw)
        return ssscan.STATUS[lib.ss_gated_scan(a["batch"], a["seq"], a["dk"], a["dv"], a["dtype"], a["q"], a["k"],
                                               a["v"], a["gamma"], a["h0"], a["y"], a["fs"], None)]
    assert call(q=None) == "SS_ERR_NULL"
    assert call(fs=None) == "SS_ERR_NULL"
    assert call(seq=0) == "SS_ERR_SHAPE"
    assert call(dtype=9) == "SS_ERR_DTYPE"
    assert call(dk=129) == "SS_ERR_UNSUPPORTED"
    assert call(q=ctypes.c_void_p(P[0].value + 1)) == "SS_ERR_ALIGN"
    assert call(y=ctypes.c_void_p(P[1].value + 64)) == "SS_ERR_ALIAS"
    assert call(fs=ctypes.c_void_p(P[4].value)) == "SS_ERR_ALIAS"


def test_huge_shapes_are_refused_without_overflow(lib):
    """Products of sizes that overflow 64 bits are refused before any pointer is used."""
    assert _scan(lib, batch=1 << 60, channels=1, seq=64) == 2
    assert _scan(lib, batch=1 << 59, channels=2, seq=1) == 2
    st = lib.ss_gated_scan(1 << 58, 1, 128, 64, ssscan.SS_BF16, P[0], P[1], P[2], P[3], None, P[4], P[5], None)
    assert ssscan.STATUS[st] == "SS_ERR_SHAPE"
    st = lib.ss_gated_scan(1, 1 << 60, 64, 64, ssscan.SS_BF16, P[0], P[1], P[2], P[3], None, P[4], P[5], None)
    assert ssscan.STATUS[st] == "SS_ERR_SHAPE"


def test_scan_conv_checks(lib):
    def call(**kw):
        a = dict(u=P[0], w=P[6], cb=None, K=4, cs=None, cso=None, xo=None, dt=P[1], A=P[2], B=P[3], C=P[4], y=P[5])
        a.update(kw)
        return ssscan.STATUS[lib.ss_scan_fwd_conv(2, 16, 16, 64, ssscan.SS_BF16, a["u"], a["w"], a["cb"], a["K"],
                                                  a["cs"], a["cso"], a["xo"], a["dt"], a["A"], a["B"], a["C"], None,
                                                  None, None, None, None, 1, a["y"], None, None, 0, None)]
    assert call(w=None) == "SS_ERR_NULL"
    assert call(K=5) == "SS_ERR_UNSUPPORTED"
    assert call(K=0) == "SS_ERR_UNSUPPORTED"
    assert call(u=None) == "SS_ERR_NULL"
    assert call(xo=ctypes.c_void_p(P[0].value + 64)) == "SS_ERR_ALIAS"      # x_out over u
    assert call(cs=P[7], cso=ctypes.c_void_p(P[7].value + 4)) == "SS_ERR_ALIAS"  # state out over state in
    assert call(xo=P[5]) == "SS_ERR_ALIAS"                                  # x_out over y
    assert call(cso=ctypes.c_void_p(P[6].value + 2)) == "SS_ERR_ALIGN"


def test_decode_conv_checks(lib):
    def call(**kw):
        a = dict(state=P[0], cs=P[7], w=P[6], K=4, u=P[1], dt=P[2], A=P[3], B=P[4], C=P[5], y=P[8])
        a.update(kw)
        return ssscan.STATUS[lib.ss_state_update_conv(4, 32, 16, ssscan.SS_F32, a["state"], a["cs"], a["w"], None,
                                                      a["K"], a["u"], a["dt"], a["A"], a["B"], a["C"], None, None,
                                                      None, 1, a["y"], None)]
    assert call(w=None) == "SS_ERR_NULL"
    assert call(K=5) == "SS_ERR_UNSUPPORTED"
    assert call(cs=None) == "SS_ERR_NULL"
    assert call(cs=ctypes.c_void_p(P[0].value + 64)) == "SS_ERR_ALIAS"   # conv state over the state
    assert call(cs=ctypes.c_void_p(P[7].value + 2)) == "SS_ERR_ALIGN"


def test_segment_decay_checks(lib):
    E = ssscan.STATUS

    def call(**kw):
        a = dict(batch=1, channels=16, state_dim=16, seq=64, dtype=ssscan.SS_BF16, dt=P[0], A=P[1],
                 dt_bias=None, reset=None, flags=1, decay=P[2])
        a.update(kw)
        return E[lib.ss_segment_decay(a["batch"], a["channels"], a["state_dim"], a["seq"], a["dtype"], a["dt"],
                                      a["A"], a["dt_bias"], a["reset"], a["flags"], a["decay"], None)]

    assert call(dt=None) == "SS_ERR_NULL"
    assert call(decay=None) == "SS_ERR_NULL"
    assert call(seq=0) == "SS_ERR_SHAPE"
    assert call(dtype=7) == "SS_ERR_DTYPE"
    assert call(state_dim=5) == "SS_ERR_UNSUPPORTED"
    assert call(flags=2) == "SS_ERR_UNSUPPORTED"
    assert call(A=ctypes.c_void_p(P[1].value + 2)) == "SS_ERR_ALIGN"
    assert call(decay=ctypes.c_void_p(P[0].value + 64)) == "SS_ERR_ALIAS"   # inside dt
    assert call(batch=1 << 40, channels=1 << 40) == "SS_ERR_SHAPE"


def test_join_segments_checks(lib):
    E = ssscan.STATUS

    def call(segments=4, count=256, comp=P[0], rank=1, carry=P[1], final=P[2]):
        return E[lib.ss_join_segments(segments, count, comp, rank, carry, final, None)]

    assert call(comp=None) == "SS_ERR_NULL"
    assert call(carry=None, final=None) == "SS_ERR_NULL"
    assert call(segments=0) == "SS_ERR_SHAPE"
    assert call(count=0) == "SS_ERR_SHAPE"
    assert call(rank=0) == "SS_ERR_SHAPE"          # segment 0's entering state is h0 itself
    assert call(rank=4) == "SS_ERR_SHAPE"
    assert call(carry=ctypes.c_void_p(P[1].value + 1)) == "SS_ERR_ALIGN"
    assert call(carry=ctypes.c_void_p(P[0].value + 1024)) == "SS_ERR_ALIAS"  # inside the composites
    assert call(final=ctypes.c_void_p(P[1].value + 512)) == "SS_ERR_ALIAS"   # overlaps carry
    assert call(count=1 << 62) == "SS_ERR_SHAPE"


def test_mufu_probe_checks(lib):
    ops = ctypes.c_int64(0)
    P = [ctypes.c_void_p(0x7f0000000000 + i * 0x100000000) for i in range(2)]
    assert lib.ss_debug_mufu_probe(0, 16, 4, None, P[1], ctypes.byref(ops), None) == 1
    assert lib.ss_debug_mufu_probe(2, 16, 4, P[0], P[1], ctypes.byref(ops), None) == 5
    assert lib.ss_debug_mufu_probe(0, 0, 4, P[0], P[1], ctypes.byref(ops), None) == 2
    assert lib.ss_debug_mufu_probe(1, 16, 0, P[0], P[1], ctypes.byref(ops), None) == 2
