"""The C-ABI library loads and exports every entry point include/ace.h
declares; host-side argument validation rejects bad calls before anything is
launched.  No GPU needed."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ace.h")


@pytest.fixture(scope="module")
def ace():
    from token_dynamic_expert_b200 import build
    build.build()
    from token_dynamic_expert_b200 import ace as mod
    return mod


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(ace_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ["ace_workspace_size", "ace_moe_forward", "ace_moe_scores", "ace_build_tables",
              "ace_tables_workspace_size", "ace_read_status", "ace_status_str", "ace_version"]:
        assert n in names


def test_library_exports_every_declared_symbol(ace):
    lib = ctypes.CDLL(ace.LIB_PATH)
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert missing == []


def test_library_exports_nothing_else(ace):
    out = os.popen("nm -D --defined-only %s" % ace.LIB_PATH).read()
    exported = sorted(set(re.findall(r" T (ace_\w+)", out)))
    assert exported == _declared_functions()


def test_status_strings(ace):
    assert ace.ace_status_str(ace.ACE_OK) == "ACE_OK"
    assert ace.ace_status_str(ace.ACE_ERR_TIMEOUT) == "ACE_ERR_TIMEOUT"
    assert ace.ace_status_str(99) == "ACE_UNKNOWN_STATUS"
    assert re.match(r"\d+\.\d+\.\d+", ace.ace_version())


def _fake_layer(ace, **kw):
    # host addresses that are never dereferenced: validation fails first
    p = 0x10000
    args = dict(d=256, E=8, m=128, k=2, dtype=ace.ACE_BF16, gamma=p, w_router=p, router_bias=None,
                w_gate=p, w_up=p, w_down=p, amax=p)
    args.update(kw)
    return ace.ace_layer(**args)


def _fwd(ace, layer, T=4, u=0x20000, y=0x40000, ws=0x80000, ws_bytes=1 << 30, opts=None):
    opts = opts or ace.ace_fwd_opts(tau=0.1, renorm_topk=1, fusion=0, eps_rms=1e-6)
    return ace.lib().ace_moe_forward(ctypes.byref(layer), u, T, ctypes.byref(opts), y, ws,
                                     ws_bytes, None, None)


@pytest.mark.parametrize("bad", [dict(d=0), dict(E=-1), dict(k=0), dict(k=9), dict(k=17, E=32),
                                 dict(dtype=7), dict(gamma=None), dict(w_router=None),
                                 dict(w_gate=None), dict(w_down=None), dict(w_up=0x10008),
                                 dict(gamma=0x10004)])
def test_forward_rejects_bad_layers(ace, bad):
    assert _fwd(ace, _fake_layer(ace, **bad)) == ace.ACE_ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [dict(d=100), dict(m=96), dict(E=1024), dict(d=320)])
def test_forward_reports_unsupported_shapes(ace, bad):
    assert _fwd(ace, _fake_layer(ace, **bad)) == ace.ACE_ERR_UNSUPPORTED


def test_forward_rejects_bad_calls(ace):
    L = _fake_layer(ace)
    assert _fwd(ace, L, T=-1) == ace.ACE_ERR_INVALID_ARG
    assert _fwd(ace, L, u=None) == ace.ACE_ERR_INVALID_ARG
    assert _fwd(ace, L, y=None) == ace.ACE_ERR_INVALID_ARG
    assert _fwd(ace, L, u=0x20008) == ace.ACE_ERR_INVALID_ARG          # misaligned input
    assert _fwd(ace, L, u=0x20000, y=0x20000 + 512) == ace.ACE_ERR_INVALID_ARG  # overlap
    assert _fwd(ace, L, ws=None) == ace.ACE_ERR_WORKSPACE
    assert _fwd(ace, L, ws=0x80010) == ace.ACE_ERR_WORKSPACE           # not 256-B aligned
    assert _fwd(ace, L, ws_bytes=1024) == ace.ACE_ERR_WORKSPACE        # too small
    for f in (-1, 5):  # no such fusion rule
        bad = ace.ace_fwd_opts(tau=0.1, renorm_topk=1, fusion=f, eps_rms=1e-6)
        assert _fwd(ace, L, opts=bad) == ace.ACE_ERR_INVALID_ARG
    assert ace.lib().ace_moe_forward(ctypes.byref(L), 0x20000, 4, None, 0x40000, 0x80000,
                                     1 << 30, None, None) == ace.ACE_ERR_INVALID_ARG


def test_workspace_size_is_monotone_and_rejects_bad_layers(ace):
    L = _fake_layer(ace)
    sizes = [ace.ace_workspace_size(L, T) for T in (1, 32, 33, 1000, 4096)]
    assert all(s > 0 for s in sizes)
    assert sizes == sorted(sizes)
    assert ace.ace_workspace_size(_fake_layer(ace, d=0), 16) == 0
    assert ace.lib().ace_workspace_size(None, 16) == 0
    # the worst case holds every slot: gathered rows, intermediates and
    # outputs, all in the storage type (bf16 here)
    big = _fake_layer(ace, d=2048, E=128, m=768, k=8)
    assert ace.ace_workspace_size(big, 1024) >= 1024 * 8 * (2048 * 2 + 768 * 2 + 2048 * 2)


def test_scores_reject_bad_calls(ace):
    L = _fake_layer(ace)
    opts = ace.ace_fwd_opts(tau=0.0, renorm_topk=1, fusion=0, eps_rms=1e-6)
    f = ace.lib().ace_moe_scores
    assert f(ctypes.byref(L), 0x20000, 4, ctypes.byref(opts), None, None, 0x80000, 1 << 30,
             None) == ace.ACE_ERR_INVALID_ARG
    assert f(None, 0x20000, 4, ctypes.byref(opts), 0x30000, None, 0x80000, 1 << 30,
             None) == ace.ACE_ERR_INVALID_ARG


def test_read_status_rejects_missing_workspace(ace):
    assert ace.lib().ace_read_status(None, 0, None, None) == ace.ACE_ERR_WORKSPACE


def test_tau_quantile_rejects_bad_calls(ace):
    f = ace.lib().ace_tau_quantile
    n = ace.ace_tau_workspace_size()
    assert n >= 256 + 4 * 256 * 4
    ws, tau, sc = 0x100000, 0x200000, 0x300000  # never dereferenced: rejected first
    assert f(sc, 4, 0, 1, tau, ws, n, None) == ace.ACE_ERR_INVALID_ARG        # k < 1
    assert f(sc, 4, 17, 1, tau, ws, n, None) == ace.ACE_ERR_INVALID_ARG       # k > 16
    assert f(sc, -1, 8, 1, tau, ws, n, None) == ace.ACE_ERR_INVALID_ARG       # n_tok < 0
    assert f(None, 4, 8, 1, tau, ws, n, None) == ace.ACE_ERR_INVALID_ARG      # no scores
    assert f(sc, 4, 8, 1, None, ws, n, None) == ace.ACE_ERR_INVALID_ARG       # no output
    assert f(sc, 4, 8, 1, tau + 2, ws, n, None) == ace.ACE_ERR_INVALID_ARG    # misaligned
    assert f(sc, 4, 8, 1, tau, ws, n - 1, None) == ace.ACE_ERR_WORKSPACE      # short
    assert f(sc, 4, 8, 1, tau, ws + 16, n, None) == ace.ACE_ERR_WORKSPACE     # misaligned
    assert f(sc, 4, 8, 1, tau, None, n, None) == ace.ACE_ERR_WORKSPACE


@pytest.mark.parametrize("fusion,tables,ok", [
    (1, {}, False), (1, dict(a_gsp=0x10000), False), (2, dict(a_rcr=0x10000), False),
    (3, dict(a_rcr=0x10000), False), (4, dict(a_gsp=0x10000), False),
    (3, dict(a_gsp=0x10002), False),                     # misaligned table
    (1, dict(a_gsp=0x10000, a_rcr=0x10000), True), (3, dict(a_gsp=0x10000), True),
    (4, dict(a_rcr=0x10000), True), (0, {}, True)])
def test_fusion_rules_need_their_tables(ace, fusion, tables, ok):
    """Each fusion rule reads the view tables it fuses; a missing one is an
    argument error found before any launch.  Valid combinations get past
    validation and stop at the (deliberately short) workspace."""
    L = _fake_layer(ace, **tables)
    opts = ace.ace_fwd_opts(tau=0.1, renorm_topk=1, fusion=fusion, eps_rms=1e-6)
    want = ace.ACE_ERR_WORKSPACE if ok else ace.ACE_ERR_INVALID_ARG
    assert _fwd(ace, L, opts=opts, ws_bytes=1024) == want


def test_stack_rejects_bad_calls(ace):
    Ls = (ace.ace_layer * 3)(_fake_layer(ace), _fake_layer(ace), _fake_layer(ace))
    opts = (ace.ace_fwd_opts * 3)(*[ace.ace_fwd_opts(tau=0.1, renorm_topk=1, fusion=0,
                                                     eps_rms=1e-6)] * 3)
    f = ace.lib().ace_moe_stack_forward
    ok = dict(u=0x20000, y=0x40000, ws=0x80000, nb=1 << 30)
    assert ace.lib().ace_stack_workspace_size(Ls, 3, 8) >= 2 * 8 * 256 * 2
    assert ace.lib().ace_stack_workspace_size(Ls, 0, 8) == 0
    assert f(Ls, 0, ok["u"], 4, opts, ok["y"], ok["ws"], ok["nb"], None) == ace.ACE_ERR_INVALID_ARG
    assert f(Ls, 3, ok["u"], 4, None, ok["y"], ok["ws"], ok["nb"], None) == ace.ACE_ERR_INVALID_ARG
    assert f(Ls, 3, ok["u"], 4, opts, ok["u"] + 64, ok["ws"], ok["nb"], None) == \
        ace.ACE_ERR_INVALID_ARG                                        # u and y overlap
    assert f(Ls, 3, ok["u"], 4, opts, ok["y"], ok["ws"], 1024, None) == ace.ACE_ERR_WORKSPACE
    assert f(Ls, 3, ok["u"], 4, opts, ok["y"], ok["ws"] + 16, ok["nb"], None) == \
        ace.ACE_ERR_WORKSPACE
    bad = (ace.ace_layer * 3)(_fake_layer(ace), _fake_layer(ace, d=512), _fake_layer(ace))
    assert f(bad, 3, ok["u"], 4, opts, ok["y"], ok["ws"], ok["nb"], None) == \
        ace.ACE_ERR_INVALID_ARG                                        # layers of different d
    opts[2].fusion = 1                                                 # min without view tables
    assert f(Ls, 3, ok["u"], 4, opts, ok["y"], ok["ws"], ok["nb"], None) == \
        ace.ACE_ERR_INVALID_ARG


def test_noalloc_rejects_bad_calls_before_any_device_call(ace):
    """ace_moe_decode_noalloc applies ace_moe_forward's layer checks and shape
    rule, and its own token range, on the host."""
    f = ace.lib().ace_moe_decode_noalloc
    opts = ace.ace_fwd_opts(tau=0.1, renorm_topk=1, fusion=0, eps_rms=1e-6)
    L = _fake_layer(ace)
    u, y = 0x20000, 0x40000
    assert f(ctypes.byref(L), u, 9, ctypes.byref(opts), y, None) == ace.ACE_ERR_INVALID_ARG
    assert f(ctypes.byref(L), u, 0, ctypes.byref(opts), y, None) == ace.ACE_ERR_INVALID_ARG
    assert f(ctypes.byref(L), u, 4, None, y, None) == ace.ACE_ERR_INVALID_ARG
    assert f(ctypes.byref(L), u, 4, ctypes.byref(opts), u + 64, None) == ace.ACE_ERR_INVALID_ARG
    assert f(ctypes.byref(L), u + 8, 4, ctypes.byref(opts), y, None) == ace.ACE_ERR_INVALID_ARG
    for bad in (dict(d=192), dict(m=192), dict(d=100), dict(E=1024)):
        assert f(ctypes.byref(_fake_layer(ace, **bad)), u, 4, ctypes.byref(opts), y,
                 None) == ace.ACE_ERR_UNSUPPORTED, bad
    assert f(ctypes.byref(_fake_layer(ace, dtype=ace.ACE_F32)), u, 4, ctypes.byref(opts), y,
             None) == ace.ACE_ERR_UNSUPPORTED
    assert f(ctypes.byref(_fake_layer(ace, k=0)), u, 4, ctypes.byref(opts), y,
             None) == ace.ACE_ERR_INVALID_ARG


def test_peer_wait_limit_setting(ace):
    """Process-wide limit of the cross-CTA waits: 2 s by default, 0 restores
    the default, the previous value is returned."""
    assert ace.ace_set_peer_wait_limit_ns(0) == 2_000_000_000
    assert ace.ace_set_peer_wait_limit_ns(5000) == 2_000_000_000
    assert ace.ace_set_peer_wait_limit_ns(0) == 5000
    assert ace.ace_set_peer_wait_limit_ns(0) == 2_000_000_000
