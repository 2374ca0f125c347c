"""The C-ABI library loads on a machine without a GPU, exports every entry
point that include/mtpv.h declares, and rejects bad arguments on the host
before any launch (no compute call is made here)."""
import ctypes
import os
import re

import pytest

import verify_step_lm_b200 as mtpv
from verify_step_lm_b200 import build as mtpv_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mtpv.h")

INVALID, WORKSPACE = 1, 3


@pytest.fixture(scope="module")
def lib():
    mtpv_build.build()
    return mtpv.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mtpv_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("mtpv_lm_head_smallm", "mtpv_verify", "mtpv_sample", "mtpv_verify_step",
                     "mtpv_verify_step_host", "mtpv_verify_workspace_bytes", "mtpv_status_string",
                     "mtpv_version"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_only_abi_symbols_are_exported(lib):
    # hidden visibility: nothing but the mtpv_ entry points in the dynamic table
    out = os.popen(f"nm -D --defined-only {mtpv.LIB_PATH}").read().split("\n")
    syms = {l.split()[-1] for l in out if l.strip() and l.split()[1] in ("T", "t")}
    extra = {s for s in syms if not s.startswith("mtpv_")}
    assert not extra, sorted(extra)[:10]


def test_version_and_status_strings(lib):
    assert mtpv.version() >= 100
    assert mtpv.status_string(0) == "ok"
    assert "workspace" in mtpv.status_string(3)
    assert mtpv.status_string(99) == "unknown status"


def test_workspace_queries(lib):
    assert mtpv.lm_head_workspace_bytes(4, 5120, 151936, mtpv.W_BF16) == 0
    w = mtpv.verify_workspace_bytes(1, 3, 151936)
    assert w > 0 and w % 256 == 0
    assert mtpv.verify_workspace_bytes(8, 3, 248320) > w
    assert mtpv.verify_workspace_bytes(0, 3, 100) == 0          # B < 1
    assert mtpv.verify_workspace_bytes(1, 17, 100) == 0         # K > 16
    assert mtpv.verify_workspace_bytes(1, 3, (1 << 24) + 1) == 0
    s = mtpv.verify_step_workspace_bytes(1, 3, 151936, 5120)
    # the step keeps both logit blocks: (4 + 3) rows x V fp32
    assert s >= 7 * 151936 * 4
    assert mtpv.verify_step_workspace_bytes(1, 3, 151936, 5000) == 0  # h % 64 != 0
    assert mtpv.verify_step_workspace_bytes(16, 3, 1000, 512) > 0     # 64 target rows: allowed
    assert mtpv.verify_step_workspace_bytes(17, 3, 1000, 512) == 0    # 68 > 64 target rows
    assert mtpv.verify_step_host_workspace_bytes(1, 3, 151936, 5120) > s
    assert mtpv.sample_workspace_bytes(3, 100) > 0


def _p(v):
    return ctypes.c_void_p(v)


def test_lm_head_pair_argument_checks(lib):
    f = lib.mtpv_lm_head_pair
    a = 1 << 20  # a fake, aligned device address: never dereferenced on these paths
    P = _p(a)
    ok = (P, 4, P, P, P, 3, P, P, P, 5120, 1000, None, 0, None)
    bad = [
        (None,) + ok[1:],                              # xt missing
        ok[:8] + (None,) + ok[9:],                     # yd missing
        ok[:1] + (0,) + ok[2:],                        # Mt = 0
        ok[:5] + (65,) + ok[6:],                       # Md > 64
        ok[:9] + (5000,) + ok[10:],                    # Kd % 64
        ok[:10] + (0,) + ok[11:],                      # N = 0
        ok[:2] + (_p(a + 8),) + ok[3:],                # w misaligned
        ok[:7] + (_p(a + 1),) + ok[8:],                # scales misaligned
    ]
    for args in bad:
        assert f(*args) == INVALID
    assert f(*ok) == 3                                           # no workspace: MTPV_ERR_WORKSPACE
    assert f(*(ok[:11] + (P, 255, None))) == 3                   # workspace too small
    assert lib.mtpv_lm_head_pair_workspace_bytes(4, 3, 5120, 151936) == 256
    assert lib.mtpv_lm_head_pair_workspace_bytes(4, 3, 5000, 151936) == 0


def test_draft_loop_argument_checks(lib):
    f = lib.mtpv_draft_loop
    a = 1 << 20  # a fake, aligned device address: never dereferenced on these paths
    P = _p(a)
    need = lib.mtpv_draft_loop_workspace_bytes(1, 3, 151936, 5120)
    assert need > 0
    assert lib.mtpv_draft_loop_workspace_bytes(65, 3, 1000, 512) == 0   # B > 64
    assert lib.mtpv_draft_loop_workspace_bytes(1, 17, 1000, 512) == 0   # K > 16
    assert lib.mtpv_draft_loop_workspace_bytes(1, 3, 1000, 500) == 0    # h % 64
    ok = (P, P, P, P, 1, 3, 151936, 5120, 0.6, 0.95, P, None, P, need, None)
    bad = [
        (None,) + ok[1:],                          # no weights
        ok[:4] + (0,) + ok[5:],                    # B = 0
        ok[:8] + (-1.0,) + ok[9:],                 # T < 0
        ok[:9] + (0.0,) + ok[10:],                 # top_p = 0
        ok[:10] + (None,) + ok[11:],               # no output
        ok[:2] + (_p(a + 8),) + ok[3:],            # h_draft misaligned
    ]
    for args in bad:
        assert f(*args) == INVALID
    assert f(*(ok[:12] + (None, need, None))) == WORKSPACE
    assert f(*(ok[:13] + (need - 1, None))) == WORKSPACE


def test_lm_head_argument_checks(lib):
    f = lib.mtpv_lm_head_smallm
    ok = 1 << 20  # a fake, aligned device address: never dereferenced on these paths
    assert f(None, 4, 512, 100, _p(ok), None, 0, _p(ok), None, 0, None) == INVALID
    assert f(_p(ok), 0, 512, 100, _p(ok), None, 0, _p(ok), None, 0, None) == INVALID      # M = 0
    assert f(_p(ok), 65, 512, 100, _p(ok), None, 0, _p(ok), None, 0, None) == INVALID     # M > 64
    assert f(_p(ok), 4, 500, 100, _p(ok), None, 0, _p(ok), None, 0, None) == INVALID      # Kd % 64
    assert f(_p(ok), 4, 512, 0, _p(ok), None, 0, _p(ok), None, 0, None) == INVALID        # N = 0
    assert f(_p(ok + 8), 4, 512, 100, _p(ok), None, 0, _p(ok), None, 0, None) == INVALID  # x align
    assert f(_p(ok), 4, 512, 100, _p(ok), None, 1, _p(ok), None, 0, None) == INVALID      # no scales
    assert f(_p(ok), 4, 512, 100, _p(ok), None, 7, _p(ok), None, 0, None) == INVALID      # bad fmt


def test_verify_argument_checks(lib):
    f = lib.mtpv_verify
    a = 1 << 20
    args = [_p(a), _p(a), _p(a), _p(a), _p(a), 1, 3, 1000, 0.6, 0.95, _p(a), _p(a), None]
    need = mtpv.verify_workspace_bytes(1, 3, 1000)
    # workspace missing / too small / misaligned
    assert f(*args, None, need, None) == WORKSPACE
    assert f(*args, _p(a), need - 1, None) == WORKSPACE
    assert f(*args, _p(a + 16), need, None) == WORKSPACE
    bad = list(args)
    bad[8] = -0.5           # temperature < 0
    assert f(*bad, _p(a), need, None) == INVALID
    bad = list(args)
    bad[8] = float("nan")
    assert f(*bad, _p(a), need, None) == INVALID
    bad = list(args)
    bad[9] = 0.0            # top_p must be > 0
    assert f(*bad, _p(a), need, None) == INVALID
    bad = list(args)
    bad[6] = 0              # K = 0
    assert f(*bad, _p(a), need, None) == INVALID
    bad = list(args)
    bad[0] = None
    assert f(*bad, _p(a), need, None) == INVALID
    bad = list(args)
    bad[0] = _p(a + 2)      # logits must be 4-byte aligned
    assert f(*bad, _p(a), need, None) == INVALID


def test_sample_and_step_argument_checks(lib):
    a = 1 << 20
    assert lib.mtpv_sample(None, 1, 10, 1.0, 1.0, _p(a), _p(a), None, _p(a), 4096, None) == INVALID
    assert lib.mtpv_sample(_p(a), 0, 10, 1.0, 1.0, _p(a), _p(a), None, _p(a), 4096, None) == INVALID
    assert lib.mtpv_sample(_p(a), 1, 10, 1.0, 1.0, _p(a), _p(a), None, None, 0, None) == WORKSPACE
    st = lib.mtpv_verify_step(_p(a), _p(a), _p(a), _p(a), _p(a), _p(a), _p(a), _p(a),
                              1, 3, 1000, 5000, 0.6, 0.95, _p(a), _p(a), None, None, None,
                              _p(a), 1 << 30, None)
    assert st == INVALID  # h not a multiple of 64
    st = lib.mtpv_verify_step_host(_p(a), _p(a), _p(a), None, _p(a), _p(a), _p(a), _p(a),
                                   1, 3, 1000, 512, 0.6, 0.95, _p(a), _p(a), None,
                                   _p(a), 1 << 30, None)
    assert st == INVALID  # missing host input
