"""The C ABI without a GPU: the library loads, exports every entry point that
include/dsa.h declares, sizes workspaces, and rejects bad arguments before
touching the device."""
import ctypes
import os
import re

import pytest

from dynamic_block_sparse_pool_b200 import _lib
from dynamic_block_sparse_pool_b200.build import LIB, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return _lib.lib()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_four_pipeline_calls():
    syms = declared_symbols()
    for name in ("dsa_pool_score", "dsa_select_topp", "dsa_attn_fwd", "dsa_block_mass"):
        assert name in syms


def declared_prototypes():
    """name -> (return type, [parameter types]) for every prototype in dsa.h."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = {}
    for ret, name, params in re.findall(
            r"^\s*((?:const\s+)?[a-z_0-9]+\s*\**)\s*(dsa_[a-z0-9_]+)\s*\(([^)]*)\)\s*;",
            text, flags=re.M):
        params = " ".join(params.split())
        types = [] if params in ("", "void") else [
            re.sub(r"\s*\b[A-Za-z_][A-Za-z_0-9]*$", "", p.strip()) for p in params.split(",")]
        protos[name] = (" ".join(ret.split()), types)
    return protos


def _ctype_of(c):
    """The ctypes type the binding must use for a C parameter or return type."""
    c = " ".join(c.replace("*", " * ").split())
    if c.endswith("*"):
        return ctypes.c_char_p if c == "const char *" else ctypes.c_void_p
    return {"int": ctypes.c_int, "float": ctypes.c_float, "size_t": ctypes.c_size_t,
            "unsigned long long": ctypes.c_ulonglong,
            "dsa_dtype": ctypes.c_int, "dsa_status": ctypes.c_int}[c]


def test_binding_signatures_match_the_header():
    # every prototype's argument count and types, and its return type, as the
    # ctypes binding declares them (a mismatch would pass a wrong value to
    # the library without any error)
    protos = declared_prototypes()
    assert set(protos) == set(_lib.SIGNATURES), set(protos) ^ set(_lib.SIGNATURES)
    for name, (ret, params) in protos.items():
        res, args = _lib.SIGNATURES[name]
        assert res == _ctype_of(ret), (name, ret, res)
        assert [_ctype_of(t) for t in params] == list(args), (name, params, args)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    # the binding declares a signature for each of them
    assert set(declared_symbols()) <= set(_lib.SIGNATURES)


def test_exports_via_nm(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (dsa_\w+)", out))
    assert set(declared_symbols()) <= exported


def test_version_and_workspace_sizes(lib):
    assert lib.dsa_version() == 101
    # pool: 2 * B*H*nB*D floats; select: B*H*nB*33 words
    assert lib.dsa_workspace_size(0, 1, 40, 75600, 128, 128) == 2 * 40 * 591 * 128 * 4
    assert lib.dsa_workspace_size(1, 1, 40, 75600, 128, 128) == 40 * 591 * 33 * 4
    assert lib.dsa_workspace_size(0, 1, 2, 256, 64, 64) == 2 * 2 * 4 * 64 * 4
    assert lib.dsa_workspace_size(0, 1, 1, 256, 96, 64) == 0      # bad D
    assert lib.dsa_workspace_size(7, 1, 1, 256, 64, 64) == 0       # bad op


FAKE = 0x10000  # never dereferenced: every call below fails validation first


@pytest.mark.parametrize("args,what", [
    (dict(q=None), "null q"),
    (dict(D=96), "D"),
    (dict(block=32), "block"),
    (dict(N=0), "N"),
    (dict(scale=0.0), "scale"),
    (dict(scale=float("inf")), "scale"),
    (dict(q=FAKE + 4), "aligned"),
    (dict(ws_bytes=16), "workspace"),
    (dict(cand_row_ptr=FAKE), "both"),
    (dict(N=1025 * 64, block=64), "nB"),
    (dict(dt=5), "dtype"),
])
def test_pool_score_rejects(lib, args, what):
    a = dict(q=FAKE, k=FAKE, dt=1, B=1, H=2, N=256, D=64, block=64, scale=0.125,
             cand_row_ptr=None, cand_col=None, probs=FAKE, ws=FAKE, ws_bytes=1 << 20,
             stream=None)
    a.update(args)
    st = lib.dsa_pool_score(a["q"], a["k"], a["dt"], a["B"], a["H"], a["N"], a["D"],
                            a["block"], a["scale"], a["cand_row_ptr"], a["cand_col"],
                            a["probs"], a["ws"], a["ws_bytes"], a["stream"])
    assert st == _lib.DSA_ERR_INVALID_ARG
    assert what.lower() in lib.dsa_last_error().decode().lower()


@pytest.mark.parametrize("p", [0.0, -0.5, 1.5, float("nan")])
def test_select_rejects_p(lib, p):
    st = lib.dsa_select_topp(FAKE, 4, 16, p, None, None, FAKE, FAKE, FAKE, 1 << 20, None)
    assert st == _lib.DSA_ERR_INVALID_ARG
    assert "p must be" in lib.dsa_last_error().decode()


def test_select_rejects_sizes(lib):
    assert lib.dsa_select_topp(FAKE, 4, 1025, 0.5, None, None, FAKE, FAKE, FAKE, 1 << 20,
                               None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_select_topp(FAKE, 0, 16, 0.5, None, None, FAKE, FAKE, FAKE, 1 << 20,
                               None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_select_topp(FAKE, 4, 16, 0.5, None, None, FAKE, FAKE, FAKE, 8,
                               None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_select_topp(FAKE, 4, 16, 0.5, FAKE, None, FAKE, FAKE, FAKE, 1 << 20,
                               None) == _lib.DSA_ERR_INVALID_ARG


def test_attn_and_mass_reject(lib):
    ok = (FAKE, FAKE, FAKE, 1, 1, 2, 256, 64, 128, 0.125, FAKE, FAKE, FAKE, None, None, None)
    bad_out = ok[:12] + (FAKE + 8,) + ok[13:]
    assert lib.dsa_attn_fwd(*bad_out) == _lib.DSA_ERR_INVALID_ARG
    # the ordered entry: the order after col_idx, the rest as above
    ordered = ok[:12] + (FAKE,) + ok[12:]
    assert lib.dsa_attn_fwd_ordered(*(ordered[:12] + (FAKE + 2,) + ordered[13:])) == \
        _lib.DSA_ERR_INVALID_ARG                                                      # order
    assert "aligned" in lib.dsa_last_error().decode()
    assert lib.dsa_attn_fwd_ordered(*(ordered[:13] + (FAKE + 8,) + ordered[14:])) == \
        _lib.DSA_ERR_INVALID_ARG                                                      # out
    assert lib.dsa_attn_fwd_ordered(*(ordered[:7] + (80,) + ordered[8:])) == _lib.DSA_ERR_INVALID_ARG
    no_v = ok[:2] + (None,) + ok[3:]
    assert lib.dsa_attn_fwd(*no_v) == _lib.DSA_ERR_INVALID_ARG
    bad_d = ok[:7] + (80,) + ok[8:]
    assert lib.dsa_attn_fwd(*bad_d) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_block_mass(None, FAKE, 1, 2, 256, 128, FAKE, FAKE, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_block_mass(FAKE, FAKE, 1, 2, 256, 100, FAKE, FAKE, None) == _lib.DSA_ERR_INVALID_ARG


def test_row_order_rejects(lib):
    assert lib.dsa_row_order(None, 1, 2, 16, FAKE, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_row_order(FAKE, 1, 2, 16, None, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_row_order(FAKE, 0, 2, 16, FAKE, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_row_order(FAKE, 1, 2, 1025, FAKE, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_row_order(FAKE, 1, 2, 0, FAKE, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_row_order(FAKE + 2, 1, 2, 16, FAKE, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_row_order(FAKE, 1 << 16, 1 << 10, 1024, FAKE, None) == _lib.DSA_ERR_INVALID_ARG


def test_mass_to_probs_rejects(lib):
    assert lib.dsa_mass_to_probs(None, FAKE, FAKE, 4, 4, FAKE, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_mass_to_probs(FAKE, FAKE, FAKE, 0, 4, FAKE, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_mass_to_probs(FAKE, FAKE, FAKE, 4, 0, FAKE, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_mass_to_probs(FAKE, FAKE, FAKE, 4, 2000, FAKE, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_mass_to_probs(FAKE, FAKE, FAKE + 2, 4, 4, FAKE, None) == _lib.DSA_ERR_INVALID_ARG


def test_pool_score_hier_rejects(lib):
    ok = (FAKE, FAKE, 1, 1, 2, 256, 64, 128, 2, 0.125, FAKE, FAKE, 1 << 30, None)
    assert lib.dsa_pool_score_hier(None, *ok[1:]) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_pool_score_hier(*ok[:8], 3, *ok[9:]) == _lib.DSA_ERR_INVALID_ARG       # sub
    assert lib.dsa_pool_score_hier(*ok[:12], 16, None) == _lib.DSA_ERR_INVALID_ARG        # workspace
    big = ok[:5] + (1 << 20,) + ok[6:8] + (4,) + ok[9:]                                  # > 2048 sub-blocks
    assert lib.dsa_pool_score_hier(*big) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_workspace_size(_lib.DSA_OP_POOL_SCORE_HIER2, 1, 2, 256, 64, 128) == \
        4 * (2 * 2 * 4 * 64 + 2 * 4 * 4)


@pytest.mark.parametrize("limit", [0, 999, 10 ** 9 + 1, 2 ** 63])
def test_selftest_wait_timeout_rejects_limits(lib, limit):
    assert lib.dsa_selftest_wait_timeout(limit, None) == _lib.DSA_ERR_INVALID_ARG
    assert "limit_ns" in lib.dsa_last_error().decode()


def test_python_wrapper_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        _lib.lib()


def test_host_pipeline_workspace_size_needs_no_gpu(lib):
    L = lib
    # bf16, 2 x 40 heads x 75,600 tokens x 128, block 128, 5 heads per chunk
    a = L.dsa_host_pipeline_workspace_size(1, 2, 40, 75600, 128, 128, 5)
    b = L.dsa_host_pipeline_workspace_size(1, 2, 40, 75600, 128, 128, 10)
    assert 0 < a < b
    # two slots of 5 heads hold at least Q, K, V and O in bf16
    assert a >= 2 * 4 * 5 * 75600 * 128 * 2
    # fp32 needs more than bf16; chunk <= 0 picks B*H / 8 heads
    assert L.dsa_host_pipeline_workspace_size(0, 2, 40, 75600, 128, 128, 5) > a
    assert L.dsa_host_pipeline_workspace_size(1, 2, 40, 75600, 128, 128, 0) == \
        L.dsa_host_pipeline_workspace_size(1, 2, 40, 75600, 128, 128, 10)
    # invalid dtype or head dimension
    assert L.dsa_host_pipeline_workspace_size(7, 1, 1, 1000, 128, 128, 1) == 0
    assert L.dsa_host_pipeline_workspace_size(1, 1, 1, 1000, 96, 128, 1) == 0
