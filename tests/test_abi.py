"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/srm_moe.h, include/srm_dsa.h and include/srm_ep.h
declare, sizes its workspaces and rejects invalid arguments before any launch."""
import ctypes
import os
import re

import pytest

from sigmoid_routed_mixture_b200 import build as B
from sigmoid_routed_mixture_b200 import dsa
from sigmoid_routed_mixture_b200 import ep
from sigmoid_routed_mixture_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    B.build()
    return moe.lib()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b((?:moe|dsa)_[a-z0-9_]+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(L):
    declared = declared_functions()
    assert {"moe_route", "moe_permute", "moe_forward"} <= declared
    for name in declared:
        assert hasattr(L, name), name
    assert set(moe.SYMBOLS) <= declared
    assert set(dsa.SYMBOLS) <= declared and "dsa_select" in declared
    assert {"moe_ep_plan", "moe_ep_dispatch", "moe_ep_return", "moe_ep_shared", "moe_workspace_offset",
            "moe_pack_router", "moe_route_packed"} <= declared
    ep.lib()  # the expert-parallel entry points resolve and take their types


def test_status_strings(L):
    for code in range(9):
        s = L.moe_status_string(code)
        assert isinstance(s, bytes) and len(s) > 0
    assert L.moe_status_string(0) == b"ok"


def cfg(**kw):
    base = dict(T=64, H=256, I=128, E=16, K=4, routed_scale=2.5, has_shared=True)
    base.update(kw)
    return moe.Config(**base)


def test_workspace_size_grows_with_tokens(L):
    small = moe.workspace_bytes(cfg(T=64))
    big = moe.workspace_bytes(cfg(T=4096))
    assert big > small > 0
    # h [rows, I] and Y [rows, H] in bf16 dominate: rows = T*(K+1)
    rows = 4096 * 5
    assert big >= 2 * rows * (128 + 256)


@pytest.mark.parametrize("bad,code", [
    (dict(K=0), 1), (dict(K=17, E=32), 2), (dict(E=300, K=8), 2), (dict(K=20, E=16), 1),
    (dict(H=200), 2), (dict(I=96), 2), (dict(T=-1), 1), (dict(routed_scale=float("nan")), 1),
    (dict(T=1 << 29, K=8), 2),
])
def test_invalid_configs_rejected(L, bad, code):
    c = cfg(**bad).c()
    assert L.moe_workspace_size(ctypes.byref(c)) == 0
    rc = L.moe_route(ctypes.byref(c), None, None, None, None, None, None, None, None, 0, None)
    assert rc == code


def test_null_pointers_rejected_before_launch(L):
    c = cfg().c()
    assert L.moe_route(ctypes.byref(c), None, None, None, None, None, None, None, None, 0, None) == 1
    assert L.moe_permute(ctypes.byref(c), None, None, None, None, None, 0, None) == 1
    assert L.moe_forward(ctypes.byref(c), None, None, None, None, None, None, None, 0, None) == 1
    assert L.moe_pack_weights(ctypes.byref(c), None, None, None, None, None, None, None, None, None, None) == 1
    st = ctypes.c_int(0)
    assert L.moe_get_device_error(None, ctypes.byref(st), None) == 1


def test_misaligned_and_small_workspace_rejected(L):
    c = cfg().c()
    fake = ctypes.c_void_p(0x10001)  # never dereferenced: validation fails first
    aligned = ctypes.c_void_p(0x100000)
    assert L.moe_route(ctypes.byref(c), fake, aligned, aligned, aligned, aligned, None, None, aligned, 1 << 40,
                       None) == 3
    need = L.moe_workspace_size(ctypes.byref(c))
    assert L.moe_permute(ctypes.byref(c), aligned, aligned, aligned, aligned, aligned, need - 1, None) == 4


def test_router_packing_and_ep_calls_validate_before_launch(L):
    c = cfg().c()
    fake = ctypes.c_void_p(0x10001)
    aligned = ctypes.c_void_p(0x100000)
    assert L.moe_router_packed_size(ctypes.byref(c)) == 2 * 3 * 64 * 256
    assert L.moe_router_packed_size(ctypes.byref(cfg(K=0).c())) == 0
    assert L.moe_pack_router(ctypes.byref(c), None, None, None) == 1
    assert L.moe_pack_router(ctypes.byref(c), fake, aligned, None) == 3
    assert L.moe_route_packed(ctypes.byref(c), aligned, fake, aligned, aligned, aligned, None, None, aligned,
                              1 << 40, None) == 3
    need = L.moe_workspace_size(ctypes.byref(c))
    assert L.moe_route_packed(ctypes.byref(c), aligned, aligned, aligned, aligned, aligned, None, None, aligned,
                              need - 1, None) == 4
    # the fp32 router path checks everything before its split kernel
    assert L.moe_route(ctypes.byref(c), aligned, aligned, aligned, aligned, aligned, None, None, aligned,
                       need - 1, None) == 4
    assert ep.workspace_offset(cfg(), ep.WS_SLOT_OUTPUTS) > ep.workspace_offset(cfg(), ep.WS_TOKEN_ROWS) > 0
    assert L.moe_workspace_offset(ctypes.byref(c), 7) == ctypes.c_size_t(-1).value
    first = (ctypes.c_int32 * 3)(0, 8, 16)
    bad_first = (ctypes.c_int32 * 3)(0, 8, 15)
    assert L.moe_ep_plan(ctypes.byref(c), 2, 0, bad_first, aligned, aligned, aligned, aligned, 16, aligned,
                         None) == 1
    assert L.moe_ep_plan(ctypes.byref(c), 2, 2, first, aligned, aligned, aligned, aligned, 16, aligned, None) == 1
    assert L.moe_ep_plan(ctypes.byref(c), 9, 0, first, aligned, aligned, aligned, aligned, 16, aligned, None) == 1
    assert L.moe_ep_plan(ctypes.byref(c), 2, 0, first, fake, aligned, aligned, aligned, 16, aligned, None) == 3
    owner = cfg(K=1, has_shared=False).c()
    assert L.moe_ep_return(ctypes.byref(c), 2, aligned, None, None, aligned, 1 << 40, None) == 1  # K != 1
    assert L.moe_ep_return(ctypes.byref(owner), 2, None, None, None, aligned, 1 << 40, None) == 1
    assert L.moe_ep_shared(ctypes.byref(cfg(has_shared=False).c()), None, None, None, 0, None) == 1


def test_zero_tokens_is_a_no_op(L):
    c = cfg(T=0).c()
    assert L.moe_route(ctypes.byref(c), None, None, None, None, None, None, None, None, 0, None) == 0
    assert L.moe_forward(ctypes.byref(c), None, None, None, None, None, None, None, 0, None) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(moe, "_lib", None)
    with pytest.raises(RuntimeError, match="not found"):
        moe.lib()


# ---------------------------------------------------------------- key selection

def dsa_cfg(**kw):
    base = dict(B=2, T=64, S=64)
    base.update(kw)
    return dsa.Config(**base)


def test_dsa_workspace_size(L):
    dsa.lib()
    small = dsa.workspace_bytes(dsa_cfg())
    big = dsa.workspace_bytes(dsa_cfg(T=4096, S=4096, B=4))
    assert big > small > 0
    assert big >= 4 * 4096 * 4096 * 4  # room for the fp32 scores


@pytest.mark.parametrize("bad,code", [
    (dict(n_heads=16), 2), (dict(head_dim=96), 2), (dict(T=0), 1), (dict(T=65, S=64), 1),
    (dict(topk=0), 1), (dict(topk=70000), 2), (dict(S=40000, T=1), 2), (dict(B=-1), 1),
])
def test_dsa_invalid_configs_rejected(L, bad, code):
    dsa.lib()
    c = dsa_cfg(**bad).c()
    assert L.dsa_workspace_size(ctypes.byref(c)) == 0
    assert L.dsa_select(ctypes.byref(c), None, None, None, None, None, None, 0, None) == code


def test_dsa_pointer_checks_before_launch(L):
    dsa.lib()
    c = dsa_cfg().c()
    need = L.dsa_workspace_size(ctypes.byref(c))
    ws = ctypes.c_void_p(0x100000)
    p16 = ctypes.c_void_p(0x200000)
    odd = ctypes.c_void_p(0x200008)  # 8-byte aligned only: q, k, w need 16
    assert L.dsa_select(ctypes.byref(c), None, p16, p16, p16, None, ws, need, None) == 1
    assert L.dsa_select(ctypes.byref(c), odd, p16, p16, p16, None, ws, need, None) == 3
    assert L.dsa_select(ctypes.byref(c), p16, p16, p16, p16, None, ws, need - 1, None) == 4
    assert L.dsa_scores(ctypes.byref(c), p16, p16, p16, None, ws, need, None) == 1
    assert L.dsa_topk(ctypes.byref(c), p16, None, ws, need, None) == 1
    assert L.dsa_select(ctypes.byref(c), p16, p16, p16, p16, None, ctypes.c_void_p(0x100010), need,
                        None) == 3


def test_dsa_no_sequences_is_a_no_op(L):
    dsa.lib()
    c = dsa_cfg(B=0).c()
    assert L.dsa_select(ctypes.byref(c), None, None, None, None, None, None, 0, None) == 0


C_CLIENT = r"""
#include <stdio.h>
#include "srm_moe.h"
#include "srm_dsa.h"
#include "srm_ep.h"

int main(void) {
    moe_cfg_t cfg = {16384, 6144, 2048, 256, 8, 2.5f, 1};
    dsa_cfg_t kcfg = {4, 4096, 4096, 32, 128, 2048};
    size_t a = moe_workspace_size(&cfg), b = dsa_workspace_size(&kcfg);
    moe_cfg_t bad = cfg;
    bad.K = 0;
    /* host validation only: no pointer is dereferenced, nothing is launched */
    moe_status_t st = moe_route(&bad, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0);
    printf("%zu %zu %d %s\n", a, b, (int)st, moe_status_string(MOE_ERR_ARG));
    return (a > 0 && b > 0 && st == MOE_ERR_ARG) ? 0 : 1;
}
"""


def test_headers_are_plain_c_and_link(L, tmp_path):
    """include/*.h compile as C99 and a C program links against the library and
    calls its host-side entry points (no GPU needed)."""
    import subprocess

    src = tmp_path / "client.c"
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    lib_dir = os.path.dirname(moe.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                        "-L", lib_dir, "-lsrm_moe", "-Wl,-rpath," + lib_dir, "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    a, b, st, msg = r.stdout.split(maxsplit=3)
    assert int(a) == moe.workspace_bytes(moe.Config(16384, 6144, 2048, 256, 8))
    assert int(st) == 1 and msg.strip() == "invalid argument"
