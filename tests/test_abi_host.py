"""Host-side checks of the C ABI: the library loads without a GPU, exports
every entry point that include/bfmoe.h declares, and rejects bad arguments
on the host before anything touches CUDA.  Every call here returns before
the first CUDA runtime call, so nothing runs on a device."""
import os
import re

import pytest

import ternary_moe_butterfly_b200 as bf
from ternary_moe_butterfly_b200 import build as bfbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_library():
    bfbuild.build()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "bfmoe.h")).read()
    return sorted(set(re.findall(r"BFMOE_API\s+[^;(]*?\b(bfmoe_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for need in ["bfmoe_pack_base", "bfmoe_route", "bfmoe_butterfly_apply", "bfmoe_forward", "bfmoe_sync_status",
                 "bfmoe_forward_workspace_bytes", "bfmoe_route_workspace_bytes", "bfmoe_packed_base_bytes"]:
        assert need in syms


def test_library_exports_every_declared_symbol():
    L = bf.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_binding_has_the_same_names():
    for name in declared_symbols():
        assert callable(getattr(bf, name)), name


def test_status_strings():
    assert bf.bfmoe_status_string(0) == "ok"
    for c in range(1, 7):
        assert bf.bfmoe_status_string(c) not in ("", "unknown status")
    assert bf.bfmoe_status_string(99) == "unknown status"


@pytest.mark.parametrize("d", [64, 128, 512, 1024, 4096])
def test_packed_size(d):
    assert bf.bfmoe_packed_base_bytes(d) == 16 + d * d // 4


@pytest.mark.parametrize("d", [0, -64, 63, 100, 32, 8192])
def test_packed_size_rejects(d):
    assert bf.bfmoe_packed_base_bytes(d) == 0


FAKE = 1 << 20  # an aligned non-null address that is never dereferenced


@pytest.mark.parametrize("d,code", [(100, bf.ERR_INVALID_ARG), (0, bf.ERR_INVALID_ARG), (32, bf.ERR_UNSUPPORTED),
                                    (8192, bf.ERR_UNSUPPORTED)])
def test_forward_rejects_width(d, code):
    assert bf.bfmoe_forward(FAKE, bf.BF16, 16, d, FAKE, 8, 2, FAKE, FAKE, FAKE, FAKE * 2, FAKE * 3, 1 << 40,
                            None) == code


@pytest.mark.parametrize("T,N,k,code", [(0, 8, 2, bf.ERR_INVALID_ARG), (16, 0, 1, bf.ERR_INVALID_ARG),
                                        (16, 4, 5, bf.ERR_INVALID_ARG), (16, 64, 9, bf.ERR_UNSUPPORTED),
                                        (16, 5000, 2, bf.ERR_UNSUPPORTED), (1 << 24, 8, 2, bf.ERR_UNSUPPORTED)])
def test_forward_rejects_routing_shape(T, N, k, code):
    assert bf.bfmoe_forward(FAKE, bf.BF16, T, 64, FAKE, N, k, FAKE, FAKE, FAKE, FAKE * 2, FAKE * 3, 1 << 40,
                            None) == code


def test_forward_rejects_pointers_and_workspace():
    T, d, N, k = 16, 64, 8, 2
    need = bf.bfmoe_forward_workspace_bytes(T, d, N, k)
    assert need > 0
    args = dict(x=FAKE, dt=bf.F32, T=T, d=d, logits=FAKE, N=N, k=k, packed_base=FAKE, theta=FAKE, phi=FAKE,
                y=FAKE * 2, ws=FAKE * 3, ws_bytes=need, stream=None)

    def call(**kw):
        a = dict(args, **kw)
        return bf.bfmoe_forward(*a.values())

    assert call(x=None) == bf.ERR_INVALID_ARG
    assert call(y=None) == bf.ERR_INVALID_ARG
    assert call(ws=None) == bf.ERR_INVALID_ARG
    assert call(x=FAKE + 8) == bf.ERR_INVALID_ARG      # not 16-byte aligned
    assert call(ws=FAKE * 3 + 128) == bf.ERR_INVALID_ARG  # not 256-byte aligned
    assert call(y=FAKE) == bf.ERR_INVALID_ARG           # aliases x
    assert call(dt=7) == bf.ERR_INVALID_ARG
    assert call(ws_bytes=need - 1) == bf.ERR_WORKSPACE


def test_route_and_butterfly_reject_on_host():
    assert bf.bfmoe_route(FAKE, 10, 4, 5, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == bf.ERR_INVALID_ARG
    need = bf.bfmoe_route_workspace_bytes(10, 4, 2)
    assert bf.bfmoe_route(FAKE, 10, 4, 2, FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, None) == bf.ERR_WORKSPACE
    assert bf.bfmoe_route(FAKE, 10, 4, 2, None, FAKE, FAKE, FAKE, FAKE, need, None) == bf.ERR_INVALID_ARG
    wn = bf.bfmoe_butterfly_workspace_bytes(64, 3)
    assert bf.bfmoe_butterfly_apply(FAKE, bf.F32, 5, 48, 3, FAKE, None, 0, FAKE * 2, FAKE * 3, wn,
                                    None) == bf.ERR_INVALID_ARG
    assert bf.bfmoe_butterfly_apply(FAKE, bf.F32, 5, 64, 3, FAKE, None, 0, FAKE, FAKE * 3, wn,
                                    None) == bf.ERR_INVALID_ARG  # x aliases y
    assert bf.bfmoe_butterfly_apply(FAKE, bf.F32, 5, 64, 3, FAKE, None, 0, FAKE * 2, FAKE * 3, wn - 1,
                                    None) == bf.ERR_WORKSPACE
    assert bf.bfmoe_pack_base(FAKE, 65, 1.0, FAKE, None) == bf.ERR_INVALID_ARG
    assert bf.bfmoe_pack_base(FAKE + 1, 64, 1.0, FAKE, None) == bf.ERR_INVALID_ARG


@pytest.mark.parametrize("T,d,N,k", [(128, 64, 8, 2), (4096, 512, 64, 2), (8192, 4096, 64, 2), (12608, 1024, 64, 1),
                                     (1, 64, 1, 1)])
def test_workspace_layout_is_aligned_and_sized(T, d, N, k):
    code, lay = bf.bfmoe_forward_ws_layout(T, d, N, k)
    assert code == bf.OK
    assert lay.total == bf.bfmoe_forward_workspace_bytes(T, d, N, k)
    offs = [lay.status, lay.topk_idx, lay.gates, lay.perm, lay.offsets]
    assert all(o % 256 == 0 for o in offs)
    assert lay.status == 0
    assert sorted(offs) == offs
    assert lay.offsets + 4 * (N + 1) <= lay.total
    # the workspace holds at least the routed fp16 rows and the fp16 products
    assert lay.total >= T * k * d * 4
