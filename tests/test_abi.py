"""CPU checks of the C ABI: the library loads, exports every entry point
the header declares, and its host-side logic (validation, sizes, capacity)
behaves - no kernel is launched."""
import ctypes
import os
import re

import pytest

from mixture_experts_routing_top_b200 import build, libmoe as M
from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "libmoe.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return M.lib()


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared()
    for n in ("moe_route_topk", "moe_route_ec", "moe_permute", "moe_expert_ffn", "moe_unpermute",
              "moe_unpermute_ec", "moe_coselect", "moe_transition", "moe_gather_rows"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    for n in declared():
        assert hasattr(L, n), n
        assert n in M.SIGNATURES, "binding lacks " + n


def test_status_strings(L):
    assert L.moe_status_string(0) == b"ok"
    for s in range(1, 9):
        assert L.moe_status_string(s) not in (b"ok", b"unknown status")
    assert L.moe_status_string(99) == b"unknown status"
    for s in range(0, 9):
        assert L.moe_status_str(s) == L.moe_status_string(s)
    assert L.moe_abi_version() == 1


@pytest.mark.parametrize("cf,T,k,E", [(1.25, 256, 2, 8), (1.25, 8192, 2, 8), (1.5, 16384, 6, 64), (0.5, 1000, 3, 7),
                                      (0.0, 100, 2, 4), (-1.0, 5, 1, 1), (0.3333, 777, 5, 13)])
def test_capacity_agrees_with_oracle(L, cf, T, k, E):
    assert M.capacity(cf, T, k, E) == O.capacity(cf, T, k, E)


def test_max_rows(L):
    assert M.permute_max_rows(256, 2, 8, 1.25) == min(512, 8 * 80)
    assert M.permute_max_rows(100, 3, 4, 0.5) == 4 * 38
    assert M.permute_max_rows(100, 8, 256, 0.0, 8) == 100 * 8
    assert M.permute_max_rows(100, 8, 256, 0.0, 4) == 100 * 4
    assert M.permute_max_rows(0, 2, 8, 1.0) == 0


def test_workspace_queries(L):
    assert M.permute_workspace_bytes(131072, 8, 256, 0) >= 2 * 4 * 256 * 512
    assert M.permute_workspace_bytes(131072, 8, 256, 64) > M.permute_workspace_bytes(131072, 8, 256, 0)
    assert M.route_ec_workspace_bytes(32768, 128, 512) >= 32768 * 128 * 8
    assert M.expert_ffn_workspace_bytes(1000, 64, 128, None) >= 1000 * 128 * 4


def test_host_validation_rejects_before_launch(L):
    vp = ctypes.c_void_p(0x1000)           # never dereferenced: validation fails first
    nul = None
    assert L.moe_route_topk(vp, 10, 4, 5, 0, vp, vp, nul) == 1          # k > E
    assert L.moe_route_topk(vp, 10, 4, 0, 0, vp, vp, nul) == 1          # k < 1
    assert L.moe_route_topk(vp, 10, 2000, 4, 0, vp, vp, nul) == 2       # E > 1024
    assert L.moe_route_topk(vp, 10, 64, 33, 0, vp, vp, nul) == 2        # k > 32
    assert L.moe_route_topk(nul, 10, 4, 2, 0, vp, vp, nul) == 1         # null logits
    assert L.moe_route_topk(nul, 0, 4, 2, 0, nul, nul, nul) == 0        # empty: nothing to do
    assert L.moe_route_ec(vp, 10, 4, 11, vp, vp, vp, vp, vp, 1 << 20, nul) == 1   # C > T
    assert L.moe_route_ec(vp, 10, 4, 2, vp, vp, vp, vp, nul, 0, nul) == 4         # no workspace
    assert L.moe_route_ec(vp, 10, 4, 2, vp, vp, vp, vp, ctypes.c_void_p(0x1001), 1 << 30, nul) == 4  # misaligned
    # permute: dtype, x/buffer pairing, row alignment, workspace
    args = lambda **kw: dict(dict(x=vp, dt=1, T=10, d=8, idx=vp, k=2, E=4, cf=1.0, goe=nul, G=0, buf=vp, rm=vp,
                                  rt=vp, cnt=vp, off=vp, drop=vp, ws=ctypes.c_void_p(0x100000), wsb=1 << 30), **kw)
    call = lambda a: L.moe_permute(a["x"], a["dt"], a["T"], a["d"], a["idx"], a["k"], a["E"], a["cf"], a["goe"],
                                   a["G"], a["buf"], a["rm"], a["rt"], a["cnt"], a["off"], a["drop"], a["ws"],
                                   a["wsb"], nul)
    assert call(args(dt=7)) == 1
    assert call(args(buf=nul)) == 1
    assert call(args(d=7)) == 2              # 14-byte bf16 rows
    assert call(args(ws=nul)) == 4
    assert call(args(wsb=16)) == 4
    assert call(args(k=5)) == 1              # k > E
    assert call(args(goe=vp, G=0)) == 1      # groups without G
    # expert FFN: bf16 needs d, F multiples of 64
    assert L.moe_expert_ffn(vp, 1, 100, 96, 128, 4, vp, vp, vp, vp, 0, vp, ctypes.c_void_p(0x100000), 1 << 30, nul) == 2
    assert L.moe_expert_ffn(vp, 1, 100, 128, 128, 4, vp, vp, nul, vp, 0, vp, ctypes.c_void_p(0x100000), 1 << 30, nul) == 1
    assert L.moe_expert_ffn(vp, 1, 100, 128, 128, 4, vp, vp, vp, vp, 3, vp, ctypes.c_void_p(0x100000), 1 << 30, nul) == 1
    assert L.moe_expert_ffn(vp, 1, 100, 128, 128, 2000, vp, vp, vp, vp, 0, vp, ctypes.c_void_p(0x100000), 1 << 30, nul) == 2
    assert L.moe_unpermute(vp, 0, 20, 10, 8, 40, vp, vp, nul, vp, 0, nul) == 2   # k > 32
    assert L.moe_unpermute(vp, 5, 20, 10, 8, 2, vp, vp, nul, vp, 0, nul) == 1    # dtype
    assert L.moe_unpermute(vp, 0, -1, 10, 8, 2, vp, vp, nul, vp, 0, nul) == 1    # R < 0
    assert L.moe_gather_rows(vp, 1, 10, 7, vp, vp, 20, vp, nul) == 2             # 14-byte rows
    assert L.moe_unpermute_ec(vp, 0, 20, 10, 8, nul, vp, vp, vp, 0, nul) == 1     # null tok_ptr
    assert L.moe_coselect(vp, 10, 2, 2000, vp, nul) == 2
    assert L.moe_transition(vp, 1, vp, 0, 10, 8, vp, nul) == 1
    assert L.moe_selftest_bounded_wait(0, 999, vp, nul) == 1                     # limit below 1 us
    assert L.moe_selftest_bounded_wait(0, 2 * 10 ** 9, vp, nul) == 1             # above 1 s
    assert L.moe_selftest_bounded_wait(0, 10 ** 6, nul, nul) == 1                # no result buffer


def test_host_validation_of_the_later_calls(L):
    """The fused router, the group-major expert path, placement and the
    shuffling statistic: bad arguments rejected on the host with the status
    the header documents, before any launch (this box has no GPU)."""
    vp, nul = ctypes.c_void_p(0x1000), None
    router = lambda dt=1, T=10, d=128, E=16, k=2, logits=vp, x=vp: L.moe_router_topk(
        x, dt, T, d, vp, E, k, 0, logits, vp, vp, nul)
    assert router(d=96) == 2                 # bf16: d % 64
    assert router(E=12) == 2                 # bf16: E % 8
    assert router(E=264) == 2                # bf16: E <= 256
    assert router(k=9) == 2                  # bf16: k <= 8
    assert router(k=17) == 1                 # k > E
    assert router(dt=7) == 1                 # dtype
    assert router(x=nul) == 1
    assert router(dt=0, logits=nul) == 1     # fp32 needs the logits buffer
    assert router(T=0) == 0
    copy = lambda dt=1, d=64, S=10, src=vp: L.moe_copy_slot_rows(src, dt, 10, d, vp, vp, S, vp, 10, nul)
    assert copy(S=-1) == 1 and copy(dt=9) == 1 and copy(src=nul) == 1
    assert copy(dt=0, d=3) == 2              # 12-byte rows
    assert copy(S=0) == 0
    pre = lambda dt=1, T=10, d=64, k=2, gate=vp: L.moe_group_precombine(vp, dt, 20, T, d, k, vp, vp, gate, vp, 20, nul)
    assert pre(k=0) == 1 and pre(k=33) == 2 and pre(gate=nul) == 1 and pre(d=4) == 2 and pre(T=0) == 0
    ug = lambda od=1, T=10, d=64, k=2, yg=vp, Rg=20: L.moe_unpermute_groups(yg, 1, Rg, T, d, k, vp, nul, vp, od, nul)
    assert ug(od=4) == 1 and ug(k=40) == 2 and ug(yg=nul) == 1 and ug(d=12) == 2 and ug(T=0) == 0
    assert L.moe_place_experts(vp, 12, 5, vp, nul) == 1                 # G does not divide E
    assert L.moe_place_experts(vp, 2000, 1, vp, nul) == 2
    assert L.moe_place_experts(nul, 12, 3, vp, nul) == 1
    assert L.moe_group_affinity(vp, 16, vp, 0, vp, nul) == 1
    assert L.moe_group_affinity(vp, 16, vp, 2000, vp, nul) == 2
    assert L.moe_group_affinity(vp, 16, nul, 4, vp, nul) == 1
    assert L.moe_predict_home(vp, 10, 0, vp, 16, 4, vp, nul) == 1
    assert L.moe_predict_home(vp, 10, 33, vp, 16, 4, vp, nul) == 2
    assert L.moe_predict_home(vp, 10, 1, vp, 16, 4, nul, nul) == 1
    assert L.moe_predict_home(vp, 0, 1, vp, 16, 4, vp, nul) == 0
    assert L.moe_count_local(vp, 10, 0, vp, 16, 4, nul, vp, nul) == 1
    assert L.moe_count_local(vp, 10, 2, vp, 16, 2000, nul, vp, nul) == 2
    assert L.moe_count_local(vp, 10, 2, vp, 16, 4, nul, nul, nul) == 1
    assert L.moe_count_local(vp, 0, 2, vp, 16, 4, nul, vp, nul) == 0


def test_noalloc_checks_arguments_before_its_scratch_size(L):
    """moe_permute_noalloc returns moe_permute's status for bad arguments,
    whatever the problem size; only valid problems too large for its fixed
    scratch get MOE_ERR_WORKSPACE.  Nothing is launched in any case."""
    vp, nul = ctypes.c_void_p(0x1000), None
    na = lambda T=10, k=2, E=4, G=0, goe=nul, dt=1, d=8, cnt=vp: L.moe_permute_noalloc(
        vp, dt, T, d, vp, k, E, 1.0, goe, G, vp, vp, vp, cnt, vp, vp, nul)
    big = 1 << 22                            # needs far more scratch than the 4 MiB array holds
    assert M.permute_workspace_bytes(big, 8, 256, 0) > 4 << 20
    assert na(k=5) == 1                      # k > E
    assert na(T=big, k=300, E=256) == 1      # k > E on a large problem: the argument error
    assert na(T=big, k=33, E=256) == 2       # k > 32
    assert na(T=big, k=8, E=2000) == 2       # E > 1024
    assert na(T=big, k=8, E=256, dt=7) == 1  # dtype
    assert na(T=big, k=8, E=256, d=7) == 2   # 14-byte bf16 rows
    assert na(T=big, k=8, E=256, cnt=nul) == 1
    assert na(T=big, k=8, E=256, goe=vp, G=0) == 1
    assert na(T=big, k=8, E=256) == 4        # valid but beyond the scratch
    assert na(T=262144, k=8, E=256, goe=vp, G=64) == 4
