"""Python face of the CPU oracle (``moe_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.  Marshals
numpy arrays into the plain C oracle; every computation happens in C, in
double precision, single-threaded.  bf16 arrays are numpy.uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_SO = os.path.join(_HERE, "libmoe_oracle.so")
CC_FLAGS = ["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-fno-fast-math", "-ffp-contract=off"]
F32, BF16 = 0, 1
SWIGLU, GELU = 0, 1
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle: plain C, one thread, no vectorising fast-math.
    MOE_ORACLE_LIB names a library built elsewhere from a variant of this
    source (the pin tests' mutation check loads a deliberately broken copy
    through it); unset, the oracle here is built and used."""
    override = os.environ.get("MOE_ORACLE_LIB")
    if override:
        return override
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call(CC_FLAGS + [_SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    vp, i64, i32, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
    sig = {
        "oracle_router_logits": (None, [vp, i32, i64, i32, vp, i32, vp]),
        "oracle_route_topk": (i32, [vp, i64, i32, i32, i32, vp, vp]),
        "oracle_capacity": (i64, [dbl, i64, i32, i32]),
        "oracle_permute": (i64, [vp, i64, i32, i32, i64, vp, i32, vp, vp, vp, vp, vp, vp]),
        "oracle_gather_rows": (None, [vp, i64, vp, i64, vp]),
        "oracle_expert_ffn_rows": (None, [vp, i32, i64, i32, i32, vp, vp, vp, vp, i32, vp]),
        "oracle_unpermute": (None, [vp, i32, i64, i32, i32, vp, vp, vp, vp]),
        "oracle_copy_slot_rows": (None, [vp, i64, vp, vp, i64, vp]),
        "oracle_group_precombine": (None, [vp, i32, i64, i32, i32, vp, vp, vp, vp]),
        "oracle_unpermute_groups": (None, [vp, i32, i64, i32, i32, vp, vp, vp]),
        "oracle_route_ec": (i32, [vp, i64, i32, i32, vp, vp, vp, vp]),
        "oracle_unpermute_ec": (None, [vp, i32, i64, i32, vp, vp, vp, vp]),
        "oracle_coselect": (None, [vp, i64, i32, i32, vp]),
        "oracle_transition": (None, [vp, i32, vp, i32, i64, i32, vp]),
        "oracle_local_fraction": (dbl, [vp, i64, i32, vp, i32]),
        "oracle_place_experts": (i32, [vp, i32, i32, vp]),
        "oracle_group_affinity": (None, [vp, i32, vp, i32, vp]),
        "oracle_predict_home": (None, [vp, i64, i32, vp, i32, vp]),
        "oracle_count_local": (i64, [vp, i64, i32, vp, i32, vp]),
        "oracle_silu": (dbl, [dbl]),
        "oracle_gelu": (dbl, [dbl]),
        "oracle_round_bf16": (dbl, [dbl]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    _lib = lib
    return lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError("activations must be float32 or bf16 bit patterns (uint16), got %s" % a.dtype)



def router_logits(x: np.ndarray, W_r: np.ndarray) -> np.ndarray:
    """The router's linear gate x W_r^T, float64 [T, E]."""
    x = np.ascontiguousarray(x)
    W_r = np.ascontiguousarray(W_r)
    dt = _dt(x)
    assert W_r.dtype == x.dtype and W_r.shape[1] == x.shape[1]
    T, d = x.shape
    E = W_r.shape[0]
    out = np.empty((T, E), np.float64)
    _load().oracle_router_logits(x.ctypes.data, dt, T, d, W_r.ctypes.data, E, out.ctypes.data)
    return out


def route_topk(logits: np.ndarray, k: int, norm_topk: bool = False):
    """TopKRouter: (expert_idx int32 [T,k], gate float32 [T,k])."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    idx = np.empty((T, k), np.int32)
    gate = np.empty((T, k), np.float32)
    if _load().oracle_route_topk(lg.ctypes.data, T, E, k, int(norm_topk), idx.ctypes.data, gate.ctypes.data):
        raise ValueError("bad top-k arguments")
    return idx, gate


def capacity(capacity_factor: float, T: int, k: int, E: int) -> int:
    return int(_load().oracle_capacity(float(capacity_factor), T, k, E))


def permute(expert_idx: np.ndarray, E: int, cap: int, group_of_expert: Optional[np.ndarray] = None):
    """token_permutation (indices).  Returns dict with row_map, row_token, counts,
    load, offsets, dropped, R."""
    idx = _c(expert_idx, np.int32)
    T, k = idx.shape
    S = T * k
    row_map = np.empty(S, np.int32)
    row_token = np.full(max(S, 1), -1, np.int32)
    counts = np.empty(E, np.int32)
    load = np.empty(E, np.int32)
    dropped = np.zeros(1, np.int64)
    if group_of_expert is None:
        goe_p, G = None, E
        offsets = np.empty(E + 1, np.int32)
    else:
        goe = _c(group_of_expert, np.int32)
        G = int(goe.max()) + 1 if goe.size else 0
        goe_p = goe.ctypes.data
        offsets = np.empty(G + 1, np.int32)
    R = _load().oracle_permute(idx.ctypes.data, T, k, E, int(cap), goe_p, G, row_map.ctypes.data,
                               row_token.ctypes.data, counts.ctypes.data, load.ctypes.data,
                               offsets.ctypes.data, dropped.ctypes.data)
    return dict(row_map=row_map.reshape(T, k), row_token=row_token[:R].copy(), counts=counts, load=load,
                offsets=offsets, dropped=int(dropped[0]), R=int(R))


def gather_rows(x: np.ndarray, row_token: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x)
    rt = _c(row_token, np.int32)
    out = np.empty((rt.size,) + x.shape[1:], x.dtype)
    row_bytes = x[0].nbytes if x.shape[0] else 0
    _load().oracle_gather_rows(x.ctypes.data, row_bytes, rt.ctypes.data, rt.size, out.ctypes.data)
    return out


def expert_ffn_rows(x_rows: np.ndarray, row_expert: np.ndarray, W1, W3, W2, act: str = "swiglu") -> np.ndarray:
    """Expert MLP on each row with its own expert; returns float64 [n, d]
    (values already rounded to the activation dtype)."""
    x = np.ascontiguousarray(x_rows)
    dt = _dt(x)
    n, d = x.shape
    W1 = np.ascontiguousarray(W1)
    W2 = np.ascontiguousarray(W2)
    F = W1.shape[1]
    a = SWIGLU if act == "swiglu" else GELU
    if a == SWIGLU:
        W3 = np.ascontiguousarray(W3)
        w3p = W3.ctypes.data
    else:
        w3p = None
    re = _c(row_expert, np.int32)
    y = np.empty((n, d), np.float64)
    _load().oracle_expert_ffn_rows(x.ctypes.data, dt, n, d, F, re.ctypes.data, W1.ctypes.data, w3p,
                                   W2.ctypes.data, a, y.ctypes.data)
    return y


def unpermute(Y: np.ndarray, row_map: np.ndarray, gate: np.ndarray, shared: Optional[np.ndarray] = None):
    """token_unpermutation: float64 [T, d]."""
    Y = np.ascontiguousarray(Y)
    dt = _dt(Y)
    rm = _c(row_map, np.int32)
    T, k = rm.shape
    d = Y.shape[1]
    g = _c(gate, np.float32)
    sp = None
    if shared is not None:
        shared = np.ascontiguousarray(shared)
        assert shared.dtype == Y.dtype
        sp = shared.ctypes.data
    out = np.empty((T, d), np.float64)
    _load().oracle_unpermute(Y.ctypes.data, dt, T, d, k, rm.ctypes.data, g.ctypes.data, sp, out.ctypes.data)
    return out


def copy_slot_rows(src: np.ndarray, src_row, dst_row, dst: np.ndarray) -> np.ndarray:
    """dst[dst_row[s]] = src[src_row[s]] where both are >= 0 (dst updated in place)."""
    src = np.ascontiguousarray(src)
    assert dst.flags.c_contiguous and dst.dtype == src.dtype and dst.shape[1:] == src.shape[1:]
    sr = _c(src_row, np.int32).reshape(-1)
    dr = _c(dst_row, np.int32).reshape(-1)
    assert sr.size == dr.size
    _load().oracle_copy_slot_rows(src.ctypes.data, src[0].nbytes if src.shape[0] else 0, sr.ctypes.data,
                                  dr.ctypes.data, sr.size, dst.ctypes.data)
    return dst


def group_precombine(Y_e: np.ndarray, row_map_e, row_map_g, gate, R_g: int) -> np.ndarray:
    """One row per (token, group): float64 [R_g, d], bf16-rounded for bf16
    inputs; rows no slot maps to are NaN."""
    Y_e = np.ascontiguousarray(Y_e)
    dt = _dt(Y_e)
    re = _c(row_map_e, np.int32)
    rg = _c(row_map_g, np.int32)
    g = _c(gate, np.float32)
    T, k = rg.shape
    assert re.shape == (T, k) and g.shape == (T, k)
    d = Y_e.shape[1]
    P = np.full((R_g, d), np.nan)
    _load().oracle_group_precombine(Y_e.ctypes.data, dt, T, d, k, re.ctypes.data, rg.ctypes.data, g.ctypes.data,
                                    P.ctypes.data)
    return P


def unpermute_groups(Y_g: np.ndarray, row_map_g, shared: Optional[np.ndarray] = None) -> np.ndarray:
    """Token outputs from their group rows: float64 [T, d]."""
    Y_g = np.ascontiguousarray(Y_g)
    dt = _dt(Y_g)
    rg = _c(row_map_g, np.int32)
    T, k = rg.shape
    d = Y_g.shape[1]
    sp = None
    if shared is not None:
        shared = np.ascontiguousarray(shared)
        assert shared.dtype == Y_g.dtype
        sp = shared.ctypes.data
    out = np.empty((T, d), np.float64)
    _load().oracle_unpermute_groups(Y_g.ctypes.data, dt, T, d, k, rg.ctypes.data, sp, out.ctypes.data)
    return out


def to_dtype_bits(v: np.ndarray, like: np.ndarray) -> np.ndarray:
    """float64 values already representable in like's dtype -> that dtype
    (float32, or bf16 bit patterns as uint16)."""
    f = np.ascontiguousarray(v, np.float64).astype(np.float32)
    if like.dtype == np.uint16:
        u = f.view(np.uint32)
        assert ((u & 0xFFFF) == 0).all(), "values are not bf16"
        return (u >> 16).astype(np.uint16)
    return f


def route_ec(logits: np.ndarray, C: int):
    """ExpertChoiceRouter: (ec_token [E,C], ec_gate [E,C], tok_ptr [T+1], tok_row [E*C])."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    ec_token = np.empty((E, C), np.int32)
    ec_gate = np.empty((E, C), np.float32)
    tok_ptr = np.empty(T + 1, np.int32)
    tok_row = np.empty(E * C, np.int32)
    if _load().oracle_route_ec(lg.ctypes.data, T, E, C, ec_token.ctypes.data, ec_gate.ctypes.data,
                               tok_ptr.ctypes.data, tok_row.ctypes.data):
        raise ValueError("bad expert-choice arguments")
    return ec_token, ec_gate, tok_ptr, tok_row


def unpermute_ec(Y: np.ndarray, tok_ptr, tok_row, ec_gate) -> np.ndarray:
    Y = np.ascontiguousarray(Y)
    dt = _dt(Y)
    tp = _c(tok_ptr, np.int32)
    tr = _c(tok_row, np.int32)
    g = _c(ec_gate, np.float32).reshape(-1)
    T = tp.size - 1
    d = Y.shape[1]
    out = np.empty((T, d), np.float64)
    _load().oracle_unpermute_ec(Y.ctypes.data, dt, T, d, tp.ctypes.data, tr.ctypes.data, g.ctypes.data,
                                out.ctypes.data)
    return out


def coselect(expert_idx: np.ndarray, E: int, into: Optional[np.ndarray] = None) -> np.ndarray:
    idx = _c(expert_idx, np.int32)
    T, k = idx.shape
    C = np.zeros((E, E), np.int32) if into is None else into
    assert C.dtype == np.int32 and C.flags.c_contiguous and C.shape == (E, E)
    _load().oracle_coselect(idx.ctypes.data, T, k, E, C.ctypes.data)
    return C


def transition(idx1: np.ndarray, idx2: np.ndarray, E: int, into: Optional[np.ndarray] = None) -> np.ndarray:
    a = _c(idx1, np.int32)
    b = _c(idx2, np.int32)
    T, k1 = a.shape
    T2, k2 = b.shape
    assert T == T2
    M = np.zeros((E, E), np.int32) if into is None else into
    _load().oracle_transition(a.ctypes.data, k1, b.ctypes.data, k2, T, E, M.ctypes.data)
    return M


def local_fraction(expert_idx: np.ndarray, group_of_expert: np.ndarray, G: int) -> float:
    idx = _c(expert_idx, np.int32)
    T, k = idx.shape
    goe = _c(group_of_expert, np.int32)
    return float(_load().oracle_local_fraction(idx.ctypes.data, T, k, goe.ctypes.data, G))


def place_experts(cosel: np.ndarray, G: int) -> np.ndarray:
    """Greedy correlated placement: group_of_expert [E]."""
    C = _c(cosel, np.int32)
    E = C.shape[0]
    goe = np.empty(E, np.int32)
    if _load().oracle_place_experts(C.ctypes.data, E, G, goe.ctypes.data):
        raise ValueError("G must divide E")
    return goe


def group_affinity(trans: np.ndarray, group_of_expert: np.ndarray, G: int) -> np.ndarray:
    M = _c(trans, np.int32)
    E = M.shape[0]
    goe = _c(group_of_expert, np.int32)
    aff = np.empty((E, G), np.int64)
    _load().oracle_group_affinity(M.ctypes.data, E, goe.ctypes.data, G, aff.ctypes.data)
    return aff


def predict_home(idx1: np.ndarray, affinity: np.ndarray) -> np.ndarray:
    i1 = _c(idx1, np.int32)
    T, k1 = i1.shape
    aff = _c(affinity, np.int64)
    home = np.empty(T, np.int32)
    _load().oracle_predict_home(i1.ctypes.data, T, k1, aff.ctypes.data, aff.shape[1], home.ctypes.data)
    return home


def count_local(expert_idx: np.ndarray, group_of_expert: np.ndarray, G: int, home=None) -> int:
    idx = _c(expert_idx, np.int32)
    T, k = idx.shape
    goe = _c(group_of_expert, np.int32)
    hp = None
    if home is not None:
        home = _c(home, np.int32)
        hp = home.ctypes.data
    return int(_load().oracle_count_local(idx.ctypes.data, T, k, goe.ctypes.data, G, hp))


def silu(z: float) -> float:
    return float(_load().oracle_silu(z))


def gelu(z: float) -> float:
    return float(_load().oracle_gelu(z))


def round_bf16(x: float) -> float:
    return float(_load().oracle_round_bf16(x))


# ------------------------------------------------------------------ layers
def topk_layer_tokens(w, logits, x, weights, shared_weights, tokens):
    """Full top-k MoE layer output for the listed tokens only, float64
    [len(tokens), d] (not rounded to the output dtype).

    Routing and capacity run over all T tokens (a token's drops depend on
    every earlier token); the expert MLPs run only on the listed tokens'
    kept assignments."""
    idx, gate = route_topk(logits, w.k, w.norm_topk)
    cap = capacity(w.capacity_factor, w.T, w.k, w.E)
    p = permute(idx, w.E, cap)
    tokens = np.asarray(tokens, np.int64)
    W1, W3, W2 = weights
    rows, experts, owner, slot = [], [], [], []
    for i, t in enumerate(tokens):
        for j in range(w.k):
            if p["row_map"][t, j] >= 0:
                rows.append(t)
                experts.append(idx[t, j])
                owner.append(i)
                slot.append(j)
    out = np.zeros((len(tokens), w.d), np.float64)
    if rows:
        y = expert_ffn_rows(x[np.asarray(rows)], np.asarray(experts, np.int32), W1, W3, W2, w.act)
        # gate-weighted sum in slot order, as in unpermute()
        for n in range(len(rows)):
            out[owner[n]] += np.float64(gate[tokens[owner[n]], slot[n]]) * y[n]
    if shared_weights is not None:
        sW1, sW3, sW2 = shared_weights
        ys = expert_ffn_rows(x[tokens], np.zeros(len(tokens), np.int32), sW1, sW3, sW2, "swiglu")
        out += ys
    return out, dict(idx=idx, gate=gate, cap=cap, perm=p)


def topk_group_layer_tokens(w, logits, x, weights, shared_weights, group_of_expert, tokens):
    """The top-k layer with the send-once dispatcher and real experts, for
    the listed tokens only: float64 [len(tokens), d].  Per token, the kept
    expert outputs of each group are gate-summed into one row (rounded to
    the activation dtype, as a returned tensor is), and the token's output
    is the sum of its group rows (+ the shared expert)."""
    idx, gate = route_topk(logits, w.k, w.norm_topk)
    cap = capacity(w.capacity_factor, w.T, w.k, w.E)
    p = permute(idx, w.E, cap)
    goe = np.asarray(group_of_expert, np.int32)
    tokens = np.asarray(tokens, np.int64)
    n = tokens.size
    W1, W3, W2 = weights
    rows, experts = [], []
    rm_e = np.full((n, w.k), -1, np.int32)          # local expert rows of the listed tokens
    rm_g = np.full((n, w.k), -1, np.int32)          # local group rows
    n_g = 0
    for i, t in enumerate(tokens):
        seen = {}
        for j in range(w.k):
            if p["row_map"][t, j] < 0:
                continue
            rm_e[i, j] = len(rows)
            rows.append(t)
            experts.append(idx[t, j])
            g = int(goe[idx[t, j]])
            if g not in seen:
                seen[g] = n_g
                n_g += 1
            rm_g[i, j] = seen[g]
    out = np.zeros((n, w.d), np.float64)
    if rows:
        y = expert_ffn_rows(x[np.asarray(rows)], np.asarray(experts, np.int32), W1, W3, W2, w.act)
        y_bits = to_dtype_bits(y, x)
        P = group_precombine(y_bits, rm_e, rm_g, gate[tokens], n_g)
        out = unpermute_groups(to_dtype_bits(P, x), rm_g)
    if shared_weights is not None:
        sW1, sW3, sW2 = shared_weights
        out = out + expert_ffn_rows(x[tokens], np.zeros(n, np.int32), sW1, sW3, sW2, "swiglu")
    return out, dict(idx=idx, gate=gate, cap=cap, perm=p)
