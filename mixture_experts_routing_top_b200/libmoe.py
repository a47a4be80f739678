"""Python binding of the libmoe C ABI (``include/libmoe.h``).

Argument marshalling only: every function checks dtypes/devices/shapes of
torch tensors, allocates outputs and workspaces with torch (device memory
is PyTorch's job here), and calls the C entry point of the same name on the
current CUDA stream.  Every step of the MoE layer runs in the library's
CUDA kernels; there is no CPU or PyTorch fallback: a missing library or a
non-zero status raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
SO_PATH = os.path.join(_HERE, "lib", "libmoe.so")

MOE_F32, MOE_BF16 = 0, 1
MOE_ACT_SWIGLU, MOE_ACT_GELU = 0, 1
STATUS = {0: "MOE_OK", 1: "MOE_ERR_ARG", 2: "MOE_ERR_SHAPE", 3: "MOE_ERR_DTYPE", 4: "MOE_ERR_WORKSPACE",
          5: "MOE_ERR_CUDA", 6: "MOE_ERR_UNSUPPORTED", 7: "MOE_ERR_TIMEOUT", 8: "MOE_ERR_DEVICE_INDEX"}

# name -> (restype, argtypes)
_vp, _i32, _i64, _dbl, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [_i32]),
    "moe_status_str": (ctypes.c_char_p, [_i32]),
    "moe_abi_version": (_i32, []),
    "moe_device_error": (_i32, [_i32]),
    "moe_kernel_launches": (ctypes.c_uint64, []),
    "moe_selftest_bounded_wait": (_i32, [_i32, ctypes.c_longlong, _vp, _vp]),
    "moe_route_topk": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_router_topk": (_i32, [_vp, _i32, _i32, _i32, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp]),
    "moe_route_ec_workspace_bytes": (_sz, [_i32, _i32, _i32]),
    "moe_route_ec": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_capacity": (_i64, [_dbl, _i32, _i32, _i32]),
    "moe_permute_max_rows": (_i64, [_i32, _i32, _i32, _dbl, _i32]),
    "moe_permute_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32]),
    "moe_permute": (_i32, [_vp, _i32, _i32, _i32, _vp, _i32, _i32, _dbl, _vp, _i32, _vp, _vp, _vp, _vp, _vp,
                           _vp, _vp, _sz, _vp]),
    "moe_permute_noalloc": (_i32, [_vp, _i32, _i32, _i32, _vp, _i32, _i32, _dbl, _vp, _i32, _vp, _vp, _vp, _vp,
                                   _vp, _vp, _vp]),
    "moe_gather_rows": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _i32, _vp, _vp]),
    "moe_expert_ffn_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32]),
    "moe_expert_ffn": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _sz, _vp]),
    "moe_unpermute": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _vp]),
    "moe_unpermute_ec": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _vp]),
    "moe_copy_slot_rows": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp, _i32, _vp, _i32, _vp]),
    "moe_group_precombine": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _i32, _vp]),
    "moe_unpermute_groups": (_i32, [_vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _i32, _vp]),
    "moe_coselect": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp]),
    "moe_transition": (_i32, [_vp, _i32, _vp, _i32, _i32, _i32, _vp, _vp]),
    "moe_place_experts": (_i32, [_vp, _i32, _i32, _vp, _vp]),
    "moe_group_affinity": (_i32, [_vp, _i32, _vp, _i32, _vp, _vp]),
    "moe_predict_home": (_i32, [_vp, _i32, _i32, _vp, _i32, _i32, _vp, _vp]),
    "moe_count_local": (_i32, [_vp, _i32, _i32, _vp, _i32, _i32, _vp, _vp, _vp]),
}

_lib = None


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__("%s failed: %s (%d)" % (fn, STATUS.get(status, "?"), status))
        self.status = status


def lib() -> ctypes.CDLL:
    """The loaded libmoe.so; raises if it was never built."""
    global _lib
    if _lib is None:
        if not os.path.exists(SO_PATH):
            raise RuntimeError("libmoe.so is missing (%s): build it first with "
                               "`python -m mixture_experts_routing_top_b200.build`" % SO_PATH)
        L = ctypes.CDLL(SO_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _check(fn: str, status: int):
    if status != 0:
        raise MoeError(fn, status)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _p(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, dtype=None, name="tensor"):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    return t


def _buf(t: torch.Tensor, dtype, min_numel: int, name: str, device=None) -> torch.Tensor:
    """A caller's buffer checked against what the library reads or writes
    through its pointer: a contiguous CUDA tensor of `dtype` (None: any) with
    at least `min_numel` elements, on `device` when given.  One combined test
    on the common path (it runs on every call of a layer); the specific
    message only on failure."""
    if (t.is_cuda and t.is_contiguous() and (dtype is None or t.dtype == dtype)
            and (device is None or t.device == device) and t.numel() >= min_numel):
        return t
    _dev(t, dtype, name)
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, the call's inputs on %s" % (name, t.device, device))
    if t.numel() < min_numel:
        raise ValueError("%s has %d elements, the call needs %d" % (name, t.numel(), min_numel))
    return t


def _out(t: Optional[torch.Tensor], shape, dtype, device, name: str) -> torch.Tensor:
    """The caller's output buffer (checked as in _buf) or a new one."""
    if t is None:
        return torch.empty(shape, dtype=dtype, device=device)
    return _buf(t, dtype, math.prod(shape), name, device)


def _ws_bytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def _act_dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MOE_F32
    if t.dtype == torch.bfloat16:
        return MOE_BF16
    raise ValueError("activations must be float32 or bfloat16, got %s" % t.dtype)


def _ws(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


# ------------------------------------------------------------- routing
def route_topk(logits: torch.Tensor, k: int, norm_topk: bool = False, expert_idx=None, gate=None, stream=None):
    _dev(logits, torch.float32, "logits")
    T, E = logits.shape
    expert_idx = _out(expert_idx, (T, k), torch.int32, logits.device, "expert_idx")
    gate = _out(gate, (T, k), torch.float32, logits.device, "gate")
    _check("moe_route_topk", lib().moe_route_topk(_p(logits), T, E, k, int(bool(norm_topk)), _p(expert_idx),
                                                  _p(gate), _stream(stream)))
    return expert_idx, gate



def router_topk(x: torch.Tensor, W_r: torch.Tensor, k: int, norm_topk: bool = False, expert_idx=None, gate=None,
                logits=None, want_logits: bool = False, stream=None):
    """Router linear gate + TopKRouter: (expert_idx [T,k] int32, gate [T,k] fp32, logits [T,E] fp32 or None)."""
    _dev(x, None, "x")
    _dev(W_r, x.dtype, "W_r")
    T, d = x.shape
    E = W_r.shape[0]
    if W_r.shape[1] != d:
        raise ValueError("W_r must be [E, d]")
    dev = x.device
    _buf(W_r, x.dtype, E * d, "W_r", dev)
    expert_idx = _out(expert_idx, (T, k), torch.int32, dev, "expert_idx")
    gate = _out(gate, (T, k), torch.float32, dev, "gate")
    if logits is not None or want_logits or x.dtype == torch.float32:
        logits = _out(logits, (T, E), torch.float32, dev, "logits")
    _check("moe_router_topk", lib().moe_router_topk(
        _p(x), _act_dtype(x), T, d, _p(W_r), E, k, int(bool(norm_topk)), _p(logits), _p(expert_idx), _p(gate),
        _stream(stream)))
    return expert_idx, gate, logits


def route_ec_workspace_bytes(T: int, E: int, C: int) -> int:
    return int(lib().moe_route_ec_workspace_bytes(T, E, C))


def route_ec(logits: torch.Tensor, C: int, workspace=None, out=None, stream=None):
    """Returns (ec_token [E,C], ec_gate [E,C], tok_ptr [T+1], tok_row [E*C])."""
    _dev(logits, torch.float32, "logits")
    T, E = logits.shape
    dev = logits.device
    ec_token, ec_gate, tok_ptr, tok_row = out if out is not None else (None, None, None, None)
    ec_token = _out(ec_token, (E, C), torch.int32, dev, "ec_token")
    ec_gate = _out(ec_gate, (E, C), torch.float32, dev, "ec_gate")
    tok_ptr = _out(tok_ptr, (T + 1,), torch.int32, dev, "tok_ptr")
    tok_row = _out(tok_row, (E * C,), torch.int32, dev, "tok_row")
    nbytes = route_ec_workspace_bytes(T, E, C)
    workspace = _ws(nbytes, dev) if workspace is None else _buf(workspace, None, 0, "workspace", dev)
    _check("moe_route_ec", lib().moe_route_ec(_p(logits), T, E, C, _p(ec_token), _p(ec_gate), _p(tok_ptr),
                                              _p(tok_row), _p(workspace), _ws_bytes(workspace), _stream(stream)))
    return ec_token, ec_gate, tok_ptr, tok_row


# --------------------------------------------------------- permutation
def capacity(capacity_factor: float, T: int, k: int, E: int) -> int:
    return int(lib().moe_capacity(float(capacity_factor), T, k, E))


def permute_max_rows(T: int, k: int, E: int, capacity_factor: float, G: int = 0) -> int:
    return int(lib().moe_permute_max_rows(T, k, E, float(capacity_factor), G))


def permute_workspace_bytes(T: int, k: int, E: int, G: int = 0) -> int:
    return int(lib().moe_permute_workspace_bytes(T, k, E, G))


def permute(x: Optional[torch.Tensor], expert_idx: torch.Tensor, E: int, capacity_factor: float,
            group_of_expert: Optional[torch.Tensor] = None, G: int = 0, out=None, workspace=None, stream=None):
    """token_permutation.  Returns dict(buffer, row_map, row_token, counts,
    offsets, dropped); buffer is [R_max, d] (R = offsets[-1] rows used)."""
    _dev(expert_idx, torch.int32, "expert_idx")
    T, k = expert_idx.shape
    dev = expert_idx.device
    if group_of_expert is not None:
        _buf(group_of_expert, torch.int32, E, "group_of_expert", dev)
        if G <= 0:
            raise ValueError("G must be given with group_of_expert")
    else:
        G = 0
    R_max = permute_max_rows(T, k, E, capacity_factor, G)
    dtype = MOE_F32
    d = 0
    if x is not None:
        _buf(x, None, 0, "x", dev)
        if x.dim() != 2 or x.shape[0] < T:
            raise ValueError("x must be [T, d] with T = %d rows" % T)
        dtype = _act_dtype(x)
        d = x.shape[1]
    if out is None:
        out = {}
    if x is not None:
        out["buffer"] = _out(out.get("buffer"), (max(R_max, 1), d), x.dtype, dev, "buffer")
        if out["buffer"].shape[-1] != d:
            raise ValueError("buffer rows must hold d = %d elements" % d)
    else:
        out.setdefault("buffer", None)
    out["row_map"] = _out(out.get("row_map"), (T, k), torch.int32, dev, "row_map")
    out["row_token"] = _out(out.get("row_token"), (max(R_max, 1),), torch.int32, dev, "row_token")
    out["counts"] = _out(out.get("counts"), (E,), torch.int32, dev, "counts")
    out["offsets"] = _out(out.get("offsets"), ((G if G else E) + 1,), torch.int32, dev, "offsets")
    out["dropped"] = _out(out.get("dropped"), (1,), torch.int32, dev, "dropped")
    workspace = (_ws(permute_workspace_bytes(T, k, E, G), dev) if workspace is None
                 else _buf(workspace, None, 0, "workspace", dev))
    _check("moe_permute", lib().moe_permute(
        _p(x), dtype, T, d, _p(expert_idx), k, E, float(capacity_factor), _p(group_of_expert), G,
        _p(out["buffer"] if x is not None else None), _p(out["row_map"]), _p(out["row_token"]), _p(out["counts"]),
        _p(out["offsets"]), _p(out["dropped"]), _p(workspace), _ws_bytes(workspace), _stream(stream)))
    out["R_max"] = R_max
    return out


def gather_rows(x: torch.Tensor, tok_ptr: torch.Tensor, tok_row: torch.Tensor, R: int, buffer=None, stream=None):
    _dev(x, None, "x")
    T, d = x.shape
    dev = x.device
    _buf(tok_ptr, torch.int32, T + 1, "tok_ptr", dev)
    _buf(tok_row, torch.int32, 0, "tok_row", dev)
    buffer = _out(buffer, (R, d), x.dtype, dev, "buffer")
    _check("moe_gather_rows", lib().moe_gather_rows(_p(x), _act_dtype(x), T, d, _p(tok_ptr), _p(tok_row), R,
                                                    _p(buffer), _stream(stream)))
    return buffer


# --------------------------------------------------------- expert MLPs
def expert_ffn_workspace_bytes(R_max: int, d: int, F: int, dtype: torch.dtype) -> int:
    return int(lib().moe_expert_ffn_workspace_bytes(R_max, d, F, MOE_BF16 if dtype == torch.bfloat16 else MOE_F32))


def expert_ffn(buffer: torch.Tensor, offsets: torch.Tensor, W1: torch.Tensor, W3: Optional[torch.Tensor],
               W2: torch.Tensor, act: str = "swiglu", y=None, workspace=None, stream=None):
    _dev(buffer, None, "buffer")
    dev = buffer.device
    dtype = _act_dtype(buffer)
    R_max, d = buffer.shape
    E, F, d1 = W1.shape
    _buf(offsets, torch.int32, E + 1, "offsets", dev)
    if d1 != d or tuple(W2.shape) != (E, d, F) or (W3 is not None and tuple(W3.shape) != (E, F, d)):
        raise ValueError("weight shapes: W1 and W3 [E,F,d], W2 [E,d,F]")
    for name, w in (("W1", W1), ("W2", W2)) + ((("W3", W3),) if W3 is not None else ()):
        _buf(w, buffer.dtype, 0, name, dev)
    if act not in ("swiglu", "gelu"):
        raise ValueError("act must be 'swiglu' or 'gelu'")
    a = MOE_ACT_SWIGLU if act == "swiglu" else MOE_ACT_GELU
    y = _out(y, (R_max, d), buffer.dtype, dev, "y")
    if y.shape[-1] != d:
        raise ValueError("y rows must hold d = %d elements" % d)
    workspace = (_ws(expert_ffn_workspace_bytes(R_max, d, F, buffer.dtype), dev) if workspace is None
                 else _buf(workspace, None, 0, "workspace", dev))
    _check("moe_expert_ffn", lib().moe_expert_ffn(
        _p(buffer), dtype, R_max, d, F, E, _p(offsets), _p(W1), _p(W3), _p(W2), a, _p(y), _p(workspace),
        _ws_bytes(workspace), _stream(stream)))
    return y


# ----------------------------------------------------- unpermutation
def unpermute(y: torch.Tensor, row_map: torch.Tensor, gate: torch.Tensor, shared: Optional[torch.Tensor] = None,
              out_dtype: Optional[torch.dtype] = None, out=None, stream=None):
    _dev(y, None, "y")
    dev = y.device
    _dev(row_map, torch.int32, "row_map")
    T, k = row_map.shape
    d = y.shape[1]
    _buf(row_map, torch.int32, T * k, "row_map", dev)
    _buf(gate, torch.float32, T * k, "gate", dev)
    out_dtype = out_dtype or (out.dtype if out is not None else y.dtype)
    if shared is not None:
        _buf(shared, y.dtype, T * d, "shared", dev)
    out = _out(out, (T, d), out_dtype, dev, "out")
    _check("moe_unpermute", lib().moe_unpermute(
        _p(y), _act_dtype(y), y.shape[0], T, d, k, _p(row_map), _p(gate), _p(shared), _p(out), _act_dtype(out),
        _stream(stream)))
    return out


# ------------------------------------------------ group-major expert path
def copy_slot_rows(src: torch.Tensor, src_row: torch.Tensor, dst_row: torch.Tensor, dst: torch.Tensor, stream=None):
    """dst[dst_row[s]] = src[src_row[s]] for the slots where both are >= 0."""
    _dev(src, None, "src")
    _dev(dst, src.dtype, "dst")
    _dev(src_row, torch.int32, "src_row")
    _dev(dst_row, torch.int32, "dst_row")
    if src_row.numel() != dst_row.numel() or src.shape[1:] != dst.shape[1:]:
        raise ValueError("copy_slot_rows: row maps or row sizes differ")
    _check("moe_copy_slot_rows", lib().moe_copy_slot_rows(
        _p(src), _act_dtype(src), src.shape[0], src.shape[1], _p(src_row), _p(dst_row), src_row.numel(), _p(dst),
        dst.shape[0], _stream(stream)))
    return dst


def group_precombine(y_e: torch.Tensor, row_map_e: torch.Tensor, row_map_g: torch.Tensor, gate: torch.Tensor,
                     y_g: torch.Tensor, stream=None):
    """y_g[r] = sum of gate * y_e over the token's slots that map to group row r."""
    _dev(y_e, None, "y_e")
    _dev(y_g, y_e.dtype, "y_g")
    for name, a, dt in (("row_map_e", row_map_e, torch.int32), ("row_map_g", row_map_g, torch.int32),
                        ("gate", gate, torch.float32)):
        _dev(a, dt, name)
    T, k = row_map_g.shape
    if tuple(row_map_e.shape) != (T, k) or tuple(gate.shape) != (T, k):
        raise ValueError("group_precombine: row_map_e, row_map_g and gate must all be [T, k]")
    _check("moe_group_precombine", lib().moe_group_precombine(
        _p(y_e), _act_dtype(y_e), y_e.shape[0], T, y_e.shape[1], k, _p(row_map_e), _p(row_map_g), _p(gate),
        _p(y_g), y_g.shape[0], _stream(stream)))
    return y_g


def unpermute_groups(y_g: torch.Tensor, row_map_g: torch.Tensor, shared: Optional[torch.Tensor] = None,
                     out_dtype: Optional[torch.dtype] = None, out=None, stream=None):
    """out[t] = sum of the token's distinct group rows (+ shared[t])."""
    _dev(y_g, None, "y_g")
    dev = y_g.device
    _buf(row_map_g, torch.int32, 0, "row_map_g", dev)
    T, k = row_map_g.shape
    d = y_g.shape[1]
    if shared is not None:
        _buf(shared, y_g.dtype, T * d, "shared", dev)
    out = _out(out, (T, d), out_dtype or (out.dtype if out is not None else y_g.dtype), dev, "out")
    _check("moe_unpermute_groups", lib().moe_unpermute_groups(
        _p(y_g), _act_dtype(y_g), y_g.shape[0], T, d, k, _p(row_map_g), _p(shared), _p(out), _act_dtype(out),
        _stream(stream)))
    return out


def unpermute_ec(y: torch.Tensor, tok_ptr: torch.Tensor, tok_row: torch.Tensor, ec_gate: torch.Tensor,
                 out_dtype: Optional[torch.dtype] = None, out=None, stream=None):
    _dev(y, None, "y")
    dev = y.device
    _buf(tok_ptr, torch.int32, 1, "tok_ptr", dev)
    _buf(tok_row, torch.int32, 0, "tok_row", dev)
    _buf(ec_gate, torch.float32, 0, "ec_gate", dev)
    T = tok_ptr.numel() - 1
    d = y.shape[1]
    out_dtype = out_dtype or (out.dtype if out is not None else y.dtype)
    out = _out(out, (T, d), out_dtype, dev, "out")
    _check("moe_unpermute_ec", lib().moe_unpermute_ec(
        _p(y), _act_dtype(y), y.shape[0], T, d, _p(tok_ptr), _p(tok_row), _p(ec_gate), _p(out), _act_dtype(out),
        _stream(stream)))
    return out


# ---------------------------------------------------------- statistics
def coselect(expert_idx: torch.Tensor, E: int, into: Optional[torch.Tensor] = None, stream=None):
    _dev(expert_idx, torch.int32, "expert_idx")
    T, k = expert_idx.shape
    if into is None:
        into = torch.zeros((E, E), dtype=torch.int32, device=expert_idx.device)
    _buf(into, torch.int32, E * E, "into", expert_idx.device)
    _check("moe_coselect", lib().moe_coselect(_p(expert_idx), T, k, E, _p(into), _stream(stream)))
    return into


def transition(idx1: torch.Tensor, idx2: torch.Tensor, E: int, into: Optional[torch.Tensor] = None, stream=None):
    _dev(idx1, torch.int32, "idx1")
    _dev(idx2, torch.int32, "idx2")
    T, k1 = idx1.shape
    T2, k2 = idx2.shape
    if T != T2:
        raise ValueError("idx1 and idx2 need the same token count")
    if into is None:
        into = torch.zeros((E, E), dtype=torch.int32, device=idx1.device)
    _buf(idx2, torch.int32, 0, "idx2", idx1.device)
    _buf(into, torch.int32, E * E, "into", idx1.device)
    _check("moe_transition", lib().moe_transition(_p(idx1), k1, _p(idx2), k2, T, E, _p(into), _stream(stream)))
    return into


# ------------------------------------------- placement and shuffling
def place_experts(cosel: torch.Tensor, G: int, out=None, stream=None):
    _dev(cosel, torch.int32, "cosel")
    E = cosel.shape[0]
    _buf(cosel, torch.int32, E * E, "cosel")
    out = _out(out, (E,), torch.int32, cosel.device, "out")
    _check("moe_place_experts", lib().moe_place_experts(_p(cosel), E, G, _p(out), _stream(stream)))
    return out


def group_affinity(trans: torch.Tensor, group_of_expert: torch.Tensor, G: int, out=None, stream=None):
    _dev(trans, torch.int32, "trans")
    E = trans.shape[0]
    _buf(trans, torch.int32, E * E, "trans")
    _buf(group_of_expert, torch.int32, E, "group_of_expert", trans.device)
    out = _out(out, (E, G), torch.int64, trans.device, "out")
    _check("moe_group_affinity", lib().moe_group_affinity(_p(trans), E, _p(group_of_expert), G, _p(out),
                                                          _stream(stream)))
    return out


def predict_home(idx1: torch.Tensor, affinity: torch.Tensor, out=None, stream=None):
    _dev(idx1, torch.int32, "idx1")
    _buf(affinity, torch.int64, 0, "affinity", idx1.device)
    T, k1 = idx1.shape
    E, G = affinity.shape
    out = _out(out, (T,), torch.int32, idx1.device, "out")
    _check("moe_predict_home", lib().moe_predict_home(_p(idx1), T, k1, _p(affinity), E, G, _p(out), _stream(stream)))
    return out


def count_local(expert_idx: torch.Tensor, group_of_expert: torch.Tensor, G: int, home=None, into=None,
                stream=None):
    _dev(expert_idx, torch.int32, "expert_idx")
    dev = expert_idx.device
    _buf(group_of_expert, torch.int32, 0, "group_of_expert", dev)
    T, k = expert_idx.shape
    E = group_of_expert.numel()
    if home is not None:
        _buf(home, torch.int32, T, "home", dev)
    if into is None:
        into = torch.zeros(1, dtype=torch.int64, device=dev)
    _buf(into, torch.int64, 1, "into", dev)
    _check("moe_count_local", lib().moe_count_local(_p(expert_idx), T, k, _p(group_of_expert), E, G, _p(home),
                                                    _p(into), _stream(stream)))
    return into


def device_error(clear: bool = True) -> int:
    """Device fault word of the current device (synchronises): 0 if clean."""
    return int(lib().moe_device_error(int(bool(clear))))


def selftest_bounded_wait(arrive: bool, limit_ns: int, stream=None) -> torch.Tensor:
    """Runs the bounded-wait check kernel: [completed (1/0), microseconds waited]."""
    out = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    _check("moe_selftest_bounded_wait", lib().moe_selftest_bounded_wait(int(bool(arrive)), int(limit_ns), _p(out),
                                                                        _stream(stream)))
    return out


def kernel_launches() -> int:
    """Kernels libmoe has launched in this process so far."""
    return int(lib().moe_kernel_launches())
