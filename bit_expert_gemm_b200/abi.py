"""ctypes binding of libmoe_b200.so (include/moe.h), one Python function per
C entry point with the same name.

The functions only marshal arguments: they check dtypes / devices / shapes of
torch tensors, allocate outputs with torch when the caller does not pass
them, and call the C ABI on torch's current CUDA stream.  Every step of the
computation runs in the library's kernels.  If the library is missing the
import of this module succeeds but every call raises, so a missing build can
never fall back to another implementation.
"""

from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "moe.h")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT = range(6)
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT"}
MOE_DTYPE_BF16, MOE_DTYPE_F16 = 0, 1
(MOE_OP_ROUTE_TOPK, MOE_OP_PERMUTE, MOE_OP_SWIGLU_BF16, MOE_OP_SWIGLU_AWQ_G32, MOE_OP_SWIGLU_NVFP4, MOE_OP_REFILL,
 MOE_OP_NVFP4_QUANTIZE, MOE_OP_EXPERTS_BF16, MOE_OP_ROUTE_PERMUTE, MOE_OP_EXPERTS_AWQ_G32) = range(10)


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn}: {STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_SIGS = {
    "moe_abi_version": (_I, []),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_device_status": (_I, [_I, _P]),
    "moe_selftest_bounded_wait": (_I, [_I, _P, _P]),
    "moe_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "moe_route_topk": (_I, [_P, _I, _I, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "moe_route_permute": (_I, [_P, _I, _I, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_norm_route_permute": (_I, [_P, _I, _I, _P, ctypes.c_float, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P,
                                    _P, _P, _P, _P, _SZ, _P]),
    "moe_permute": (_I, [_P, _I, _I, _I, _P, _P, _P, _P, _SZ, _P]),
    "moe_ep_plan": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "moe_gather_rows": (_I, [_P, _I, _I, _P, _I, _P, _P]),
    "moe_permute_noalloc": (_I, [_P, _I, _I, _I, _P, _P, _P, _P]),
    "moe_grouped_swiglu_bf16": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _I, _I, _P, _P, _SZ, _P]),
    "moe_experts_bf16": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _I, _I, _P, _P, _P, _SZ, _P]),
    "moe_experts_awq_g32": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P,
                                 _P, _SZ, _P]),
    "moe_experts_awq_g32_prepacked": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I,
                                           _P, _P, _P, _SZ, _P]),
    "moe_awq_packed_bytes": (_SZ, [_I, _I, _I]),
    "moe_awq_prepack_g32": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P, _SZ, _P]),
    "moe_grouped_swiglu_awq_g32": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _I, _I, _P, _P, _SZ,
                                        _P]),
    "moe_awq_dequant_g32": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "moe_nvfp4_quantize": (_I, [_P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_grouped_swiglu_nvfp4": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P, _SZ,
                                      _P]),
    "moe_nvfp4_packed_sf_bytes": (_SZ, [_I, _I, _I, _I]),
    "moe_nvfp4_prepack_sf": (_I, [_P, _I, _I, _I, _I, _P, _SZ, _P]),
    "moe_grouped_swiglu_nvfp4_prepacked": (_I, [_P, _P, _P, _I, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _I,
                                                _P, _P, _SZ, _P]),
    "moe_combine": (_I, [_P, _I, _P, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P]),
    "razor_refill_rms_accumulate": (_I, [_P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _I, _P, _SZ, _P]),
    "razor_select": (_I, [_P, _P, _I, _I, _P, _P, _P, _P]),
    "razor_router_norm": (_I, [_P, _I, _I, _I, _P, _P, _P]),
    "moe_shared_gate": (_I, [_P, _I, _I, _P, _I, _P, _P]),
    "moe_rmsnorm": (_I, [_P, _I, _I, _P, ctypes.c_float, _I, _P, _P]),
    "razor_slice": (_I, [_P, _I, _SZ, _P, _I, _P, _P]),
}

_lib = None


def header_symbols():
    """Names of the entry points declared in include/moe.h."""
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b((?:moe|razor)_\w+)\s*\(", src, flags=re.M)))


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m bit_expert_gemm_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _call(name: str, *args) -> None:
    lib = load()
    rc = getattr(lib, name)(*args)
    if rc != MOE_OK:
        raise MoEError(name, rc, lib.moe_last_error().decode())


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MOE_DTYPE_BF16
    if t.dtype == torch.float16:
        return MOE_DTYPE_F16
    raise ValueError(f"16-bit tensor expected, got {t.dtype}")


def _need(t: torch.Tensor, dtype, name: str):
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")


def abi_version() -> int:
    return load().moe_abi_version()


def moe_device_status(clear: bool = True, stream=None) -> int:
    return load().moe_device_status(int(clear), _stream(stream))


def moe_selftest_bounded_wait(limit_us: int, result: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Launches the bounded-wait self-test (a wait that nothing completes runs
    out after limit_us); returns result [2] int32 (1 = that role's wait gave
    up).  Read moe_device_status afterwards: MOE_ERR_TIMEOUT."""
    if result is None:
        result = torch.zeros(2, dtype=torch.int32, device="cuda")
    _need(result, torch.int32, "result")
    _call("moe_selftest_bounded_wait", int(limit_us), _p(result), _stream(stream))
    return result


def moe_workspace_size(op: int, T: int, H: int, E: int, k_slots: int, I: int) -> int:
    return int(load().moe_workspace_size(op, T, H, E, k_slots, I))


def workspace(op: int, T: int, H: int, E: int, k_slots: int, I: int, device) -> torch.Tensor:
    return torch.empty(max(256, moe_workspace_size(op, T, H, E, k_slots, I)), dtype=torch.uint8, device=device)


def moe_route_topk(x, w_router, bias, k: int, extra: int = 0, topk_idx=None, topk_w=None, topk_logit=None, ws=None,
                   stream=None):
    T, H = x.shape
    E = w_router.shape[0]
    dev = x.device
    if topk_idx is None:
        topk_idx = torch.empty((T, k + extra), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    if topk_logit is None:
        topk_logit = torch.empty((T, k + extra), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(MOE_OP_ROUTE_TOPK, T, H, E, k + extra, 0, dev)
    if bias is not None:
        _need(bias, torch.float32, "bias")
    _call("moe_route_topk", _p(x), T, H, _p(w_router), _p(bias), E, k, extra, _dtype_code(x), _p(topk_idx),
          _p(topk_w), _p(topk_logit), _p(ws), ws.numel(), _stream(stream))
    return topk_idx, topk_w, topk_logit


def moe_route_permute(x, w_router, bias, k: int, extra: int = 0, topk_idx=None, topk_w=None, topk_logit=None,
                      expert_offsets=None, row_token=None, slot_row=None, ws=None, stream=None):
    """moe_route_topk then moe_permute of its selection, in one call (one
    kernel for T <= 128).  Returns (topk_idx, topk_w, topk_logit,
    expert_offsets, row_token, slot_row)."""
    T, H = x.shape
    E = w_router.shape[0]
    ks = k + extra
    dev = x.device
    if topk_idx is None:
        topk_idx = torch.empty((T, ks), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    if topk_logit is None:
        topk_logit = torch.empty((T, ks), dtype=torch.float32, device=dev)
    if expert_offsets is None:
        expert_offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    if row_token is None:
        row_token = torch.empty((T * ks,), dtype=torch.int32, device=dev)
    if slot_row is None:
        slot_row = torch.empty((T, ks), dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(MOE_OP_ROUTE_PERMUTE, T, H, E, ks, 0, dev)
    if bias is not None:
        _need(bias, torch.float32, "bias")
    _call("moe_route_permute", _p(x), T, H, _p(w_router), _p(bias), E, k, extra, _dtype_code(x), _p(topk_idx),
          _p(topk_w), _p(topk_logit), _p(expert_offsets), _p(row_token), _p(slot_row), _p(ws), ws.numel(),
          _stream(stream))
    return topk_idx, topk_w, topk_logit, expert_offsets, row_token, slot_row


def moe_norm_route_permute(x, norm_w, w_router, bias, k: int, extra: int = 0, eps: float = 1e-6,
                           w_shared_gate=None, x_norm=None, shared_gate=None, topk_idx=None, topk_w=None,
                           topk_logit=None, expert_offsets=None, row_token=None, slot_row=None, ws=None, stream=None):
    """Pre-MoE RMSNorm (gain 1 + norm_w) into x_norm, the shared-expert gate
    when w_shared_gate is given, and moe_route_permute of x_norm, in one
    call.  Returns (x_norm, shared_gate or None, topk_idx, topk_w,
    topk_logit, expert_offsets, row_token, slot_row)."""
    T, H = x.shape
    E = w_router.shape[0]
    ks = k + extra
    dev = x.device
    if norm_w.dtype != x.dtype or tuple(norm_w.shape) != (H,):
        raise ValueError("moe_norm_route_permute: norm_w must be [H] of x's dtype")
    if w_shared_gate is not None and (w_shared_gate.dtype != x.dtype or tuple(w_shared_gate.shape) != (H,)):
        raise ValueError("moe_norm_route_permute: w_shared_gate must be [H] of x's dtype")
    if x_norm is None:
        x_norm = torch.empty_like(x)
    if w_shared_gate is not None and shared_gate is None:
        shared_gate = torch.empty((T,), dtype=torch.float32, device=dev)
    if w_shared_gate is None:
        shared_gate = None
    if topk_idx is None:
        topk_idx = torch.empty((T, ks), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    if topk_logit is None:
        topk_logit = torch.empty((T, ks), dtype=torch.float32, device=dev)
    if expert_offsets is None:
        expert_offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    if row_token is None:
        row_token = torch.empty((T * ks,), dtype=torch.int32, device=dev)
    if slot_row is None:
        slot_row = torch.empty((T, ks), dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(MOE_OP_ROUTE_PERMUTE, T, H, E, ks, 0, dev)
    if bias is not None:
        _need(bias, torch.float32, "bias")
    _call("moe_norm_route_permute", _p(x), T, H, _p(norm_w), float(eps), _p(w_shared_gate), _p(w_router), _p(bias), E,
          k, extra, _dtype_code(x), _p(x_norm), _p(shared_gate), _p(topk_idx), _p(topk_w), _p(topk_logit),
          _p(expert_offsets), _p(row_token), _p(slot_row), _p(ws), ws.numel(), _stream(stream))
    return x_norm, shared_gate, topk_idx, topk_w, topk_logit, expert_offsets, row_token, slot_row


def moe_ep_plan(expert_offsets, world: int, rows: int, row_local_expert=None, send_counts=None, stream=None):
    """Expert-parallel dispatch plan of `rows` permuted rows: the local
    expert index of each row at its destination rank and the rows per rank."""
    _need(expert_offsets, torch.int32, "expert_offsets")
    E = expert_offsets.numel() - 1
    dev = expert_offsets.device
    if row_local_expert is None:
        row_local_expert = torch.empty((rows,), dtype=torch.int32, device=dev)
    if send_counts is None:
        send_counts = torch.empty((world,), dtype=torch.int32, device=dev)
    _call("moe_ep_plan", _p(expert_offsets), E, world, rows, _p(row_local_expert), _p(send_counts), _stream(stream))
    return row_local_expert, send_counts


def moe_gather_rows(src, index, out=None, stream=None):
    """out[r] = src[index[r]] for whole 16-bit rows."""
    _need(index, torch.int32, "index")
    src_rows, H = src.shape
    rows = index.numel()
    if src.element_size() != 2:
        raise ValueError("moe_gather_rows: 16-bit rows expected")
    if out is None:
        out = torch.empty((rows, H), dtype=src.dtype, device=src.device)
    _call("moe_gather_rows", _p(src), src_rows, H, _p(index), rows, _p(out), _stream(stream))
    return out


def moe_permute(topk_idx, E: int, expert_offsets=None, row_token=None, slot_row=None, ws=None, stream=None):
    _need(topk_idx, torch.int32, "topk_idx")
    T, ks = topk_idx.shape
    dev = topk_idx.device
    if expert_offsets is None:
        expert_offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    if row_token is None:
        row_token = torch.empty((T * ks,), dtype=torch.int32, device=dev)
    if slot_row is None:
        slot_row = torch.empty((T, ks), dtype=torch.int32, device=dev)
    if ws is None:
        ws = workspace(MOE_OP_PERMUTE, T, 0, E, ks, 0, dev)
    _call("moe_permute", _p(topk_idx), T, ks, E, _p(expert_offsets), _p(row_token), _p(slot_row), _p(ws), ws.numel(),
          _stream(stream))
    return expert_offsets, row_token, slot_row


def moe_permute_noalloc(topk_idx, E: int, expert_offsets=None, row_token=None, slot_row=None, stream=None):
    """moe_permute with the library's fixed scratch array instead of a
    workspace, for callers that cannot allocate device memory."""
    _need(topk_idx, torch.int32, "topk_idx")
    T, ks = topk_idx.shape
    dev = topk_idx.device
    if expert_offsets is None:
        expert_offsets = torch.empty((E + 1,), dtype=torch.int32, device=dev)
    if row_token is None:
        row_token = torch.empty((T * ks,), dtype=torch.int32, device=dev)
    if slot_row is None:
        slot_row = torch.empty((T, ks), dtype=torch.int32, device=dev)
    _call("moe_permute_noalloc", _p(topk_idx), T, ks, E, _p(expert_offsets), _p(row_token), _p(slot_row),
          _stream(stream))
    return expert_offsets, row_token, slot_row


def moe_grouped_swiglu_bf16(x, row_token, expert_offsets, rows: int, w_gate_up, w_down, out_fp32: bool = False, f=None,
                            ws=None, stream=None):
    T, H = x.shape
    E, I2, _ = w_gate_up.shape
    I = I2 // 2
    dev = x.device
    if f is None:
        f = torch.empty((rows, H), dtype=torch.float32 if out_fp32 else x.dtype, device=dev)
    if ws is None:
        ws = workspace(MOE_OP_SWIGLU_BF16, rows, H, E, 1, I, dev)
    _need(expert_offsets, torch.int32, "expert_offsets")
    _call("moe_grouped_swiglu_bf16", _p(x), _p(row_token), _p(expert_offsets), T, rows, H, I, E, _p(w_gate_up),
          _p(w_down), _dtype_code(x), int(out_fp32), _p(f), _p(ws), ws.numel(), _stream(stream))
    return f


def moe_experts_bf16(x, row_token, expert_offsets, rows: int, w_gate_up, w_down, w_sh_gate_up, w_sh_down,
                     out_fp32: bool = False, f=None, shared_out=None, ws=None, stream=None):
    """Routed experts (f [rows, H]) and the shared expert (shared_out [T, H]) in one call."""
    T, H = x.shape
    E, I2, _ = w_gate_up.shape
    I = I2 // 2
    dev = x.device
    if f is None:
        f = torch.empty((rows, H), dtype=torch.float32 if out_fp32 else x.dtype, device=dev)
    if shared_out is None:
        shared_out = torch.empty((T, H), dtype=x.dtype, device=dev)
    if ws is None:
        ws = workspace(MOE_OP_EXPERTS_BF16, T, H, E, max(1, rows // max(T, 1)), I, dev)
    _call("moe_experts_bf16", _p(x), _p(row_token), _p(expert_offsets), T, rows, H, I, E, _p(w_gate_up), _p(w_down),
          _p(w_sh_gate_up), _p(w_sh_down), _dtype_code(x), int(out_fp32), _p(f), _p(shared_out), _p(ws), ws.numel(),
          _stream(stream))
    return f, shared_out


def moe_experts_awq_g32(x, row_token, expert_offsets, rows: int, qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d, w_sh_gate_up,
                        w_sh_down, out_fp32: bool = False, f=None, shared_out=None, ws=None, stream=None):
    """Routed AWQ experts (f [rows, H]) and the 16-bit shared expert (shared_out [T, H]) in one call; x FP16,
    or BF16 for the BF16 mode (scales rounded to BF16, BF16 weights; the shared expert in x's dtype)."""
    T, H = x.shape
    E = qw_gu.shape[0]
    I = qw_gu.shape[2] * 8 // 2
    dev = x.device
    dcode = _dtype_code(x)
    if f is None:
        f = torch.empty((rows, H), dtype=torch.float32 if out_fp32 else x.dtype, device=dev)
    if shared_out is None:
        shared_out = torch.empty((T, H), dtype=x.dtype, device=dev)
    if ws is None:
        ws = workspace(MOE_OP_EXPERTS_AWQ_G32, T, H, E, max(1, rows // max(T, 1)), I, dev)
    _call("moe_experts_awq_g32", _p(x), _p(row_token), _p(expert_offsets), T, rows, H, I, E, _p(qw_gu), _p(qz_gu),
          _p(sc_gu), _p(qw_d), _p(qz_d), _p(sc_d), _p(w_sh_gate_up), _p(w_sh_down), dcode, int(out_fp32), _p(f),
          _p(shared_out), _p(ws), ws.numel(), _stream(stream))
    return f, shared_out


def moe_awq_prepack_g32(qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d, out=None, stream=None):
    """Tile-packed copy of one layer's routed AWQ weights (uint8 device buffer) for moe_experts_awq_g32_prepacked."""
    E, H = qw_gu.shape[0], qw_gu.shape[1]
    I = qw_gu.shape[2] * 8 // 2
    nbytes = int(load().moe_awq_packed_bytes(E, H, I))
    if nbytes == 0:
        raise ValueError(f"moe_awq_prepack_g32: unsupported sizes E={E} H={H} I={I}")
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=qw_gu.device)
    _call("moe_awq_prepack_g32", _p(qw_gu), _p(qz_gu), _p(sc_gu), _p(qw_d), _p(qz_d), _p(sc_d), E, H, I, _p(out),
          out.numel(), _stream(stream))
    return out


def moe_experts_awq_g32_prepacked(x, row_token, expert_offsets, rows: int, qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d,
                                  awq_packed, w_sh_gate_up, w_sh_down, out_fp32: bool = False, f=None,
                                  shared_out=None, ws=None, stream=None):
    """moe_experts_awq_g32 with the routed weights also tile-packed: the decode kernel reads only the packed
    copy, the grouped prefill GEMMs read it for 128- and 256-column tiles and then gather the x rows
    themselves."""
    T, H = x.shape
    E = qw_gu.shape[0]
    I = qw_gu.shape[2] * 8 // 2
    dev = x.device
    dcode = _dtype_code(x)
    if f is None:
        f = torch.empty((rows, H), dtype=torch.float32 if out_fp32 else x.dtype, device=dev)
    if shared_out is None:
        shared_out = torch.empty((T, H), dtype=x.dtype, device=dev)
    if ws is None:
        ws = workspace(MOE_OP_EXPERTS_AWQ_G32, T, H, E, max(1, rows // max(T, 1)), I, dev)
    _call("moe_experts_awq_g32_prepacked", _p(x), _p(row_token), _p(expert_offsets), T, rows, H, I, E, _p(qw_gu),
          _p(qz_gu), _p(sc_gu), _p(qw_d), _p(qz_d), _p(sc_d), _p(awq_packed), _p(w_sh_gate_up), _p(w_sh_down),
          dcode, int(out_fp32), _p(f), _p(shared_out), _p(ws), ws.numel(), _stream(stream))
    return f, shared_out


def moe_grouped_swiglu_awq_g32(x, row_token, expert_offsets, rows: int, qw_gu, qz_gu, sc_gu, qw_d, qz_d, sc_d,
                               out_fp32: bool = False, f=None, ws=None, stream=None):
    T, H = x.shape
    E = qw_gu.shape[0]
    I = qw_gu.shape[2] * 8 // 2
    dev = x.device
    dcode = _dtype_code(x)  # FP16, or BF16 for the BF16 mode
    if f is None:
        f = torch.empty((rows, H), dtype=torch.float32 if out_fp32 else x.dtype, device=dev)
    if ws is None:
        ws = workspace(MOE_OP_SWIGLU_AWQ_G32, rows, H, E, 1, I, dev)
    _call("moe_grouped_swiglu_awq_g32", _p(x), _p(row_token), _p(expert_offsets), T, rows, H, I, E, _p(qw_gu),
          _p(qz_gu), _p(sc_gu), _p(qw_d), _p(qz_d), _p(sc_d), dcode, int(out_fp32), _p(f), _p(ws), ws.numel(),
          _stream(stream))
    return f


def moe_awq_dequant_g32(qweight, qzeros, scales, out=None, dtype=torch.float16, stream=None):
    """qweight [B, K, N/8] (or [K, N/8]) -> [B, K, N] of dtype (FP16, or BF16
    for the BF16 mode): the exact weights the AWQ GEMM multiplies with."""
    squeeze = qweight.dim() == 2
    qw = qweight.unsqueeze(0) if squeeze else qweight
    qz = qzeros.unsqueeze(0) if squeeze else qzeros
    sc = scales.unsqueeze(0) if squeeze else scales
    B, K, W = qw.shape
    N = W * 8
    _need(qw, torch.int32, "qweight")
    _need(qz, torch.int32, "qzeros")
    _need(sc, torch.float16, "scales")
    if out is None:
        out = torch.empty((B, K, N), dtype=dtype, device=qw.device)
    _call("moe_awq_dequant_g32", _p(qw), _p(qz), _p(sc), B, K, N, _dtype_code(out), _p(out), _stream(stream))
    return out[0] if squeeze else out


def moe_nvfp4_quantize(v, global_scale_in=None, codes=None, sf=None, global_scale_out=None, ws=None, stream=None):
    """v [batch, rows, K] (or [rows, K]) 16-bit -> (codes [.., K/2] u8, sf [.., K/16] u8, gs [batch] f32)."""
    squeeze = v.dim() == 2
    v3 = v.unsqueeze(0) if squeeze else v
    B, R, K = v3.shape
    dev = v.device
    if codes is None:
        codes = torch.empty((B, R, K // 2), dtype=torch.uint8, device=dev)
    if sf is None:
        sf = torch.empty((B, R, K // 16), dtype=torch.uint8, device=dev)
    if global_scale_out is None:
        global_scale_out = torch.empty((B,), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.empty(max(256, int(load().moe_workspace_size(MOE_OP_NVFP4_QUANTIZE, R, K, 0, 0, 0)) * max(1, B)),
                         dtype=torch.uint8, device=dev)
    _call("moe_nvfp4_quantize", _p(v3), B, R, K, _dtype_code(v), _p(global_scale_in), _p(codes), _p(sf),
          _p(global_scale_out), _p(ws), ws.numel(), _stream(stream))
    if squeeze:
        return codes[0], sf[0], global_scale_out
    return codes, sf, global_scale_out


def moe_grouped_swiglu_nvfp4(x, row_token, expert_offsets, rows: int, w_gu, sf_gu, gs_gu, w_d, sf_d, gs_d,
                             act_gs_in=None, act_gs_out=None, out_fp32: bool = False, f=None, ws=None, stream=None):
    T, H = x.shape
    E = w_gu.shape[0]
    I = w_gu.shape[1] // 2
    dev = x.device
    if f is None:
        f = torch.empty((rows, H), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=dev)
    if ws is None:
        ws = workspace(MOE_OP_SWIGLU_NVFP4, rows, H, E, 1, I, dev)
    _call("moe_grouped_swiglu_nvfp4", _p(x), _p(row_token), _p(expert_offsets), T, rows, H, I, E, _p(w_gu),
          _p(sf_gu), _p(gs_gu), _p(w_d), _p(sf_d), _p(gs_d), _p(act_gs_in), _p(act_gs_out), int(out_fp32), _p(f),
          _p(ws), ws.numel(), _stream(stream))
    return f


def moe_nvfp4_prepack_sf(sf, swiglu: bool, out=None, stream=None):
    """Rearrange one projection's weight scales sf [E, rows, K/16] into the FP4 GEMM's tile order."""
    E, R, K16 = sf.shape
    K = K16 * 16
    nbytes = int(load().moe_nvfp4_packed_sf_bytes(E, R, K, int(swiglu)))
    if nbytes == 0:
        raise ValueError(f"moe_nvfp4_prepack_sf: unsupported sizes E={E} rows={R} K={K}")
    if out is None:
        out = torch.empty(nbytes, dtype=torch.uint8, device=sf.device)
    _call("moe_nvfp4_prepack_sf", _p(sf), E, R, K, int(swiglu), _p(out), out.numel(), _stream(stream))
    return out


def moe_grouped_swiglu_nvfp4_prepacked(x, row_token, expert_offsets, rows: int, w_gu, sf_gu_packed, gs_gu, w_d,
                                       sf_d_packed, gs_d, act_gs_in=None, act_gs_out=None, out_fp32: bool = False,
                                       f=None, ws=None, stream=None):
    T, H = x.shape
    E = w_gu.shape[0]
    I = w_gu.shape[1] // 2
    dev = x.device
    if f is None:
        f = torch.empty((rows, H), dtype=torch.float32 if out_fp32 else torch.bfloat16, device=dev)
    if ws is None:
        ws = workspace(MOE_OP_SWIGLU_NVFP4, rows, H, E, 1, I, dev)
    _call("moe_grouped_swiglu_nvfp4_prepacked", _p(x), _p(row_token), _p(expert_offsets), T, rows, H, I, E,
          _p(w_gu), _p(sf_gu_packed), _p(gs_gu), _p(w_d), _p(sf_d_packed), _p(gs_d), _p(act_gs_in),
          _p(act_gs_out), int(out_fp32), _p(f), _p(ws), ws.numel(), _stream(stream))
    return f


def moe_combine(f, slot_row, topk_w, shared_out=None, shared_gate=None, y=None, dtype=None, stream=None):
    T, k = topk_w.shape
    ks = slot_row.shape[1]
    H = f.shape[1]
    f_fp32 = f.dtype == torch.float32
    if dtype is None:
        dtype = shared_out.dtype if shared_out is not None else (torch.bfloat16 if f_fp32 else f.dtype)
    if y is None:
        y = torch.empty((T, H), dtype=dtype, device=f.device)
    _call("moe_combine", _p(f), int(f_fp32), _p(slot_row), ks, _p(topk_w), _p(shared_out), _p(shared_gate), T, k, H,
          _dtype_code(y), _p(y), _stream(stream))
    return y


def razor_refill_rms_accumulate(f, slot_row, topk_idx, topk_logit, expert_offsets, sum_sq, count, shared_out=None,
                                y_out=None, dtype=torch.bfloat16, ws=None, stream=None):
    T, ks = slot_row.shape
    k = ks - 1
    H = f.shape[1]
    E = sum_sq.shape[0]
    _need(sum_sq, torch.float64, "sum_sq")
    _need(count, torch.int64, "count")
    if ws is None:
        ws = workspace(MOE_OP_REFILL, T, H, E, ks, 0, f.device)
    dcode = _dtype_code(y_out) if y_out is not None else (MOE_DTYPE_F16 if dtype == torch.float16 else MOE_DTYPE_BF16)
    _call("razor_refill_rms_accumulate", _p(f), int(f.dtype == torch.float32), _p(slot_row), _p(topk_idx),
          _p(topk_logit), _p(expert_offsets), T, k, H, E, _p(sum_sq), _p(count), _p(shared_out), _p(y_out), dcode,
          _p(ws), ws.numel(), _stream(stream))
    return sum_sq, count


def razor_select(sum_sq, count, keep: int, kept=None, ranking=None, score=None, stream=None):
    E = sum_sq.shape[0]
    dev = sum_sq.device
    if kept is None:
        kept = torch.empty((max(keep, 1),), dtype=torch.int32, device=dev)
    if ranking is None:
        ranking = torch.empty((E,), dtype=torch.int32, device=dev)
    if score is None:
        score = torch.empty((E,), dtype=torch.float64, device=dev)
    _call("razor_select", _p(sum_sq), _p(count), E, keep, _p(kept), _p(ranking), _p(score), _stream(stream))
    return kept[:keep], ranking, score


def moe_shared_gate(x, w_gate, gate=None, stream=None):
    """gate [T] FP32 = sigmoid(x . w_gate) for x [T, H], w_gate [H]."""
    T, H = x.shape
    if w_gate.dtype != x.dtype or tuple(w_gate.shape) != (H,):
        raise ValueError("moe_shared_gate: w_gate must be [H] of x's dtype")
    if gate is None:
        gate = torch.empty((T,), dtype=torch.float32, device=x.device)
    _need(gate, torch.float32, "gate")
    _call("moe_shared_gate", _p(x), T, H, _p(w_gate), _dtype_code(x), _p(gate), _stream(stream))
    return gate


def moe_rmsnorm(x, w, eps: float = 1e-6, y=None, stream=None):
    """Pre-MoE RMSNorm with the (1 + w) gain: y [T, H] (may be x)."""
    T, H = x.shape
    if w.dtype != x.dtype or tuple(w.shape) != (H,):
        raise ValueError("moe_rmsnorm: w must be [H] of x's dtype")
    if y is None:
        y = torch.empty_like(x)
    _call("moe_rmsnorm", _p(x), T, H, _p(w), float(eps), _dtype_code(x), _p(y), _stream(stream))
    return y


def razor_router_norm(w_router, sum_sq=None, count=None, stream=None):
    """Router-norm keep statistics: sum_sq[e] = ||w_router[e]||^2 (FP64),
    count[e] = 1, ready for razor_select."""
    E, H = w_router.shape
    dev = w_router.device
    if sum_sq is None:
        sum_sq = torch.empty((E,), dtype=torch.float64, device=dev)
    if count is None:
        count = torch.empty((E,), dtype=torch.int64, device=dev)
    _need(sum_sq, torch.float64, "sum_sq")
    _need(count, torch.int64, "count")
    _call("razor_router_norm", _p(w_router), E, H, _dtype_code(w_router), _p(sum_sq), _p(count), _stream(stream))
    return sum_sq, count


def razor_slice(src, kept, out=None, stream=None):
    """out[j] = src[kept[j]] along the leading (expert) dimension, byte-exact.
    src [E, ...] contiguous of any dtype, kept [keep] int32 on the device."""
    _need(kept, torch.int32, "kept")
    E = src.shape[0]
    keep = kept.shape[0]
    if out is None:
        out = torch.empty((keep, *src.shape[1:]), dtype=src.dtype, device=src.device)
    if out.dtype != src.dtype or tuple(out.shape) != (keep, *src.shape[1:]):
        raise ValueError("razor_slice: out must be [keep, ...] of src's dtype")
    bpe = src[0].numel() * src.element_size() if E else 0
    _call("razor_slice", _p(src), E, bpe, _p(kept), keep, _p(out), _stream(stream))
    return out
