"""Thin Python binding of libe4b (the C ABI in include/e4b.h).

Argument marshalling only: every function checks tensor placement, dtype and
shape, passes raw device pointers and sizes to the C call of the same name and
raises :class:`E4BError` on a non-OK status.  All arithmetic runs in the CUDA
library; nothing here computes on the tensors.  PyTorch supplies device memory
and streams.

The library must have been built (``python -m quantized_moe_expert_nf4_b200.build``
or ``__graft_entry__.build()``); loading fails loudly otherwise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libe4b.so")

E4B_OK = 0
STATUS_NAMES = {0: "E4B_OK", 1: "E4B_ERR_INVALID_ARGUMENT", 2: "E4B_ERR_UNSUPPORTED",
                3: "E4B_ERR_WORKSPACE", 4: "E4B_ERR_CUDA"}
E4B_F32, E4B_BF16 = 0, 1
E4B_EPI_NONE, E4B_EPI_SWIGLU = 0, 1
E4B_PATH_AUTO, E4B_PATH_DECODE, E4B_PATH_GROUPED = 0, 1, 2
E4B_QUANT_NF4, E4B_QUANT_FP4 = 0, 1
# The E4B_VERSION this binding marshals for (e4b_expert_stack's layout among others).
ABI_VERSION = 3

# Every symbol include/e4b.h declares.
EXPORTED = (
    "e4b_status_string", "e4b_last_error", "e4b_last_path", "e4b_version", "e4b_last_launches",
    "e4b_workspace_error", "e4b_workspace_clear_error",
    "e4b_timing_enable", "e4b_timing_kernels", "e4b_timing_get",
    "e4b_nf4_quantize_stack", "e4b_quantize_stack",
    "e4b_moe_route_permute_workspace_size", "e4b_moe_route_permute",
    "e4b_grouped_nf4_gemm_workspace_size", "e4b_grouped_nf4_gemm", "e4b_grouped_4bit_gemm",
    "e4b_grouped_nf4_gemm_dgrad_workspace_size", "e4b_grouped_nf4_gemm_dgrad", "e4b_grouped_4bit_gemm_dgrad",
    "e4b_grouped_lora_grads_workspace_size", "e4b_grouped_lora_grads",
    "e4b_grouped_mxfp4_gemm_workspace_size", "e4b_grouped_mxfp4_gemm",
    "e4b_moe_expert_forward_workspace_size", "e4b_moe_expert_forward",
    "e4b_moe_expert_forward_path", "e4b_moe_expert_forward_decode_noalloc",
    "e4b_moe_expert_backward_workspace_size", "e4b_moe_expert_backward",
)


class E4BError(RuntimeError):
    def __init__(self, status: int, fn: str, detail: str):
        self.status = status
        super().__init__(f"{fn}: {STATUS_NAMES.get(status, status)}: {detail}")


class ExpertStackC(ctypes.Structure):
    _fields_ = [
        ("gu_packed", ctypes.c_void_p), ("gu_absmax", ctypes.c_void_p),
        ("dn_packed", ctypes.c_void_p), ("dn_absmax", ctypes.c_void_p),
        ("lora_A", ctypes.c_void_p), ("lora_B", ctypes.c_void_p),
        ("lora_r", ctypes.c_int), ("lora_alpha", ctypes.c_float),
        ("E", ctypes.c_int64), ("H", ctypes.c_int64), ("I", ctypes.c_int64),
        ("quant_type", ctypes.c_int32),
    ]


_lib: Optional[ctypes.CDLL] = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libe4b.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libe4b.so not built at {path}: run __graft_entry__.build()")
    lib = ctypes.CDLL(path)
    i64, i32, vp, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    lib.e4b_status_string.restype = ctypes.c_char_p
    lib.e4b_status_string.argtypes = [i32]
    lib.e4b_last_error.restype = ctypes.c_char_p
    lib.e4b_last_error.argtypes = []
    lib.e4b_last_path.restype = ctypes.c_char_p
    lib.e4b_last_path.argtypes = []
    lib.e4b_version.restype = i32
    lib.e4b_version.argtypes = []
    if lib.e4b_version() != ABI_VERSION:
        raise RuntimeError(f"{path} is ABI version {lib.e4b_version()}, this binding expects {ABI_VERSION}: "
                           "rebuild it with __graft_entry__.build()")
    lib.e4b_last_launches.restype = i32
    lib.e4b_last_launches.argtypes = []
    lib.e4b_timing_enable.restype = i32
    lib.e4b_timing_enable.argtypes = [i32]
    lib.e4b_timing_kernels.restype = i32
    lib.e4b_timing_kernels.argtypes = []
    lib.e4b_timing_get.restype = i32
    lib.e4b_timing_get.argtypes = [i32, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                   ctypes.POINTER(ctypes.c_int)]
    lib.e4b_nf4_quantize_stack.restype = i32
    lib.e4b_nf4_quantize_stack.argtypes = [vp, i32, i64, i64, i64, i32, vp, vp, vp]
    lib.e4b_quantize_stack.restype = i32
    lib.e4b_quantize_stack.argtypes = [vp, i32, i64, i64, i64, i32, i32, vp, vp, vp]
    lib.e4b_moe_route_permute_workspace_size.restype = sz
    lib.e4b_moe_route_permute_workspace_size.argtypes = [i64, i64, i32]
    lib.e4b_moe_route_permute.restype = i32
    lib.e4b_moe_route_permute.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.e4b_grouped_nf4_gemm_workspace_size.restype = sz
    lib.e4b_grouped_nf4_gemm_workspace_size.argtypes = [i64, i64, i64, i32]
    lib.e4b_grouped_nf4_gemm.restype = i32
    lib.e4b_grouped_nf4_gemm.argtypes = [vp, i64, i64, vp, vp, i64, i64, vp, vp, i64, i64, vp, vp, i32,
                                         ctypes.c_float, i32, vp, i32, vp, sz, vp]
    lib.e4b_grouped_4bit_gemm.restype = i32
    lib.e4b_grouped_4bit_gemm.argtypes = [vp, i64, i64, vp, vp, i64, i64, vp, vp, i32, i64, i64, vp, vp, i32,
                                          ctypes.c_float, i32, vp, i32, vp, sz, vp]
    lib.e4b_grouped_nf4_gemm_dgrad_workspace_size.restype = sz
    lib.e4b_grouped_nf4_gemm_dgrad_workspace_size.argtypes = [i64, i64, i64, i32]
    lib.e4b_grouped_nf4_gemm_dgrad.restype = i32
    lib.e4b_grouped_nf4_gemm_dgrad.argtypes = [vp, i64, i64, vp, vp, i64, i64, vp, vp, i64, i64, vp, vp, i32,
                                               ctypes.c_float, vp, i32, vp, sz, vp]
    lib.e4b_grouped_4bit_gemm_dgrad.restype = i32
    lib.e4b_grouped_4bit_gemm_dgrad.argtypes = [vp, i64, i64, vp, vp, i64, i64, vp, vp, i32, i64, i64, vp, vp,
                                                i32, ctypes.c_float, vp, i32, vp, sz, vp]
    lib.e4b_grouped_lora_grads_workspace_size.restype = sz
    lib.e4b_grouped_lora_grads_workspace_size.argtypes = [i64, i32]
    lib.e4b_grouped_lora_grads.restype = i32
    lib.e4b_grouped_lora_grads.argtypes = [vp, i64, i64, vp, vp, i64, i64, vp, i64, i64, i64, vp, vp, i32,
                                           ctypes.c_float, vp, vp, vp, sz, vp]
    lib.e4b_grouped_mxfp4_gemm.restype = i32
    lib.e4b_grouped_mxfp4_gemm_workspace_size.restype = sz
    lib.e4b_grouped_mxfp4_gemm_workspace_size.argtypes = [i64, i64, i64]
    lib.e4b_grouped_mxfp4_gemm.argtypes = [vp, i64, i64, vp, vp, i64, i64, vp, vp, i64, i64, i32, vp, i32, vp, sz,
                                           vp]
    lib.e4b_moe_expert_forward_workspace_size.restype = sz
    lib.e4b_moe_expert_forward_workspace_size.argtypes = [i64, ctypes.POINTER(ExpertStackC), i32]
    lib.e4b_moe_expert_forward.restype = i32
    lib.e4b_moe_expert_forward.argtypes = [vp, i64, vp, i32, i32, ctypes.POINTER(ExpertStackC), vp, vp, sz, vp]
    lib.e4b_moe_expert_forward_decode_noalloc.restype = i32
    lib.e4b_moe_expert_forward_decode_noalloc.argtypes = [vp, i64, vp, i32, i32, ctypes.POINTER(ExpertStackC), vp,
                                                          vp]
    lib.e4b_workspace_error.restype = i32
    lib.e4b_workspace_error.argtypes = [vp, ctypes.POINTER(ctypes.c_int32)]
    lib.e4b_workspace_clear_error.restype = i32
    lib.e4b_workspace_clear_error.argtypes = [vp, vp]
    lib.e4b_moe_expert_backward_workspace_size.restype = sz
    lib.e4b_moe_expert_backward_workspace_size.argtypes = [i64, ctypes.POINTER(ExpertStackC), i32]
    lib.e4b_moe_expert_backward.restype = i32
    lib.e4b_moe_expert_backward.argtypes = [vp, i64, vp, i32, i32, ctypes.POINTER(ExpertStackC), vp, vp, vp, vp,
                                            vp, vp, sz, vp]
    lib.e4b_moe_expert_forward_path.restype = i32
    lib.e4b_moe_expert_forward_path.argtypes = [vp, i64, vp, i32, i32, ctypes.POINTER(ExpertStackC), vp, vp,
                                                sz, i32, vp]
    _lib = lib
    return lib


def _check(status: int, fn: str) -> None:
    if status != E4B_OK:
        raise E4BError(status, fn, load_library().e4b_last_error().decode())


def last_path() -> str:
    return load_library().e4b_last_path().decode()


def last_launches() -> int:
    return int(load_library().e4b_last_launches())


def timing_enable(on: bool) -> None:
    load_library().e4b_timing_enable(int(bool(on)))


def timing_read() -> dict:
    """{kernel name: (total ms, launches)} recorded since timing_enable(True)."""
    lib = load_library()
    out = {}
    for i in range(lib.e4b_timing_kernels()):
        name, ms, n = ctypes.c_char_p(), ctypes.c_double(), ctypes.c_int()
        _check(lib.e4b_timing_get(i, ctypes.byref(name), ctypes.byref(ms), ctypes.byref(n)), "e4b_timing_get")
        out[name.value.decode()] = (ms.value, n.value)
    return out


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, name: str, dtype=None) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _quantize_args(W, packed, absmax):
    _dev(W, "W")
    _dev(packed, "packed", torch.uint8)
    _dev(absmax, "absmax", torch.float32)
    if W.dim() != 3:
        raise ValueError("W must be [E, N, K]")
    E, N, K = W.shape
    dt = {torch.float32: E4B_F32, torch.bfloat16: E4B_BF16}.get(W.dtype)
    if dt is None:
        raise ValueError("W must be float32 or bfloat16")
    if packed.numel() < E * N * K // 2 or absmax.numel() < E * N * K // 64:
        raise ValueError("packed/absmax too small")
    return dt, E, N, K


def e4b_nf4_quantize_stack(W: torch.Tensor, packed: torch.Tensor, absmax: torch.Tensor,
                           blocksize: int = 64, stream=None) -> None:
    """W [E, N, K] fp32/bf16 -> packed [E, N*K/2] uint8, absmax [E, N*K/64] fp32."""
    dt, E, N, K = _quantize_args(W, packed, absmax)
    _check(load_library().e4b_nf4_quantize_stack(W.data_ptr(), dt, E, N, K, blocksize, packed.data_ptr(),
                                                 absmax.data_ptr(), _stream(stream)),
           "e4b_nf4_quantize_stack")


def e4b_quantize_stack(W: torch.Tensor, packed: torch.Tensor, absmax: torch.Tensor,
                       quant_type: int = E4B_QUANT_NF4, blocksize: int = 64, stream=None) -> None:
    """As e4b_nf4_quantize_stack, for either 4-bit storage (E4B_QUANT_NF4 or E4B_QUANT_FP4)."""
    dt, E, N, K = _quantize_args(W, packed, absmax)
    _check(load_library().e4b_quantize_stack(W.data_ptr(), dt, E, N, K, blocksize, int(quant_type),
                                             packed.data_ptr(), absmax.data_ptr(), _stream(stream)),
           "e4b_quantize_stack")


def e4b_moe_route_permute_workspace_size(M: int, E: int, k: int) -> int:
    return int(load_library().e4b_moe_route_permute_workspace_size(M, E, k))


def e4b_moe_route_permute(logits: torch.Tensor, k: int, renormalize: bool, topk_ids: torch.Tensor,
                          topk_w: torch.Tensor, expert_offsets: torch.Tensor, perm: torch.Tensor,
                          inv_perm: torch.Tensor, workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    _dev(logits, "logits", torch.float32)
    M, E = logits.shape
    for t, n, d in ((topk_ids, "topk_ids", torch.int32), (topk_w, "topk_w", torch.float32),
                    (expert_offsets, "expert_offsets", torch.int32), (perm, "perm", torch.int32),
                    (inv_perm, "inv_perm", torch.int32)):
        _dev(t, n, d)
    if topk_ids.numel() < M * k or topk_w.numel() < M * k or perm.numel() < M * k or inv_perm.numel() < M * k:
        raise ValueError("route outputs too small")
    if expert_offsets.numel() < E + 1:
        raise ValueError("expert_offsets must hold E+1 entries")
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().e4b_moe_route_permute(
        logits.data_ptr(), M, E, k, int(bool(renormalize)), topk_ids.data_ptr(), topk_w.data_ptr(),
        expert_offsets.data_ptr(), perm.data_ptr(), inv_perm.data_ptr(), _ptr(workspace), ws, _stream(stream)),
        "e4b_moe_route_permute")


def e4b_grouped_nf4_gemm_workspace_size(total_rows: int, N: int, K: int, r: int = 0) -> int:
    return int(load_library().e4b_grouped_nf4_gemm_workspace_size(total_rows, N, K, r))


def _gemm(fn: str, quant_type: Optional[int], A, row_index, expert_offsets, total_rows, packed, absmax, N, K,
          out, epi, lora_A, lora_B, lora_scale, workspace, stream) -> None:
    if A.dim() != 2 or A.dtype != torch.bfloat16 or not A.is_cuda or A.stride(1) != 1:
        raise ValueError("A must be a 2-D bf16 CUDA tensor with unit column stride")
    _dev(expert_offsets, "expert_offsets", torch.int32)
    _dev(packed, "packed", torch.uint8)
    _dev(absmax, "absmax", torch.float32)
    _dev(out, "out")
    if row_index is not None:
        _dev(row_index, "row_index", torch.int32)
    E = expert_offsets.numel() - 1
    r = 0
    if lora_A is not None:
        _dev(lora_A, "lora_A", torch.bfloat16)
        _dev(lora_B, "lora_B", torch.bfloat16)
        r = lora_A.shape[1]
    od = {torch.float32: E4B_F32, torch.bfloat16: E4B_BF16}.get(out.dtype)
    if od is None:
        raise ValueError("out must be float32 or bfloat16")
    ncols = N // 2 if epi == E4B_EPI_SWIGLU else N
    if out.numel() < total_rows * ncols:
        raise ValueError("out too small")
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    q = [] if quant_type is None else [int(quant_type)]
    _check(getattr(load_library(), fn)(
        A.data_ptr(), A.shape[0], A.stride(0), _ptr(row_index), expert_offsets.data_ptr(), E, total_rows,
        packed.data_ptr(), absmax.data_ptr(), *q, N, K, _ptr(lora_A), _ptr(lora_B), r, float(lora_scale), epi,
        out.data_ptr(), od, _ptr(workspace), ws, _stream(stream)), fn)


def e4b_grouped_nf4_gemm(A: torch.Tensor, row_index: Optional[torch.Tensor], expert_offsets: torch.Tensor,
                         total_rows: int, packed: torch.Tensor, absmax: torch.Tensor, N: int, K: int,
                         out: torch.Tensor, epi: int = E4B_EPI_NONE, lora_A: Optional[torch.Tensor] = None,
                         lora_B: Optional[torch.Tensor] = None, lora_scale: float = 0.0,
                         workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    _gemm("e4b_grouped_nf4_gemm", None, A, row_index, expert_offsets, total_rows, packed, absmax, N, K, out, epi,
          lora_A, lora_B, lora_scale, workspace, stream)


def e4b_grouped_4bit_gemm(A: torch.Tensor, row_index: Optional[torch.Tensor], expert_offsets: torch.Tensor,
                          total_rows: int, packed: torch.Tensor, absmax: torch.Tensor, N: int, K: int,
                          out: torch.Tensor, quant_type: int = E4B_QUANT_NF4, epi: int = E4B_EPI_NONE,
                          lora_A: Optional[torch.Tensor] = None, lora_B: Optional[torch.Tensor] = None,
                          lora_scale: float = 0.0, workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """e4b_grouped_nf4_gemm on a stack of either 4-bit storage (quant_type)."""
    _gemm("e4b_grouped_4bit_gemm", quant_type, A, row_index, expert_offsets, total_rows, packed, absmax, N, K, out,
          epi, lora_A, lora_B, lora_scale, workspace, stream)


def e4b_grouped_nf4_gemm_dgrad_workspace_size(total_rows: int, N: int, K: int, r: int = 0) -> int:
    return int(load_library().e4b_grouped_nf4_gemm_dgrad_workspace_size(total_rows, N, K, r))


def _dgrad(fn: str, quant_type: Optional[int], dY, row_index, expert_offsets, total_rows, packed, absmax, N, K,
           out, lora_A, lora_B, lora_scale, workspace, stream) -> None:
    if dY.dim() != 2 or dY.dtype != torch.bfloat16 or not dY.is_cuda or dY.stride(1) != 1:
        raise ValueError("dY must be a 2-D bf16 CUDA tensor with unit column stride")
    _dev(expert_offsets, "expert_offsets", torch.int32)
    _dev(packed, "packed", torch.uint8)
    _dev(absmax, "absmax", torch.float32)
    _dev(out, "out")
    if row_index is not None:
        _dev(row_index, "row_index", torch.int32)
    E = expert_offsets.numel() - 1
    r = 0
    if lora_A is not None:
        _dev(lora_A, "lora_A", torch.bfloat16)
        _dev(lora_B, "lora_B", torch.bfloat16)
        r = lora_A.shape[1]
    od = {torch.float32: E4B_F32, torch.bfloat16: E4B_BF16}.get(out.dtype)
    if od is None:
        raise ValueError("out must be float32 or bfloat16")
    if out.numel() < total_rows * K:
        raise ValueError("out too small")
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    q = [] if quant_type is None else [int(quant_type)]
    _check(getattr(load_library(), fn)(
        dY.data_ptr(), dY.shape[0], dY.stride(0), _ptr(row_index), expert_offsets.data_ptr(), E, total_rows,
        packed.data_ptr(), absmax.data_ptr(), *q, N, K, _ptr(lora_A), _ptr(lora_B), r, float(lora_scale),
        out.data_ptr(), od, _ptr(workspace), ws, _stream(stream)), fn)


def e4b_grouped_nf4_gemm_dgrad(dY: torch.Tensor, row_index: Optional[torch.Tensor], expert_offsets: torch.Tensor,
                               total_rows: int, packed: torch.Tensor, absmax: torch.Tensor, N: int, K: int,
                               out: torch.Tensor, lora_A: Optional[torch.Tensor] = None,
                               lora_B: Optional[torch.Tensor] = None, lora_scale: float = 0.0,
                               workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """out[p] = dY[row_index[p]] . W_e (+ lora_scale * (dY . lora_B[e]) . lora_A[e]), [total_rows, K]."""
    _dgrad("e4b_grouped_nf4_gemm_dgrad", None, dY, row_index, expert_offsets, total_rows, packed, absmax, N, K, out,
           lora_A, lora_B, lora_scale, workspace, stream)


def e4b_grouped_4bit_gemm_dgrad(dY: torch.Tensor, row_index: Optional[torch.Tensor], expert_offsets: torch.Tensor,
                                total_rows: int, packed: torch.Tensor, absmax: torch.Tensor, N: int, K: int,
                                out: torch.Tensor, quant_type: int = E4B_QUANT_NF4,
                                lora_A: Optional[torch.Tensor] = None, lora_B: Optional[torch.Tensor] = None,
                                lora_scale: float = 0.0, workspace: Optional[torch.Tensor] = None,
                                stream=None) -> None:
    """e4b_grouped_nf4_gemm_dgrad on a stack of either 4-bit storage (quant_type)."""
    _dgrad("e4b_grouped_4bit_gemm_dgrad", quant_type, dY, row_index, expert_offsets, total_rows, packed, absmax, N,
           K, out, lora_A, lora_B, lora_scale, workspace, stream)


def e4b_grouped_lora_grads_workspace_size(total_rows: int, r: int) -> int:
    return int(load_library().e4b_grouped_lora_grads_workspace_size(total_rows, r))


def e4b_grouped_lora_grads(x: torch.Tensor, row_index: Optional[torch.Tensor], expert_offsets: torch.Tensor,
                           total_rows: int, da: torch.Tensor, N: int, K: int, lora_A: torch.Tensor,
                           lora_B: torch.Tensor, lora_scale: float, dA: torch.Tensor, dB: torch.Tensor,
                           workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """dA [E, r, K], dB [E, N, r] (fp32) of one grouped projection's adapter."""
    for t, n in ((x, "x"), (da, "da")):
        if t.dim() != 2 or t.dtype != torch.bfloat16 or not t.is_cuda or t.stride(1) != 1:
            raise ValueError(f"{n} must be a 2-D bf16 CUDA tensor with unit column stride")
    _dev(expert_offsets, "expert_offsets", torch.int32)
    _dev(lora_A, "lora_A", torch.bfloat16)
    _dev(lora_B, "lora_B", torch.bfloat16)
    _dev(dA, "dA", torch.float32)
    _dev(dB, "dB", torch.float32)
    if row_index is not None:
        _dev(row_index, "row_index", torch.int32)
    E = expert_offsets.numel() - 1
    r = lora_A.shape[1]
    if dA.numel() < E * r * K or dB.numel() < E * N * r:
        raise ValueError("dA/dB too small")
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().e4b_grouped_lora_grads(
        x.data_ptr(), x.shape[0], x.stride(0), _ptr(row_index), expert_offsets.data_ptr(), E, total_rows,
        da.data_ptr(), da.stride(0), N, K, lora_A.data_ptr(), lora_B.data_ptr(), r, float(lora_scale),
        dA.data_ptr(), dB.data_ptr(), _ptr(workspace), ws, _stream(stream)), "e4b_grouped_lora_grads")


def e4b_grouped_mxfp4_gemm_workspace_size(total_rows: int, N: int, K: int) -> int:
    return int(load_library().e4b_grouped_mxfp4_gemm_workspace_size(total_rows, N, K))


def e4b_grouped_mxfp4_gemm(A: torch.Tensor, row_index: Optional[torch.Tensor], expert_offsets: torch.Tensor,
                           total_rows: int, blocks: torch.Tensor, scales: torch.Tensor, N: int, K: int,
                           out: torch.Tensor, epi: int = E4B_EPI_NONE, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> None:
    """y[p] = A[row_index[p]] . W_e^T with W_e given as MXFP4 code bytes and e8m0 scales."""
    if A.dim() != 2 or A.dtype != torch.bfloat16 or not A.is_cuda or A.stride(1) != 1:
        raise ValueError("A must be a 2-D bf16 CUDA tensor with unit column stride")
    _dev(expert_offsets, "expert_offsets", torch.int32)
    _dev(blocks, "blocks", torch.uint8)
    _dev(scales, "scales", torch.uint8)
    _dev(out, "out")
    if row_index is not None:
        _dev(row_index, "row_index", torch.int32)
    E = expert_offsets.numel() - 1
    od = {torch.float32: E4B_F32, torch.bfloat16: E4B_BF16}.get(out.dtype)
    if od is None:
        raise ValueError("out must be float32 or bfloat16")
    ncols = N // 2 if epi == E4B_EPI_SWIGLU else N
    if out.numel() < total_rows * ncols:
        raise ValueError("out too small")
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().e4b_grouped_mxfp4_gemm(
        A.data_ptr(), A.shape[0], A.stride(0), _ptr(row_index), expert_offsets.data_ptr(), E, total_rows,
        blocks.data_ptr(), scales.data_ptr(), N, K, epi, out.data_ptr(), od, _ptr(workspace), ws, _stream(stream)),
        "e4b_grouped_mxfp4_gemm")


class ExpertStack:
    """Device tensors of one MoE layer's packed stacks (and optional adapter)."""

    def __init__(self, gu_packed, gu_absmax, dn_packed, dn_absmax, E, H, I,
                 lora_A=None, lora_B=None, lora_alpha=0.0, quant_type=E4B_QUANT_NF4):
        for t, n, d in ((gu_packed, "gu_packed", torch.uint8), (gu_absmax, "gu_absmax", torch.float32),
                        (dn_packed, "dn_packed", torch.uint8), (dn_absmax, "dn_absmax", torch.float32)):
            _dev(t, n, d)
        if gu_packed.numel() < E * 2 * I * H // 2 or dn_packed.numel() < E * H * I // 2:
            raise ValueError("packed stacks too small")
        if gu_absmax.numel() < E * 2 * I * H // 64 or dn_absmax.numel() < E * H * I // 64:
            raise ValueError("absmax too small")
        r = 0
        if lora_A is not None:
            _dev(lora_A, "lora_A", torch.bfloat16)
            _dev(lora_B, "lora_B", torch.bfloat16)
            r = lora_A.shape[1]
            if tuple(lora_A.shape) != (E, r, H) or tuple(lora_B.shape) != (E, 2 * I, r):
                raise ValueError("lora_A must be [E, r, H] and lora_B [E, 2I, r]")
        self.tensors = (gu_packed, gu_absmax, dn_packed, dn_absmax, lora_A, lora_B)
        self.E, self.H, self.I, self.r = E, H, I, r
        self.quant_type = int(quant_type)
        self.c = ExpertStackC(gu_packed.data_ptr(), gu_absmax.data_ptr(), dn_packed.data_ptr(),
                              dn_absmax.data_ptr(), _ptr(lora_A), _ptr(lora_B), r, float(lora_alpha), E, H, I,
                              self.quant_type)


def e4b_moe_expert_forward_workspace_size(M: int, stack: ExpertStack, k: int) -> int:
    return int(load_library().e4b_moe_expert_forward_workspace_size(M, ctypes.byref(stack.c), k))


def e4b_moe_expert_forward(x: torch.Tensor, router_logits: torch.Tensor, k: int, renormalize: bool,
                           stack: ExpertStack, out: torch.Tensor, workspace: Optional[torch.Tensor],
                           path: int = E4B_PATH_AUTO, stream=None) -> None:
    _dev(x, "x", torch.bfloat16)
    _dev(router_logits, "router_logits", torch.float32)
    _dev(out, "out", torch.bfloat16)
    M = x.shape[0]
    if x.shape[1] != stack.H or router_logits.shape != (M, stack.E) or out.shape != (M, stack.H):
        raise ValueError("x [M, H], router_logits [M, E] and out [M, H] required")
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().e4b_moe_expert_forward_path(
        x.data_ptr(), M, router_logits.data_ptr(), k, int(bool(renormalize)), ctypes.byref(stack.c),
        out.data_ptr(), _ptr(workspace), ws, path, _stream(stream)), "e4b_moe_expert_forward")


def e4b_moe_expert_backward_workspace_size(M: int, stack: "ExpertStack", k: int) -> int:
    return int(load_library().e4b_moe_expert_backward_workspace_size(M, ctypes.byref(stack.c), k))


def e4b_moe_expert_backward(x: torch.Tensor, router_logits: torch.Tensor, k: int, renormalize: bool,
                            stack: "ExpertStack", dout: torch.Tensor, dx: torch.Tensor, dlogits: torch.Tensor,
                            dA: Optional[torch.Tensor], dB: Optional[torch.Tensor], workspace: Optional[torch.Tensor],
                            stream=None) -> None:
    """Gradients of sum(dout * forward(x, router_logits)): dx [M, H], dlogits [M, E] and, with an
    adapter, dA [E, r, H], dB [E, 2I, r] (all fp32); routing ids held fixed (see include/e4b.h)."""
    _dev(x, "x", torch.bfloat16)
    _dev(router_logits, "router_logits", torch.float32)
    _dev(dout, "dout", torch.bfloat16)
    _dev(dx, "dx", torch.float32)
    _dev(dlogits, "dlogits", torch.float32)
    M = x.shape[0]
    if (x.shape[1] != stack.H or router_logits.shape != (M, stack.E) or dout.shape != (M, stack.H)
            or dx.shape != (M, stack.H) or dlogits.shape != (M, stack.E)):
        raise ValueError("x, dout, dx [M, H] and router_logits, dlogits [M, E] required")
    for t, n in ((dA, "dA"), (dB, "dB")):
        if t is not None:
            _dev(t, n, torch.float32)
    ws = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load_library().e4b_moe_expert_backward(
        x.data_ptr(), M, router_logits.data_ptr(), k, int(bool(renormalize)), ctypes.byref(stack.c),
        dout.data_ptr(), dx.data_ptr(), dlogits.data_ptr(), _ptr(dA), _ptr(dB), _ptr(workspace), ws,
        _stream(stream)), "e4b_moe_expert_backward")


def e4b_moe_expert_forward_decode_noalloc(x: torch.Tensor, router_logits: torch.Tensor, k: int, renormalize: bool,
                                          stack: ExpertStack, out: torch.Tensor, stream=None) -> None:
    """The layer forward for 1..8 tokens without a workspace (see include/e4b.h)."""
    _dev(x, "x", torch.bfloat16)
    _dev(router_logits, "router_logits", torch.float32)
    _dev(out, "out", torch.bfloat16)
    M = x.shape[0]
    if x.shape[1] != stack.H or router_logits.shape != (M, stack.E) or out.shape != (M, stack.H):
        raise ValueError("x [M, H], router_logits [M, E] and out [M, H] required")
    _check(load_library().e4b_moe_expert_forward_decode_noalloc(
        x.data_ptr(), M, router_logits.data_ptr(), k, int(bool(renormalize)), ctypes.byref(stack.c),
        out.data_ptr(), _stream(stream)), "e4b_moe_expert_forward_decode_noalloc")


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zeroed device byte buffer of at least nbytes (at least 256 B, 256-B aligned
    by torch); its first 4 bytes are the error word the kernels report through."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


E4B_KERNEL_ERR_NONE, E4B_KERNEL_ERR_WAIT_FULL, E4B_KERNEL_ERR_WAIT_EMPTY, E4B_KERNEL_ERR_WAIT_DRAIN = 0, 1, 2, 3
E4B_KERNEL_ERR_GRID_BARRIER = 4


def workspace_error(ws: torch.Tensor) -> int:
    """The error word of a workspace (0: no kernel gave up a bounded wait).
    Synchronises the device."""
    code = ctypes.c_int32(-1)
    _check(load_library().e4b_workspace_error(_ptr(ws), ctypes.byref(code)), "e4b_workspace_error")
    return int(code.value)


def workspace_clear_error(ws: torch.Tensor, stream=None) -> None:
    _check(load_library().e4b_workspace_clear_error(_ptr(ws), _stream(stream)), "e4b_workspace_clear_error")
