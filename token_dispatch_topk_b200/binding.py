"""Thin ctypes binding of libmoe_route.so (include/moe_route.h), same names as the C ABI.

Argument marshalling only: every step of the routing path runs in the library's
CUDA kernels.  torch tensors supply device memory and the stream
(``torch.cuda.current_stream().cuda_stream`` unless one is given).  There is no
CPU fallback: a missing library, a CPU tensor or a non-OK status raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import NamedTuple, Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_route.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_BAD_EXPERT_ID = 6
MOE_ERR_BAD_ROW = 7

MOE_DTYPE_F32 = 0
MOE_DTYPE_BF16 = 1
MOE_RENORMALIZE = 1
MOE_GATHER_ZERO_PAD = 2
MOE_GATHER_HIDDEN_READY = 4
MOE_DISPATCH_GIVEN_IDS = 8
MOE_SCORING_SIGMOID = 16

# Every symbol include/moe_route.h declares, with (restype, argtypes).
_P, _I32, _I64, _U32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_size_t
SIGNATURES = {
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_version": (_I32, []),
    "moe_topk_softmax": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I32, _I32, _U32, _P, _P, _P]),
    "moe_align_capacity": (_I64, [_I64, _I32, _I32, _I32]),
    "moe_align_num_blocks": (_I64, [_I64, _I32, _I32, _I32]),
    "moe_align_workspace_bytes": (_SZ, [_I64, _I32, _I32]),
    "moe_workspace_init": (ctypes.c_int, [_P, _SZ, _P]),
    "moe_align_permute": (ctypes.c_int, [_P, _I64, _I32, _I32, _P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_align_permute_noalloc": (ctypes.c_int, [_P, _I64, _I32, _I32, _P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P,
                                                  _P]),
    "moe_gather": (ctypes.c_int, [_P, _I64, _I32, _I32, _P, _P, _P, _I64, _U32, _P, _P, _P]),
    "moe_combine": (ctypes.c_int, [_P, _P, _P, _I64, _I32, _I32, _I64, _P, _P, _P]),
    "moe_read_status": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_int)]),
    "moe_route_dispatch_workspace_bytes": (_SZ, [_I64, _I32, _I32]),
    "moe_route_dispatch": (ctypes.c_int, [_P, ctypes.c_int, _P, _I64, _I32, _I32, _I32, _U32, _P, _I32, _I32, _P, _P,
                                          _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "moe_reduce_partials": (ctypes.c_int, [_P, _I32, _I64, _I32, _P, _P]),
}

_lib: Optional[ctypes.CDLL] = None


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoe_route.so (built by token_dispatch_topk_b200.build); raises if it is missing."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m token_dispatch_topk_b200.build` "
                           "(the routing path has no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().moe_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, where)


def _dev(t: Optional[torch.Tensor], name: str):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the routing path runs only on the GPU)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


# ----------------------------------------------------------------- host-only queries --
def moe_version() -> int:
    return int(load_library().moe_version())


def moe_align_capacity(T: int, k: int, E_local: int, block_size: int) -> int:
    return int(load_library().moe_align_capacity(T, k, E_local, block_size))


def moe_align_num_blocks(T: int, k: int, E_local: int, block_size: int) -> int:
    return int(load_library().moe_align_num_blocks(T, k, E_local, block_size))


def moe_align_workspace_bytes(T: int, k: int, E_local: int) -> int:
    return int(load_library().moe_align_workspace_bytes(T, k, E_local))


# --------------------------------------------------------------------------- stages --
def moe_workspace_init(workspace: torch.Tensor, stream=None) -> None:
    _check(load_library().moe_workspace_init(_dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
                                             _stream(stream)), "moe_workspace_init")


def alloc_workspace(T: int, k: int, E_local: int, device) -> torch.Tensor:
    """A zeroed align workspace (int32 words; word 0 is the device status word)."""
    nbytes = moe_align_workspace_bytes(T, k, E_local)
    return torch.zeros((nbytes + 3) // 4, dtype=torch.int32, device=device)


def _scoring_flag(scoring: str) -> int:
    if scoring == "softmax":
        return 0
    if scoring == "sigmoid":
        return MOE_SCORING_SIGMOID
    raise ValueError(f"scoring must be 'softmax' or 'sigmoid', got {scoring!r}")


def moe_topk_softmax(logits: torch.Tensor, k: int, renormalize: bool, topk_weights: Optional[torch.Tensor] = None,
                     topk_ids: Optional[torch.Tensor] = None, stream=None, scoring: str = "softmax"):
    """logits [T, E] bf16/fp32 -> (topk_weights [T, k] fp32, topk_ids [T, k] int32).

    ``scoring``: "softmax" (default) or "sigmoid" (each selected expert weighs 1/(1+exp(-x)))."""
    if logits.dim() != 2:
        raise ValueError("logits must be [T, E]")
    T, E = logits.shape
    if logits.dtype == torch.bfloat16:
        dt = MOE_DTYPE_BF16
    elif logits.dtype == torch.float32:
        dt = MOE_DTYPE_F32
    else:
        raise ValueError(f"logits dtype {logits.dtype} unsupported (bf16 or fp32)")
    if topk_weights is None:
        topk_weights = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    if topk_ids is None:
        topk_ids = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    assert topk_weights.dtype == torch.float32 and topk_ids.dtype == torch.int32
    assert topk_weights.numel() == T * k and topk_ids.numel() == T * k
    st = load_library().moe_topk_softmax(_dev(logits, "logits"), dt, T, E, k,
                                         (MOE_RENORMALIZE if renormalize else 0) | _scoring_flag(scoring),
                                         _dev(topk_weights, "topk_weights"), _dev(topk_ids, "topk_ids"),
                                         _stream(stream))
    _check(st, "moe_topk_softmax")
    return topk_weights, topk_ids


class AlignResult(NamedTuple):
    counts: torch.Tensor
    offsets: torch.Tensor
    sorted_token_ids: torch.Tensor
    expert_ids: torch.Tensor
    num_tokens_post_pad: torch.Tensor
    inv_perm: torch.Tensor
    capacity: int


def alloc_align_outputs(T: int, k: int, E_local: int, block_size: int, device) -> AlignResult:
    C = moe_align_capacity(T, k, E_local, block_size)
    NB = moe_align_num_blocks(T, k, E_local, block_size)
    if C < 0:
        raise ValueError("invalid align sizes")
    z = dict(dtype=torch.int32, device=device)
    return AlignResult(torch.empty(E_local, **z), torch.empty(E_local + 1, **z), torch.empty(C, **z),
                       torch.empty(NB, **z), torch.empty(1, **z), torch.empty(T * k, **z), C)


def moe_align_permute(topk_ids: torch.Tensor, E_global: int, block_size: int,
                      expert_map: Optional[torch.Tensor] = None, E_local: Optional[int] = None,
                      out: Optional[AlignResult] = None, workspace: Optional[torch.Tensor] = None,
                      stream=None) -> AlignResult:
    """topk_ids [T, k] int32 (+ optional expert_map [E_global] int32) -> AlignResult on the device."""
    T, k = topk_ids.shape
    if E_local is None:
        E_local = E_global
    if out is None:
        out = alloc_align_outputs(T, k, E_local, block_size, topk_ids.device)
    if workspace is None:
        workspace = alloc_workspace(T, k, E_local, topk_ids.device)
    assert topk_ids.dtype == torch.int32 and (expert_map is None or expert_map.dtype == torch.int32)
    st = load_library().moe_align_permute(
        _dev(topk_ids, "topk_ids"), T, k, E_global, _dev(expert_map, "expert_map"), E_local, block_size,
        _dev(out.counts, "counts"), _dev(out.offsets, "offsets"), _dev(out.sorted_token_ids, "sorted_token_ids"),
        _dev(out.expert_ids, "expert_ids"), _dev(out.num_tokens_post_pad, "num_tokens_post_pad"),
        _dev(out.inv_perm, "inv_perm"), _dev(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "moe_align_permute")
    return out


def moe_align_permute_noalloc(topk_ids: torch.Tensor, E_global: int, block_size: int,
                              expert_map: Optional[torch.Tensor] = None, E_local: Optional[int] = None,
                              out: Optional[AlignResult] = None, device_status: Optional[torch.Tensor] = None,
                              stream=None) -> AlignResult:
    """moe_align_permute without a workspace: the library's fixed per-device scratch is used instead
    (for callers that cannot allocate; calls must not overlap on the GPU).  ``out`` may be preallocated."""
    T, k = topk_ids.shape
    if E_local is None:
        E_local = E_global
    if out is None:
        out = alloc_align_outputs(T, k, E_local, block_size, topk_ids.device)
    assert topk_ids.dtype == torch.int32 and (expert_map is None or expert_map.dtype == torch.int32)
    st = load_library().moe_align_permute_noalloc(
        _dev(topk_ids, "topk_ids"), T, k, E_global, _dev(expert_map, "expert_map"), E_local, block_size,
        _dev(out.counts, "counts"), _dev(out.offsets, "offsets"), _dev(out.sorted_token_ids, "sorted_token_ids"),
        _dev(out.expert_ids, "expert_ids"), _dev(out.num_tokens_post_pad, "num_tokens_post_pad"),
        _dev(out.inv_perm, "inv_perm"), _dev(device_status, "device_status"), _stream(stream))
    _check(st, "moe_align_permute_noalloc")
    return out


def moe_gather(hidden: torch.Tensor, k: int, inv_perm: torch.Tensor, capacity: int,
               sorted_token_ids: Optional[torch.Tensor] = None, num_tokens_post_pad: Optional[torch.Tensor] = None,
               zero_pad: bool = False, permuted: Optional[torch.Tensor] = None,
               device_status: Optional[torch.Tensor] = None, stream=None, hidden_ready: bool = False) -> torch.Tensor:
    """hidden [T, H] bf16 -> permuted [capacity, H] bf16 (expert-grouped rows).

    hidden_ready: hidden was complete before the previous kernel in the stream was launched
    (MOE_GATHER_HIDDEN_READY), so the kernel may start loading it before that kernel finishes."""
    T, H = hidden.shape
    assert hidden.dtype == torch.bfloat16
    if permuted is None:
        permuted = torch.empty((capacity, H), dtype=torch.bfloat16, device=hidden.device)
    st = load_library().moe_gather(_dev(hidden, "hidden"), T, H, k, _dev(inv_perm, "inv_perm"),
                                   _dev(sorted_token_ids, "sorted_token_ids"),
                                   _dev(num_tokens_post_pad, "num_tokens_post_pad"), capacity,
                                   (MOE_GATHER_ZERO_PAD if zero_pad else 0) |
                                   (MOE_GATHER_HIDDEN_READY if hidden_ready else 0), _dev(permuted, "permuted"),
                                   _dev(device_status, "device_status"), _stream(stream))
    _check(st, "moe_gather")
    return permuted


def moe_combine(expert_out: torch.Tensor, topk_weights: torch.Tensor, inv_perm: torch.Tensor,
                out: Optional[torch.Tensor] = None, device_status: Optional[torch.Tensor] = None,
                stream=None) -> torch.Tensor:
    """expert_out [capacity, H] bf16, topk_weights [T, k] fp32, inv_perm [T*k] -> out [T, H] bf16."""
    T, k = topk_weights.shape
    capacity, H = expert_out.shape
    assert expert_out.dtype == torch.bfloat16
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=expert_out.device)
    st = load_library().moe_combine(_dev(expert_out, "expert_out"), _dev(topk_weights, "topk_weights"),
                                    _dev(inv_perm, "inv_perm"), T, k, H, capacity, _dev(out, "out"),
                                    _dev(device_status, "device_status"), _stream(stream))
    _check(st, "moe_combine")
    return out


def moe_reduce_partials(partials, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """partials: the ranks' bf16 partial combines [rows, H] in rank order (tensors on this GPU or,
    with peer access, on others) -> out [rows, H] bf16: their fp32 sum in rank order, rounded once."""
    partials = list(partials)
    if not partials:
        raise ValueError("moe_reduce_partials needs at least one partial")
    rows, H = partials[0].shape
    for p in partials:
        assert p.dtype == torch.bfloat16 and tuple(p.shape) == (rows, H), "partials must all be bf16 [rows, H]"
    if out is None:
        out = torch.empty((rows, H), dtype=torch.bfloat16, device=partials[0].device)
    ptrs = (ctypes.c_void_p * len(partials))(*[_dev(p, "partial") for p in partials])
    st = load_library().moe_reduce_partials(ctypes.cast(ptrs, ctypes.c_void_p), len(partials), rows, H,
                                            _dev(out, "out"), _stream(stream))
    _check(st, "moe_reduce_partials")
    return out


def moe_route_dispatch_workspace_bytes(T: int, k: int, E_local: int) -> int:
    return int(load_library().moe_route_dispatch_workspace_bytes(T, k, E_local))


def alloc_dispatch_workspace(T: int, k: int, E_local: int, device) -> torch.Tensor:
    """A zeroed workspace for moe_route_dispatch (int32 words; word 0 is the device status word)."""
    nbytes = moe_route_dispatch_workspace_bytes(T, k, E_local)
    return torch.zeros((nbytes + 3) // 4, dtype=torch.int32, device=device)


def moe_route_dispatch(logits: Optional[torch.Tensor], hidden: torch.Tensor, k: int, renormalize: bool,
                       block_size: int, expert_map: Optional[torch.Tensor] = None, E_local: Optional[int] = None,
                       topk_weights: Optional[torch.Tensor] = None, topk_ids: Optional[torch.Tensor] = None,
                       align: Optional[AlignResult] = None, permuted: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None, given_ids: bool = False,
                       E: Optional[int] = None, scoring: str = "softmax"):
    """Gating + align + permute-gather in one call.  Returns (topk_weights, topk_ids, AlignResult, permuted).

    With ``given_ids`` the routes in ``topk_ids`` are the input (no gating): ``logits`` may be None (then
    ``E`` gives the number of global experts) and ``topk_weights`` is neither read nor written."""
    T, H = hidden.shape
    if logits is not None:
        assert logits.shape[0] == T
        E = logits.shape[1]
    if E is None:
        raise ValueError("E is needed when logits is None")
    if logits is None or logits.dtype == torch.bfloat16:
        dt = MOE_DTYPE_BF16
    elif logits.dtype == torch.float32:
        dt = MOE_DTYPE_F32
    else:
        raise ValueError(f"logits dtype {logits.dtype} unsupported (bf16 or fp32)")
    if logits is None and not given_ids:
        raise ValueError("logits are needed unless the routes are given")
    assert hidden.dtype == torch.bfloat16
    if E_local is None:
        E_local = E
    dev = hidden.device
    if topk_weights is None and not given_ids:
        topk_weights = torch.empty((T, k), dtype=torch.float32, device=dev)
    if topk_ids is None:
        if given_ids:
            raise ValueError("given_ids needs topk_ids")
        topk_ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    if align is None:
        align = alloc_align_outputs(T, k, E_local, block_size, dev)
    if permuted is None:
        permuted = torch.empty((align.capacity, H), dtype=torch.bfloat16, device=dev)
    if workspace is None:
        workspace = alloc_dispatch_workspace(T, k, E_local, dev)
    assert expert_map is None or expert_map.dtype == torch.int32
    flags = (MOE_RENORMALIZE if renormalize else 0) | (MOE_DISPATCH_GIVEN_IDS if given_ids else 0) | \
        _scoring_flag(scoring)
    st = load_library().moe_route_dispatch(
        _dev(logits, "logits"), dt, _dev(hidden, "hidden"), T, E, k, H, flags,
        _dev(expert_map, "expert_map"), E_local, block_size, _dev(topk_weights, "topk_weights"),
        _dev(topk_ids, "topk_ids"), _dev(align.counts, "counts"), _dev(align.offsets, "offsets"),
        _dev(align.sorted_token_ids, "sorted_token_ids"), _dev(align.expert_ids, "expert_ids"),
        _dev(align.num_tokens_post_pad, "num_tokens_post_pad"), _dev(align.inv_perm, "inv_perm"),
        _dev(permuted, "permuted"), _dev(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(st, "moe_route_dispatch")
    return topk_weights, topk_ids, align, permuted


def moe_read_status(device_status_word: torch.Tensor, stream=None) -> int:
    """Read (and reset) a device status word; returns the recorded moe_status_t (0 = none)."""
    v = ctypes.c_int(0)
    _check(load_library().moe_read_status(_dev(device_status_word, "device_status_word"), _stream(stream),
                                          ctypes.byref(v)), "moe_read_status")
    return int(v.value)
