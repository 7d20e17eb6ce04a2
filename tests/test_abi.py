"""The C-ABI library on the CPU: it loads, exports every symbol include/moe_route.h declares,
and its host-side logic (sizes, validation, status strings) behaves as documented.
No call here reaches a CUDA launch: each one is rejected (or is a no-op) before that."""
import ctypes
import os
import re

import pytest

import oracle
import token_dispatch_topk_b200 as tdt
from token_dispatch_topk_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_route.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_four_stages():
    names = declared_symbols()
    for stage in ("moe_topk_softmax", "moe_align_permute", "moe_gather", "moe_combine"):
        assert stage in names


def test_library_exports_every_declared_symbol():
    lib = B.load_library()
    names = declared_symbols()
    assert names, "no MOE_API declarations found"
    for n in names:
        assert hasattr(lib, n), f"{n} declared in moe_route.h but not exported"
    assert set(names) == set(B.SIGNATURES), "binding signatures out of sync with the header"


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        B.load_library(str(tmp_path / "absent.so"))


def test_sizes_match_the_oracle():
    for T, k, El, bs in [(64, 2, 8, 16), (4096, 8, 128, 64), (2, 6, 40, 8), (16384, 4, 60, 64),
                         (65536, 8, 256, 128), (0, 3, 5, 7), (1, 1, 1, 1)]:
        assert tdt.moe_align_capacity(T, k, El, bs) == oracle.align_capacity(T, k, El, bs)
        C = tdt.moe_align_capacity(T, k, El, bs)
        assert tdt.moe_align_num_blocks(T, k, El, bs) == -(-C // bs)
        assert tdt.moe_align_workspace_bytes(T, k, El) >= 256
    assert tdt.moe_align_capacity(-1, 2, 3, 4) == -1
    assert tdt.moe_align_capacity(4, 0, 3, 4) == -1


def test_status_strings():
    for code in range(8):
        assert B.status_string(code).startswith("MOE_")
    assert "UNKNOWN" in B.status_string(99)
    assert tdt.moe_version() >= 100


N = None


def test_topk_validation_before_launch():
    lib = B.load_library()
    f = lib.moe_topk_softmax
    assert f(N, B.MOE_DTYPE_BF16, 4, 8, 9, 0, N, N, N) == B.MOE_ERR_INVALID_ARG       # k > E
    assert f(N, B.MOE_DTYPE_BF16, 4, 8, 0, 0, N, N, N) == B.MOE_ERR_INVALID_ARG       # k < 1
    assert f(N, B.MOE_DTYPE_BF16, -1, 8, 2, 0, N, N, N) == B.MOE_ERR_INVALID_ARG      # T < 0
    assert f(N, 7, 4, 8, 2, 0, N, N, N) == B.MOE_ERR_INVALID_ARG                      # dtype
    assert f(N, B.MOE_DTYPE_F32, 4, 8, 2, 0x20, N, N, N) == B.MOE_ERR_INVALID_ARG     # flags
    assert f(N, B.MOE_DTYPE_F32, 0, 8, 2, B.MOE_SCORING_SIGMOID | B.MOE_RENORMALIZE, N, N, N) == B.MOE_OK
    assert f(N, B.MOE_DTYPE_F32, 4, 2048, 2, 0, N, N, N) == B.MOE_ERR_UNSUPPORTED     # E > 1024
    assert f(N, B.MOE_DTYPE_F32, 4, 64, 33, 0, N, N, N) == B.MOE_ERR_UNSUPPORTED      # k > 32
    assert f(N, B.MOE_DTYPE_F32, 4, 64, 8, 0, N, N, N) == B.MOE_ERR_INVALID_ARG       # null pointers
    assert f(N, B.MOE_DTYPE_F32, 0, 64, 8, 1, N, N, N) == B.MOE_OK                    # T == 0: no-op


def test_align_validation_before_launch():
    lib = B.load_library()
    f = lib.moe_align_permute
    buf = ctypes.c_void_p(16)  # never dereferenced: every call below is rejected on the host
    args = lambda T=4, k=2, Eg=8, emap=N, El=8, bs=4, ws=buf, wsb=1 << 20: (
        buf, T, k, Eg, emap, El, bs, buf, buf, buf, buf, buf, buf, ws, wsb, N)
    assert f(*args(El=9)) == B.MOE_ERR_INVALID_ARG            # E_local > E_global
    assert f(*args(El=4)) == B.MOE_ERR_INVALID_ARG            # identity map needs E_local == E_global
    assert f(*args(bs=0)) == B.MOE_ERR_INVALID_ARG
    assert f(*args(T=-1)) == B.MOE_ERR_INVALID_ARG
    assert f(*args(Eg=2048, El=2048)) == B.MOE_ERR_UNSUPPORTED
    assert f(*args(ws=N)) == B.MOE_ERR_WORKSPACE
    assert f(*args(wsb=8)) == B.MOE_ERR_WORKSPACE
    assert f(*args(T=1 << 28, k=8)) == B.MOE_ERR_INVALID_ARG  # T*k >= 2^30
    assert f(*args(ws=ctypes.c_void_p(20))) == B.MOE_ERR_INVALID_ARG  # misaligned workspace


def test_gather_combine_validation_before_launch():
    lib = B.load_library()
    buf = ctypes.c_void_p(16)
    odd = ctypes.c_void_p(24)
    g = lib.moe_gather
    assert g(buf, 4, 12, 2, buf, N, N, 100, 0, buf, N, N) == B.MOE_ERR_INVALID_ARG    # H % 8
    assert g(odd, 4, 16, 2, buf, N, N, 100, 0, buf, N, N) == B.MOE_ERR_INVALID_ARG    # misaligned hidden
    assert g(buf, 4, 16, 2, buf, N, N, 100, 0x8, buf, N, N) == B.MOE_ERR_INVALID_ARG  # flags
    assert g(buf, 4, 16, 2, buf, N, N, 100, B.MOE_GATHER_ZERO_PAD, buf, N, N) == B.MOE_ERR_INVALID_ARG
    assert g(buf, 4, 16, 33, buf, N, N, 100, 0, buf, N, N) == B.MOE_ERR_UNSUPPORTED
    assert g(N, 0, 16, 2, N, N, N, 0, 0, N, N, N) == B.MOE_OK                         # nothing to do
    c = lib.moe_combine
    assert c(buf, buf, buf, 4, 2, 12, 100, buf, N, N) == B.MOE_ERR_INVALID_ARG        # H % 8
    assert c(buf, buf, buf, 4, 2, 16, 100, odd, N, N) == B.MOE_ERR_INVALID_ARG        # misaligned out
    assert c(buf, N, buf, 4, 2, 16, 100, buf, N, N) == B.MOE_ERR_INVALID_ARG          # null weights
    assert c(N, N, N, 0, 2, 16, 0, N, N, N) == B.MOE_OK                               # T == 0
    assert lib.moe_read_status(N, N, N) == B.MOE_ERR_INVALID_ARG


def test_binding_rejects_cpu_tensors():
    import torch
    with pytest.raises(ValueError, match="CUDA tensor"):
        tdt.moe_topk_softmax(torch.zeros(4, 8, dtype=torch.bfloat16), 2, True)


def test_flag_values_match_the_header():
    text = open(HEADER).read()
    defined = {m.group(1): int(m.group(2)) for m in re.finditer(r"^#define\s+(MOE_\w+)\s+(\d+)u", text, flags=re.M)}
    for name in ("MOE_RENORMALIZE", "MOE_GATHER_ZERO_PAD", "MOE_GATHER_HIDDEN_READY", "MOE_DISPATCH_GIVEN_IDS",
                 "MOE_SCORING_SIGMOID"):
        assert getattr(B, name) == defined[name], name


def test_dispatch_validation_before_launch():
    lib = B.load_library()
    buf = ctypes.c_void_p(16)
    d = lib.moe_route_dispatch

    def call(logits, flags, weights, workspace=N, ws_bytes=0, H=16):
        return d(logits, B.MOE_DTYPE_BF16, buf, 2, 160, 6, H, flags, buf, 40, 8, weights, buf, buf, buf, buf, buf,
                 buf, buf, buf, workspace, ws_bytes, N)

    given = B.MOE_DISPATCH_GIVEN_IDS
    assert call(N, 0, buf) == B.MOE_ERR_INVALID_ARG                 # gating needs logits
    assert call(buf, 0, N) == B.MOE_ERR_INVALID_ARG                 # and somewhere for the weights
    assert call(N, given, N) == B.MOE_ERR_WORKSPACE                 # given routes: neither is needed
    assert call(buf, 0x20, buf) == B.MOE_ERR_INVALID_ARG            # unknown flag
    assert call(buf, B.MOE_SCORING_SIGMOID, buf) == B.MOE_ERR_WORKSPACE  # sigmoid scoring accepted
    assert call(buf, B.MOE_GATHER_ZERO_PAD, buf) == B.MOE_ERR_INVALID_ARG
    assert call(buf, B.MOE_RENORMALIZE | given, buf, H=12) == B.MOE_ERR_INVALID_ARG  # H % 8


def test_reduce_partials_host_validation():
    """moe_reduce_partials rejects bad arguments before any CUDA call (no GPU needed)."""
    lib = B.load_library()
    aligned = ctypes.c_void_p(1 << 20)
    arr = (ctypes.c_void_p * 17)(*([aligned] * 17))
    p = ctypes.cast(arr, ctypes.c_void_p)
    assert lib.moe_reduce_partials(p, 0, 4, 8, aligned, None) == B.MOE_ERR_INVALID_ARG      # no partial
    assert lib.moe_reduce_partials(p, 17, 4, 8, aligned, None) == B.MOE_ERR_UNSUPPORTED     # more than 16
    assert lib.moe_reduce_partials(p, 2, 4, 12, aligned, None) == B.MOE_ERR_INVALID_ARG     # H % 8 != 0
    assert lib.moe_reduce_partials(p, 2, -1, 8, aligned, None) == B.MOE_ERR_INVALID_ARG     # rows < 0
    assert lib.moe_reduce_partials(p, 2, 0, 8, aligned, None) == B.MOE_OK                   # nothing to do
    assert lib.moe_reduce_partials(p, 2, 4, 8, ctypes.c_void_p(0x1002), None) == B.MOE_ERR_INVALID_ARG  # out
    bad = (ctypes.c_void_p * 2)(aligned, ctypes.c_void_p(0x1008))
    assert lib.moe_reduce_partials(ctypes.cast(bad, ctypes.c_void_p), 2, 4, 8, aligned, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_reduce_partials(None, 2, 4, 8, aligned, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_reduce_partials(p, 2, 1 << 40, 1 << 20, aligned, None) == B.MOE_ERR_INVALID_ARG  # rows * H too large
    assert lib.moe_reduce_partials(p, 2, 1 << 40, (1 << 31) - 8, aligned, None) == B.MOE_ERR_INVALID_ARG


def test_noalloc_rejects_sizes_beyond_its_scratch_on_the_host():
    """moe_align_permute_noalloc checks the size of its fixed scratch before any CUDA call: 255 tiles
    of 8192 slots with 1024 local experts fit the 1 MiB array, 256 tiles do not."""
    lib = B.load_library()
    buf = (ctypes.c_int32 * 16)()
    p = ctypes.addressof(buf)  # never dereferenced: every call below is rejected on the host
    f = lib.moe_align_permute_noalloc
    assert f(p, 522241, 4, 1024, N, 1024, 16, p, p, p, p, p, p, N, N) == B.MOE_ERR_UNSUPPORTED
    assert f(p, 1 << 18, 4, 1024, N, 1024, 64, p, p, p, p, p, p, N, N) == B.MOE_ERR_UNSUPPORTED
    # every size whose tiles number 256 (of 2048, 4096 or 8192 slots) is beyond the array
    for slots in (522241, 524288, 1044481, 1048576, 2088961):
        assert f(p, slots, 1, 1024, N, 1024, 16, p, p, p, p, p, p, N, N) == B.MOE_ERR_UNSUPPORTED, slots
    assert f(p, 4, 4, 2048, N, 2048, 16, p, p, p, p, p, p, N, N) == B.MOE_ERR_UNSUPPORTED  # E_local > 1024
    assert f(p, 4, 4, 8, N, 4, 16, p, p, p, p, p, p, N, N) == B.MOE_ERR_INVALID_ARG  # identity map, E_local != E
