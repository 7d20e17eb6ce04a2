"""Helpers shared by the GPU parity tests (conversions between torch and the oracle's numpy arrays)."""
import numpy as np
import torch

TOPK_WEIGHT_ATOL = 2e-6   # fp32 gating weights vs the double-precision softmax rounded to fp32
COMBINE_MAX_ULP = 1       # combine output, bf16 ulps (ordered-integer distance, +0 == -0)


def require_gpu():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda")


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits_to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def logits_for_oracle(logits: torch.Tensor) -> np.ndarray:
    return bf16_bits(logits) if logits.dtype == torch.bfloat16 else logits.detach().cpu().numpy()


def np_i32(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy().astype(np.int32)


def ulp_distance_bf16(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    def ordered(x):
        i = x.astype(np.int64)
        return np.where(i >= 0x8000, -(i & 0x7FFF), i)
    return np.abs(ordered(a_bits) - ordered(b_bits))


def assert_align_equal(gpu, ref: dict, what: str = "") -> None:
    """Bit-exact comparison of every align output (GPU AlignResult vs oracle dict)."""
    for name in ("counts", "offsets", "num_tokens_post_pad", "expert_ids", "sorted_token_ids", "inv_perm"):
        g = np_i32(getattr(gpu, name))
        r = ref[name]
        assert g.shape == r.shape, (what, name, g.shape, r.shape)
        bad = np.nonzero(g != r)[0]
        assert bad.size == 0, f"{what} {name}: {bad.size} mismatches, first at {bad[:5]}: gpu {g[bad[:5]]} ref {r[bad[:5]]}"


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at |x| (8 significant bits); the smallest normal spacing at 0."""
    ax = np.abs(x.astype(np.float64))
    e = np.floor(np.log2(np.maximum(ax, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def assert_combine_within_weight_tolerance(out_gpu_bits, out_ref_bits, y_bits, inv_perm, k, what=""):
    """Full-pipeline combine check: the GPU combined its own gating weights, which may differ from the
    oracle's by TOPK_WEIGHT_ATOL each, so |out_gpu - out_ref| <= TOPK_WEIGHT_ATOL * sum_j |y_j|
    + two bf16 ulps at the largest admissible magnitude + fp32 accumulation slack.  Every term of the
    bound is computed from oracle-side values."""
    T = out_ref_bits.shape[0]
    got = (out_gpu_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = (out_ref_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    yv = (y_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    inv = np.asarray(inv_perm).reshape(T, k)
    mag = np.zeros_like(ref)
    for j in range(k):
        r = inv[:, j]
        ok = r >= 0
        mag[ok] += np.abs(yv[r[ok]])
    slack = TOPK_WEIGHT_ATOL * mag + k * 2.0 ** -23 * mag
    bound = slack + 2 * bf16_ulp(np.abs(ref) + slack)
    excess = np.abs(got - ref) - bound
    assert excess.max() <= 0, f"{what}: combine beyond the propagated weight tolerance by {excess.max()}"
