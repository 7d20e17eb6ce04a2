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
