"""Comparison helpers shared by the GPU parity tests (test-side only)."""
import numpy as np

import oracle as O

SCORE_ATOL = 1e-3      # fp32 accumulation of bf16 inputs
TOPK_GAP = 2e-3        # indices must match exactly where the score gap exceeds this
ATTN_ATOL = 2e-2       # bf16 attention outputs, absolute ...
ATTN_RTOL = 2e-2       # ... and relative


def bf16_of(x) -> np.ndarray:
    """Round float64 oracle values to bf16 bits (test-side, for feeding later stages)."""
    from long_context_memory_b200.workloads import f32_to_bf16_bits

    return f32_to_bf16_bits(np.asarray(x, dtype=np.float32))


def torch_bits(t) -> np.ndarray:
    """bf16 torch tensor -> uint16 numpy bits."""
    import torch

    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def check_topk(gpu_idx, gpu_score, s_oracle, k, where=""):
    """Gap-aware top-k parity for one query.

    * every returned score matches the oracle score of the returned doc (1e-3);
    * rank r of the GPU list has an oracle score within TOPK_GAP of the oracle's
      r-th best score (order agrees up to near-ties);
    * when the k-th / (k+1)-th oracle gap exceeds TOPK_GAP the index sets are equal;
    * indices are identical at every rank whose neighbours are separated by more
      than TOPK_GAP on both sides.
    """
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    assert len(set(gpu_idx.tolist())) == k, f"{where}: duplicate ids {gpu_idx}"
    assert np.all((gpu_idx >= 0) & (gpu_idx < len(s_oracle))), where
    o_idx, o_val = O.topk(s_oracle, min(k + 1, len(s_oracle)))
    assert np.allclose(np.asarray(gpu_score, dtype=np.float64), s_oracle[gpu_idx], atol=SCORE_ATOL, rtol=0), (
        f"{where}: scores differ by {np.max(np.abs(gpu_score - s_oracle[gpu_idx]))}")
    assert np.all(np.abs(s_oracle[gpu_idx] - o_val[:k]) <= TOPK_GAP), f"{where}: rank-wise score mismatch"
    if len(o_val) > k and o_val[k - 1] - o_val[k] > TOPK_GAP:
        assert set(gpu_idx.tolist()) == set(o_idx[:k].tolist()), f"{where}: top-k sets differ"
    for r in range(k):
        left = r == 0 or o_val[r - 1] - o_val[r] > TOPK_GAP
        right = (r + 1 >= len(o_val)) or o_val[r] - o_val[r + 1] > TOPK_GAP
        if left and right:
            assert gpu_idx[r] == o_idx[r], f"{where}: rank {r}: {gpu_idx[r]} vs {o_idx[r]}"


def check_attention(gpu_out, ref, where=""):
    g = np.asarray(gpu_out, dtype=np.float64)
    err = np.abs(g - ref)
    bound = ATTN_ATOL + ATTN_RTOL * np.abs(ref)
    worst = np.argmax(err - bound)
    assert np.all(err <= bound), (
        f"{where}: max excess {np.max(err - bound):.3e} at {np.unravel_index(worst, g.shape)}: "
        f"gpu {g.flat[worst]:.5f} oracle {ref.flat[worst]:.5f}")
