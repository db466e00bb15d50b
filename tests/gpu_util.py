"""Helpers for the GPU parity tests: host <-> device moves and the parity rules."""
from __future__ import annotations

import numpy as np
import torch

DEV = "cuda:0"


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 BF16 bit patterns -> bf16 CUDA tensor (same bits)."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(DEV)


def f32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def u8_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(DEV)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    if t.dtype == torch.float16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def flags_dev() -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def hessian_rel_err(H_gpu: np.ndarray, H_ref: np.ndarray) -> float:
    return float(np.linalg.norm(H_gpu.astype(np.float64) - H_ref) / max(np.linalg.norm(H_ref), 1e-300))


def sweep_parity(codes_gpu, q_gpu, c1_gpu, ref, rel_tie=1e-5, c2_gpu=None):
    """Apply the sweep parity rule; returns a dict of counts, asserts the hard parts.

    Codes must match wherever the oracle's best and second-best costs differ by more
    than rel_tie relative (and wherever c1 == c2 == 0 or the dequantized blocks are
    identical -- both covered by cost2 == inf or cost1 == cost2 == 0).  Near-tie
    blocks may differ; their mismatches are counted.
    """
    c1, c2 = ref["cost1"], ref["cost2"]
    clear = (c2 - c1) > rel_tie * c2
    zero_tie = (c1 == 0) & (c2 == 0)
    unique = np.isinf(c2)
    must = clear | zero_tie | unique
    near = ~must
    mism = codes_gpu != ref["codes"]
    n = codes_gpu.size
    bad = np.argwhere(mism & must)
    assert bad.size == 0, f"{len(bad)} sweep code mismatches outside near ties, first {bad[:5].tolist()}"
    # nibbles of blocks whose code matches are bit-exact
    nb = codes_gpu.shape[1]
    qm = q_gpu.reshape(-1, nb, 8) == ref["q"].reshape(-1, nb, 8)
    same = ~mism
    assert np.all(qm.all(-1)[same]), "packed nibbles differ on a block with the same code"
    # winning costs agree with the exact ones (FP32 evaluation)
    ok = same & (c1 > 0)
    if ok.any():
        rel = np.abs(c1_gpu[ok].astype(np.float64) - c1[ok]) / c1[ok]
        assert rel.max() < 2e-5, rel.max()
    if c2_gpu is not None:
        # runner-up: the smallest cost above the winner's; on blocks with a clear winner
        # it is the oracle's best cost among different dequantized blocks
        fin = same & clear & np.isfinite(c2)
        if fin.any():
            rel2 = np.abs(c2_gpu[fin].astype(np.float64) - c2[fin]) / c2[fin]
            assert rel2.max() < 2e-5, rel2.max()
        assert np.all(np.isinf(c2_gpu[same & unique])), "runner-up cost must be +inf when no other block exists"
    return {"blocks": n, "near_ties": int(near.sum()), "near_tie_mismatches": int((mism & near).sum()),
            "mismatch_frac": float((mism & near).sum()) / max(n, 1)}
