"""Host-side arithmetic of bench.py against brute force (CPU): the executed
FLOPs of a mask (4 d x query rows x pooled key rows over the non-skipped
pairs, causal blocks above the diagonal left out) and the FlashAttention
convention for causal masks (only the key <= query pairs of the diagonal
blocks)."""
import numpy as np
import pytest
import torch

import bench as B

SKIP = 255


def brute(mask, N, block, d, causal, pairs_only):
    total = 0
    nb = mask.shape[-1]
    for b in range(mask.shape[0]):
        for h in range(mask.shape[1]):
            for I in range(nb):
                q0, q1 = I * block, min((I + 1) * block, N)
                for J in range(nb):
                    l = int(mask[b, h, I, J])
                    if l == SKIP or (causal and J > I):
                        continue
                    k0, k1 = J * block, min((J + 1) * block, N)
                    krows = (k1 - k0) >> l
                    if causal and pairs_only and J == I:
                        total += sum(1 for i in range(q0, q1) for j in range(k0, k1) if j <= i)
                    else:
                        total += (q1 - q0) * krows
    return 4 * d * total


@pytest.mark.parametrize("causal", [False, True])
def test_executed_flops_brute_force(causal):
    g = torch.Generator().manual_seed(3)
    N, block, d, L, nb = 300, 64, 16, 3, 5
    m = torch.randint(0, L + 1, (2, 2, nb, nb), generator=g)
    mask = torch.where(m == L, torch.full_like(m, SKIP), m).to(torch.uint8)
    if causal:
        idx = torch.arange(nb)
        mask[:, :, idx, idx] = 0
    got = B.executed_flops(mask, N, block, d, L, causal)
    assert got == brute(mask.numpy(), N, block, d, causal, False)
    if causal:
        fa = got - B.diagonal_excess_flops(mask, N, block, d)
        assert fa == brute(mask.numpy(), N, block, d, True, True)
