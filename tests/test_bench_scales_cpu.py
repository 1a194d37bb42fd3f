"""The library comparator in the benchmark runs RFQ as one MXFP4 GEMM over the operands
concatenated along K, [QX | QR] . [QW | QW]^T.  Its scale arrays are joined in the
block-scaled MMA layout by `bench.concat_scales_along_k`; this checks, on the CPU, that
the join equals the oracle's layout of the concatenated matrix's scales, on ragged row
counts (padding row tiles) and several K."""
import numpy as np
import pytest

import bench
import oracle
from block_scaled_gemm_rfq_b200 import workloads as wl


@pytest.mark.parametrize("rows,K", [(1, 128), (130, 256), (300, 512), (128, 1024)])
def test_concat_scales_matches_layout_of_concatenated_operand(rows, K):
    a = oracle.quantize_bf16(wl.random_matrix(rows, K, seed=rows + K, scale=2.0), residual=True)
    s1, s2 = a["scales_x"], a["scales_r"]                      # plain [rows][K/32]
    joined = bench.concat_scales_along_k(oracle.scales_to_mma_layout(s1), oracle.scales_to_mma_layout(s2), rows, K)
    expected = oracle.scales_to_mma_layout(np.concatenate([s1, s2], axis=1))
    assert np.array_equal(joined, expected)


def test_concat_scales_rejects_partial_atoms():
    with pytest.raises(ValueError):
        bench.concat_scales_along_k(np.zeros(512, np.uint8), np.zeros(512, np.uint8), 128, 96)
