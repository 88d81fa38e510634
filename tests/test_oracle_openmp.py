"""The OpenMP build of the oracle (used only to time it on all host cores) is the same
oracle: on ragged shapes its codes, scales, 1/s and fp64 GEMM (all rows and a row
subset) are bit-identical to the single-threaded build's."""
import numpy as np
import pytest

import oracle
from mxfp4_w4a4_post_b200 import workloads as wl


@pytest.mark.parametrize("M,N,K", [(37, 70, 96), (5, 129, 800)])
def test_openmp_build_matches_serial(M, N, K):
    L = wl.with_shape(wl.tiny_layer(), M=M, N=N, K=K)
    x, W, s = wl.draw_x(L), wl.draw_W(L), wl.draw_s(L)
    rows = np.array([M - 1, 0, M // 2], dtype=np.int64)
    out = {}
    try:
        for omp in (False, True):
            oracle.set_openmp(omp)
            wc, ws, inv = oracle.prepare_weight(W, s)
            ac, as_ = oracle.quant_rows(x, inv)
            out[omp] = (wc, ws, inv.view(np.uint32), ac, as_, oracle.gemm_fp64(ac, as_, wc, ws, K),
                        oracle.gemm_fp64(ac, as_, wc, ws, K, rows=rows))
    finally:
        oracle.set_openmp(False)
    for a, b in zip(out[False], out[True]):
        assert np.array_equal(a, b)
