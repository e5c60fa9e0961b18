"""The work-item order shared by both persistent kernels (`grouped_order` in
csrc/saf_common.cuh), compiled for the host from the same header and checked
exhaustively: every item maps to a distinct (slice, block rank), all of them
are covered, slices come in groups of 1024 // nblk (at least one) in order,
and inside a group the ranks never decrease (rank 0 is the longest block: the forward visits
nqb - rank key blocks for its query block, the backward nqb - rank query
blocks for its key block)."""
import ctypes
import os
import subprocess

import pytest

from mixed_head_causal_b200 import build as saf_build

DRIVER = r"""
#include "saf_common.cuh"
extern "C" void order_all(int BH, int nblk, int* bh, int* rank) {
    for (unsigned b = 0; b < (unsigned)(BH * nblk); ++b) saf::grouped_order(b, BH, nblk, bh[b], rank[b]);
}
"""
GROUP_ITEMS = 1024


def group(nblk):
    return max(1, GROUP_ITEMS // nblk)


@pytest.fixture(scope="module")
def order_lib(tmp_path_factory):
    d = tmp_path_factory.mktemp("grouped_order")
    src = d / "order.cu"
    src.write_text(DRIVER)
    so = d / "order.so"
    subprocess.check_call([saf_build.nvcc(), "-std=c++17", "-O2", "-shared", "-Xcompiler", "-fPIC",
                           "-gencode", "arch=compute_100a,code=sm_100a",
                           "-I", saf_build.CSRC, "-I", saf_build.INCLUDE, str(src), "-o", str(so)])
    return ctypes.CDLL(str(so))


def order(lib, BH, nblk):
    n = BH * nblk
    bh, rank = (ctypes.c_int * n)(), (ctypes.c_int * n)()
    lib.order_all(BH, nblk, bh, rank)
    return list(bh), list(rank)


@pytest.mark.parametrize("BH", [1, 2, 15, 16, 17, 31, 32, 33, 96, 100, 384])
@pytest.mark.parametrize("nblk", [1, 2, 3, 8, 32, 64, 100, 128, 1024, 1500])
def test_grouped_order_is_a_longest_first_bijection(order_lib, BH, nblk):
    bh, rank = order(order_lib, BH, nblk)
    pairs = list(zip(bh, rank))
    assert sorted(pairs) == [(h, r) for h in range(BH) for r in range(nblk)]
    G = group(nblk)
    for b, (h, r) in enumerate(pairs):
        g = b // (G * nblk)
        assert g * G <= h < min(BH, (g + 1) * G)  # its group, in order
        if b > 0 and (b - 1) // (G * nblk) == g:
            assert r >= rank[b - 1]  # longest first inside the group
