"""Index arithmetic of the kernels' work splits, checked on the CPU.

The formulas below restate, term for term, how the CUDA kernels divide
their work (K ranges of a cluster, the units of the cluster sums, the 3-D
scale box of the few-token GEMM).  The checks are the invariants the
kernels rely on: every K step, chunk, output element and scale block is
covered exactly once and every coordinate stays inside its buffer.
"""

import itertools

import pytest

BMW, NT = 128, 64          # few-token GEMM: weight rows per tile, token columns


def ks_k_range(num_k, split, rank):
    k0 = num_k * rank // split
    return k0, num_k * (rank + 1) // split - k0


@pytest.mark.parametrize("split", [1, 2, 4, 8])
def test_few_token_k_ranges_partition_the_k_steps(split):
    for num_k in range(split, 65):
        seen = []
        for rank in range(split):
            k0, nk = ks_k_range(num_k, split, rank)
            assert nk >= 1
            seen += list(range(k0, k0 + nk))
        assert seen == list(range(num_k))


@pytest.mark.parametrize("split", [2, 4, 8])
def test_few_token_cluster_sum_covers_the_tile_once(split):
    r0 = BMW // split                 # rows a rank sums
    groups = r0 // 4                  # 4-row float4 units per token
    covered = {}
    for rank in range(split):
        for et in range(128):         # the four epilogue warps
            for u in range(et, groups * NT, 128):
                m = u // groups
                row = rank * r0 + 4 * (u % groups)
                assert 0 <= m < NT and row % 4 == 0 and rank * r0 <= row < (rank + 1) * r0
                for k in range(4):
                    key = (m, row + k)
                    assert key not in covered
                    covered[key] = rank
    assert len(covered) == NT * BMW
    # the partial tiles [64 tokens][128 columns] fp32: a float4 at
    # (m * 128 + row) * 4 bytes is 16-byte aligned and inside 32 KB
    for (m, row) in covered:
        off = (m * BMW + (row - row % 4)) * 4
        assert off % 16 == 0 and off + 16 <= NT * BMW * 4


def test_few_token_weight_scale_box_stays_in_the_repacked_buffer():
    # 3-D view of the repacked weight scales: {128 u32, 2 halves,
    # ceil(N/256) * K/64 blocks}; tile t of 128 rows reads half t & 1 of
    # block rows (t >> 1) * kblocks + 4 k .. + 3
    for N in range(32, 2049, 32):
        for K in (256, 512, 3840):
            kblocks = K // 64
            extent = -(-N // 256) * kblocks
            for t in range(-(-N // BMW)):
                for kk in range(K // 256):
                    z = (t >> 1) * kblocks + 4 * kk
                    assert 0 <= z and z + 4 <= extent
                    assert (t & 1) in (0, 1)


def kq_split_ok(split, chunks):
    return split == 1 or (4 * split <= chunks if split <= 8 else 2 * split <= chunks)


@pytest.mark.parametrize("split", [1, 2, 4, 8, 16])
def test_activation_chunk_ranges_and_stages(split):
    for chunks in range(1, 200):
        if not kq_split_ok(split, chunks):
            continue
        covered = []
        for rank in range(split):
            c_begin = rank * chunks // split
            c_end = (rank + 1) * chunks // split
            assert c_end - c_begin >= (2 if split > 1 else 1)
            nstages = (c_end - c_begin + 1) // 2
            # stage i holds chunks c_begin + 2 i and, if present, the next
            for i in range(nstages):
                kc0 = c_begin + 2 * i
                nc = 1 if c_end - kc0 < 2 else 2
                covered += list(range(kc0, kc0 + nc))
        assert covered == list(range(chunks))


@pytest.mark.parametrize("bm,split", list(itertools.product([64, 128], [2, 4, 8, 16])))
def test_activation_cluster_sum_units_partition(bm, split):
    units = bm * (128 // 4)          # BM rows x 32 float4 of L
    seen = []
    for rank in range(split):
        seen += list(range(rank * units // split, (rank + 1) * units // split))
    assert seen == list(range(units))
