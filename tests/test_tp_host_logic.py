"""Host-side arithmetic of the vocab-parallel glue (tp.py), checked over many
vocabularies and group sizes without a GPU: the shards partition [0, V) in
order, start on the split / chunk grid, and the split counts satisfy the
conditions rlk_linear_logp_fwd_shard and rlk_linear_logp_combine check."""
import itertools

from invariant_lm_head_gemm_b200 import tp


def _cdiv(a, b):
    return -(-a // b)


def _chunk(V):
    # the backward chunk width rlk_bwd_chunk_width returns: min(8192, V rounded up to 256)
    return min(8192, _cdiv(V, 256) * 256)


VOCABS = (1, 2, 255, 256, 257, 511, 512, 513, 1537, 8191, 8192, 8193, 20000, 40000, 151936,
          152064, 262144)
WORLDS = (1, 2, 3, 4, 5, 7, 8, 16)


def test_shards_partition_the_vocabulary_on_the_grid():
    for V, world in itertools.product(VOCABS, WORLDS):
        align = tp.shard_alignment(V, 512, _chunk(V))
        assert align % 512 == 0 and align % _chunk(V) == 0
        bounds = [tp.shard_rows(V, world, r, align) for r in range(world)]
        assert bounds[0][0] == 0 and bounds[-1][1] == V
        per = tp.per_shard(V, world, align)
        seen_empty = False
        for r, (v0, v1) in enumerate(bounds):
            assert 0 <= v0 <= v1 <= V
            if r:
                assert v0 == bounds[r - 1][1]               # contiguous, in rank order
            if v1 == v0:
                seen_empty = True
                continue
            assert not seen_empty                           # empty shards only at the end
            assert v0 % align == 0                          # on the split and chunk grid
            assert v1 - v0 <= per
            assert v1 == V or v1 - v0 == per                # only the last one is short


def test_split_counts_meet_the_shard_and_combine_conditions():
    for V, world in itertools.product(VOCABS, WORLDS):
        split = 512
        align = tp.shard_alignment(V, split, _chunk(V))
        Gs = _cdiv(tp.per_shard(V, world, align), split)
        G = _cdiv(V, split)
        nshards = _cdiv(G, Gs)
        # rlk_linear_logp_combine: (nshards - 1) * Gs < G <= nshards * Gs
        assert (nshards - 1) * Gs < G <= nshards * Gs
        for r in range(world):
            v0, v1 = tp.shard_rows(V, world, r, align)
            if v1 > v0:
                # rlk_linear_logp_fwd_shard: ceil(V_shard / 512) <= Gs <= ceil(V / 512)
                assert _cdiv(v1 - v0, split) <= Gs <= G
                assert r < nshards                          # its block is in the combine's range


def test_chunk_slots_meet_the_backward_shard_condition():
    for V, world in itertools.product(VOCABS, WORLDS):
        chunk = _chunk(V)
        align = tp.shard_alignment(V, 512, chunk)
        cps = _cdiv(tp.per_shard(V, world, align), chunk)
        owners = []
        for r in range(world):
            v0, v1 = tp.shard_rows(V, world, r, align)
            if v1 > v0:
                # rlk_linear_logp_bwd_shard: ceil(V_shard / w) <= part_chunks <= ceil(V / w)
                assert _cdiv(v1 - v0, chunk) <= cps <= _cdiv(V, chunk)
                owners += [(r, k) for k in range(_cdiv(v1 - v0, chunk))]
        # (rank, local chunk) order over the all-to-all's blocks is global chunk order,
        # and the first ceil(V / chunk) blocks are exactly those chunks
        assert len(owners) == _cdiv(V, chunk)
        flat = [(r, k) for r in range(world) for k in range(cps)]
        assert flat[:len(owners)] == owners
