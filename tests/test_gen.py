"""The seeded workload generator: determinism, structure, bf16 exactness."""
import numpy as np

from workloads import gen


def test_deterministic_and_chunk_local():
    w = gen.scaled("cfg3", context_lens=(20000, 9000))
    a = gen.prefix_chunk(w, 0, 1)
    b = gen.prefix_chunk(w, 0, 1)
    np.testing.assert_array_equal(a[0], b[0])
    K, V = gen.prefix_seq(w, 0)
    np.testing.assert_array_equal(K[8192:16384], a[0])
    assert K.shape == (20000, 8, 128)


def test_bf16_values_are_exact():
    w = gen.scaled("cfg2", context_lens=(1000,))
    K, V = gen.prefix_seq(w, 0)
    for x in (K, V, gen.query(w, 0)):
        u = x.view(np.uint32)
        assert np.all((u & 0xFFFF) == 0)


def test_fp32_workload_is_not_rounded():
    w = gen.get("cfg1")
    K, _ = gen.prefix_seq(w, 0)
    assert np.any((K.view(np.uint32) & 0xFFFF) != 0)


def test_ragged_lengths_and_paged_table():
    w = gen.get("cfg5")
    assert len(w.context_lens) == 16
    assert all(4096 <= L < 262144 for L in w.context_lens)
    t = gen.block_table(w)
    used = t[t >= 0]
    assert len(used) == w.num_phys_blocks
    assert np.array_equal(np.sort(used), np.arange(w.num_phys_blocks))
    for b in range(w.batch):
        assert np.all(t[b, :w.seq_capacity(b)] >= 0)


def test_planted_counts():
    w = gen.get("cfg2")
    p = gen.plan(w, 3)
    nb = w.n_blocks(w.context_lens[3])
    assert np.all(p.planted[:nb].sum(axis=0) == round(0.01 * nb))
    w1 = gen.get("cfg1")
    assert gen.plan(w1, 0).planted[:, 0].sum() == 3


def test_step_tokens_continue_block_offsets():
    w = gen.scaled("cfg3", context_lens=(128 + 3,))
    p = gen.plan(w, 0)
    k, v = gen.step_tokens(w, 0)             # position 131, block 2
    assert k.shape == (1, 8, 128)
    # V noise is N(0,1) around the block's value offset
    assert abs(float((v[0] - p.offsets[2, 1]).mean())) < 0.3
