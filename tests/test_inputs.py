"""The seeded input recipe (no GPU): each generator in synth.py does what the
recipe says, and the prefill chunk's Zipf load has the shape the measurements
quote (max 7,426 pairs on one expert, median 44, 96 experts with >= 128)."""
import numpy as np

from bit_expert_ffn_router_b200 import synth


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 lies halfway between bf16 neighbours 1 and 1 + 2^-7: ties go to even (1.0)
    vals = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, np.nan], dtype=np.float32)
    bits = synth.f32_to_bf16_bits(vals)
    assert bits[0] == 0x3F80 and bits[1] == 0x3F80 and bits[2] == 0x3F82
    assert synth.bf16_bits_to_f32(bits[3:4])[0] == np.float32(-2.5)
    assert bits[4] == 0x7FC0
    x = synth.activations(64, 256, seed=3)
    assert x.dtype == np.uint16 and x.shape == (64, 256)
    back = synth.bf16_bits_to_f32(x)
    assert np.array_equal(synth.f32_to_bf16_bits(back), x)  # bf16 values round-trip exactly
    assert abs(back.std() - 1.0) < 0.03 and abs(back.mean()) < 0.03


def test_router_weights_and_expert_sections():
    w = synth.router_weights(64, 512, seed=1)
    assert w.dtype == np.float32 and w.shape == (64, 512) and abs(w.std() - 0.02) < 0.001
    for bits in (2, 3):
        s = synth.expert_sections(256, 128, bits, seed=5)
        assert s["gu_codes"].shape == (256, 256 * bits // 8) and s["dn_codes"].shape == (256, 128 * bits // 8)
        assert s["gu_scales"].shape == (256, 8) and s["dn_scales"].shape == (256, 4)
        sc = np.concatenate([s["gu_scales"].ravel(), s["dn_scales"].ravel()]).astype(np.float64)
        assert sc.min() >= float(np.float16(0.005)) and sc.max() <= float(np.float16(0.02))
        # uniform bytes make every 2-bit field uniform over 0..3
        fields = np.concatenate([(s["gu_codes"] >> (2 * i)) & 3 for i in range(4)]).ravel()
        freq = np.bincount(fields, minlength=4) / fields.size
        assert np.all(np.abs(freq - 0.25) < 0.01)


def test_zipf_sets_are_k_distinct_experts_and_seeded():
    a = synth.zipf_sets(500, 512, 10, seed=7)
    assert a.shape == (500, 10) and a.min() >= 0 and a.max() < 512
    assert all(len(set(r)) == 10 for r in a.tolist())
    assert np.array_equal(a, synth.zipf_sets(500, 512, 10, seed=7))
    assert not np.array_equal(a, synth.zipf_sets(500, 512, 10, seed=8))


def test_prefill_chunk_load_shape():
    counts = np.bincount(synth.zipf_sets(8192, 512, 10, seed=0).ravel(), minlength=512)
    assert counts.sum() == 81920
    assert counts.max() == 7426 and np.median(counts) == 44 and (counts >= 128).sum() == 96
    assert counts.min() >= 1 and (counts < 16).sum() == 7


def test_zipf_concentration_matches_the_hot_set_calibration():
    # Zipf(1.1) puts about three quarters of the selections in each layer's 94
    # most popular experts (4,500 hot slots / 48 layers)
    shares = []
    for seed in (0, 1000, 2000, 3000):
        sets = synth.zipf_sets(2000, 512, 10, seed)
        shares.append((synth.zipf_ranks(512, seed)[sets] <= 94).mean())
    assert 0.74 < np.mean(shares) < 0.78


def test_bias_marks_exactly_the_sets():
    sets = synth.zipf_sets(16, 64, 4, seed=2)
    b = synth.bias_from_sets(sets, 64)
    assert b.dtype == np.float32 and b.shape == (16, 64)
    for t in range(16):
        assert set(np.nonzero(b[t])[0].tolist()) == set(sets[t].tolist())
        assert np.all(b[t][sets[t]] == np.float32(synth.BIAS))


def test_correlated_sets_keep_the_stated_reuse():
    s = synth.correlated_sets(steps=20, T=4, E=512, k=10, keep=7, seed=9)
    assert s.shape == (20, 4, 10)
    for i in range(20):
        for t in range(4):
            assert len(set(s[i, t].tolist())) == 10
            if i:
                # the first `keep` entries come from the previous step's set
                assert set(s[i, t, :7].tolist()) <= set(s[i - 1, t].tolist())


def test_hot_slot_table_is_a_permutation_with_the_popular_experts_first():
    L, E, n_hot = 6, 64, 100
    slot_of = synth.hot_slot_table(L, E, n_hot, seed=4)
    assert np.array_equal(np.sort(slot_of), np.arange(L * E))
    rank = np.stack([synth.zipf_ranks(E, 4 + 1000 * l) for l in range(L)]).ravel()
    hot = slot_of < n_hot
    assert hot.sum() == n_hot and rank[hot].max() <= rank[~hot].min()
    # within the hot set, slots ascend with rank
    order = np.argsort(slot_of[hot])
    assert np.all(np.diff(rank[hot][order]) >= 0)
