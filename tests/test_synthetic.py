"""The seeded input generators (CPU): determinism, independence of the worker
count, bf16 rounding, and the statistics the recipes promise."""
import numpy as np

import synthetic as SY


def test_bf16_round_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -9, -2.5, 3.0e38], dtype=np.float32)
    back = SY.bf16_to_f32(SY.bf16_round(x))
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa -> 1
    assert back[0] == 1.0 and back[1] == 1.0
    assert back[2] == np.float32(1.0 + 2 ** -7)
    assert back[3] == -2.5
    assert np.all(np.abs(back - x) <= np.abs(x) * 2 ** -8)


def test_logits_do_not_depend_on_worker_count():
    a = SY.make_logits(3, [40, 300], 700, 3.0, 1.5, "bf16")
    b = SY.make_logits(3, [40, 300], 700, 3.0, 1.5, "bf16", workers=2)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_lm_head_case_does_not_depend_on_worker_count():
    for hd, ht in ((128, 128), (64, 192)):
        a = SY.make_lm_head_case("w", 2, 4, 1000, hd, ht, 3.0, 1.5, seed=1)
        b = SY.make_lm_head_case("w", 2, 4, 1000, hd, ht, 3.0, 1.5, seed=1, workers=3)
        for k in ("h_draft", "w_draft", "h_teacher", "w_teacher"):
            assert np.array_equal(getattr(a, k), getattr(b, k)), (hd, ht, k)


def test_lm_head_recipe_statistics():
    c = SY.make_lm_head_case("s", 4, 16, 4096, 256, 256, sig_t=3.0, sig_n=1.5, seed=0)
    assert c.h_draft.shape == (64, 256) and c.w_draft.shape == (4096, 256)
    f = lambda a: SY.to_f64(a, "bf16")
    t = f(c.h_teacher) @ f(c.w_teacher).T
    z = f(c.h_draft) @ f(c.w_draft).T
    assert abs(t.std() - 3.0) < 0.15            # teacher logits of deviation sig_t
    assert abs((z - t).std() - 1.5) < 0.1       # draft = teacher + noise of deviation sig_n
    assert np.array_equal(c.h_draft, c.h_teacher)  # equal hidden sizes: the same hidden states


def test_seeds_give_different_inputs():
    a = SY.make_lm_head_case("d", 1, 2, 300, 64, 64, 3.0, 1.5, seed=0)
    b = SY.make_lm_head_case("d", 1, 2, 300, 64, 64, 3.0, 1.5, seed=1)
    assert not np.array_equal(a.w_teacher, b.w_teacher)
