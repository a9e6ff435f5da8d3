"""Pins of the oracle's argmax and greedy draft acceptance against hand-derived cases."""
import numpy as np

from conftest import golden


def test_argmax_first_index_of_the_maximum(orc):
    assert orc.argmax(np.array([1.0, 3.0, 3.0, 2.0])) == 1
    assert orc.argmax(np.array([-5.0, -1.0, -1.0])) == 1
    assert orc.argmax(np.zeros(7)) == 0
    assert orc.argmax(np.array([2.5])) == 0
    v = np.random.default_rng(3).standard_normal(1000)
    assert orc.argmax(v) == int(np.argmax(v))


def test_accept_greedy_hand_cases(orc):
    g = golden("accept_greedy.json")
    lens, out, acc = orc.accept_greedy(g["row_argmax"], g["row_tokens"], g["ars"], g["lens"])
    assert acc.tolist() == g["expect_n_accept"]
    assert out.tolist() == g["expect_out_tokens"]
    assert lens.tolist() == g["expect_lens"]
