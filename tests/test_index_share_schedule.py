"""IndexShare layer schedule (host logic, no GPU): ik_llama.cpp PR #2063's IndexShare commit has layers
il <= 1 and every il % 4 == 2 compute their own selection; the others reuse the last one computed."""
from sparse_attention_sum_b200 import runner


def test_schedule_of_the_first_layers():
    own = [il for il in range(16) if runner.computes_own_selection(il)]
    assert own == [0, 1, 2, 6, 10, 14]


def test_78_layer_stack_computes_21_selections():
    assert sum(runner.computes_own_selection(il) for il in range(78)) == 21


def test_every_reusing_layer_follows_a_computing_layer_at_most_three_back():
    for il in range(78):
        if not runner.computes_own_selection(il):
            assert any(runner.computes_own_selection(j) for j in range(max(0, il - 3), il))
