"""Host logic of the per-layer alpha / k search (no GPU): candidate order and
the choice of the smallest error, ties to the earlier candidate."""
from outlier_split_mixed_b200.search import pick_best, search_alpha_k


def test_search_order_and_choice():
    seen = []

    def fake(alpha, k):
        seen.append((alpha, k))
        return abs(alpha - 0.6) + 1.0 / (1 + k)

    r = search_alpha_k(None, None, [0.4, 0.6, 0.8], [0, 32, 128], evaluate=fake)
    assert seen == [(a, k) for k in (0, 32, 128) for a in (0.4, 0.6, 0.8)]
    assert (r.alpha, r.k) == (0.6, 128)
    assert [t[:2] for t in r.table] == seen


def test_ties_go_to_the_earlier_candidate():
    assert pick_best([(0.5, 0, 1.0), (0.6, 0, 0.5), (0.7, 0, 0.5)]) == (0.6, 0, 0.5)
