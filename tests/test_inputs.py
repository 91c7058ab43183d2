"""Host-side bookkeeping of the seeded workloads: the pair counts behind the flop figures."""
import itertools

from exact_io_aware_81_b200 import inputs


def _brute(Nq, Nk, causal, window):
    off = Nk - Nq
    return sum(1 for i in range(Nq) for j in range(Nk)
               if not causal or (j <= i + off and (window == 0 or j > i + off - window)))


def test_allowed_pairs_brute_force():
    for Nq, Nk, W in itertools.product([1, 5, 17, 64], [17, 64, 100], [0, 1, 3, 16, 17, 50, 100, 200]):
        if Nq > Nk:
            continue
        assert inputs.allowed_pairs(Nq, Nk, True, W) == _brute(Nq, Nk, True, W), (Nq, Nk, W)
    assert inputs.allowed_pairs(7, 3, False) == 21


def test_named_window_workloads_are_consistent():
    # the sliding-window workloads count N x W pairs once every row's window is full
    W, N = 4096, 32768
    assert inputs.allowed_pairs(N, N, True, W) == W * (W + 1) // 2 + (N - W) * W
    assert inputs.allowed_pairs(2048, 16384, True, W) == 2048 * W
