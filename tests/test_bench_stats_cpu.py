"""Host-side selection statistics the benchmark reports beside its rates: the
per-query-tile union of kept blocks and the tensor work the gathered-row
kernels execute, on a selection small enough to count by hand."""
import importlib.util
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_selection_stats_by_hand():
    # T 256, block 64, K 2, G 4: tile 0 keeps nothing, tile 1 keeps {0}, tile 2
    # keeps {0, 1}, tile 3 keeps {0, 2} (even t) or {1, 2} (odd t)
    T, bs, K = 256, 64, 2
    idx = np.full((1, 1, T, K), -1, np.int32)
    n = np.zeros((1, 1, T), np.int32)
    for t in range(T):
        tau = t // bs
        if tau == 1:
            idx[0, 0, t, 0], n[0, 0, t] = 0, 1
        elif tau == 2:
            idx[0, 0, t, :], n[0, 0, t] = (0, 1), 2
        elif tau == 3:
            idx[0, 0, t, :], n[0, 0, t] = ((0, 2) if t % 2 == 0 else (1, 2)), 2
    st = _bench().selection_stats(idx, n, T, bs, G=4)
    # unions 1, 2, 3 blocks; selections per visited block 64/1, 128/2, 128/3
    assert st["union_blocks_per_tile"] == 2.0
    assert abs(st["selections_per_visited_block"] - (64 + 64 + 128 / 3) / 3) < 1e-12
    # tokens walked per block: 64 own + 128, 96, 64, 0 later ones; 32 tokens per
    # chunk -> 7 + 5 + 4 + 2 chunks of 128 rows x 64 keys
    assert st["executed_pairs"] == 18 * 128 * 64


def test_selection_stats_ignores_padding_slots():
    # slots at or past n_sel hold stale ids that must not count
    T, bs, K = 128, 64, 3
    idx = np.zeros((1, 1, T, K), np.int32)
    n = np.zeros((1, 1, T), np.int32)
    n[0, 0, 64:] = 1                          # tile 1 keeps block 0 once; slots 1, 2 are padding
    st = _bench().selection_stats(idx, n, T, bs, G=1)
    assert st["union_blocks_per_tile"] == 1.0
    assert st["selections_per_visited_block"] == 64.0
    # block 0: 64 own + 64 later tokens, 128 tokens per chunk -> 1 chunk; block 1: 1 chunk
    assert st["executed_pairs"] == 2 * 128 * 64
