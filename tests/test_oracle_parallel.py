"""The oracle's OpenMP variants (token loops over host threads, used to time
the oracle on all host cores) give exactly the serial oracle's results."""
import numpy as np

from combine_moe_layout_06_b200 import inputs


def test_parallel_variants_equal_serial(oracle_mod):
    assert oracle_mod.parallel_threads() >= 1
    for T, H, E, k, R, N, seed in ((1, 8, 4, 1, 1, 1, 1), (777, 72, 64, 8, 8, 2, 2),
                                   (3000, 40, 60, 4, 7, 7, 3)):
        d = inputs.make_random(T, H, E, k, seed=seed, zipf_s=0.8)
        x, topk, w = d["x"], d["topk_idx"], d["topk_w"]
        lay = oracle_mod.layout(topk, E, R, N, nodes=True)
        assert np.array_equal(oracle_mod.dispatch_flat_par(x, lay["slot"]),
                              oracle_mod.dispatch_flat(x, lay["slot"]))
        st_p, recv_p = oracle_mod.dispatch_two_level_par(x, lay, R, N)
        st_s, recv_s = oracle_mod.dispatch_two_level(x, lay, R, N)
        assert np.array_equal(st_p, st_s) and np.array_equal(recv_p, recv_s)
        eo = inputs.random_bf16_bits((T * k, H), seed=seed + 5)
        assert np.array_equal(oracle_mod.combine_par(eo, w, lay["slot"]),
                              oracle_mod.combine(eo, w, lay["slot"]))
