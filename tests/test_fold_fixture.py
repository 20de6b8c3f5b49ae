"""The fp32 fold-order fixture (tests/golden/fold_order_f32.json) on the CPU:
its hand-derived values equal the plain host fp32 folds it describes, the
order shows in them, and the fp64 oracle on the same inputs returns the exact
sums (so the fixture's construction makes every expert output D[e], as it
says)."""
import numpy as np

import fold_fixture as ff
import workloads


def test_fixture_values_are_the_host_fp32_folds():
    """The hand-derived values of the fixture equal the host fp32 folds it
    describes (pins the fixture itself; runs without a GPU)."""
    fx = ff.load()
    c = ff.contributions(fx)
    S = np.broadcast_to(np.asarray(fx["S"], dtype=np.float32), (c.shape[0], c.shape[2]))
    y = ff.host_fold_f32(c, fx["ids"], 4, S)
    assert y[:, 0].tolist() == fx["expected_column0"]
    assert y[:3, 1].tolist() == fx["expected_column1_tokens0to2"]
    for case in fx["band_form"]["cases"]:
        yb = ff.host_band_form_f32(c[:1], fx["ids"][:1], case["band_start"], S[:1])
        assert float(yb[0, 0]) == case["y"], case
    # and the order matters: the slot order of token 0 gives another value
    order = [0, 1, 2, 3]
    acc = c[0, order[0], 0]
    for j in order[1:]:
        acc = np.float32(acc + c[0, j, 0])
    assert np.float32(acc + np.float32(0.5)) != y[0, 0]


def test_oracle_on_the_fixture_gives_the_exact_sums(oracle_lib):
    """In fp64 every sum of the fixture is exact: column 0 of tokens 0..2 is
    2^24 + 1 + 1 - 2^24 + 0.5 = 2.5, token 3's is 2^24 + 1 + 2 - 2^24 + 0.5 =
    3.5; so the fp32 values differ from the exact ones by rounding alone, and
    f_e(x) = D[e] as constructed."""
    import torch
    fx = ff.load()
    x, wg, wu, wd, sh = ff.tensors(fx)

    def b(a):
        return workloads.bits(torch.from_numpy(a).to(torch.bfloat16))
    ids = np.asarray(fx["ids"], dtype=np.int32)
    w = np.asarray(fx["weights"], dtype=np.float64)
    y = oracle_lib.moe_ffn_monolith(b(x), ids, w, b(wg), b(wu), b(wd), 4,
                                    shared=tuple(b(a) for a in sh))
    D = np.asarray(fx["D"], dtype=np.float64)
    exact = np.stack([sum(w[t, j] * D[ids[t, j]] for j in range(4)) for t in range(4)])
    exact = exact + np.asarray(fx["S"], dtype=np.float64)
    assert np.array_equal(y, exact)
    assert y[:, 0].tolist() == [2.5, 2.5, 2.5, 3.5]
