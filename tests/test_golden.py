"""The oracle against hand-derived closed-form cases (tests/golden/)."""
import json
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
with open(os.path.join(HERE, "golden", "hand_cases.json")) as f:
    CASES = json.load(f)["cases"]


def arr(x):
    return np.array([[np.nan if v is None else v for v in row] for row in np.array(x, dtype=object).reshape(-1, np.array(x, dtype=object).shape[-1])], dtype=np.float32).reshape(np.array(x, dtype=object).shape)


@pytest.mark.parametrize("case", CASES, ids=[c["name"] for c in CASES])
def test_hand_case(oracle_mod, case):
    q, kn, vn = arr(case["q"]), arr(case["k_new"]), arr(case["v_new"])
    kc, vc = arr(case["k_cache"]), arr(case["v_cache"])
    cu = np.concatenate([[0], np.cumsum(case["q_lens"])]).astype(np.int32)
    out, lse = oracle_mod.forward(q, kn, vn, kc, vc, np.array(case["page_table"], np.int32), cu,
                                  np.array(case["kv_lens"], np.int32), case["scale"],
                                  case["causal"], oracle_mod.F32)
    np.testing.assert_allclose(out, np.array(case["expected_out"]), rtol=0, atol=case["tol"])
    np.testing.assert_allclose(lse, np.array(case["expected_lse"]), rtol=0, atol=case["tol"])
    if "expected_k_page0_slot0" in case:
        np.testing.assert_array_equal(kc[0, 0, 0], np.array(case["expected_k_page0_slot0"], np.float32))
        assert np.isnan(kc[0, 1]).all() and np.isnan(kc[1]).all()
