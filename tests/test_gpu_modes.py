"""Output variants on the GPU: both-parity outputs and per-path-retained
outputs, against the oracle (FlashCart, arXiv 2610.06409, App. B: opposite
parity products; App. D: path retention or summation).

Every case goes through the C ABI (eqconv_plan_create_ex) in both backward
modes; the layout the library reports (D_out, each path's first output row)
must equal the oracle's, and y, dx, dw, dr must agree element by element
within the convolution's tolerance.
"""
import numpy as np
import pytest

from equivariant_gnn_message_edge_b200 import binding as B
from equivariant_gnn_message_edge_b200.workloads import both_parity_irreps, natural_irreps
from oracle import conv as oconv
from tests.gpu_common import check_all, oracle_full, run_gpu

pytestmark = pytest.mark.gpu

# (L_in, L_sh, L_out, C, N, E): several channel tiles with a ragged last one,
# every l = 3 combination the variants compile, scalar inputs
CASES = [
    (1, 1, 1, 36, 40, 700),
    (2, 2, 2, 132, 90, 2500),
    (0, 3, 3, 68, 50, 900),
    (3, 2, 3, 40, 60, 1200),
    (2, 3, 1, 64, 70, 1500),
    (3, 3, 3, 100, 64, 1600),
]
MODES = {"both": (True, False), "per_path": (False, True), "both_per_path": (True, True)}


def _inputs(prob, N, E, seed):
    rng = np.random.default_rng(seed)
    s = rng.integers(0, N, E).astype(np.int32)
    rcv = rng.integers(0, N, E).astype(np.int32)
    r = (rng.standard_normal((E, 3)) * 2).astype(np.float32)
    r[1] = 0.0                                           # a zero-length edge
    x = rng.standard_normal((N, prob.D_in, prob.C)).astype(np.float32)
    w = (rng.standard_normal((E, prob.P, prob.C)) / np.sqrt(prob.P)).astype(np.float32)
    gy = rng.standard_normal((N, prob.D_out, prob.C)).astype(np.float32)
    return s, rcv, r, x, w, gy


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("case", CASES)
def test_output_variants_match_oracle(case, mode):
    L_in, L_sh, L_out, C, N, E = case
    all_parity, per_path = MODES[mode]
    ins = natural_irreps(L_in)
    outs = both_parity_irreps(L_out) if all_parity else natural_irreps(L_out)
    prob = oconv.Problem(ins, L_sh, outs, C, per_path=per_path)
    s, rcv, r, x, w, gy = _inputs(prob, N, E, seed=10 * CASES.index(case) + list(MODES).index(mode))
    ref = oracle_full(ins, L_sh, outs, C, N, s, rcv, r, x, w, gy, per_path=per_path)
    for det in (True, False):
        res = run_gpu(ins, L_sh, outs, C, N, s, rcv, r, x, w, gy, det=det, all_parity=all_parity,
                      per_path=per_path)
        assert res["status"] == 0
        assert res["D_out"] == prob.D_out
        assert res["paths"] == [(q["l1"], q["l2"], q["l3"]) for q in prob.paths]
        assert res["path_rows"] == [q["off3"] for q in prob.paths]
        check_all(res, ref)


def test_variant_plans_reject_what_they_do_not_cover():
    with pytest.raises(B.EqconvError) as e:          # L_sh = 0 has no variant instances
        B.eqconv_plan_create_ex("0e+1o", 0, "0e+1o", 8, B.EQCONV_OUT_PER_PATH)
    assert e.value.status == B.EQCONV_ERR_UNSUPPORTED
    plan = B.eqconv_plan_create_ex("0e+1o+2e", 2, "0e+1o+2e", 8, B.EQCONV_OUT_PER_PATH)
    try:
        B.eqconv_plan_set_vec(plan, 2, 2)            # the compiled width
        with pytest.raises(B.EqconvError):
            B.eqconv_plan_set_vec(plan, 4, 4)
    finally:
        B.eqconv_plan_destroy(plan)
