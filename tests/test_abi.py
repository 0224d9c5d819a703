"""The C-ABI library on the CPU: it loads, exports every declared symbol, its
host-side planner agrees with the oracle, and bad arguments are rejected
before any device work.  No kernel runs here."""
import os
import re

import numpy as np
import pytest

from equivariant_gnn_message_edge_b200 import binding as B
from equivariant_gnn_message_edge_b200.workloads import natural_irreps
from oracle.cg import real_cg
from oracle.irreps import enumerate_paths

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "eqconv.h")


@pytest.fixture(scope="module", autouse=True)
def built_library():
    if not os.path.exists(B.LIB_PATH):
        from equivariant_gnn_message_edge_b200 import build_lib
        build_lib.build()
    return B.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"EQCONV_API\s+[\w\s\*]+?\b(eqconv_\w+)\s*\(", text)))


def exported_symbols():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True).stdout
    return {ln.split()[-1] for ln in out.splitlines() if " T " in ln}


def test_every_declared_function_is_exported():
    decl = declared_functions()
    assert len(decl) >= 15
    exported = exported_symbols()
    missing = [f for f in decl if f not in exported]
    assert not missing, missing
    for f in decl:
        getattr(B.lib(), f)


def test_binding_covers_the_header():
    assert sorted(B.ABI_FUNCTIONS) == declared_functions()


def declared_arities():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for name, params in re.findall(r"EQCONV_API\s+[\w\s\*]+?\b(eqconv_\w+)\s*\(([^)]*)\)", text):
        params = params.strip()
        out[name] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_signatures_match_the_header_arity():
    """Every ctypes signature has as many arguments as the C declaration (a
    short list would pass trailing arguments with default conversions)."""
    ar = declared_arities()
    for name, (_, args) in B._SIGS.items():
        assert len(args) == ar[name], (name, len(args), ar[name])


def test_only_the_abi_is_exported():
    extra = [s for s in exported_symbols() if not s.startswith("eqconv_") and not s.startswith("_")]
    # the static CUDA runtime may export nothing else of ours
    assert all(not s.startswith("eqc") for s in extra)


@pytest.mark.parametrize("l1,l2,l3", [(a, b, c) for a in range(4) for b in range(4) for c in range(4)
                                      if abs(a - b) <= c <= a + b])
def test_library_cg_matches_oracle(l1, l2, l3):
    """The library's compile-time Racah evaluation vs the oracle's exact
    rationals: same real basis, phase and sign convention; odd l1 + l2 + l3
    (both-parity outputs) included."""
    assert np.max(np.abs(B.eqconv_cg_table(l1, l2, l3) - real_cg(l1, l2, l3))) < 1e-12


def test_library_rejects_inadmissible_cg():
    for t in [(1, 1, 3), (4, 0, 4), (0, 2, 1)]:
        with pytest.raises(B.EqconvError) as e:
            B.eqconv_cg_table(*t)
        assert e.value.status == B.EQCONV_ERR_UNSUPPORTED


@pytest.mark.parametrize("all_parity", [False, True])
@pytest.mark.parametrize("per_path", [False, True])
@pytest.mark.parametrize("lin,lsh,lout", [(a, b, c) for a in range(4) for b in range(4) for c in range(4)])
def test_library_variant_layouts_match_oracle(lin, lsh, lout, all_parity, per_path):
    """Both-parity and per-path layouts: the library's paths, the first
    output row of each path and D_out equal the oracle's."""
    from equivariant_gnn_message_edge_b200.workloads import both_parity_irreps
    from oracle.conv import Problem
    ins = natural_irreps(lin)
    outs = both_parity_irreps(lout) if all_parity else natural_irreps(lout)
    mode = (B.EQCONV_OUT_ALL_PARITY if all_parity else 0) | (B.EQCONV_OUT_PER_PATH if per_path else 0)
    prob = Problem(ins, lsh, outs, 4, per_path=per_path)
    got = B.eqconv_enumerate_paths_ex(ins, lsh, outs, mode)
    assert got["paths"] == [(q["l1"], q["l2"], q["l3"]) for q in prob.paths]
    assert got["rows"] == [q["off3"] for q in prob.paths]
    assert got["D_out"] == prob.D_out


def test_variant_plans_validate_before_device_work():
    cases = [("0e+1o", 1, "0e+1o", B.EQCONV_OUT_ALL_PARITY, B.EQCONV_ERR_UNSUPPORTED),  # natural string
             ("0e+1o", 1, "0e+1o+1e", 0, B.EQCONV_ERR_UNSUPPORTED),                     # both-parity string
             ("0e+1o", 1, "0e+1o", 4, B.EQCONV_ERR_INVALID_ARG)]                        # unknown bit
    for ins, lsh, outs, mode, status in cases:
        with pytest.raises(B.EqconvError) as e:
            B.eqconv_plan_create_ex(ins, lsh, outs, 8, mode)
        assert e.value.status == status


@pytest.mark.parametrize("lin,lsh,lout", [(a, b, c) for a in range(4) for b in range(4) for c in range(4)])
def test_library_paths_match_oracle(lin, lsh, lout):
    ins, outs = natural_irreps(lin), natural_irreps(lout)
    lib_paths = B.eqconv_enumerate_paths(ins, lsh, outs)
    ref = [(q["l1"], q["l2"], q["l3"]) for q in enumerate_paths(ins, lsh, outs)]
    assert lib_paths == ref


def test_irreps_parsing():
    assert len(B.eqconv_enumerate_paths(" 1x0e + 1x1o ", 2, "0e+1o+2e")) == 7
    for bad in ["", "0x", "0e++1o", "2q", "abc"]:
        with pytest.raises(B.EqconvError) as e:
            B.eqconv_enumerate_paths(bad, 2, "0e")
        assert e.value.status == B.EQCONV_ERR_INVALID_ARG
    for unsupported in ["1o", "0e+2e", "0o", "0e+1e", "0e+1o+2e+3o+4e"]:
        with pytest.raises(B.EqconvError) as e:
            B.eqconv_enumerate_paths(unsupported, 2, "0e")
        assert e.value.status == B.EQCONV_ERR_UNSUPPORTED


def test_plan_create_validates_before_device_work():
    cases = [("0e+1o", 2, "0e", 30, B.EQCONV_ERR_UNSUPPORTED),     # C % 4
             ("0e+1o", 2, "0e", 0, B.EQCONV_ERR_INVALID_ARG),
             ("0e+1o", 4, "0e", 32, B.EQCONV_ERR_UNSUPPORTED),     # L_sh > 3
             ("0e+2e", 2, "0e", 32, B.EQCONV_ERR_UNSUPPORTED),     # not a natural prefix
             ("0e+1o", 2, "bad", 32, B.EQCONV_ERR_INVALID_ARG)]
    for ins, lsh, outs, C, status in cases:
        with pytest.raises(B.EqconvError) as e:
            B.eqconv_plan_create(ins, lsh, outs, C)
        assert e.value.status == status


def test_plan_create_without_a_gpu_fails_loudly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    with pytest.raises(B.EqconvError) as e:
        B.eqconv_plan_create("0e+1o", 2, "0e+1o+2e", 32)
    assert e.value.status == B.EQCONV_ERR_CUDA


def test_workspace_sizes():
    assert B.eqconv_graph_workspace_bytes(10, 0) > 0
    a = B.eqconv_graph_workspace_bytes(1000, 10000)
    b = B.eqconv_graph_workspace_bytes(1000, 20000)
    assert b > a >= 4 * 4 * 10000
    assert B.eqconv_graph_workspace_bytes(-1, 5) == 0


def test_status_strings():
    for s in range(6):
        assert B.eqconv_status_string(s).startswith("EQCONV_")
    assert "unknown" in B.eqconv_status_string(99)


def test_binding_rejects_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        B._ptr(torch.zeros(4))


def test_node_product_plans_validate_before_device_work():
    cases = [("0e+1o", 1, "0e+1o+1e", B.EQCONV_OUT_ALL_PARITY, B.EQCONV_ERR_UNSUPPORTED),  # both parities
             ("0e+2e", 1, "0e+1o", 0, B.EQCONV_ERR_UNSUPPORTED),                        # u not a prefix
             ("0e+1o", 4, "0e+1o", 0, B.EQCONV_ERR_UNSUPPORTED),                        # L_v > 3
             ("0e+1o", 1, "0e+1o", 8, B.EQCONV_ERR_INVALID_ARG)]                        # unknown bit
    for ins, lv, outs, mode, status in cases:
        with pytest.raises(B.EqconvError) as e:
            B.eqconv_node_product_plan_create(ins, lv, outs, 8, mode)
        assert e.value.status == status
    assert B.eqconv_node_product_workspace_bytes(0, 10) == 0
    assert B.eqconv_double_backward_workspace_bytes(0, 10) == 0


def test_header_is_plain_c_and_links(tmp_path):
    """include/eqconv.h compiles as C99 with warnings as errors, and a C
    program links against libeqconv.so and calls the host-only entry points
    (no device needed)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use.c"
    src.write_text(r"""
#include <stdio.h>
#include "eqconv.h"
int main(void) {
    int P = 0, paths[3 * 64];
    double cg[7 * 7 * 7];
    if (eqconv_enumerate_paths("0e+1o+2e", 2, "0e+1o+2e", &P, paths, 64) != EQCONV_OK || P != 11) return 1;
    if (eqconv_cg_table(1, 1, 0, cg, 343) != EQCONV_OK) return 2;
    if (eqconv_graph_workspace_bytes(10, 100) == 0) return 3;
    printf("%d %s\n", P, eqconv_status_string(EQCONV_ERR_UNSUPPORTED));
    return 0;
}
""")
    libdir = os.path.dirname(B.LIB_PATH)
    exe = tmp_path / "use"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src),
                    "-o", str(exe), "-L", libdir, "-leqconv", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    assert out.startswith("11 EQCONV_ERR_UNSUPPORTED")
