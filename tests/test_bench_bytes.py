"""The bench's algorithmic byte counts equal the per-unit figures the
roofline is stated in (no GPU): forward 4PC + 20 B per edge plus
4(D_in + D_out)C + 4 B per node, deterministic backward 8PC + 32 B per edge
plus 4(2 D_in + D_out)C + 4 B per node (each tensor a kernel reads or writes
counted once; the CSR offset arrays have N + 1 entries)."""
import pytest

import bench


@pytest.mark.parametrize("N,E,C,D_in,D_out,P", [(32768, 1475558, 128, 9, 9, 11), (16384, 737620, 128, 16, 16, 23),
                                               (256, 11674, 32, 4, 9, 7), (10, 0, 4, 1, 1, 1)])
def test_byte_counts_match_per_unit_figures(N, E, C, D_in, D_out, P):
    bc = bench.byte_counts(N, E, C, D_in, D_out, P)
    assert bc["fwd"] == E * (4 * P * C + 20) + N * (4 * (D_in + D_out) * C + 4) + 4
    assert bc["bwd"] == E * (8 * P * C + 32) + N * (4 * (2 * D_in + D_out) * C + 4) + 4
    assert bc["kernels"] == bc["graph"] + bc["fwd"] + bc["bwd"]
    assert bc["graph"] == 16 * E + 8 * (N + 1)        # senders, receivers, two offset arrays, two permutations


def test_double_backward_bytes_per_unit():
    N, E, C, D_in, D_out, P, T, G = 32768, 1475558, 128, 9, 9, 11, 4, 8
    part = E * T * 2 * G * 4
    nb = bench.dbl_bytes(N, E, C, D_in, D_out, P, part)
    per_edge = 8 * P * C + 32 + 12 * P * C + 32 + 36
    per_node = 4 * (2 * D_in + D_out) * C + 4 + 4 * (3 * D_in + D_out) * C + 4
    assert nb == E * per_edge + N * per_node + 8 + 2 * part


def test_kernel_code_hash_ignores_comments_only(tmp_path, monkeypatch):
    src = tmp_path / "k.cuh"
    src.write_text("// header\nint f(int a) {  // note\n    return a + 1; /* inline */\n}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.kernel_code_hash(["k.cuh"])
    src.write_text("// a longer header\n// over two lines\nint f(int a) {\n\n    return a + 1;\n}\n")
    assert bench.kernel_code_hash(["k.cuh"]) == h0
    src.write_text("int f(int a) {\n    return a + 2;\n}\n")
    assert bench.kernel_code_hash(["k.cuh"]) != h0
