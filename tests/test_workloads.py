"""The seeded input generators (no GPU)."""
import numpy as np

from equivariant_gnn_message_edge_b200 import workloads as wl


def test_weights_prefix_stable():
    a = wl.weights(1000, 11, 16, chunk_edges=128)
    b = wl.weights(300, 11, 16, chunk_edges=77)
    assert np.array_equal(a[:300], b)
    assert abs(float(a.var()) - 1.0 / 11) < 0.01


def test_poisson_graph_shape():
    s, r = wl.poisson_graph(4096, 45.0)
    assert s.dtype == np.int32 and r.dtype == np.int32
    assert np.all(np.diff(r) >= 0)
    assert abs(len(s) / 4096 - 45.0) < 1.0
    assert s.min() >= 0 and s.max() < 4096


def test_box_graph_is_sorted_and_symmetric():
    s, r, vec = wl.periodic_box_graph(256, 10.0, 3.5)
    assert np.all(np.diff(r) >= 0)
    key = r.astype(np.int64) * 256 + s
    assert np.all(np.diff(key) > 0)              # stable on sender, no duplicates
    assert np.all(s != r)
    d = np.linalg.norm(vec, axis=1)
    assert d.max() < 3.5 and d.min() > 0
    pairs = set(zip(s.tolist(), r.tolist()))
    assert all((b, a) in pairs for a, b in pairs)
    mean_deg = len(s) / 256
    assert 40 < mean_deg < 52                    # 0.256 / A^3 * 4/3 pi 3.5^3 ~ 46


def test_edge_vector_lengths():
    v = wl.random_edge_vectors(10000)
    n = np.linalg.norm(v, axis=1)
    assert n.min() >= 0.5 - 1e-5 and n.max() <= 5.0 + 1e-5


def test_weights_into_matches_weights():
    out = np.empty((500, 7, 12), dtype=np.float32)
    wl.weights_into(out, chunk_edges=64)
    assert np.array_equal(out, wl.weights(500, 7, 12, chunk_edges=200))


def test_water_box_workload():
    from equivariant_gnn_message_edge_b200 import workloads as wl
    W = wl.WORKLOADS["waterbox"]
    s, rcv, r = wl.make_graph(W)
    _, _, _, dummy = wl.water_box_graph()
    assert len(s) == 82909 and int(dummy.sum()) == 7537
    assert np.all(np.diff(rcv) >= 0)                       # receiver-sorted
    w = wl.water_box_weights(23, W.C)
    assert w.shape == (82909, 23, 128) and np.all(w[dummy] == 0.0) and np.all(np.isfinite(w))
