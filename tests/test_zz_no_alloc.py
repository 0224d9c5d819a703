"""The allocation-free graph build (eqconv_graph_build_noalloc), on the GPU.

Some callers cannot allocate device memory, for example a plugin that runs
inside another program's simulation step where that program owns every device
allocation.  For them the library builds the edge layout with scratch from a
fixed device array instead of a caller workspace.  This checks, through the C
ABI, that it gives exactly what the allocating eqconv_graph_build gives, on
two calls in a row with different graphs (the shared scratch keeps the first
call's contents), and that a graph too large for the fixed scratch is refused
with a clear error before anything runs.

The file name sorts last so that a run stopping at the first failure has run
every other test already; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from equivariant_gnn_message_edge_b200 import binding as B

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 8 << 20


def _arrays(N, E, seed):
    rng = np.random.default_rng(seed)
    s = torch.from_numpy(rng.integers(0, N, E).astype(np.int32)).cuda()
    r = torch.from_numpy(np.sort(rng.integers(0, N, E)).astype(np.int32)).cuda()
    return s, r


def _graph(N, E, s, r):
    outs = [torch.full((N + 1,), -7, dtype=torch.int32, device="cuda"),
            torch.full((max(E, 1),), -7, dtype=torch.int32, device="cuda"),
            torch.full((N + 1,), -7, dtype=torch.int32, device="cuda"),
            torch.full((max(E, 1),), -7, dtype=torch.int32, device="cuda")]
    g = B.eqconv_graph_t(N, E, s.data_ptr(), r.data_ptr(), outs[0].data_ptr(), outs[1].data_ptr(),
                         outs[2].data_ptr(), outs[3].data_ptr())
    return g, outs


def _with_workspace(plan, N, E, s, r):
    g, outs = _graph(N, E, s, r)
    nbytes = B.eqconv_graph_workspace_bytes(N, E)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    B.eqconv_graph_build(plan, g, ws, nbytes)
    torch.cuda.synchronize()
    return [o.cpu() for o in outs]


def _no_alloc(plan, N, E, s, r):
    g, outs = _graph(N, E, s, r)
    B.eqconv_graph_build_noalloc(plan, g)
    torch.cuda.synchronize()
    return [o.cpu() for o in outs]


def test_noalloc_matches_allocating_build_twice():
    plan = B.eqconv_plan_create("0e+1o+2e", 2, "0e+1o+2e", 128)
    try:
        # two different graphs, the second one smaller, so stale scratch from
        # the first call would show up in the second
        for N, E, seed in [(70000, 300000, 1), (1503, 83325, 2)]:
            assert B.eqconv_graph_workspace_bytes(N, E) <= SCRATCH_BYTES
            s, r = _arrays(N, E, seed)
            ref = _with_workspace(plan, N, E, s, r)
            got = _no_alloc(plan, N, E, s, r)
            for a, b in zip(got, ref):
                assert torch.equal(a, b)       # integer CSR: bit-exact
            assert B.eqconv_get_device_error(plan) == B.EQCONV_OK
    finally:
        B.eqconv_plan_destroy(plan)


def test_noalloc_refuses_graphs_beyond_the_fixed_scratch():
    plan = B.eqconv_plan_create("0e+1o", 1, "0e+1o", 8)
    try:
        N, E = 32768, 1_000_000
        assert B.eqconv_graph_workspace_bytes(N, E) > SCRATCH_BYTES
        s, r = _arrays(N, E, 3)
        g, outs = _graph(N, E, s, r)
        with pytest.raises(B.EqconvError) as e:
            B.eqconv_graph_build_noalloc(plan, g)
        assert e.value.status == B.EQCONV_ERR_WORKSPACE
        assert "fixed scratch" in B.eqconv_last_error()
        torch.cuda.synchronize()
        assert int(outs[0][0].item()) == -7     # nothing ran
    finally:
        B.eqconv_plan_destroy(plan)
