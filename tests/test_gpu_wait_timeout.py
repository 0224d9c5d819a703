"""The bounded wait of the row-staging pipeline gives up, reports and
returns (needs a B200).

A test-only build of the forward kernel (csrc/testing/eqc_wait_probe.cu: the
library's code with every stage fill expecting 16 bytes more than its copies
carry, and a 2 ms wait limit) can never see a stage complete.  It must set
status bit 4 (a wait gave up), drain the copies it has in flight and return,
so the launch finishes promptly and the context stays usable: the library's
own forward on the same inputs afterwards still matches the oracle.  Nothing
here faults or hangs the GPU: the copies are in bounds and land; only the
byte count the barrier waits for is never reached, and every wait is bounded
in time.
"""
import ctypes
import os
import time

import numpy as np
import pytest
import torch

from equivariant_gnn_message_edge_b200 import workloads as wl
from oracle import conv as oconv
from tests.gpu_common import assert_close, run_gpu, to_dev

pytestmark = pytest.mark.gpu

PROBE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                     "equivariant_gnn_message_edge_b200", "libeqc_wait_probe.so")


def test_unfinished_stage_wait_times_out_sets_status_and_returns():
    assert os.path.exists(PROBE), "libeqc_wait_probe.so not built (python -m equivariant_gnn_message_edge_b200.build_lib)"
    lib = ctypes.CDLL(PROBE)
    f = lib.eqc_probe_forward_short_fill
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 3 + [ctypes.c_void_p] * 6
    ins, L, C, N = "0e+1o", 1, 64, 256
    s, rcv, r = wl.periodic_box_graph(N, 10.0, 3.5)
    prob = oconv.Problem(ins, L, ins, C)
    assert lib.eqc_probe_paths() == prob.P
    x = wl.features(N, prob.D_in, C, wl.SEED_X)
    w = wl.weights(len(s), prob.P, C)
    # the CSR of the receiver-sorted box is its identity order
    recv_ptr = np.concatenate([[0], np.cumsum(np.bincount(rcv, minlength=N))]).astype(np.int32)
    recv_perm = np.argsort(rcv, kind="stable").astype(np.int32)
    d = {k: to_dev(v) for k, v in dict(rp=recv_ptr, perm=recv_perm, s=s, x=x, r=r, w=w).items()}
    y = torch.zeros((N, prob.D_out, C), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    t0 = time.monotonic()
    rc = f(d["rp"].data_ptr(), d["perm"].data_ptr(), d["s"].data_ptr(), N, len(s), C, d["x"].data_ptr(),
           d["r"].data_ptr(), d["w"].data_ptr(), y.data_ptr(), status.data_ptr(), ctypes.c_void_p(stream.cuda_stream))
    assert rc == 0, f"launch failed: {rc}"
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    st = int(status.item())
    assert st & 4, f"status {st:#x}: the timed-out wait was not reported"
    assert elapsed < 5.0, f"the kernel took {elapsed:.1f} s to give up"

    # the context is still usable: the library's forward gives the oracle's result
    got = run_gpu(ins, L, ins, C, N, s, rcv, r, x, w)
    assert got["status"] == 0
    assert_close("y after timeout", got["y"], oconv.full(prob, N, s, rcv, r, x, w))
