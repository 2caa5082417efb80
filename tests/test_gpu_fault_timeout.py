"""A kernel wait that runs out, on the GPU, through the C ABI: failure detection without a fault.

Every pipeline wait in the library is an mbarrier wait bounded in time; when the limit passes, the
kernel records DSA_ERR_TIMEOUT in the plan's status word, lets the copies and MMAs it issued land,
frees its TMEM and returns, so the context stays usable. This test uses a separate, test-only build
of the library (libdsa_testfaults.so: -DDSA_TEST_FAULTS, waits limited to 20 ms; the product library
has no switch) in which dsa_test_set_fault(1) makes every indexer CTA leave the keys of its first
tile unloaded. Nothing faults or hangs: the MMA issuer's wait for those keys runs out.

Checked: the launch itself succeeds, dsa_status_read then reports DSA_ERR_TIMEOUT (and clears it),
and a normal call on the same context afterwards returns the oracle's scores with status DSA_OK.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_12_b200 as dsa
from oracle import dsa_oracle as O
from sparse_attention_12_b200 import build as dsa_build
from sparse_attention_12_b200 import synth
from tests import gpu_helpers as G

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def faults_lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    lib = ctypes.CDLL(dsa_build.build_faults())
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    BP = ctypes.POINTER(dsa.DsaBatchC)
    for name, res, args in (("dsa_test_set_fault", I, [I]),
                            ("dsa_plan_workspace_size", SZ, [BP, I]),
                            ("dsa_plan", I, [BP, I, P, SZ, P]),
                            ("dsa_status_read", I, [P, P]),
                            ("dsa_index_scores", I, [BP, P, P, P, P, I, P, P, P, I64, P])):
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    return lib


def test_indexer_wait_runs_out_and_reports_timeout(faults_lib):
    lib = faults_lib
    wl = synth.custom("fault", [300, 1000, 64], [1, 2, 1], n_heads_index=64, topk=64, n_heads=16)
    hb = synth.make_batch(wl, seed=3, extra_pages=1)
    db = dsa.DeviceBatch(hb)
    stream = torch.cuda.current_stream().cuda_stream
    plan = torch.empty(max(16, lib.dsa_plan_workspace_size(db.batch.ref(), db.nhI)), dtype=torch.uint8,
                       device="cuda")
    ld = (hb.max_seq_len + 127) // 128 * 128
    T = hb.total_q
    scores = torch.full((T, ld), float("nan"), dtype=torch.float32, device="cuda")

    def run():
        assert lib.dsa_plan(db.batch.ref(), db.nhI, plan.data_ptr(), plan.numel(), stream) == 0
        return lib.dsa_index_scores(db.batch.ref(), plan.data_ptr(), db.qI.data_ptr(), db.qI_scale.data_ptr(),
                                    db.wI.data_ptr(), db.nhI, db.kI_cache.data_ptr(), db.kI_scale.data_ptr(),
                                    scores.data_ptr(), ld, stream)

    try:
        assert lib.dsa_test_set_fault(1) == 0
        assert run() == 0                                     # the launch itself is fine
        assert lib.dsa_status_read(plan.data_ptr(), stream) == 5  # DSA_ERR_TIMEOUT, read back and cleared
        assert lib.dsa_status_read(plan.data_ptr(), stream) == 0
    finally:
        lib.dsa_test_set_fault(0)
    # the same context, a normal call: status OK and the oracle's scores
    assert run() == 0
    assert lib.dsa_status_read(plan.data_ptr(), stream) == 0
    rows = list(range(T))
    _, pos = O.query_positions(hb.seq_lens, hb.cu_q)
    G.check_scores(G.oracle_scores(hb, rows), G.rows_to_host(scores, rows), pos)
