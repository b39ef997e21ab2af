"""Failure detection on the GPU without a fault: the router's waits are bounded. A testing hook
makes the producer withhold every tile; the other warps' waits run out, the kernel records a
timeout in the device error word and returns, and the context keeps working afterwards."""
import time

import numpy as np
import pytest
import torch

from msa_inputs import rng
from msa_inputs.device import upload

pytestmark = pytest.mark.gpu


def test_router_wait_timeout_is_reported_and_context_survives():
    import oracle as O
    import routed_long_context_b200 as m
    from routed_long_context_b200 import _lib
    from routed_long_context_b200.bank import BankLayout

    counts = np.full(64, 8, dtype=np.int64)
    lay = BankLayout(counts)
    C = int(counts.sum())
    index = rng.round_to(O.unit(rng.normal(7, 1, 0, C * 1024).reshape(C, 8, 128)).astype(np.float32), "bf16")
    qr = rng.normal(7, 2, 0, 16 * 1024, 1.0, "bf16").reshape(1, 16, 8, 128)
    idx_d, qr_d = upload(index, "bf16"), upload(qr, "bf16")
    assert m.device_status() == 0
    _lib.check(_lib.lib.msa_route_inject_stall(1), "inject")
    try:
        t0 = time.time()
        m.msa_route_scores(idx_d, lay.chunk_doc, lay.n_docs, qr_d)
        code = m.device_status()              # synchronises: the launch returns after its bounded waits
        waited = time.time() - t0
    finally:
        _lib.check(_lib.lib.msa_route_inject_stall(0), "inject")
    assert code == 2, code                     # MSA_DEV_WAIT_TIMEOUT
    assert 1.0 < waited < 30.0, waited
    # the same context still routes correctly
    ds = m.msa_route_scores(idx_d, lay.chunk_doc, lay.n_docs, qr_d)
    ref, _ = O.route(index, lay.doc_chunk_off_host, qr)
    assert np.abs(ds.float().cpu().numpy() - ref).max() <= 2e-3
    assert m.device_status() == 0
