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


def test_host_wait_deadline_reports_timeout_and_the_next_round_is_correct():
    """A round whose host-side wait (fetch mode 0) cannot be met returns MSA_ERR_TIMEOUT instead of
    blocking: the router is made to withhold its tiles (bounded, about 2 s), the round is given a
    deadline of 0. After the stalled launch has given up, the next round selects the planted
    documents and reports no device error."""
    import routed_long_context_b200 as m
    from msa_inputs import workloads
    from msa_inputs.device import memory_tensor, small_tensors
    from routed_long_context_b200 import _lib
    from routed_long_context_b200.bank import BankLayout, index_from_prepooled

    w = workloads.mem_100m(layers=1, n_host_banks=1, n_docs=2000)
    lay = BankLayout(w.doc_chunks)
    index = index_from_prepooled(lay, memory_tensor(w, 0, "krbar"))
    dev = memory_tensor(w, 0, "bank")
    bank = torch.empty(dev.shape, dtype=dev.dtype, pin_memory=True)
    bank.copy_(dev)
    sm = small_tensors(w, 0)
    cs = m.rope_table(4096, w.d, w.rope_base)
    local = [torch.zeros((1, w.T0, w.hkv, w.d), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    out = torch.empty((1, w.T0, w.hq, w.d), dtype=torch.bfloat16, device="cuda")
    idx_host = torch.empty((1, w.k), dtype=torch.int32, pin_memory=True)
    layer = dict(kr_index=index, host_bank=bank, qr=sm["qr"], q_new=sm["q"], k_new=sm["k_new"], v_new=sm["v_new"],
                 local_k=local[0], local_v=local[1], out=out, topk_idx_host=idx_host)
    rnd = m.InterleaveRound([layer], n_chunks=lay.n_chunks, n_docs=lay.n_docs, doc_chunk_off=lay.doc_chunk_off,
                            doc_chunk_off_host=lay.doc_chunk_off_host, chunk_doc=lay.chunk_doc, n_q=1, H=w.H, d=w.d,
                            hq=w.hq, hkv=w.hkv, k=w.k, L_prev=0, T_new=w.T0, new_q_stride=w.T0, L_max=w.T0,
                            max_mem=w.max_mem, cos_sin=cs, fetch_mode=0)
    compute, copy = torch.cuda.Stream(), torch.cuda.Stream()
    assert m.device_status() == 0
    # one plain round first: under lazy module loading the first launch of a kernel can block the host
    # until the running kernels end, which would let the stalled router finish before the host waits
    rnd.run(compute, copy)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    _lib.check(_lib.lib.msa_route_inject_stall(1), "inject")
    try:
        with pytest.raises(m.MSAError) as err:
            rnd.run(compute, copy, timeout_us=0)
    finally:
        _lib.check(_lib.lib.msa_route_inject_stall(0), "inject")
        torch.cuda.synchronize()               # the stalled router returns after its bounded waits
        code = m.device_status()               # read and cleared even when the round did not raise
    assert err.value.status == _lib.MSA_ERR_TIMEOUT
    assert code == 2                           # MSA_DEV_WAIT_TIMEOUT
    idx_host.fill_(-1)
    rnd.run(compute, copy)
    torch.cuda.synchronize()
    assert m.device_status() == 0
    assert set(w.expected(0, 0, 0)) <= set(idx_host[0].tolist())
