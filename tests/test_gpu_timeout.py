"""The kernels' bounded-wait path on the GPU, without a fault.

A self-test kernel waits on a pipeline barrier that nothing arrives on, with the wait
every pipeline of the library uses.  Under a short limit it gives up, records a timeout
in the device error word and returns; qlora_sync_status then reports QLORA_ERR_TIMEOUT
(and clears it), and the context stays usable for a normal layer call afterwards.
"""
import time

import pytest
import torch

import bit_quantized_base_nf4_b200 as q
from bit_quantized_base_nf4_b200 import synthetic as syn
from oracle import nf4_oracle as O

pytestmark = pytest.mark.gpu

DEV = "cuda"


def test_wait_limit_runs_out_and_is_reported():
    q.qlora_sync_status()                                  # nothing pending
    q.qlora_set_wait_limit_ns(50_000_000)                  # 50 ms
    try:
        t0 = time.perf_counter()
        q.qlora_probe_wait_timeout()
        with pytest.raises(q.QloraError) as e:
            q.qlora_sync_status()
        elapsed = time.perf_counter() - t0
        assert e.value.status == 6, e.value                # QLORA_ERR_TIMEOUT
        assert "timed out" in str(e.value)
        assert 0.04 <= elapsed < 30.0, elapsed             # the wait gave up at its limit
        q.qlora_sync_status()                              # the error word was cleared
    finally:
        q.qlora_set_wait_limit_ns(2_000_000_000)

    # the context is still usable: a normal layer call gives the oracle's result
    c = syn.LayerCase("after-timeout-m128-n256-k512-r8", M=128, N=256, K=512, r=8, alpha=16.0, seed=401)
    W = c.weight()
    w = q.NF4Weight.empty(c.N, c.K)
    q.qlora_quantize_nf4_dq(W.to(DEV), w)
    X, A, B = c.x().to(DEV), c.lora_a().to(DEV), c.lora_b().to(DEV)
    ws = torch.empty(q.qlora_workspace_bytes(c.M, c.N, c.K, c.r), dtype=torch.uint8, device=DEV)
    Y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=DEV)
    q.qlora_lora_linear_fwd(w, X, A, B, c.r, c.scaling, Y, None, ws)
    q.qlora_sync_status()
    ref = O.quantize_nf4_dq(W.numpy())
    Wd = O.dequant(ref["codes"], ref["scales"], ref["scales2"]).reshape(c.N, c.K)
    Yref, _ = O.lora_linear_fwd(Wd, X.cpu(), A.cpu(), B.cpu(), c.scaling)
    assert O.within_tolerance(Y.float().cpu(), Yref), O.rel_errors(Y.float().cpu(), Yref)
