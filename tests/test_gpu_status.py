"""Bounded device waits and host-side errors, on the GPU, without any fault.

The self-test kernel waits on a shared-memory barrier that nothing completes;
its wait gives up after a short poll limit and records the give-up in the
workspace status word, which the host reads.  The context stays usable."""
import pytest
import torch

import gpu_helpers as H
import workloads as W

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    m = H.ts()
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    m.ts_workspace_init(ws)
    assert m.ts_get_device_status(ws) == (m.TS_OK, 0)
    m.ts_selftest_expire_wait(ws, 2000)
    status, site = m.ts_get_device_status(ws)
    assert status == m.TS_ERR_DEVICE_TIMEOUT and site == 99
    assert m.ts_get_device_status(ws) == (m.TS_OK, 0)      # read clears it
    # the context is still fine: a full step runs and matches the oracle
    k, v = W.random_kv(600, 2, 64, 1, device="cuda")
    q = torch.randn((1, 4, 64)).to(torch.bfloat16).cuda()
    case = H.Case(k, v, [0, 600], q)
    buf = H.run_step(case, 32, 4, 16)
    H.check_step(case, buf, 32, 4, 16)
    assert m.ts_get_device_status(buf.ws)[0] == m.TS_OK


def test_host_errors():
    m = H.ts()
    k, v = W.random_kv(100, 2, 64, 2, device="cuda")
    q = torch.randn((1, 4, 64)).to(torch.bfloat16).cuda()
    kv = m.KVCache(k, v, [0, 100], 4)
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    votes = torch.zeros(100, device="cuda")
    with pytest.raises(m.TsError) as e:
        m.ts_score(kv, q, None, votes, small)
    assert e.value.status == m.TS_ERR_WORKSPACE
    bad = m.KVCache(k, v, [0, 100], 3)                       # 3 % 2 != 0
    with pytest.raises(m.TsError) as e:
        m.ts_workspace_bytes(bad, 8, 1, 1)
    assert e.value.status == m.TS_ERR_INVALID_ARG
    k3, v3 = W.random_kv(100, 3, 64, 2, device="cuda")      # h_kv = 3 unsupported
    kv3 = m.KVCache(k3, v3, [0, 100], 6)
    with pytest.raises(m.TsError) as e:
        m.ts_workspace_bytes(kv3, 8, 1, 1)                   # sizing reports failure as 0 bytes
    big = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    q6 = torch.randn((1, 6, 64)).to(torch.bfloat16).cuda()
    with pytest.raises(m.TsError) as e:
        m.ts_score_logits(kv3, q6, None, big)
    assert e.value.status == m.TS_ERR_UNSUPPORTED
