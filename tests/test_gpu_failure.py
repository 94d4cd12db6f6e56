"""Failure detection on the GPU without a fault: a kernel's bounded wait on a barrier
that nothing arrives at runs out, the device status word reports the timeout (with the
wait's site), reading it clears it, and the context stays usable."""
import pytest
import torch

import query_aware_selective_b200 as qas
from query_aware_selective_b200 import _abi
from oracle import esa as oesa
from tests.parity import check_selection

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def test_bounded_wait_runs_out_and_is_reported():
    torch.cuda.set_device(0)
    qas.device_status()                                    # nothing pending
    _abi.wait_selftest(10_000_000)                         # 10 ms
    with pytest.raises(qas.EsaError, match="9901"):
        qas.device_status()
    qas.device_status()                                    # the read cleared it
    # the context still works: a small selection matches the oracle
    g = torch.Generator().manual_seed(7)
    q_c = torch.randn(1, 1, 64, generator=g)
    k_c = torch.randn(1, 3000, 64, generator=g)
    p = qas.params(16, 256, 64, 2, 10.0)
    idx, cnt, _ = qas.score_select(q_c.to(DEV), k_c.to(DEV), 2999, p)
    qas.device_status()
    ref_idx, ref_cnt, ref_sp = oesa.score_select(q_c.double().numpy(), k_c.double().numpy(), 2999, 16, 256, 64, 2,
                                                 10.0)
    check_selection(idx[0].cpu().numpy(), int(cnt[0]), ref_idx[0], ref_cnt[0], ref_sp[0], 16, 64)
