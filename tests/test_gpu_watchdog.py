"""Bounded pipeline waits: a wait that can never complete gives up with a
status the host reads, and the CUDA context stays usable (needs a B200)."""
import pytest
import torch

import gqa_flash_attention_attn_b200 as ga
from gqa_flash_attention_attn_b200.inputs import make_qkv

pytestmark = pytest.mark.gpu


def test_wait_that_never_completes_reports_timeout():
    assert ga.last_status() == ga.ATTN_OK            # clears any earlier status
    ga.watchdog_selftest(2_000_000)                  # 2 ms limit on an mbarrier nobody completes
    assert ga.last_status() == ga.ATTN_ERR_TIMEOUT
    assert ga.last_status() == ga.ATTN_OK            # reading clears it
    # the context still runs real work afterwards
    q, k, v = make_qkv(1, 4, 2, 128, 128, 128, seed=0)
    out, lse = ga.prefill(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    assert torch.isfinite(out).all()
    assert ga.last_status() == ga.ATTN_OK
