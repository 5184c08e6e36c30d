"""A wait of the fused index kernel's CTAs on one another gives up without a fault.

The multi-CTA selection meets twice (the sample threshold, then the candidate list). Each meeting
is a bounded poll; when it runs out, the kernel sets bit 8 of the status word at the workspace
tail, leaves its selection outputs alone and returns, and the device stays usable. The test
lowers the poll limit to 0 through the library's test hook, so that the waits run out at once
(no flag is left unset, nothing faults or traps), checks the status bit, then restores the limit
and checks that the next call's results equal the first call's.
"""
import numpy as np
import pytest
import torch

import kpool_indexer_int8_b200 as kp

pytestmark = pytest.mark.gpu


def test_cross_cta_wait_gives_up_with_a_status_and_no_fault():
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev).manual_seed(11)
    ld, sel, width = 65536, 512, 2176     # one query over 65,536 pools: its selection spans the SMs
    dims = kp.make_dims(64)
    pooled = torch.randn(1, ld, 128, device=dev, generator=g)
    q_idx = torch.randn(1, 32, 128, device=dev, generator=g).to(torch.bfloat16)
    w = torch.rand(1, 32, device=dev, generator=g)
    i32 = lambda v: torch.tensor(v, dtype=torch.int32, device=dev)  # noqa: E731
    q_seq, q_pos, pad, length = i32([0]), i32([4 * ld - 1]), i32([0]), i32([4 * ld])
    need = kp.glm_dsa_workspace_size(dims, kp.GLM_OP_INDEX_SCORES_TOPK, 1, ld, sel)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    status = ws[need - 256:need - 252].view(torch.int32)
    topk = torch.empty(1, sel, dtype=torch.int32, device=dev)
    tok = torch.empty(1, width, dtype=torch.int32, device=dev)

    def call():
        status.zero_()
        topk.fill_(-7)
        tok.fill_(-7)
        kp.glm_index_topk_expand(dims, q_idx, w, pooled, q_seq, q_pos, pad, length, sel, topk, width, tok=tok,
                                 workspace=ws)
        torch.cuda.synchronize()
        return int(status.item())

    assert call() == 0
    ref_topk, ref_tok = topk.clone(), tok.clone()
    assert (ref_topk >= 0).all()
    try:
        kp.glm_debug_set_cross_cta_wait_limit(0)
        st = call()                      # every meeting gives up at once
    finally:
        kp.glm_debug_set_cross_cta_wait_limit(kp.GLM_CROSS_CTA_WAIT_LIMIT)
    assert st & 8, st
    assert (topk == -7).all()            # the selection was not written
    assert call() == 0                   # the device is usable and the default limit is back
    assert torch.equal(topk, ref_topk) and torch.equal(tok, ref_tok)
