"""The in-kernel wait limit turns a wait that nothing satisfies into an
ATTN_ERR_TIMEOUT status instead of a hang; the context stays usable."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_watchdog_reports_timeout_and_context_survives(cuda_lib):
    assert cuda_lib.attn_check_status() == 0
    cuda_lib.attn_watchdog_selftest(20_000_000)       # 20 ms limit
    assert cuda_lib.attn_check_status() == -5
    assert cuda_lib.attn_check_status() == 0          # cleared after the read
    q = torch.randn(1, 1, 64, 64, device="cuda").to(torch.bfloat16)
    o, lse = cuda_lib.forward(q, q, q, False, 0.125)
    assert cuda_lib.attn_check_status() == 0 and torch.isfinite(lse).all()
