"""Device-side failure reporting without a GPU fault: a bounded wait of the
fused batch-1 kernel runs out, the kernel records PI_ERR_TIMEOUT in the
workspace status word and completes, and the context stays usable.

The wait is made to run out through the library's test hook
(pi_debug_wait_fault): entry 0 of the predictor's h is never published, and
every wait is limited to 2 ms.  Nothing traps, faults or hangs: the
other CTAs stop waiting at the limit, publish their (meaningless) partials so
that every reduction completes, and exit.  After the hook is cleared and the
workspace re-initialised, the next call on the same workspace must match the
CPU oracle again.
"""
import pytest
import torch

from activation_sparse_decode_gemv_b200 import binding as pb
from activation_sparse_decode_gemv_b200 import inputs
from parity import Gpu, check_layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("want_ids", [False, True])
def test_withheld_h_slice_times_out_and_recovers(cuda_device, want_ids):
    cfg = inputs.CONFIGS["opt7b_f16"].scaled(d=512, f=2085, r=128)
    lt = inputs.make_layer(cfg, 0, seed=51)
    g = Gpu(lt, 1)
    u_host = inputs.layer_input(cfg, inputs.make_tokens(cfg, 0, 1, seed=53))
    u = u_host.to(cuda_device)
    y = torch.zeros((1, cfg.d), device=cuda_device)
    idx = torch.zeros((1, cfg.f), dtype=torch.int32, device=cuda_device) if want_ids else None
    cnt = torch.zeros((1,), dtype=torch.int32, device=cuda_device) if want_ids else None
    try:
        pb.pi_debug_wait_fault(0, 2000)
        pb.pi_decode_ffn(g.layer, u, y, g.ws, idx=idx, count=cnt)
        torch.cuda.synchronize()  # the kernel completed
    finally:
        pb.pi_debug_wait_fault(-1, 0)
    assert g.status() == pb.PI_ERR_TIMEOUT
    assert g.status() == pb.PI_OK  # reading clears it
    # the context and the workspace are usable again
    pb.pi_workspace_init(g.ws)
    check_layer(lt, u_host, g)
    assert g.status() == pb.PI_OK

