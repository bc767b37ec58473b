"""Device-side failure detection without a GPU fault: a wait that nothing
completes gives up after its cycle budget, records the timeout bit, and the
host reads CSA2_ERR_TIMEOUT from csa2_sync_status; the context stays usable
(a following pack is still bit-exact)."""
import numpy as np
import pytest
import torch

from fp4_kv_cache_quantize_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fp4_kv_cache_quantize_b200 import csa2
    return csa2


def test_expired_wait_is_reported_and_the_context_survives(lib, orc):
    ws = lib.workspace(lib.WS_HEADER)
    lib.csa2_workspace_init(ws)
    lib.csa2_selftest_bounded_wait(ws, 2_000_000)      # about a millisecond
    with pytest.raises(lib.Csa2Error) as e:
        lib.csa2_sync_status(ws)
    assert e.value.status == 6
    lib.csa2_sync_status(ws)                            # the status word was cleared
    x = synth.to_bf16_bits(np.random.default_rng(3).standard_normal((32, 512)).astype(np.float32))
    xt = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    codes = torch.empty((32, 256), dtype=torch.uint8, device="cuda")
    scales = torch.empty((32, 32), dtype=torch.uint8, device="cuda")
    lib.csa2_quantize_fp4(xt, codes, scales)
    oc, os_ = orc.quantize_fp4(x)
    assert np.array_equal(codes.cpu().numpy(), oc) and np.array_equal(scales.cpu().numpy(), os_)


def test_wait_budget_is_checked_on_the_host(lib, orc):
    ws = lib.workspace(lib.WS_HEADER)
    for bad in (10, 3_000_000_000):
        with pytest.raises(lib.Csa2Error) as e:
            lib.csa2_selftest_bounded_wait(ws, bad)
        assert e.value.status == 1
