"""The bounded-wait exit path of the tensor-core kernels, made to run out on purpose with
a short limit set at run time (msa_route_wait_selftest): the wait gives up, the kernel
reports MSA_DEVERR_TIMEOUT, frees its tensor memory and returns, and the context stays
usable.  No GPU fault, trap or hang is involved: the wait is bounded by the GPU's timer."""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def msa():
    import top_kv_routing_b200 as m
    return m


def test_wait_that_nothing_completes_times_out_cleanly(msa):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    msa.msa_route_wait_selftest(20_000_000, False, err)  # 20 ms
    b.record()
    torch.cuda.synchronize()
    assert int(err.item()) == msa.MSA_DEVERR_TIMEOUT
    assert a.elapsed_time(b) >= 19.0   # the wait lasted its limit, then gave up


def test_completed_wait_reports_nothing(msa):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    msa.msa_route_wait_selftest(20_000_000, True, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0


def test_context_usable_after_a_timeout(msa):
    # a timed-out wait, then the tensor-core routing path on the same stream
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    msa.msa_route_wait_selftest(1_000_000, False, err)
    torch.cuda.synchronize()
    assert int(err.item()) == msa.MSA_DEVERR_TIMEOUT
    H, HQ, D, C, k = 8, 32, 128, 200, 4
    torch.manual_seed(3)
    kr = torch.nn.functional.normalize(torch.randn((1, C, H, D), device="cuda"), dim=-1).to(torch.bfloat16)
    coffs = torch.arange(0, C + 1, 2, dtype=torch.int64, device="cuda")
    T = 40
    ws = torch.empty(msa.msa_route_topk_workspace_size(1, 1, T, H, C, C // 2, k), dtype=torch.uint8, device="cuda")
    ids = torch.empty((1, 1, k), dtype=torch.int32, device="cuda")
    sc = torch.empty((1, 1, k), device="cuda")
    err2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    msa.msa_route_topk(torch.randn((1, T, HQ, D), device="cuda"), [0, T], kr, coffs, C // 2, C, 1, HQ, H, D, k, ids,
                       sc, ws, flags=msa.MSA_ROUTE_TENSOR, dev_err=err2)
    torch.cuda.synchronize()
    assert int(err2.item()) == 0
    got = ids.cpu().numpy()[0, 0]
    assert len(set(got.tolist())) == k and min(got) >= 0


def test_bad_limit_is_rejected(msa):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(msa.MsaError):
        msa.msa_route_wait_selftest(0, False, err)
