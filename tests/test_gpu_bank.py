"""GPU: appending documents to a resident bank equals encoding all documents at once (bit
for bit, including the E4M3 filter keys and routing over the result), the appended part
matches the oracle's pooling, and device arrays survive a bank file round trip."""
import numpy as np
import pytest
import torch

import msa_synth as syn
import oracle
from tests.helpers import POOL_TOL, bf16_to_np

pytestmark = pytest.mark.gpu

H, HQ, D = 8, 32, 128
THETA = 1e6


@pytest.fixture(scope="module")
def msa():
    import top_kv_routing_b200 as m
    return m


@pytest.fixture(scope="module")
def raw():
    """14 documents (ragged lengths, one shorter than a block), 2 layers of bf16 K, V, K_r."""
    lens = np.array([130, 64, 7, 700, 65, 300, 1, 128, 900, 64, 257, 33, 500, 191])
    L = 2
    bank = syn.make_bank(21, len(lens), lens, L)
    n = bank.n_tokens
    toks = {s: np.stack([syn.raw_tokens(bank, l, s, 0, n, dtype="bf16") for l in range(L)])
            for s in (syn.STREAM_K, syn.STREAM_V, syn.STREAM_KR)}
    return bank, toks


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _split(bank, toks, n_a):
    offs = bank.doc_tok_offsets
    cut = int(offs[n_a])
    a = [_dev(toks[s][:, :cut]) for s in (syn.STREAM_K, syn.STREAM_V, syn.STREAM_KR)]
    b = [_dev(toks[s][:, cut:]) for s in (syn.STREAM_K, syn.STREAM_V, syn.STREAM_KR)]
    return a, offs[:n_a + 1], b, offs[n_a:] - cut


def _same(x, y):
    return torch.equal(x.view(torch.uint8) if x.dtype != torch.uint8 else x,
                       y.view(torch.uint8) if y.dtype != torch.uint8 else y)


@pytest.mark.parametrize("n_a", [9, 0, 14])
def test_append_equals_encoding_everything(msa, raw, n_a):
    from top_kv_routing_b200 import bank as mb
    bank, toks = raw
    full_toks = [_dev(toks[s]) for s in (syn.STREAM_K, syn.STREAM_V, syn.STREAM_KR)]
    whole = mb.encode(*full_toks, bank.doc_tok_offsets, THETA)
    a, offs_a, b, offs_b = _split(bank, toks, n_a)
    part = mb.encode(*a, offs_a, THETA, content_on_host=True)
    grown = mb.append(part, *b, offs_b, THETA)
    torch.cuda.synchronize()
    assert np.array_equal(grown.doc_chunk_offsets, whole.doc_chunk_offsets)
    for name in ("kr_hat", "kr_f8", "kr_norm"):
        assert _same(getattr(grown, name), getattr(whole, name)), name
    assert grown.content.device.type == "cpu" and grown.content.is_pinned()
    assert _same(grown.content, whole.content.cpu())


def test_appended_blocks_match_oracle(msa, raw):
    from top_kv_routing_b200 import bank as mb
    bank, toks = raw
    n_a = 9
    a, offs_a, b, offs_b = _split(bank, toks, n_a)
    grown = mb.append(mb.encode(*a, offs_a, THETA), *b, offs_b, THETA)
    C0 = int(grown.doc_chunk_offsets[n_a])
    f = syn.bf16_bits_to_f32
    cut = int(bank.doc_tok_offsets[n_a])
    for l in range(2):
        ref = oracle.pool(f(toks[syn.STREAM_K][l, cut:]), f(toks[syn.STREAM_V][l, cut:]),
                          f(toks[syn.STREAM_KR][l, cut:]), offs_b, H, D, 64, THETA)
        content = bf16_to_np(grown.content[l, C0:])
        assert np.abs(content[:, 0] - ref["k_bar"]).max() <= POOL_TOL
        assert np.abs(content[:, 1] - ref["v_bar"]).max() <= POOL_TOL
        assert np.abs(bf16_to_np(grown.kr_hat[l, C0:]) - ref["kr_unit"]).max() <= POOL_TOL
        nr = grown.kr_norm[l, C0:].cpu().numpy()
        assert np.allclose(nr, ref["kr_norm"], rtol=1e-4, atol=1e-6)


def test_routing_over_appended_bank(msa, raw):
    from top_kv_routing_b200 import bank as mb
    bank, toks = raw
    full_toks = [_dev(toks[s]) for s in (syn.STREAM_K, syn.STREAM_V, syn.STREAM_KR)]
    whole = mb.encode(*full_toks, bank.doc_tok_offsets, THETA)
    a, offs_a, b, offs_b = _split(bank, toks, 9)
    grown = mb.append(mb.encode(*a, offs_a, THETA), *b, offs_b, THETA)
    L, T, k, target = 2, 16, 4, 12  # a document of the appended part
    q = np.stack([syn.fill(5, syn.STREAM_QR, l, 0, 0, T * HQ, D, sigma=0.5, topic=bank.topic,
                           row_topic=np.full(T * HQ, target)).reshape(T, HQ, D) for l in range(L)])
    qd = torch.from_numpy(q.astype(np.float32)).cuda()
    res = []
    for bk in (whole, grown):
        n_docs, C = bk.n_docs, bk.n_blocks
        ws = torch.empty(msa.msa_route_topk_workspace_size(L, 1, T, H, C, n_docs, k), dtype=torch.uint8,
                         device="cuda")
        ids = torch.full((1, L, k), -7, dtype=torch.int32, device="cuda")
        sc = torch.full((1, L, k), float("nan"), device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        coffs = torch.from_numpy(bk.doc_chunk_offsets).cuda()
        msa.msa_route_topk(qd, [0, T], bk.kr_hat, coffs, n_docs, C, L, HQ, H, D, k, ids, sc, ws,
                           flags=msa.MSA_ROUTE_TENSOR_F8, dev_err=err, kr_f8=bk.kr_f8)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        res.append((ids.cpu().numpy(), sc.cpu().numpy()))
    assert np.array_equal(res[0][0], res[1][0]) and np.array_equal(res[0][1], res[1][1])
    assert (res[1][0][0, :, 0] == target).all()


@pytest.mark.parametrize("content_on_host", [True, False])
def test_device_bank_file_round_trip(msa, tmp_path, content_on_host):
    from top_kv_routing_b200 import bank as mb
    L, C = 2, 600  # content 9.8 MB, routing keys 4.9 MB: several halves of a 2 MB staging buffer each
    g = torch.Generator(device="cuda").manual_seed(3)
    rnd = lambda shape, dt, hi: torch.randint(0, hi, shape, generator=g, device="cuda", dtype=torch.int32).to(dt)
    kr_hat = rnd((L, C, H, D), torch.int16, 1 << 15).view(torch.bfloat16)
    kr_f8 = rnd((L, C, H, D), torch.uint8, 256)
    content = rnd((L, C, 2, H, D), torch.int16, 1 << 15).view(torch.bfloat16)
    if content_on_host:
        content = content.cpu().pin_memory()
    kr_norm = torch.rand((L, C, H), generator=g, device="cuda")
    offs = np.array([0, 1, 599, 600], dtype=np.int64)
    info = msa.MsaBankInfo(n_layers=L, n_heads=H, head_dim=D, block_tokens=64, n_docs=3, n_blocks=C,
                           fields=msa.MSA_BANK_KR | msa.MSA_BANK_KR_F8 | msa.MSA_BANK_KV | msa.MSA_BANK_NORM)
    staging = torch.empty(2 << 20, dtype=torch.uint8, pin_memory=True)
    p = tmp_path / "bank.msab"
    msa.msa_bank_save(p, info, offs, kr_hat, kr_f8, content, kr_norm, staging)
    back = mb.load(p, content_on_host=not content_on_host)
    assert np.array_equal(back.doc_chunk_offsets, offs)
    assert _same(back.kr_hat, kr_hat) and _same(back.kr_f8, kr_f8) and _same(back.kr_norm, kr_norm)
    assert _same(back.content.cpu(), content.cpu())
    # a host destination reads the same file identically
    kr_host = np.zeros((L, C, H, D), np.uint16)
    msa.msa_bank_load(p, np.zeros(4, np.int64), kr_hat=kr_host)
    assert np.array_equal(kr_host, kr_hat.cpu().view(torch.int16).numpy().view(np.uint16))
    # and a whole bank saved by the module loads back equal
    q = tmp_path / "bank2.msab"
    mb.save(back, q)
    again = mb.load(q, device="cuda", content_on_host=True)
    assert _same(again.kr_hat, kr_hat) and _same(again.content.cpu(), content.cpu())
