"""Bank files on the host (no GPU needed): the library's writer against an independent
reader of the documented format, round trips, damaged files, the append offsets and the
host re-layout."""
import os
import struct

import numpy as np
import pytest

H, D = 8, 128


@pytest.fixture(scope="module")
def msa():
    import top_kv_routing_b200 as m
    return m


def _checksum(data: bytes) -> int:
    """The section checksum as msa_bank.h defines it, written out independently."""
    M = (1 << 64) - 1
    pad = (-len(data)) % 32
    words = struct.unpack(f"<{(len(data) + pad) // 8}Q", data + b"\0" * pad)
    h = [0xcbf29ce484222325 ^ j for j in range(4)]
    for i, w in enumerate(words):
        h[i & 3] = ((h[i & 3] ^ w) * 0x100000001b3) & M
    rotl = lambda v, r: ((v << r) | (v >> (64 - r))) & M
    return h[0] ^ rotl(h[1], 16) ^ rotl(h[2], 32) ^ rotl(h[3], 48)


def _parse(path):
    """Header and sections of a bank file, read with struct/numpy from the documented layout."""
    raw = open(path, "rb").read()
    magic, version, hbytes, L, Hh, d, bt, n_docs, n_blocks, fields, _ = struct.unpack_from("<8sIIiiiiqqII", raw, 0)
    sec = [struct.unpack_from("<QQQ", raw, 56 + 24 * i) for i in range(5)]
    return dict(magic=magic, version=version, header_bytes=hbytes, L=L, H=Hh, d=d, block_tokens=bt, n_docs=n_docs,
                n_blocks=n_blocks, fields=fields, sections=sec, raw=raw)


def _bank(seed, L, offsets):
    rng = np.random.default_rng(seed)
    C = int(offsets[-1])
    kr = rng.integers(0, 1 << 16, size=(L, C, H, D), dtype=np.uint16)
    f8 = rng.integers(0, 256, size=(L, C, H, D), dtype=np.uint8)
    kv = rng.integers(0, 1 << 16, size=(L, C, 2, H, D), dtype=np.uint16)
    nr = rng.random((L, C, H), dtype=np.float32)
    return kr, f8, kv, nr


def _info(msa, L, n_docs, C, fields):
    return msa.MsaBankInfo(n_layers=L, n_heads=H, head_dim=D, block_tokens=64, n_docs=n_docs, n_blocks=C,
                           fields=fields)


def test_file_matches_documented_format(msa, tmp_path):
    offs = np.array([0, 3, 3, 7, 12], dtype=np.int64)
    L = 2
    kr, f8, kv, nr = _bank(1, L, offs)
    p = tmp_path / "a.msab"
    fields = msa.MSA_BANK_KR | msa.MSA_BANK_KR_F8 | msa.MSA_BANK_KV | msa.MSA_BANK_NORM
    msa.msa_bank_save(p, _info(msa, L, 4, 12, fields), offs, kr, f8, kv, nr)
    f = _parse(p)
    assert f["magic"] == b"MSABANK1" and f["version"] == 1 and f["header_bytes"] == 256
    assert (f["L"], f["H"], f["d"], f["block_tokens"], f["n_docs"], f["n_blocks"]) == (L, H, D, 64, 4, 12)
    assert f["fields"] == fields
    arrays = [offs, kr, f8, kv, nr]
    last_end = 256
    for (off, nbytes, ck), a in zip(f["sections"], arrays):
        assert off % 4096 == 0 and off >= last_end and nbytes == a.nbytes
        body = f["raw"][off:off + nbytes]
        assert body == a.tobytes()
        assert ck == _checksum(body)
        last_end = off + nbytes
    assert len(f["raw"]) == last_end


def test_round_trip_and_partial_load(msa, tmp_path):
    offs = np.array([0, 5, 6, 6, 40], dtype=np.int64)
    L = 3
    kr, f8, kv, nr = _bank(2, L, offs)
    p = tmp_path / "b.msab"
    msa.msa_bank_save(p, _info(msa, L, 4, 40, msa.MSA_BANK_KR | msa.MSA_BANK_KV), offs, kr_hat=kr, content_kv=kv)
    info = msa.msa_bank_read_info(p)
    assert (info.n_layers, info.n_docs, info.n_blocks, info.fields) == (L, 4, 40, msa.MSA_BANK_KR | msa.MSA_BANK_KV)
    o2 = np.zeros(5, np.int64)
    kr2 = np.zeros_like(kr)
    kv2 = np.zeros_like(kv)
    msa.msa_bank_load(p, o2, kr_hat=kr2, content_kv=kv2)
    assert np.array_equal(o2, offs) and np.array_equal(kr2, kr) and np.array_equal(kv2, kv)
    kr3 = np.zeros_like(kr)
    msa.msa_bank_load(p, o2, kr_hat=kr3)  # content skipped
    assert np.array_equal(kr3, kr)
    with pytest.raises(msa.MsaError) as e:  # the file has no E4M3 section
        msa.msa_bank_load(p, o2, kr_f8=np.zeros_like(f8))
    assert e.value.status == msa.MSA_ERR_INVALID_ARG


def test_empty_bank_round_trip(msa, tmp_path):
    p = tmp_path / "e.msab"
    msa.msa_bank_save(p, _info(msa, 1, 0, 0, msa.MSA_BANK_KR), np.zeros(1, np.int64), kr_hat=np.zeros(0, np.uint16))
    info = msa.msa_bank_read_info(p)
    assert info.n_docs == 0 and info.n_blocks == 0
    o = np.full(1, 7, np.int64)
    msa.msa_bank_load(p, o, kr_hat=np.zeros(1, np.uint16))
    assert o.tolist() == [0]


def test_damaged_files_are_rejected(msa, tmp_path):
    offs = np.array([0, 2, 9], dtype=np.int64)
    kr, _, _, _ = _bank(3, 1, offs)
    p = tmp_path / "c.msab"
    msa.msa_bank_save(p, _info(msa, 1, 2, 9, msa.MSA_BANK_KR), offs, kr_hat=kr)
    raw = bytearray(open(p, "rb").read())
    kr_off = struct.unpack_from("<Q", raw, 56 + 24)[0]
    cases = {"flip": (kr_off + 1000, None), "magic": (0, None), "truncate": (None, len(raw) - 100),
             "offsets": (4096, None)}
    for name, (pos, cut) in cases.items():
        bad = bytearray(raw)
        if pos is not None:
            bad[pos] ^= 0x40
        if cut is not None:
            bad = bad[:cut]
        q = tmp_path / f"bad_{name}.msab"
        q.write_bytes(bytes(bad))
        with pytest.raises(msa.MsaError) as e:
            msa.msa_bank_load(q, np.zeros(3, np.int64), kr_hat=np.zeros_like(kr))
        assert e.value.status == msa.MSA_ERR_IO, name
    with pytest.raises(msa.MsaError) as e:
        msa.msa_bank_read_info(tmp_path / "missing.msab")
    assert e.value.status == msa.MSA_ERR_IO


def test_save_rejects_bad_offsets(msa, tmp_path):
    kr = np.zeros((1, 4, H, D), np.uint16)
    for offs in ([0, 3, 2, 4], [1, 2, 3, 4], [0, 1, 2, 3]):
        with pytest.raises(msa.MsaError) as e:
            msa.msa_bank_save(tmp_path / "x.msab", _info(msa, 1, 3, 4, msa.MSA_BANK_KR), np.array(offs), kr_hat=kr)
        assert e.value.status == msa.MSA_ERR_INVALID_ARG


def test_append_offsets(msa):
    out = msa.msa_bank_append_offsets([0, 2, 2, 5], [0, 1, 4])
    assert out.tolist() == [0, 2, 2, 5, 6, 9]
    assert msa.msa_bank_append_offsets([0], [0, 3]).tolist() == [0, 3]
    assert msa.msa_bank_append_offsets([0, 4], [0]).tolist() == [0, 4]
    with pytest.raises(msa.MsaError):
        msa.msa_bank_append_offsets([0, 4, 3], [0, 1])


def test_host_relayout_leaves_room_per_layer(msa):
    L, old, new, row = 3, 5, 8, 16
    src = np.arange(L * old * row, dtype=np.uint8).reshape(L, old, row)
    dst = np.full((L, new, row), 0xEE, np.uint8)
    msa.msa_bank_relayout(src, dst, L, old, new, row)
    assert np.array_equal(dst[:, :old], src) and (dst[:, old:] == 0xEE).all()
    grow = np.full(L * new * row, 0xEE, np.uint8)  # grown in place
    grow[:src.size] = src.reshape(-1)
    msa.msa_bank_relayout(grow, grow, L, old, new, row)
    assert np.array_equal(grow.reshape(L, new, row)[:, :old], src)
