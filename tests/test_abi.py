"""The C ABI library on a machine without a GPU: it loads, exports every symbol
include/mala.h declares, and rejects invalid arguments on the host before any
CUDA call. No compute call is made here."""
import os
import re

import pytest

import mass_gated_causal_b200 as mala

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mala.h")
S = 0  # stream handle; never reached by the rejected calls


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MALA_API\s+[\w\s\*]+?\b(mala_\w+)\s*\(", text)))


def test_header_symbols_exported():
    names = declared_symbols()
    assert len(names) >= 11
    for n in names:
        assert hasattr(mala._lib, n), n
    assert set(names) == set(mala.EXPORTED)


def test_status_strings_and_version():
    assert mala.mala_abi_version() == 1
    for code, name in ((0, "MALA_OK"), (1, "MALA_ERR_INVALID_ARG"), (2, "MALA_ERR_UNSUPPORTED"),
                       (3, "MALA_ERR_WORKSPACE"), (4, "MALA_ERR_CUDA"), (5, "MALA_ERR_DEVICE_TIMEOUT"),
                       (6, "MALA_ERR_RANGE")):
        assert mala.mala_status_string(code) == name
    assert mala.mala_status_string(99) == "MALA_ERR_UNKNOWN"


P = 256  # a fake, 256-byte aligned "device pointer": never dereferenced by the rejected calls


def fwd(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, Hq=2, Hkv=1, L=100, d=128, scale=0.1, tau=1.0, Bq=128, Bk=128,
             workspace=P, workspace_bytes=1 << 30, kept_tiles=P, keep_map=None, stream=S)
    a.update(kw)
    return mala.mala_fwd(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(lse=None), 1), (dict(kept_tiles=None), 1),
    (dict(B=0), 1), (dict(L=0), 1), (dict(Hq=3, Hkv=2), 1),
    (dict(scale=0.0), 1), (dict(scale=float("nan")), 1), (dict(tau=-1.0), 1), (dict(tau=float("inf")), 1),
    (dict(d=96), 2), (dict(Bq=96, Bk=128), 2), (dict(Bq=128, Bk=256), 2), (dict(Bq=32, Bk=32), 2),
    (dict(q=P + 8), 2),
    (dict(workspace=None), 3), (dict(workspace_bytes=100), 3), (dict(workspace=P + 16), 3),
])
def test_fwd_rejects(kw, code):
    assert fwd(**kw) == code


def pre(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, Hq=2, Hkv=1, Lq=100, Lk=300, d=128, scale=0.1, tau=1.0, Bq=128,
             Bk=64, workspace=P, workspace_bytes=1 << 30, kept_tiles=P, keep_map=None, stream=S)
    a.update(kw)
    return mala.mala_prefill(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(v=None), 1), (dict(o=None), 1), (dict(kept_tiles=None), 1), (dict(Lq=0), 1), (dict(Lk=99), 1),
    (dict(Lq=0, Lk=0), 1), (dict(Hq=4, Hkv=3), 1), (dict(tau=float("nan")), 1),
    (dict(d=256), 2), (dict(Bq=256), 2), (dict(Bk=32), 2), (dict(lse=P + 4), 2),
    (dict(workspace=None), 3), (dict(workspace=P + 128), 3),
    # the fp16 V copy covers all Lk keys, not only the new ones
    (dict(workspace_bytes=(300 * 128 * 2 + 255) // 256 * 256 - 1), 3),
])
def test_prefill_rejects(kw, code):
    assert pre(**kw) == code


def fvl(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, cu_seqlens_q=P, cu_seqlens_k=P, num_seqs=3, max_seqlen_q=100,
             max_seqlen_k=200, total_q=250, total_k=400, Hq=4, Hkv=2, d=128, scale=0.1, tau=1.0, Bq=128, Bk=64,
             workspace=P, workspace_bytes=1 << 30, kept_tiles=P, keep_map=None, stream=S)
    a.update(kw)
    return mala.mala_fwd_varlen(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(cu_seqlens_q=None), 1), (dict(cu_seqlens_k=None), 1), (dict(lse=None), 1), (dict(num_seqs=0), 1),
    (dict(max_seqlen_q=0), 1), (dict(total_k=0), 1), (dict(max_seqlen_q=300), 1), (dict(max_seqlen_k=500), 1),
    (dict(Hq=3), 1), (dict(tau=-1.0), 1),
    (dict(d=32), 2), (dict(Bq=32), 2), (dict(v=P + 8), 2),
    (dict(workspace=None), 3), (dict(workspace=P + 64), 3),
    # the fp16 V copy covers all total_k key rows
    (dict(workspace_bytes=(400 * 2 * 128 * 2 + 255) // 256 * 256 - 1), 3),
])
def test_fwd_varlen_rejects(kw, code):
    assert fvl(**kw) == code


def bvl(**kw):
    a = dict(q=P, k=P, v=P, o=P, do=P, lse=P, dq=P, dk=P, dv=P, cu_seqlens=P, num_seqs=2, max_seqlen=300, total=400,
             Hq=4, Hkv=2, d=64, scale=0.1, tau=1.0, Bq=64, Bk=128, workspace=P, workspace_bytes=1 << 30,
             kept_tiles=P, keep_map=None, stream=S)
    a.update(kw)
    return mala.mala_bwd_varlen(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(cu_seqlens=None), 1), (dict(dk=None), 1), (dict(num_seqs=0), 1), (dict(max_seqlen=401), 1),
    (dict(total=0), 1), (dict(Hq=5), 1), (dict(d=100), 2), (dict(Bk=96), 2), (dict(dq=P + 2), 2),
    (dict(workspace=None), 3),
    (dict(workspace_bytes=(400 * 4 * 64 * 4 + 255) // 256 * 256 + (4 * 400 * 4 + 255) // 256 * 256 - 1), 3),
])
def test_bwd_varlen_rejects(kw, code):
    assert bvl(**kw) == code


def dpg(**kw):
    a = dict(q=P, k_pages=P, v_pages=P, block_table=P, seqlens_k=P, o=P, lse=P, B=4, Hq=8, Hkv=2, num_pages=100,
             page_size=128, max_pages_per_seq=40, d=128, scale=0.1, tau=1.0, n_splits=4, workspace=P,
             workspace_bytes=1 << 30, kept_tiles=P, keep_map=None, stream=S)
    a.update(kw)
    return mala.mala_decode_paged(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(block_table=None), 1), (dict(seqlens_k=None), 1), (dict(num_pages=0), 1), (dict(max_pages_per_seq=0), 1),
    (dict(q=None), 1), (dict(Hq=6, Hkv=4), 1), (dict(n_splits=-2), 1),
    (dict(page_size=32), 2), (dict(page_size=256), 2), (dict(d=96), 2), (dict(Hq=64, Hkv=2), 2),
    (dict(max_pages_per_seq=1 << 24), 2), (dict(k_pages=P + 8), 2),
    (dict(workspace=None), 3), (dict(workspace_bytes=64), 3),
])
def test_decode_paged_rejects(kw, code):
    assert dpg(**kw) == code


def bwd(**kw):
    a = dict(q=P, k=P, v=P, o=P, do=P, lse=P, dq=P, dk=P, dv=P, B=1, Hq=2, Hkv=1, L=100, d=128, scale=0.1,
             tau=1.0, Bq=128, Bk=128, workspace=P, workspace_bytes=1 << 30, kept_tiles=P, keep_map=None, stream=S)
    a.update(kw)
    return mala.mala_bwd(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(do=None), 1), (dict(dq=None), 1), (dict(Hq=3, Hkv=2), 1), (dict(d=80), 2),
    (dict(dv=P + 4), 2), (dict(workspace=None), 3), (dict(workspace_bytes=10), 3), (dict(workspace=P + 16), 3),
])
def test_bwd_rejects(kw, code):
    assert bwd(**kw) == code


def test_fwd_workspace_size():
    a256 = lambda x: (x + 255) // 256 * 256
    assert mala.mala_fwd_workspace_size(2, 4, 1000, 128) == a256(2 * 1000 * 4 * 128 * 2)
    assert mala.mala_fwd_workspace_size(2, 4, 1000, 96) == 0


def test_bwd_workspace_size():
    B, Hq, L, d = 2, 4, 1000, 128
    a256 = lambda x: (x + 255) // 256 * 256
    assert mala.mala_bwd_workspace_size(B, Hq, L, d) == a256(B * L * Hq * d * 4) + a256(B * Hq * L * 4)
    assert mala.mala_bwd_workspace_size(0, Hq, L, d) == 0
    assert mala.mala_bwd_workspace_size(B, Hq, L, 100) == 0


def dec(**kw):
    a = dict(q=P, kcache=P, vcache=P, o=P, lse=P, B=2, Hq=8, Hkv=2, Lk=1000, d=128, scale=0.1, tau=1.0, Bk=128,
             n_splits=4, workspace=P, workspace_bytes=1 << 30, kept_tiles=P, keep_map=None, stream=S)
    a.update(kw)
    return mala.mala_decode(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(Hq=6, Hkv=4), 1), (dict(n_splits=-1), 1), (dict(tau=-0.5), 1),
    (dict(d=32), 2), (dict(Bk=256), 2), (dict(Hq=32, Hkv=2), 2), (dict(o=P + 2), 2),
    (dict(workspace=None), 3), (dict(workspace_bytes=100), 3),
])
def test_decode_rejects(kw, code):
    assert dec(**kw) == code


def dex(**kw):
    a = dict(q=P, kcache=P, vcache=P, o=P, lse=P, B=2, Hq=8, Hkv=2, Lk=1000, d=128, scale=0.1, tau=1.0, Bk=128,
             n_splits=4, workspace=P, workspace_bytes=1 << 30, kept_tiles=P, keep_map=None, stream=S)
    a.update(kw)
    return mala.mala_decode_exact(**a)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), 1), (dict(lse=None), 1), (dict(Hq=6, Hkv=4), 1), (dict(n_splits=-1), 1), (dict(tau=-0.5), 1),
    (dict(d=32), 2), (dict(Bk=256), 2), (dict(Hq=32, Hkv=2), 2), (dict(vcache=P + 2), 2),
    (dict(workspace=None), 3), (dict(workspace_bytes=1000), 3), (dict(workspace=P + 32), 3),
])
def test_decode_exact_rejects(kw, code):
    assert dex(**kw) == code


def test_decode_exact_workspace_size():
    a256 = lambda x: (x + 255) // 256 * 256
    B, Hq, Lk, d, Bk, S = 2, 8, 1000, 128, 128, 5
    nk = -(-Lk // Bk)
    want = a256(B * Hq * nk * Bk * 4) + a256(B * Hq * nk * 8) + a256(B * Hq * nk) + a256(B * Hq * S * d * 4) + \
        a256(B * Hq * S * 4)
    assert mala.mala_decode_exact_workspace_size(B, Hq, Lk, d, Bk, S) == want
    assert mala.mala_decode_exact_workspace_size(B, Hq, Lk, d, 96, S) == 0
    assert mala.mala_decode_exact_workspace_size(B, Hq, Lk, d, Bk, 0) == 0


def test_decode_sizes_and_default_splits():
    a256 = lambda x: (x + 255) // 256 * 256
    assert mala.mala_decode_workspace_size(2, 8, 128, 5) == a256(2 * 8 * 5 * 128 * 4) + a256(2 * 8 * 5 * 4)
    assert mala.mala_decode_workspace_size(2, 8, 128, 0) == 0
    s = mala.mala_decode_default_splits(8, 8, 131072, 128)
    nk = 1024
    T = -(-nk // s)
    assert 1 <= s <= nk and -(-nk // T) == s  # every split non-empty
    assert mala.mala_decode_default_splits(1, 1, 1, 128) == 1
    assert mala.mala_decode_noalloc_max_bytes() == 8 << 20


def test_noalloc_rejects_on_host():
    kw = dict(q=P, kcache=P, vcache=P, o=P, lse=P, B=64, Hq=64, Hkv=8, Lk=65536, d=128, scale=0.1, tau=1.0,
              Bk=128, n_splits=512, kept_tiles=P, keep_map=None, stream=S)
    assert mala.mala_decode_noalloc(**kw) == 3  # partials beyond the fixed 8 MiB scratch
    kw.update(q=None)
    assert mala.mala_decode_noalloc(**kw) == 1
