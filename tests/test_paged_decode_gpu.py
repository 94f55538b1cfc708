"""MALA decode against a paged KV cache on the GPU (C ABI mala_decode_paged)
against the fp64 oracle.

Each sequence's cache is drawn with the decode recipe on its own seed, then
scattered page by page into shuffled K and V pools that also hold unrelated
pages; the block table's entries past a sequence's pages point at unrelated
pages (they must not be read). Lengths end inside and on page boundaries.
Decision rule and tolerances as for mala_decode (tests/test_decode_gpu.py,
tests/parity.py).
"""
import numpy as np
import pytest
import torch

import oracle
from parity import LSE_ABS, O_REL_L2, rel_l2
from test_decode_gpu import compare_decode_decisions
from workloads import DecodeWorkload, bf16_bits_to_f64, make_decode_inputs

pytestmark = pytest.mark.gpu


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def paged_inputs(lens, Hq, Hkv, d, page, seed, extra_pages=5):
    """bf16 bits: q [B,Hq,d]; pools [num_pages,page,Hkv,d]; int32 block table and lengths."""
    rng = np.random.default_rng(seed)
    qs, kcs, vcs = [], [], []
    for b, L in enumerate(lens):
        t = make_decode_inputs(DecodeWorkload("paged", 1, Hq, Hkv, L, d, page, seed=seed + 1 + b))
        qs.append(t["q"][0])
        kcs.append(t["kcache"][0])
        vcs.append(t["vcache"][0])
    npg = [-(-L // page) for L in lens]
    total = sum(npg) + extra_pages
    kp = rng.integers(0, 1 << 16, size=(total, page, Hkv, d), dtype=np.uint16) & 0xBFFF  # finite filler
    vp = rng.integers(0, 1 << 16, size=(total, page, Hkv, d), dtype=np.uint16) & 0xBFFF
    ids = rng.permutation(total)
    maxp = max(npg) + 2
    table = np.full((len(lens), maxp), ids[-1], dtype=np.int32)
    n = 0
    for b, L in enumerate(lens):
        for j in range(npg[b]):
            pid = ids[n]
            n += 1
            table[b, j] = pid
            rows = kcs[b][j * page:(j + 1) * page]
            kp[pid, :len(rows)] = rows
            vp[pid, :len(rows)] = vcs[b][j * page:(j + 1) * page]
    return {"q": np.stack(qs), "k_pages": kp, "v_pages": vp, "table": table,
            "seqlens": np.asarray(lens, dtype=np.int32), "kc": kcs, "vc": vcs}


CASES = [
    # lens, Hq, Hkv, d, page, tau, n_splits
    ([5000, 1, 128, 3333], 8, 2, 128, 128, 1.0, 3),
    ([5000, 1, 128, 3333], 8, 2, 128, 128, 0.0, 0),
    ([700, 4096, 65], 4, 4, 64, 64, 1.0, 5),
    ([2000, 2000], 32, 8, 128, 128, 4.0, 1),
]


@pytest.mark.parametrize("lens,Hq,Hkv,d,page,tau,n_splits", CASES)
def test_decode_paged(cuda_lib, lens, Hq, Hkv, d, page, tau, n_splits):
    inp = paged_inputs(lens, Hq, Hkv, d, page, seed=7000 + sum(lens))
    q, kp, vp = _dev(inp["q"]), _dev(inp["k_pages"]), _dev(inp["v_pages"])
    table = torch.from_numpy(inp["table"]).cuda()
    sl = torch.from_numpy(inp["seqlens"]).cuda()
    scale = d ** -0.5
    o, lse, kept, km, ns = cuda_lib.decode_paged(q, kp, vp, table, sl, scale, tau, n_splits=n_splits, keep_map=True)
    assert cuda_lib.mala_check_status() == 0
    ref = oracle.paged_decode(bf16_bits_to_f64(inp["q"]), bf16_bits_to_f64(inp["k_pages"]),
                              bf16_bits_to_f64(inp["v_pages"]), inp["table"], inp["seqlens"], scale, tau, ns)
    km_h, kept_h = km.cpu().numpy(), kept.cpu().numpy()
    B = len(lens)
    for b, L in enumerate(lens):
        nk = -(-L // page)
        assert np.isin(km_h[b, :, :nk], (0, 1)).all() and (km_h[b, :, nk:] == 255).all()
        dec = compare_decode_decisions(km_h[b:b + 1, :, :nk], ref["keep"][b:b + 1, :, :nk],
                                       ref["margin"][b:b + 1, :, :nk], nk, ns, [(0, h) for h in range(Hq)])
        assert dec["bad"] == 0, (b, dec["bad_sites"][:10])
        assert dec["in_margin"] + dec["cascaded"] <= 2, dec
        assert (kept_h[b * Hq:(b + 1) * Hq] == (km_h[b, :, :nk] == 1).sum(1)).all()
    e_o = rel_l2(o.float().cpu().numpy().astype(np.float64), ref["o"])
    e_lse = float(np.abs(lse.cpu().numpy().astype(np.float64) - ref["lse"]).max())
    print(f"[paged decode parity] lens={lens} H={Hq}/{Hkv} d={d} page={page} tau={tau} splits={ns}: "
          f"o_rel_l2={e_o:.3e} lse_abs={e_lse:.3e}")
    assert e_o <= O_REL_L2, e_o
    assert e_lse <= LSE_ABS, e_lse


def test_decode_paged_identity_table_is_contiguous_decode(cuda_lib):
    """Pages in order, equal lengths: exactly mala_decode on the contiguous cache."""
    w = DecodeWorkload("paged_eq", 3, 8, 2, 1536, 128, 128, seed=7101)
    t = make_decode_inputs(w)
    q, kc, vc = (_dev(t[x]) for x in ("q", "kcache", "vcache"))
    o1, lse1, kept1, km1, ns = cuda_lib.decode(q, kc, vc, w.scale, 1.0, 128, n_splits=4, keep_map=True)
    kp = kc.reshape(3 * 12, 128, 2, 128)
    vp = vc.reshape(3 * 12, 128, 2, 128)
    table = torch.arange(36, dtype=torch.int32, device="cuda").reshape(3, 12)
    sl = torch.full((3,), 1536, dtype=torch.int32, device="cuda")
    o2, lse2, kept2, km2, _ = cuda_lib.decode_paged(q, kp, vp, table, sl, w.scale, 1.0, n_splits=4, keep_map=True)
    assert cuda_lib.mala_check_status() == 0
    assert torch.equal(o1, o2) and torch.equal(lse1, lse2)
    assert torch.equal(kept1, kept2) and torch.equal(km1, km2)


def test_decode_paged_bad_tables_are_reported(cuda_lib):
    """A length above the table's capacity, or a page id outside the pool, is
    reported by mala_check_status (the kernel checks both before using them;
    an id outside the pool reads as zeros)."""
    inp = paged_inputs([300, 200], 4, 2, 64, 64, seed=7200)
    q, kp, vp = _dev(inp["q"]), _dev(inp["k_pages"]), _dev(inp["v_pages"])
    table = torch.from_numpy(inp["table"]).cuda()
    sl = torch.from_numpy(inp["seqlens"]).cuda()
    bad_len = sl.clone()
    bad_len[1] = table.shape[1] * 64 + 1
    cuda_lib.decode_paged(q, kp, vp, table, bad_len, 0.125, 1.0, n_splits=2)
    assert cuda_lib.mala_check_status() == cuda_lib.MALA_ERR_INVALID_ARG
    bad_pg = table.clone()
    bad_pg[0, 1] = kp.shape[0] + 7
    cuda_lib.decode_paged(q, kp, vp, bad_pg, sl, 0.125, 1.0, n_splits=2)
    assert cuda_lib.mala_check_status() == cuda_lib.MALA_ERR_INVALID_ARG
    cuda_lib.decode_paged(q, kp, vp, table, sl, 0.125, 1.0, n_splits=2)
    assert cuda_lib.mala_check_status() == 0
