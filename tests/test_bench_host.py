"""Host-side accounting of the benchmark (FLOPs, bytes), checked on the CPU."""
import numpy as np

import bench


def test_live_pairs_sum_is_causal_triangle():
    for L, Bt in ((1024, 64), (1000, 128), (777, 64), (1, 128), (129, 128)):
        lp = bench.live_pairs(L, Bt, Bt)
        assert lp.sum() == L * (L + 1) // 2
        # brute force on the tile grid
        i = np.arange(L)[:, None]
        j = np.arange(L)[None, :]
        live = (j <= i).astype(np.int64)
        nq = -(-L // Bt)
        for qb in range(nq):
            for kb in range(nq):
                assert lp[qb, kb] == live[qb * Bt:(qb + 1) * Bt, kb * Bt:(kb + 1) * Bt].sum()


def test_train_flops_tau0_conventions():
    d, B, Hq, L = 128, 1, 4, 1000
    lp = bench.live_pairs(L, 128, 128)
    f = bench.train_flops(d, B, Hq, L, lp, None, None)
    n = B * Hq * L * (L + 1) // 2
    assert f["fwd"] == 4 * d * n
    assert f["bwd"] == 10 * d * n
    keep = np.zeros((B, Hq) + lp.shape, dtype=np.uint8)
    g = bench.train_flops(d, B, Hq, L, lp, keep, keep)
    assert g["fwd"] == 2 * d * n and g["bwd"] == 2 * d * n


def test_decode_bytes():
    B, Hq, Hkv, Lk, d, Bk = 2, 8, 2, 1000, 128, 128
    nk = -(-Lk // Bk)
    full = bench.decode_bytes(B, Hq, Hkv, Lk, d, Bk, None)
    assert full["k_all"] == B * Lk * Hkv * d * 2
    assert full["v_kept"] == full["k_all"]
    km = np.zeros((B, Hq, nk), dtype=np.uint8)
    km[0, 5, 3] = 1  # KV head 1 of batch 0, tile 3
    one = bench.decode_bytes(B, Hq, Hkv, Lk, d, Bk, km)
    assert one["v_kept"] == Bk * d * 2
    km[0, 4, 3] = 1  # same group, same tile: V still loaded once
    assert bench.decode_bytes(B, Hq, Hkv, Lk, d, Bk, km)["v_kept"] == Bk * d * 2
    km[0, 4, nk - 1] = 1  # ragged last tile
    assert bench.decode_bytes(B, Hq, Hkv, Lk, d, Bk, km)["v_kept"] == (Bk + Lk - (nk - 1) * Bk) * d * 2


def test_peaks_present():
    p = bench.peaks()
    assert p["hbm_gbs"] > 1000 and p["bf16_tflops"] > 100


def test_profiled_traffic_tracks_kernel_sources(tmp_path, monkeypatch):
    csrc = tmp_path / "mass_gated_causal_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "mala_bwd.cuh").write_text("kernel v1\n")
    (csrc / "mala_ptx.cuh").write_text("helpers\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("mala_bwd_kernel", "w") is None  # no summary
    h = bench.kernel_sources_sha256("mala_bwd_kernel")
    (tmp_path / "profiles" / "mala_bwd_kernel_w_dram.md").write_text(
        f"# dram\n\n- sources-sha256: `{h}`\n- dram-bytes-per-launch: 1234.5\n")
    assert bench.profiled_traffic("mala_bwd_kernel", "w") == 1234.5
    (csrc / "mala_bwd.cuh").write_text("kernel v2\n")  # the kernel changed since the capture
    assert bench.profiled_traffic("mala_bwd_kernel", "w") is None


def test_packed_flops_sum_per_sequence():
    """Packed accounting: at tau = 0 every sequence contributes its causal
    triangle (L(L+1)/2 live pairs per head); with keep maps, exactly the live
    pairs of the kept tiles of each sequence's corner count."""
    lens, Hq, d, Bt = [5, 17, 0, 9], 2, 8, 4
    fl0 = bench.packed_flops(lens, Hq, d, Bt, Bt, None, None)
    tri = sum(L * (L + 1) // 2 for L in lens) * Hq
    assert fl0["n_legal"] == fl0["n_f"] == fl0["n_b"] == tri
    assert fl0["fwd"] == 4 * d * tri and fl0["bwd"] == 10 * d * tri
    assert fl0["tiles"] == fl0["kept_f"] == Hq * sum(n * (n + 1) // 2 for n in (2, 5, 0, 3))
    rng = np.random.default_rng(0)
    km = rng.integers(0, 2, size=(4, Hq, 5, 5)).astype(np.uint8)
    fl = bench.packed_flops(lens, Hq, d, Bt, Bt, km, km)
    want = 0
    for s, L in enumerate(lens):  # live pairs (i, j <= i) of kept tiles, counted one by one
        for h in range(Hq):
            for i in range(L):
                for j in range(i + 1):
                    want += int(km[s, h, i // Bt, j // Bt] == 1)
    assert fl["n_f"] == fl["n_b"] == want
    assert fl["fwd"] == 2 * d * tri + 2 * d * want and fl["bwd"] == 2 * d * tri + 8 * d * want


def test_matched_work_sample_equals_the_oracle_analysis():
    # the bench's torch fp64 matched-work diagnostic (run on the GPU there) gives,
    # on the CPU, the per-row figures of oracle/matched_work.py for the same keep map
    import math

    import torch

    from oracle import fwd
    from oracle.matched_work import matched_work
    from workloads import TrainWorkload, bf16_bits_to_f64, make_train_inputs

    w = TrainWorkload("mw_host", 1, 2, 1, 300, 32, 16, 16, seed=9100)
    inp = make_train_inputs(w)
    qf, kf, vf = (bf16_bits_to_f64(inp[x]) for x in ("q", "k", "v"))
    keep = fwd(qf, kf, vf, w.scale, 1.0, w.Bq, w.Bk)["keep"]
    t = lambda a: torch.from_numpy(a)
    out = bench.matched_work_sample(torch, "cpu", t(qf), t(kf), t(vf), keep, w, n_blocks=6, seed=5)
    blocks = [tuple(int(x) for x in s.strip("() ").split(",")) for s in
              out["sample"].split(": ", 1)[1].strip("[]").split("), (")]
    ref = matched_work(qf, kf, vf, w.scale, 1.0, w.Bq, w.Bk, keep=keep)
    nq = -(-w.L // w.Bq)
    rows = np.concatenate([np.arange(h * w.L + qb * w.Bq, h * w.L + min((qb + 1) * w.Bq, w.L))
                           for (b, h, qb) in blocks])
    assert out["rows"] == rows.size
    assert math.isclose(out["slot_frac"], round(ref["slots"][rows].sum() / ref["live"][rows].sum(), 4))
    for key, name in (("omitted_mass_mala_mean", "omit_mala"), ("omitted_mass_ref_mean", "omit_ref"),
                      ("out_rel_err_mala_mean", "err_mala"), ("out_rel_err_ref_mean", "err_ref")):
        assert math.isclose(out[key], ref[name][rows].mean(), rel_tol=1e-3, abs_tol=1e-12), key
    assert nq == keep.shape[2]


def test_both_arms_report_the_same_config():
    from workloads import C2
    a = bench.bench_config(C2, 1.0, 1)
    assert a == bench.bench_config(C2, 1.0, 1) and a["workload"] == C2.name and a["tau"] == 1.0


def test_pair_v_tiles_counts_key_tiles_some_block_of_a_pair_keeps():
    # brute force over CTAs: a pair of 128-row query tiles (256 rows) loads a
    # key tile's V once if any of its query blocks keeps that tile
    rng = np.random.default_rng(5)
    for L, Bq in ((1000, 128), (777, 64), (300, 64)):
        nq, nk = -(-L // Bq), -(-L // 128)
        km = rng.choice(np.array([0, 1, 255], dtype=np.uint8), size=(2, 3, nq, nk))
        want = 0
        for b in range(2):
            for h in range(3):
                for r0 in range(0, L, 256):
                    blocks = [qb for qb in range(nq) if r0 <= qb * Bq < r0 + 256]
                    for kb in range(nk):
                        want += int(any(km[b, h, qb, kb] == 1 for qb in blocks))
        assert bench.pair_v_tiles(km, L, Bq) == want


def test_walked_key_tiles_brute_force():
    # every (b, hq, pair of 128-row tiles) walks the key tiles up to the one
    # holding its last row's key: the union over the pair's rows of the causal range
    for L, Bk in ((1, 128), (128, 64), (1000, 128), (777, 64), (4096, 128)):
        want = 0
        for r0 in range(0, L, 256):
            last = min(r0 + 256, L) - 1
            want += len({k // Bk for k in range(last + 1)})
        assert bench.walked_key_tiles(2, 3, L, Bk) == 6 * want
