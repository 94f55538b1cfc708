// mala_fwd.cuh -- MALA forward kernel for sm_100a.
//
// Method (agihunt.info, "MassAlloc Attention: Let Attention Allocate Its Own
// Compute", method paragraphs): every legal causal tile is scored; after the
// QK tile, the largest per-key contribution ratio exp(s - m)/l against the
// evolving online-softmax state is compared with tau/Lq (Lq = i + 1); tiles run
// from the diagonal toward earlier keys; the first legal tile is kept; one
// row that fails to skip keeps the tile for the whole query block; a skipped
// tile loads no V and does no softmax update and no PV; LSE is written.
//
// One CTA owns 128 query rows of one (b, hq) -- one query block when Bq = 128,
// two when Bq = 64 -- and walks key tiles kb = last ... 0.
//   warps 0-3  softmax / gate / epilogue: thread t owns row t, which is TMEM
//              lane t of the S and O accumulators
//   warp  4    TMA producer: Q once, K tiles through an NK-stage ring
//   warp  5    MMA issuer (one thread): S = Q K^T into a double-buffered TMEM
//              S, the V TMA of a tile once its keep vote is known, and
//              O += P V into TMEM
// The vote of tile t is published before V(t) is requested, so a skipped
// tile costs no V traffic. QK(t+1) is issued before the vote of t, so the
// tensor core scores the next tile while the gate of this one runs.
//
// Precision: S = Q K^T is bf16 x bf16 -> fp32. The PV product runs in fp16 x
// fp16 -> fp32: P (at most 2^8 thanks to the lazy-rescale bound) is rounded
// to fp16, and the softmax warps convert each landed V tile from bf16 to fp16
// in place in shared memory (exact for |v| inside the fp16 range). bf16 P
// would add an error as large as the bf16 rounding of O itself.
#pragma once

#include "mala_ptx.cuh"

namespace mala {

struct FwdParams {
  int B, Hq, Hkv, L, G;
  int nq, nk, n_super;
  float scale_log2;  // scale * log2(e): scores are kept in log2 units
  float log2_tau;    // log2(tau), used only when the gate is on
  float* lse;        // [B, Hq, L]
  int32_t* kept_tiles;
  uint8_t* keep_map;
  unsigned* status;
};

constexpr uint32_t kDecPV = 1u;     // some query block of the CTA keeps the tile
constexpr uint32_t kDecAbort = 2u;  // a wait gave up somewhere in the CTA

template <int D, int BK>
struct FwdLayout {
  static constexpr int BM = 128;
  static constexpr int NK = 3;
  static constexpr int NV = 2;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BK * D * 2;
  static constexpr int P_BYTES = BM * BK * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * KV_BYTES;
  static constexpr int OFF_P = OFF_V + NV * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  // barriers: q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV],
  //           s_full[2], sm_done[2], dec[2], pv_done, mma_final
  static constexpr int N_BARS = 1 + 2 * NK + 2 * NV + 2 + 2 + 2 + 1 + 1;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int MISC_BYTES = 64;
  static constexpr int BYTES = OFF_MISC + MISC_BYTES;
  static constexpr int ALLOC_BYTES = BYTES + 1024;  // slack for 1024-B alignment
  static constexpr int TMEM_NEED = 2 * BK + D;
  static constexpr int TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
  static_assert(ALLOC_BYTES <= 232448, "forward shared memory exceeds the per-CTA limit");
};

template <int D, int BK, bool kGate>
__global__ void __launch_bounds__(192, 1)
    mala_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const FwdParams p) {
  using Lay = FwdLayout<D, BK>;
  constexpr int BM = Lay::BM, BQ = BK, QPB = BM / BQ;
  constexpr int NK = Lay::NK, NV = Lay::NV;
  constexpr uint32_t IDESC_QK = idesc_bf16(128, BK, false, false);
  constexpr uint32_t IDESC_PV = idesc_f16(128, D, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Lay::OFF_Q;
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  uint8_t* sP = smem + Lay::OFF_P;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* k_full = bar_q + 1;
  uint64_t* k_empty = k_full + NK;
  uint64_t* v_full = k_empty + NK;
  uint64_t* v_empty = v_full + NV;
  uint64_t* s_full = v_empty + NV;
  uint64_t* sm_done = s_full + 2;
  uint64_t* dec_bar = sm_done + 2;
  uint64_t* pv_done = dec_bar + 2;
  uint64_t* mma_final = pv_done + 1;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  uint32_t* tmem_slot = misc + 0;
  int* abort_flag = reinterpret_cast<int*>(misc + 1);
  uint32_t* dec_flags = misc + 2;  // [2]
  uint32_t* vote = misc + 4;       // [2][4] per-tile keep/abort votes
  uint32_t* evote = misc + 12;     // [4] epilogue votes

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int nbh = p.B * p.Hq;
  const int bh = blockIdx.x % nbh;
  const int sb = p.n_super - 1 - static_cast<int>(blockIdx.x / nbh);  // longest rows first
  const int b = bh / p.Hq, hq = bh % p.Hq, hkv = hq / p.G;
  const int r0 = sb * BM;
  const int last_row = min(r0 + BM, p.L) - 1;
  const int kb_hi = last_row / BK;
  const int T = kb_hi + 1;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < NK; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < NV; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&sm_done[i], 128);
      mbar_init(&dec_bar[i], 1);
    }
    mbar_init(pv_done, 1);
    mbar_init(mma_final, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_o);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const FailState fs{abort_flag, p.status};

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, Lay::Q_BYTES);
      for (int h = 0; h < D / 64; ++h) tma_load_4d(&tm_q, bar_q, sQ + h * (BM * 128), h * 64, hq, r0, b);
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t % NK;
        if (t >= NK && !mbar_wait(&k_empty[st], ((t / NK) - 1) & 1, fs)) break;
        const int kb = kb_hi - t;
        mbar_arrive_expect_tx(&k_full[st], Lay::KV_BYTES);
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(&tm_k, &k_full[st], sK + st * Lay::KV_BYTES + h * (BK * 128), h * 64, hkv, kb * BK, b);
        issued = t + 1;
      }
      // let every load this thread issued land before the CTA can exit
      mbar_wait_drain(bar_q, 0);
      for (int t = max(0, issued - NK); t < issued; ++t) mbar_wait_drain(&k_full[t % NK], (t / NK) & 1);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV), sPa = smem_u32(sP);
      const uint32_t tO = tmem + 2 * BK;
      int nv = 0, npv = 0;
      bool ok = mbar_wait(bar_q, 0, fs);
      for (int t = 0; ok && t <= T; ++t) {
        if (t < T) {
          const int st = t % NK;
          if (!mbar_wait(&k_full[st], (t / NK) & 1, fs)) break;
          if (t >= 2 && !mbar_wait(&sm_done[t & 1], ((t - 2) >> 1) & 1, fs)) break;
          tc_fence_after();
          const uint32_t tS = tmem + (t & 1) * BK;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sdesc_sw128(sQa + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024);
            const uint64_t bd =
                sdesc_sw128(sKa + st * Lay::KV_BYTES + (kk >> 2) * (BK * 128) + (kk & 3) * 32, 16, 1024);
            umma_bf16_ss(tS, a, bd, IDESC_QK, kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[t & 1]);
          umma_commit(&k_empty[st]);
          if (!kGate) {  // no gate: V(t) is always needed, fetch it ahead
            const int slot = t % NV;
            if (t >= NV && !mbar_wait(&v_empty[slot], ((t / NV) - 1) & 1, fs)) break;
            mbar_arrive_expect_tx(&v_full[slot], Lay::KV_BYTES);
            for (int h = 0; h < D / 64; ++h)
              tma_load_4d(&tm_v, &v_full[slot], sV + slot * Lay::KV_BYTES + h * (BK * 128), h * 64, hkv,
                          (kb_hi - t) * BK, b);
            nv = t + 1;
          }
        }
        if (t >= 1) {
          const int u = t - 1;
          if (!mbar_wait(&dec_bar[u & 1], (u >> 1) & 1, fs)) break;
          const uint32_t dec = *reinterpret_cast<volatile uint32_t*>(&dec_flags[u & 1]);
          if (dec & kDecAbort) break;
          if (dec & kDecPV) {
            int vi;
            if (kGate) {  // the keep vote is known: only now request V(u)
              const int slot = nv % NV;
              if (nv >= NV && !mbar_wait(&v_empty[slot], ((nv / NV) - 1) & 1, fs)) break;
              mbar_arrive_expect_tx(&v_full[slot], Lay::KV_BYTES);
              for (int h = 0; h < D / 64; ++h)
                tma_load_4d(&tm_v, &v_full[slot], sV + slot * Lay::KV_BYTES + h * (BK * 128), h * 64, hkv,
                            (kb_hi - u) * BK, b);
              vi = nv++;
            } else {
              vi = u;
            }
            const int slot = vi % NV;
            if (!mbar_wait(&sm_done[u & 1], (u >> 1) & 1, fs)) break;  // P(u) written, O rescaled
            if (!mbar_wait(&v_full[slot], (vi / NV) & 1, fs)) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint64_t a = sdesc_sw128(sPa + (kk >> 2) * (BM * 128) + (kk & 3) * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(sVa + slot * Lay::KV_BYTES + kk * 2048, BK * 128, 1024);
              umma_bf16_ss(tO, a, bd, IDESC_PV, (npv > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(pv_done);
            umma_commit(&v_empty[slot]);
            ++npv;
          }
        }
      }
      umma_commit(mma_final);  // completes once every MMA above has finished
      for (int i = max(0, nv - NV); i < nv; ++i) mbar_wait_drain(&v_full[i % NV], (i / NV) & 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int tid = threadIdx.x;  // 0..127: row within the CTA
    const int row = r0 + tid;
    const bool row_ok = row < p.L;
    const int qi = tid / BQ;
    const int qb = sb * QPB + qi;
    const bool blk_exists = qb < p.nq;
    const int kbf = blk_exists ? (min((qb + 1) * BQ, p.L) - 1) / BK : -1;
    const float thr = kGate ? p.log2_tau - lg2_approx(static_cast<float>(row + 1)) : 0.f;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tO = tmem + 2 * BK + lane_base;
    const uint32_t sPa = smem_u32(sP), sQa = smem_u32(sQ);
    const float sl2 = p.scale_log2;
    float m_use = -INFINITY, l = 0.f;
    int npv = 0, kept_count = 0;
    bool local_abort = false, all_abort = false;
    uint32_t r[32];

    for (int t = 0; t < T; ++t) {
      const int kb = kb_hi - t;
      const bool ok = mbar_wait_warp(&s_full[t & 1], (t >> 1) & 1, fs);
      local_abort |= !ok;
      tc_fence_after();
      const uint32_t tS = tmem + (t & 1) * BK + lane_base;
      const bool diag = kb * BK + BK - 1 > r0;
      float M = -INFINITY;
      if (ok) {
#pragma unroll
        for (int ch = 0; ch < BK / 32; ++ch) {
          tmem_ld32(tS + ch * 32, r);
          tmem_ld_wait();
          if (!diag) {
#pragma unroll
            for (int j = 0; j < 32; ++j) M = fmaxf(M, __uint_as_float(r[j]));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (kb * BK + ch * 32 + j <= row) M = fmaxf(M, __uint_as_float(r[j]));
          }
        }
      }
      const bool legal = blk_exists && kb <= kbf;
      bool keep_r;
      if (!legal || !row_ok) keep_r = false;
      else if (kb == kbf || !kGate) keep_r = true;  // first legal tile / full attention
      else keep_r = M * sl2 >= m_use + lg2_approx(l) + thr;  // ratio >= tau/Lq, ties keep
      const unsigned bal = __ballot_sync(0xffffffffu, keep_r);
      if (lane == 0) vote[(t & 1) * 4 + warp] = (bal ? 1u : 0u) | (local_abort ? 2u : 0u);
      named_bar_sync(1, 128);
      const uint32_t v0 = vote[(t & 1) * 4 + 0], v1 = vote[(t & 1) * 4 + 1];
      const uint32_t v2 = vote[(t & 1) * 4 + 2], v3 = vote[(t & 1) * 4 + 3];
      const bool any_abort = ((v0 | v1 | v2 | v3) & 2u) != 0;
      const bool bk0 = QPB == 1 ? (((v0 | v1 | v2 | v3) & 1u) != 0) : (((v0 | v1) & 1u) != 0);
      const bool bk1 = QPB == 1 ? false : (((v2 | v3) & 1u) != 0);
      const bool my_keep = qi == 0 ? bk0 : bk1;
      const bool need_pv = bk0 || bk1;
      if (tid == 0) {
        dec_flags[t & 1] = (need_pv ? kDecPV : 0u) | (any_abort ? kDecAbort : 0u);
        mbar_arrive(&dec_bar[t & 1]);
      }
      if (any_abort) {
        all_abort = true;
        break;
      }
      if ((tid % BQ) == 0 && legal) {
        if (p.keep_map) p.keep_map[(static_cast<size_t>(bh) * p.nq + qb) * p.nk + kb] = my_keep ? 1 : 0;
        kept_count += my_keep ? 1 : 0;
      }
      if (need_pv) {
        if (npv > 0) local_abort |= !mbar_wait_warp(pv_done, (npv - 1) & 1, fs);
        tc_fence_after();
        if (my_keep) {  // warp-uniform: a warp's rows are in one query block
          const float mt = row_ok ? M * sl2 : -INFINITY;
          const float m_new = fmaxf(m_use, mt);
          // lazy rescale: move the offset only when the max grew by > 2^8
          const bool resc = m_new > m_use + 8.f;
          const float alpha = resc ? ex2_approx(m_use - m_new) : 1.f;
          const bool need_o = resc && l > 0.f;
          if (resc) {
            l *= alpha;
            m_use = m_new;
          }
          if (__any_sync(0xffffffffu, need_o)) {
            const float a = need_o ? alpha : 1.f;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
              tmem_ld32(tO + ch * 32, r);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * a);
              tmem_st32(tO + ch * 32, r);
            }
            tmem_st_wait();
          }
          float rs = 0.f;
#pragma unroll
          for (int ch = 0; ch < BK / 32; ++ch) {
            tmem_ld32(tS + ch * 32, r);
            tmem_ld_wait();
            uint32_t pk[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int key = kb * BK + ch * 32 + 2 * jj;
              const bool l0 = row_ok && (!diag || key <= row);
              const bool l1 = row_ok && (!diag || key + 1 <= row);
              const float p0 = l0 ? ex2_approx(fmaf(__uint_as_float(r[2 * jj]), sl2, -m_use)) : 0.f;
              const float p1 = l1 ? ex2_approx(fmaf(__uint_as_float(r[2 * jj + 1]), sl2, -m_use)) : 0.f;
              pk[jj] = pack_f16x2(p0, p1);
              rs += p0 + p1;  // the normaliser sums the fp32 probabilities
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int col = ch * 32 + c * 8;
              const uint32_t addr = sPa + (col >> 6) * (BM * 128) + sw128_offset(tid, (col & 63) >> 3);
              st_shared_v4(addr, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
            }
          }
          l += rs;
        } else {  // the other query block keeps this tile: my rows add nothing
#pragma unroll
          for (int c = 0; c < BK / 8; ++c) {
            const int col = c * 8;
            st_shared_v4(sPa + (col >> 6) * (BM * 128) + sw128_offset(tid, (col & 63) >> 3), 0u, 0u, 0u, 0u);
          }
        }
        // V of this tile (the npv-th V load of the CTA): bf16 -> fp16 in place
        {
          const int vslot = npv % NV;
          const bool vok = mbar_wait_warp(&v_full[vslot], (npv / NV) & 1, fs);
          local_abort |= !vok;
          if (vok) {
            const uint32_t vb = smem_u32(sV) + vslot * Lay::KV_BYTES;
#pragma unroll 4
            for (int c = tid; c < Lay::KV_BYTES / 16; c += 128) {
              uint32_t a0, a1, a2, a3;
              ld_shared_v4(vb + c * 16, a0, a1, a2, a3);
              st_shared_v4(vb + c * 16, bf16x2_to_f16x2(a0), bf16x2_to_f16x2(a1), bf16x2_to_f16x2(a2),
                           bf16x2_to_f16x2(a3));
            }
          }
        }
        fence_proxy_async_smem();
        ++npv;
      }
      tc_fence_before();
      mbar_arrive(&sm_done[t & 1]);
    }

    if (!all_abort) {
      // ---------------------------------------------------------- epilogue
      const bool okf = mbar_wait_warp(mma_final, 0, fs);
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      if (okf) {
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          tmem_ld32(tO + ch * 32, r);
          tmem_ld_wait();
          uint32_t pk[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj)
            pk[jj] = pack_bf16x2(__uint_as_float(r[2 * jj]) * inv_l, __uint_as_float(r[2 * jj + 1]) * inv_l);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int col = ch * 32 + c * 8;
            const uint32_t addr = sQa + (col >> 6) * (BM * 128) + sw128_offset(tid, (col & 63) >> 3);
            st_shared_v4(addr, pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
          }
        }
        fence_proxy_async_smem();
        if (row_ok) p.lse[static_cast<size_t>(bh) * p.L + row] = (m_use + lg2_approx(l)) * 0.69314718055994531f;
      }
      const unsigned okall = __ballot_sync(0xffffffffu, okf);
      if (lane == 0) evote[warp] = okall == 0xffffffffu ? 1u : 0u;
      named_bar_sync(1, 128);
      const bool store = (evote[0] & evote[1] & evote[2] & evote[3]) != 0;
      if (tid == 0 && store) {
        for (int h = 0; h < D / 64; ++h) tma_store_4d(&tm_o, sQ + h * (BM * 128), h * 64, hq, r0, b);
        tma_store_commit_and_wait();
      }
      if ((tid % BQ) == 0 && blk_exists && store) atomicAdd(&p.kept_tiles[bh], kept_count);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    if (lane == 0) mbar_wait_drain(mma_final, 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

}  // namespace mala
