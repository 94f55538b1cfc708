// mala_bwd.cuh -- MALA backward kernels for sm_100a.
//
// Method (agihunt.info, "MassAlloc Attention: Let Attention Allocate Its Own
// Compute", method paragraphs): the backward recomputes the scores of every
// legal tile and tests each tile against the FINAL log-normaliser written by
// the forward -- keep iff some live (i, j) has exp(s_ij - LSE_i) >= tau/(i+1)
// -- with no stored mask and no forced tile. A skipped tile does no
// probability reconstruction, no dP, dS, dQ, dK or dV.
//
// Kernels:
//   mala_bwd_pre_kernel   D_i = <dO_i, O_i>, clears the fp32 dQ accumulator
//                         and the per-head counters
//   mala_bwd_kernel       dK/dV-stationary main loop (below)
//   mala_dq_convert_kernel fp32 dQ accumulator -> bf16 dQ
//
// mala_bwd_kernel: one CTA owns 128 keys (one key block when Bk = 128, two
// when Bk = 64) of one (b, KV head) and walks the query tiles of every query
// head of the GQA group, 128 queries at a time, from the diagonal tile to the
// last, each tile for all heads of the group in turn. dK and dV accumulate in
// TMEM across the whole walk. 14 warps:
//   warps 0-7   compute: thread t owns query row t % 128 of the current tile
//               and key columns [64h, 64h + 64), h = t / 128 (TMEM lane row of
//               S and dP), so its LSE, gate threshold and D are scalars: gate,
//               P (kept in registers), dS; at the end, key row t % 128, half h
//               of the dK and dV columns
//   warps 8-11  dQ drain: thread t owns query row t of a kept tile's dQ and
//               adds it to the fp32 accumulator by TMA reduce-add, while the
//               compute warps move on
//   warp  12    producer: K, V once; Q and dO tiles ahead (dO before the gate
//               has decided: nearly every tile is kept)
//   warp  13    MMA issuer: S = Q K^T, then for kept tiles dP = dO V^T,
//               dV += P^T dO, the next tile's S, dK += dS^T Q, dQ = dS K
// TMEM: two 128-column regions taken by tiles in turn (S, then dP over S,
// then dQ over dP), then dK and dV. P and dS share one shared-memory tile
// (query rows, 128-byte swizzle): dS overwrites P once the dV MMA that reads
// P^T (MN-major) has finished.
#pragma once

#include "mala_ptx.cuh"

namespace mala {

struct BwdParams {
  int B, Hq, Hkv, L, G;
  int nq, nk, n_super;
  int chunk_kb;  // CTA schedule: key blocks per chunk (see mala_bwd_kernel)
  float scale, scale_log2, log2_tau;
  const float* lse;   // [B, Hq, L]; packed batches: [Hq, total]
  const float* dvec;  // same layout as lse: D_i
  const int* cu;      // packed batch (else null): sequence b owns rows cu[b] .. cu[b+1]; L is the longest
  int total;          // packed batch: rows in all
  uint16_t* dk_out;   // dK, dV (bf16), for the row-wise stores of a packed batch's partial key tiles
  uint16_t* dv_out;
  float* dq_acc;      // [B, L, Hq, d] fp32 (the kernel adds into it through its tensor map)
  int32_t* kept_tiles;
  uint8_t* keep_map;
  unsigned* status;
  uint64_t wait_ns;  // limit of each bounded wait
  int stall_tile;    // test hook (-1: off): the MMA thread stalls before this tile
};

// bf16x2 of (lo, hi) by integer ops on the ALU pipe: nearest, halfway cases
// away from zero (the conversion instruction shares the pipe that computes
// exp2, which the P pass keeps busy; measured 2-4% faster on the backward)
__device__ __forceinline__ uint32_t pack_bf16x2_alu(float lo, float hi) {
  return __byte_perm(__float_as_uint(lo) + 0x8000u, __float_as_uint(hi) + 0x8000u, 0x7632);
}

constexpr uint32_t kBwdAny = 1u << 4;
constexpr uint32_t kBwdAbort = 1u << 5;

template <int D>
struct BwdLayout {
  static constexpr int T_BYTES = 128 * D * 2;  // a 128-row tile of K, V, Q or dO
  static constexpr int PS_BYTES = 128 * 128 * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + T_BYTES;
  static constexpr int OFF_Q = OFF_V + T_BYTES;  // 2 stages
  static constexpr int OFF_DO = OFF_Q + 2 * T_BYTES;
  static constexpr int OFF_PS = OFF_DO + T_BYTES;
  static constexpr int STG_BUF = 32 * 32 * 4;   // dQ staging block: [32 rows x 32] fp32
  static constexpr int STG_WARP = 2 * STG_BUF;  // two blocks per drain warp
  static constexpr int OFF_STG = OFF_PS + PS_BYTES;  // 1024-aligned (128-byte swizzle)
  static constexpr int OFF_BAR = OFF_STG + 4 * STG_WARP;
  // kv_full, q_full[2], q_empty[2], s_full, dec, do_full, do_empty, p_ready,
  // dv_done, ds_ready, dq_full, dq_free, ps_free, mma_final, info_full
  static constexpr int N_BARS = 17;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int BYTES = OFF_MISC + 128;
  static constexpr int ALLOC_BYTES = BYTES + 1024;
  static constexpr int TMEM_COLS = 512;  // S 128 | dP/dQ 128 | dK D | dV D
  static_assert(ALLOC_BYTES <= 232448, "backward shared memory exceeds the per-CTA limit");
};

// kPacked: a packed batch (p.cu set); the dense instantiation keeps every
// length and offset a kernel parameter.
template <int D, int BQ, int BK, bool kGate, bool kPacked>
__global__ void __launch_bounds__(448, 1)
    mala_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                    const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using Lay = BwdLayout<D>;
  constexpr int QPB = 128 / BQ, KPB = 128 / BK;
  constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
  constexpr uint32_t IDESC_KN = idesc_bf16(128, D, false, true);  // A K-major, B MN-major
  constexpr uint32_t IDESC_MN = idesc_bf16(128, D, true, true);   // A, B MN-major
  constexpr int TB = Lay::T_BYTES;
  constexpr uint32_t kNegInfBits = 0xff800000u;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  uint8_t* sQ = smem + Lay::OFF_Q;
  uint8_t* sDO = smem + Lay::OFF_DO;
  uint8_t* sPS = smem + Lay::OFF_PS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* q_full = bars + 1;   // [2]
  uint64_t* q_empty = bars + 3;  // [2]
  uint64_t* s_full = bars + 5;
  uint64_t* dec_bar = bars + 6;  // also tells the MMA issuer that S(t) is out of TMEM
  uint64_t* do_full = bars + 7;
  uint64_t* do_empty = bars + 8;
  uint64_t* p_ready = bars + 9;
  uint64_t* dv_done = bars + 10;  // dP(t) was issued before dV(t): its completion too
  uint64_t* ds_ready = bars + 11;
  uint64_t* dq_full = bars + 12;
  uint64_t* dq_free = bars + 13;
  uint64_t* ps_free = bars + 14;
  uint64_t* mma_final = bars + 15;
  uint64_t* info_full = bars + 16;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  uint32_t* tmem_slot = misc + 0;
  int* abort_flag = reinterpret_cast<int*>(misc + 1);
  uint32_t* dec_flags = misc + 2;
  uint32_t* vote = misc + 4;    // [2][8]
  uint32_t* evote = misc + 20;  // [8]
  int* info = reinterpret_cast<int*>(misc + 28);  // {hq, i0, TMEM region} of the next kept tile to drain

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA schedule: the grid is cut into chunks of chunk_kb key blocks, longest
  // walks (lowest key blocks) first; inside a chunk the (b, KV head) units
  // follow one another. The CTAs resident at one time then read the Q / dO
  // tiles and add into the dQ rows of one or two KV heads' query heads, which
  // stay in L2. The last chunk may be padded with empty CTAs.
  const int per_chunk = p.B * p.Hkv * p.chunk_kb;
  const int chunk = static_cast<int>(blockIdx.x) / per_chunk;
  const int in_chunk = static_cast<int>(blockIdx.x) % per_chunk;
  const int bk = in_chunk / p.chunk_kb;
  const int ks = chunk * p.chunk_kb + in_chunk % p.chunk_kb;
  const int b = bk / p.Hkv, hkv = bk % p.Hkv;
  // This CTA's sequence: L rows; a packed batch gives each sequence its own
  // length and row offset (the grid covers the longest sequence, and a CTA past
  // its sequence's rows leaves at once).
  int L = p.L, off = 0, bt = b;
  if (kPacked) {
    off = __ldg(p.cu + b);
    L = __ldg(p.cu + b + 1) - off;
    bt = 0;
    if (off < 0 || L < 0 || L > p.L || off + L > p.total) {  // nothing of this sequence is touched
      if (threadIdx.x == 0 && ks == 0) atomicOr(p.status, kStatusSeqTable);
      return;
    }
  }
  const int n_super = (L + 127) / 128;
  const int nq_b = (L + BQ - 1) / BQ, nk_b = (L + BK - 1) / BK;
  if (ks >= n_super) return;  // padding (uniform across the CTA, before any shared state)
  const int k0 = ks * 128;
  const int nqs = n_super - ks;
  const int T = p.G * nqs;
  // Walk order: query tiles from the diagonal to the last, and for each the G
  // query heads of the group in turn, so the CTAs of a KV head move through
  // the query rows G times slower and their Q / dO / dQ lines stay in L2
  // longer (1-3% faster than one head after the other, measured at 32K GQA
  // across tau). Walking every CTA of a KV head through the same tiles in
  // step was measured slower (their dQ additions then hit the same lines at
  // once), and so were staggered groups. The backward decisions do not depend
  // on the order.
  auto walk_hq = [&](int t) { return hkv * p.G + t % p.G; };
  auto walk_qs = [&](int t) { return ks + t / p.G; };

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dec_bar, 1);
    mbar_init(do_full, 1);
    mbar_init(do_empty, 1);
    mbar_init(p_ready, 256);
    mbar_init(dv_done, 1);
    mbar_init(ds_ready, 256);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(ps_free, 1);
    mbar_init(mma_final, 1);
    mbar_init(info_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(tmem_slot, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const FailState fs{abort_flag, p.status, p.wait_ns};
  // TMEM: two 128-column regions taken by tiles in turn (tile t uses region
  // t & 1 for S, then dP, then dQ), then dK and dV.
  const uint32_t tDK = tmem + 256, tDV = tmem + 256 + D;

  if (warp == 12) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, 2 * TB);
      for (int h = 0; h < D / 64; ++h) {
        tma_load_4d(&tm_k, kv_full, sK + h * 16384, h * 64, hkv, off + k0, bt);
        tma_load_4d(&tm_v, kv_full, sV + h * 16384, h * 64, hkv, off + k0, bt);
      }
    }
    int issued_q = 0, issued_do = 0;
    for (int t = 0; t < T; ++t) {
      const int st = t & 1;
      if (t >= 2 && !mbar_wait_warp(&q_empty[st], ((t >> 1) - 1) & 1, fs)) break;
      const int hq = walk_hq(t);
      const int i0 = walk_qs(t) * 128;
      if (lane == 0) {
        mbar_arrive_expect_tx(&q_full[st], TB);
        for (int h = 0; h < D / 64; ++h) tma_load_4d(&tm_q, &q_full[st], sQ + st * TB + h * 16384, h * 64, hq, off + i0, bt);
      }
      issued_q = t + 1;
      // dO of the same tile, before the gate has decided: the buffer is free as
      // soon as the previous tile's dP and dV have read it, and nearly every
      // tile is kept
      if (t >= 1 && !mbar_wait_warp(do_empty, (t - 1) & 1, fs)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(do_full, TB);
        for (int h = 0; h < D / 64; ++h) tma_load_4d(&tm_do, do_full, sDO + h * 16384, h * 64, hq, off + i0, bt);
      }
      issued_do = t + 1;
    }
    if (lane == 0) {
      mbar_wait_drain(kv_full, 0);
      for (int t = max(0, issued_q - 2); t < issued_q; ++t) mbar_wait_drain(&q_full[t & 1], (t >> 1) & 1);
      if (issued_do >= 1) mbar_wait_drain(do_full, (issued_do - 1) & 1);
    }
    __syncwarp();
  } else if (warp == 13) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // operand descriptors, built once: K-major (k-steps inside 64-column
      // atoms) and MN-major (k-steps of 16 rows) views of each tile
      const uint64_t dKk = sdesc_sw128(smem_u32(sK), 16, 1024), dKm = sdesc_sw128(smem_u32(sK), 16384, 1024);
      const uint64_t dVk = sdesc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dQk = sdesc_sw128(smem_u32(sQ), 16, 1024), dQm = sdesc_sw128(smem_u32(sQ), 16384, 1024);
      const uint64_t dOk = sdesc_sw128(smem_u32(sDO), 16, 1024), dOm = sdesc_sw128(smem_u32(sDO), 16384, 1024);
      const uint64_t dPk = sdesc_sw128(smem_u32(sPS), 16, 1024), dPm = sdesc_sw128(smem_u32(sPS), 16384, 1024);
      int nd = 0;
      int reg_kept0 = -1, reg_kept1 = -1;  // kept-tile index whose dQ still occupies region 0 / 1
      int dq_seen = -1;                    // highest kept-tile index whose dQ is known drained
      // S(t) = Q K^T into region t & 1, once Q(t) has landed and the dQ that
      // last used the region has been drained (one wait for both)
      auto issue_qk = [&](int t) -> bool {
        const int r = t & 1;
        const int pend = r ? reg_kept1 : reg_kept0;
        if (pend >= 0) {
          if (!mbar_wait2(&q_full[t & 1], (t >> 1) & 1, dq_free, pend & 1, fs)) return false;
          dq_seen = max(dq_seen, pend);
          if (r) reg_kept1 = -1; else reg_kept0 = -1;
        } else if (!mbar_wait(&q_full[t & 1], (t >> 1) & 1, fs)) {
          return false;
        }
        tc_fence_after();
        const uint64_t qa = sdesc_add(dQk, (t & 1) * TB);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_bf16_ss(tmem + r * 128, sdesc_add(qa, off), sdesc_add(dKk, off), IDESC_S, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full);
        return true;
      };
      bool ok = mbar_wait(kv_full, 0, fs);
      if (ok) ok = issue_qk(0);
      for (int t = 0; ok && t < T; ++t) {
        const int st = t & 1;
        const int hq = walk_hq(t);
        const int i0 = walk_qs(t) * 128;
        const uint32_t tR = tmem + (t & 1) * 128;
        // test hook: wait on a barrier only this thread completes (after the
        // loop), so the bounded wait expires and the CTA takes its abort path
        if (t == p.stall_tile && !mbar_wait(mma_final, 0, fs)) break;
        // the gate's decision (the compute warps have read S(t) out of the
        // region before voting) and dO(t), loaded ahead: one wait for both
        if (!mbar_wait2(dec_bar, t & 1, do_full, t & 1, fs)) break;
        const uint32_t dec = *reinterpret_cast<volatile uint32_t*>(dec_flags);
        if (dec & kBwdAbort) break;
        const bool keep = (dec & kBwdAny) != 0;
        if (keep) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {  // dP = dO V^T, over S in the same region
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16_ss(tR, sdesc_add(dOk, off), sdesc_add(dVk, off), IDESC_S, kk > 0 ? 1u : 0u);
          }
          if (!mbar_wait(p_ready, nd & 1, fs)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {  // dV += P^T dO (P^T read MN-major from the P tile)
            umma_bf16_ss(tDV, sdesc_add(dPm, kk * 2048), sdesc_add(dOm, kk * 2048), IDESC_MN,
                         (nd > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(do_empty);  // dO(t): read by dP and dV
          umma_commit(dv_done);
        } else {
          mbar_arrive(do_empty);  // dO(t) is not needed
        }
        if (t + 1 < T && !issue_qk(t + 1)) break;  // the next tile's scores, into the other region
        if (keep) {
          if (!mbar_wait(ds_ready, nd & 1, fs)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {  // dK += dS^T Q (dS^T read MN-major from the dS tile)
            umma_bf16_ss(tDK, sdesc_add(dPm, kk * 2048), sdesc_add(dQm, st * TB + kk * 2048), IDESC_MN,
                         (nd > 0 || kk > 0) ? 1u : 0u);
          }
          // the drain warps have taken the previous kept tile (info slot free)
          if (nd >= 1 && dq_seen < nd - 1) {
            if (!mbar_wait(dq_free, (nd - 1) & 1, fs)) break;
            dq_seen = nd - 1;
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {  // dQ = dS K, over dP in the same region
            umma_bf16_ss(tR, sdesc_add(dPk, (kk >> 2) * 16384 + (kk & 3) * 32), sdesc_add(dKm, kk * 2048), IDESC_KN,
                         kk > 0 ? 1u : 0u);
          }
          umma_commit(dq_full);
          umma_commit(ps_free);
          info[0] = hq;
          info[1] = i0;
          info[2] = t & 1;
          mbar_arrive(info_full);
          if (t & 1) reg_kept1 = nd; else reg_kept0 = nd;
          ++nd;
        }
        umma_commit(&q_empty[st]);  // Q(t): QK(t) and dK(t) issued
      }
      // tell the drain warps there is nothing more, once they have taken the last tile
      if (nd >= 1) mbar_wait(dq_free, (nd - 1) & 1, fs);
      info[0] = -1;
      mbar_arrive(info_full);
      umma_commit(mma_final);
    }
    __syncwarp();
  } else if (warp >= 8) {
    // ------------------------------------------------------------ dQ drain warps
    // Warp 8 + w owns query rows [32w, 32w+32) of each kept tile (TMEM lanes of
    // the dQ accumulator). It reads its rows out of TMEM, hands the region back
    // to the MMA issuer, and adds them to the fp32 workspace 32 columns at a
    // time: a swizzled [32 x 32] fp32 block in shared memory, reduced into
    // global memory by one TMA add (whole 128-byte lines, element-wise atomic;
    // per-thread atomics from registers are several times slower at the L2).
    const int wq = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    uint8_t* stg = smem + Lay::OFF_STG + wq * Lay::STG_WARP;
    for (int n = 0;; ++n) {
      if (!mbar_wait_warp(info_full, n & 1, fs)) break;
      const int hq = *reinterpret_cast<volatile int*>(&info[0]);
      const int i0 = *reinterpret_cast<volatile int*>(&info[1]);
      const int reg = *reinterpret_cast<volatile int*>(&info[2]);
      if (hq < 0) break;
      if (!mbar_wait_warp(dq_full, n & 1, fs)) break;
      tc_fence_after();
      const int row0 = i0 + wq * 32;
#pragma unroll
      for (int hb = 0; hb < D / 64; ++hb) {  // 64 columns at a time
        uint32_t qh[64];
        tmem_ld32_at(tmem + reg * 128 + lane_base + hb * 64, qh);
        tmem_ld32_at(tmem + reg * 128 + lane_base + hb * 64 + 32, qh + 32);
        tmem_ld_wait();
        if (hb == D / 64 - 1) {  // the region goes back to the MMA issuer
          tc_fence_before();
          mbar_arrive(dq_free);
        }
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          const int c = hb * 2 + c2;
          uint8_t* buf = stg + (c & 1) * Lay::STG_BUF;
          const uint32_t buf_s = smem_u32(buf);
          if (lane == 0) bulk_wait_read1();  // the block two steps back has left this buffer
          __syncwarp();
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(buf_s + sw128_offset(lane, j),
                         __float_as_uint(p.scale * __uint_as_float(qh[c2 * 32 + 4 * j])),
                         __float_as_uint(p.scale * __uint_as_float(qh[c2 * 32 + 4 * j + 1])),
                         __float_as_uint(p.scale * __uint_as_float(qh[c2 * 32 + 4 * j + 2])),
                         __float_as_uint(p.scale * __uint_as_float(qh[c2 * 32 + 4 * j + 3])));
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            // rows past the tensor are clipped; rows past a packed sequence add exact zeros
            if (row0 < L) tma_reduce_add_4d(&tm_dq, buf, c * 32, hq, off + row0, bt);
            bulk_commit();  // one group per block, empty when skipped, so the counting above holds
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else {
    // ------------------------------------------------------------ compute warps
    // Thread tid owns query row (tid % 128) of the current tile, key columns
    // [64h, 64h + 64) with h = tid / 128 (TMEM lane row, 64 columns of S and dP
    // in the tile's region): its LSE, gate threshold and D are scalars. At the
    // end, thread tid writes key row (tid % 128), half h of the columns of dK
    // and dV.
    const int tid = threadIdx.x;
    const int row = tid & 127;
    const int kh = tid >> 7;
    const int qi = row / BQ;        // my query block inside the tile
    const int kx = (kh * 64) / BK;  // my key block inside the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t psa = smem_u32(sPS) + kh * 16384;  // my 64-column atom of the P / dS tile
    const float sl2 = p.scale_log2;
    int nd = 0;
    bool local_abort = false, all_abort = false;
    // LSE and D of query head hq start at row_base(hq): [B, Hq, L], or [Hq, total] for a packed batch
    auto row_base = [&](int hq_) {
      return kPacked ? static_cast<size_t>(hq_) * p.total + off : static_cast<size_t>(b * p.Hq + hq_) * L;
    };
    // LSE and D of my row, loaded one tile ahead (rows at or past L: LSE +inf, D 0)
    auto row_lse = [&](int t) {
      const int i = walk_qs(t) * 128 + row;
      return i < L ? __ldg(p.lse + row_base(walk_hq(t)) + i) : INFINITY;
    };
    auto row_d = [&](int t) {
      const int i = walk_qs(t) * 128 + row;
      return i < L ? __ldg(p.dvec + row_base(walk_hq(t)) + i) : 0.f;
    };
    float lse_next = row_lse(0), d_next = row_d(0);

    for (int t = 0; t < T; ++t) {
      const int hq = walk_hq(t);
      const int qs = walk_qs(t);
      const bool diag = qs == ks;  // then key column c is live for my row iff c <= row
      const float lse2_row = lse_next * 1.4426950408889634f, d_row = d_next;
      if (t + 1 < T) {
        lse_next = row_lse(t + 1);
        d_next = row_d(t + 1);
      }
      const uint32_t tR = tmem + (t & 1) * 128 + kh * 64 + lane_base;
      const bool ok = mbar_wait_warp(s_full, t & 1, fs);
      local_abort |= !ok;
      tc_fence_after();
      uint32_t sh[64];
      tmem_ld32_at(tR, sh);
      tmem_ld32_at(tR + 32, sh + 32);
      tmem_ld_wait();
      tc_fence_before();  // S(t) is in registers: after the vote the MMA may write dP over it
      if (diag) {
        const int lim = row - kh * 64;  // live columns: c <= lim
#pragma unroll
        for (int c = 0; c < 64; ++c) sh[c] = c <= lim ? sh[c] : kNegInfBits;
      }
      bool hit;
      if (kGate) {
        float m8[8];  // eight independent partial maxima, two columns per step
#pragma unroll
        for (int e = 0; e < 8; ++e) m8[e] = fmaxf(__uint_as_float(sh[2 * e]), __uint_as_float(sh[2 * e + 1]));
#pragma unroll
        for (int c = 16; c < 64; c += 2)
          m8[(c >> 1) & 7] = fmax3(m8[(c >> 1) & 7], __uint_as_float(sh[c]), __uint_as_float(sh[c + 1]));
        const float m = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        // max_c(s_c) * sl2 == max_c(s_c * sl2): rounding is monotone
        const float thr = lse2_row + p.log2_tau - lg2_approx(static_cast<float>(qs * 128 + row + 1));
        hit = ok && m * sl2 >= thr;
      } else {
        const int qb = qs * QPB + qi, kb = ks * KPB + kx;
        hit = qb < nq_b && kb < nk_b && kb * BK <= min((qb + 1) * BQ, L) - 1;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, hit);
      if (lane == 0) vote[(t & 1) * 8 + warp] = (bal ? 1u : 0u) | (local_abort ? 8u : 0u);
      named_bar_sync(1, 256);
      uint32_t kept = 0;  // bit (qi * 2 + kx): sub-tile kept
      bool any_abort = false;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const uint32_t vw = vote[(t & 1) * 8 + w];
        any_abort |= (vw & 8u) != 0;
        if (vw & 1u) kept |= 1u << ((((w & 3) * 32) / BQ) * 2 + ((w >> 2) * 64) / BK);
      }
      if (tid == 0) {
        *dec_flags = kept | (kept ? kBwdAny : 0u) | (any_abort ? kBwdAbort : 0u);
        mbar_arrive(dec_bar);
      }
      if (any_abort) {
        all_abort = true;
        break;
      }
      if (tid == 0) {
        int cnt = 0;
        for (int qx = 0; qx < QPB; ++qx)
          for (int kz = 0; kz < KPB; ++kz) {
            const int qb = qs * QPB + qx, kb = ks * KPB + kz;
            if (qb < nq_b && kb < nk_b && kb * BK <= min((qb + 1) * BQ, L) - 1) {
              const int kp = (kept >> (qx * 2 + kz)) & 1u;
              if (p.keep_map) p.keep_map[(static_cast<size_t>(b * p.Hq + hq) * p.nq + qb) * p.nk + kb] = kp;
              cnt += kp;
            }
          }
        if (cnt) atomicAdd(&p.kept_tiles[b * p.Hq + hq], cnt);
      }
      if (!kept) continue;
      // ---- kept: P of my row and columns; a sub-tile that is not kept gives 0
      // (LSE taken as +inf), so do masked entries (-inf scores)
      const float lse2 = ((kept >> (qi * 2 + kx)) & 1u) ? lse2_row : INFINITY;
      uint32_t pk[32];
#pragma unroll
      for (int jj = 0; jj < 32; ++jj)
        pk[jj] = pack_bf16x2_alu(ex2_approx(fmaf(__uint_as_float(sh[2 * jj]), sl2, -lse2)),
                             ex2_approx(fmaf(__uint_as_float(sh[2 * jj + 1]), sl2, -lse2)));
      if (nd >= 1) local_abort |= !mbar_wait_warp(ps_free, (nd - 1) & 1, fs);  // dK, dQ of the last tile done
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(psa + sw128_offset(row, c), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_smem();
      mbar_arrive(p_ready);
      // ---- dS = P * (dP - D), written over P once the dV MMA has read it
      const float dsub = d_row;
      local_abort |= !mbar_wait_warp(dv_done, nd & 1, fs);  // dP(t) and dV(t) done
      tc_fence_after();
      uint32_t dh[64];
      tmem_ld32_at(tR, dh);
      tmem_ld32_at(tR + 32, dh + 32);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t addr = psa + sw128_offset(row, c);
        uint32_t ds[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)  // P of the same entries, still in registers
          ds[e] = pack_bf16x2_alu(bf16lo_to_f32(pk[4 * c + e]) * (__uint_as_float(dh[c * 8 + 2 * e]) - dsub),
                              bf16hi_to_f32(pk[4 * c + e]) * (__uint_as_float(dh[c * 8 + 2 * e + 1]) - dsub));
        st_shared_v4(addr, ds[0], ds[1], ds[2], ds[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(ds_ready);
      ++nd;
    }

    if (!all_abort) {
      // ---------------------------------------------------------- epilogue
      // dK (times the softmax scale) and dV of key row `row`, column half kh,
      // staged over the Q ring and stored by TMA.
      const bool okf = mbar_wait_warp(mma_final, 0, fs);
      tc_fence_after();
      const uint32_t sQa = smem_u32(sQ);
      if (okf) {
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          const uint32_t tsrc = (which == 0 ? tDK : tDV) + lane_base;
          const float mul = which == 0 ? p.scale : 1.f;
          const uint32_t dst = sQa + which * TB;
#pragma unroll
          for (int cc = 0; cc < D / 64; ++cc) {
            const int ch = kh * (D / 64) + cc;  // 32-column chunk
            uint32_t r[32];
            if (nd > 0) {
              tmem_ld32(tsrc + ch * 32, r);
              tmem_ld_wait();
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) r[j] = 0u;
            }
            uint32_t pk[16];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj)
              pk[jj] = pack_bf16x2(__uint_as_float(r[2 * jj]) * mul, __uint_as_float(r[2 * jj + 1]) * mul);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int col = ch * 32 + c * 8;
              st_shared_v4(dst + (col >> 6) * 16384 + sw128_offset(row, (col & 63) >> 3), pk[4 * c], pk[4 * c + 1],
                           pk[4 * c + 2], pk[4 * c + 3]);
            }
          }
        }
        fence_proxy_async_smem();
      }
      const unsigned okall = __ballot_sync(0xffffffffu, okf);
      if (lane == 0) evote[warp] = okall == 0xffffffffu ? 1u : 0u;
      named_bar_sync(1, 256);
      uint32_t all_ok = 1u;
#pragma unroll
      for (int w = 0; w < 8; ++w) all_ok &= evote[w];
      // A packed batch's partial key tile is stored row by row: a tile store
      // would write the next sequence's rows.
      const bool whole = !kPacked || k0 + 128 <= L;
      if (whole && tid == 0 && all_ok) {
        for (int h = 0; h < D / 64; ++h) {
          tma_store_4d(&tm_dk, sQ + h * 16384, h * 64, hkv, off + k0, bt);
          tma_store_4d(&tm_dv, sQ + TB + h * 16384, h * 64, hkv, off + k0, bt);
        }
        tma_store_commit_and_wait();
      }
      if (!whole && all_ok && k0 + row < L) {
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          uint4* dst = reinterpret_cast<uint4*>((which == 0 ? p.dk_out : p.dv_out) +
                                                (static_cast<size_t>(off + k0 + row) * p.Hkv + hkv) * D);
#pragma unroll
          for (int c = 0; c < D / 16; ++c) {
            const int col = kh * (D / 2) + c * 8;
            uint32_t a0, a1, a2, a3;
            ld_shared_v4(sQa + which * TB + (col >> 6) * 16384 + sw128_offset(row, (col & 63) >> 3), a0, a1, a2, a3);
            dst[col / 8] = make_uint4(a0, a1, a2, a3);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    if (lane == 0) mbar_wait_drain(mma_final, 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

// D_i = <dO_i, O_i> for every (b, i, hq); clears dq_acc and the counters.
// 8 elements (16 bytes) per thread; D/8 threads per row.
template <int D>
__global__ void __launch_bounds__(256) mala_bwd_pre_kernel(const uint4* __restrict__ o, const uint4* __restrict__ dO,
                                                          float* __restrict__ dvec, float4* __restrict__ dq_acc,
                                                          int32_t* __restrict__ kept, int n_kept, int B, int L,
                                                          int Hq) {
  constexpr int TPR = D / 8;
  const long long total = static_cast<long long>(B) * L * Hq * TPR;
  const long long nthreads = static_cast<long long>(gridDim.x) * blockDim.x;
  const int lane = threadIdx.x & 31;
  // the loop bound is taken at the warp's first lane so that every lane of a
  // warp runs the same iterations (the row reduction shuffles across lanes)
  for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g - lane < total;
       g += nthreads) {
    const bool active = g < total;
    float s = 0.f;
    if (active) {
      const uint4 a = o[g];
      const uint4 c = dO[g];
      const uint32_t av[4] = {a.x, a.y, a.z, a.w};
      const uint32_t cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s = fmaf(bf16lo_to_f32(av[e]), bf16lo_to_f32(cv[e]), s);
        s = fmaf(bf16hi_to_f32(av[e]), bf16hi_to_f32(cv[e]), s);
      }
    }
#pragma unroll
    for (int off = TPR / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off, TPR);
    if (active) {
      if ((g % TPR) == 0) {
        const long long row = g / TPR;  // (b * L + i) * Hq + hq
        const int hq = static_cast<int>(row % Hq);
        const long long bi = row / Hq;
        const int i = static_cast<int>(bi % L);
        const int bb = static_cast<int>(bi / L);
        dvec[(static_cast<long long>(bb) * Hq + hq) * L + i] = s;
      }
      dq_acc[2 * g] = make_float4(0.f, 0.f, 0.f, 0.f);
      dq_acc[2 * g + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < n_kept; i += blockDim.x) kept[i] = 0;
}

// bf16 dQ from the fp32 accumulator (the softmax scale is already applied).
__global__ void __launch_bounds__(256) mala_dq_convert_kernel(const float4* __restrict__ acc, uint4* __restrict__ dq,
                                                             long long n8) {
  const long long nthreads = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g < n8; g += nthreads) {
    const float4 a = acc[2 * g], c = acc[2 * g + 1];
    dq[g] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(c.x, c.y), pack_bf16x2(c.z, c.w));
  }
}

}  // namespace mala
