// mala_fwd.cuh -- MALA forward kernel for sm_100a.
//
// Method (agihunt.info, "MassAlloc Attention: Let Attention Allocate Its Own
// Compute", method paragraphs): every legal causal tile is scored; after the
// QK tile, the largest per-key contribution ratio exp(s - m)/l against the
// evolving online-softmax state is compared with tau/Lq (Lq = i + 1); tiles run
// from the diagonal toward earlier keys; the first legal tile is kept; one
// row that fails to skip keeps the tile for the whole query block; a skipped
// tile does no softmax update and no PV; LSE is written.
//
// One CTA owns two 128-row query tiles (A = rows r0..r0+127, B = the next 128)
// of one (b, hq) and walks key tiles kb = last ... 0. A 128-row tile holds one
// query block when Bq = 128 and two when Bq = 64; decisions are per block.
// The same kernel runs prefill against an existing cache: query row r sits at
// position P0 + r (P0 = Lk - Lq), sees keys 0 .. P0 + r and uses Lq = P0 + r + 1
// in its threshold; the training forward is P0 = 0, Lq = Lk. In a packed batch
// (device cu_seqlens) each CTA takes its sequence's lengths and row offsets
// from the tables, and a partial last tile of O is stored row by row so that
// the next sequence's rows are not written.
//   warps 0-3  softmax warpgroup of tile A (thread t = row t = TMEM lane t)
//   warps 4-7  softmax warpgroup of tile B
//   warp  8    TMA producer: both Q tiles once, K tiles through an NK ring
//              (and, with the gate off or V fetched ahead, every V tile
//              through the NV ring)
//   warp  9    MMA issuer (one thread)
//   warp  10   V issuer (one thread, gate on, V on demand)
// TMEM: S_A | S_B | O_A | O_B. P (fp16) is written over the first half of its
// tile's S columns and read from TMEM by the PV MMA (A operand in TMEM).
// The MMA thread alternates between the tiles -- PV_A(t), QK_A(t+1), PV_B(t),
// QK_B(t+1) -- so the tensor core works on one tile while the other tile's
// warpgroup runs its gate and softmax.
//
// With the gate on, a V tile is requested only once a query block has voted
// to keep it, so a skipped tile costs no V traffic. Both warpgroups vote on
// every key tile t and post their votes to a mailbox in shared memory (a flag
// ring and an mbarrier ring per warpgroup). The V issuer reads tile A's vote
// on t as soon as it is posted and, if A keeps t, requests V(t) at once, so
// the load overlaps A's probability pass; otherwise it waits for B's vote. If
// neither keeps t, nothing is loaded. V tiles take the NV slots in load order
// (the n-th loaded tile uses slot n % NV); the MMA thread, which sees both
// decisions of every tile, counts the loads the same way, and no barrier phase
// stands for a tile that was not loaded. As an opt-in (kMode 2) the gated
// kernel instead fetches every V tile ahead like the ungated one: decisions
// and outputs are the same, skipped tiles cost their V traffic, and no PV
// waits for a V load requested after a vote.
//
// Precision: S = Q K^T is bf16 x bf16 -> fp32. PV runs in fp16 x fp16 -> fp32:
// P is at most 2^8 (lazy-rescale bound) and V is read from an fp16 copy made
// by mala_v_to_f16_kernel (exact for |v| < 65504); bf16 P would add an error
// as large as the bf16 rounding of O itself.
#pragma once

#include "mala_ptx.cuh"

namespace mala {

struct FwdParams {
  int B, Hq, Hkv, G;
  int Lq, Lk, P0;       // Lq queries at positions P0 .. P0 + Lq - 1 of Lk keys (P0 = Lk - Lq)
  int nq, nk, n_pairs;  // nq = ceil(Lq / Bq), nk = ceil(Lk / Bk), n_pairs = ceil(Lq / 256)
  int chunk_pairs;      // CTA schedule: pairs per chunk (see mala_fwd_kernel)
  float scale_log2;     // scale * log2(e): scores are kept in log2 units
  float log2_tau;       // log2(tau), used only when the gate is on
  float* lse;           // [B, Hq, Lq]; packed batches: [Hq, total_q]
  uint16_t* o;          // the output (bf16), for the row-wise stores of a packed batch's partial tiles
  const int* cu_q;      // packed batch (else null): sequence b owns query rows cu_q[b] .. cu_q[b+1]
  const int* cu_k;      //   and key rows cu_k[b] .. cu_k[b+1] of the packed tensors
  int total_q, total_k; // packed batch: query and key rows in all
  int32_t* kept_tiles;
  uint8_t* keep_map;
  unsigned* status;
  unsigned long long* v_tiles;  // nullable test counter: V tiles loaded (one per load)
  uint64_t wait_ns;             // limit of each bounded wait
  int stall_tile;               // test hook (-1: off): the MMA thread stalls before this tile
};

constexpr int kVoteRing = 8;        // V mailbox depth (tiles a warpgroup may vote ahead of the V issuer)
constexpr uint32_t kDecPV = 1u;     // some query block of the tile keeps it
constexpr uint32_t kDecAbort = 2u;  // a wait gave up somewhere in the CTA
constexpr unsigned kStatusRange = 2u;

template <int D, int BK>
struct FwdLayout {
  static constexpr int BM = 128;
  static constexpr int NK = 3;
  static constexpr int NV = 2;
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BK * D * 2;
  static constexpr int OFF_Q = 0;  // Q_A, Q_B
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NK * KV_BYTES;
  static constexpr int OFF_BAR = OFF_V + NV * KV_BYTES;
  // q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[2],
  // sm_done[2], dec[2], pv_done[2], mma_final, vote_bar[2][kVoteRing]
  static constexpr int N_BARS = 1 + 2 * NK + 2 * NV + 2 + 2 + 2 + 2 + 1 + 2 * kVoteRing;
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int MISC_BYTES = 192;
  static constexpr int BYTES = OFF_MISC + MISC_BYTES;
  static constexpr int ALLOC_BYTES = BYTES + 1024;  // slack for 1024-B alignment
  static constexpr int COL_S = 0;                   // S_A at 0, S_B at BK
  static constexpr int COL_O = 2 * BK;              // O_A at 2BK, O_B at 2BK + D
  static constexpr int TMEM_NEED = 2 * BK + 2 * D;
  static constexpr int TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
  static_assert(ALLOC_BYTES <= 232448, "forward shared memory exceeds the per-CTA limit");
};

// D[tmem] (+)= A[tmem] * B[smem], kind::f16 (A in tensor memory).
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// kMode: 0 = no gate (tau = 0: every legal tile kept, V fetched ahead);
// 1 = gate, V requested only for tiles a query block keeps (the default);
// 2 = gate, V of every tile fetched ahead whatever the vote (opt-in: skipped
// tiles then cost their V traffic, but no V load waits behind a vote).
template <int D, int BQ, int BK, int kMode>
__global__ void __launch_bounds__(352, 1)
    mala_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const FwdParams p) {
  using Lay = FwdLayout<D, BK>;
  constexpr bool kGate = kMode != 0;
  constexpr bool kPrefetchV = kMode != 1;  // V(t) fetched ahead by the producer into slot t % NV
  constexpr int BM = Lay::BM, QPB = BM / BQ;
  constexpr int NK = Lay::NK, NV = Lay::NV;
  constexpr uint32_t IDESC_QK = idesc_bf16(128, BK, false, false);
  constexpr uint32_t IDESC_PV = idesc_f16(128, D, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Lay::OFF_Q;
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* bar_q = bars;
  uint64_t* k_full = bar_q + 1;
  uint64_t* k_empty = k_full + NK;
  uint64_t* v_full = k_empty + NK;
  uint64_t* v_empty = v_full + NV;
  uint64_t* s_full = v_empty + NV;   // [2]
  uint64_t* sm_done = s_full + 2;    // [2]
  uint64_t* dec_bar = sm_done + 2;   // [2]
  uint64_t* pv_done = dec_bar + 2;   // [2]
  uint64_t* mma_final = pv_done + 2;
  uint64_t* vote_bar = mma_final + 1;  // [2][kVoteRing]: vote of tile t posted, at t % kVoteRing
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  uint32_t* tmem_slot = misc + 0;
  int* abort_flag = reinterpret_cast<int*>(misc + 1);
  uint32_t* dec_flags = misc + 2;  // [2] per tile
  uint32_t* vote = misc + 4;       // [2 tiles][2 parity][4 warps]
  uint32_t* evote = misc + 20;     // [2 tiles][4 warps]
  uint32_t* vflag = misc + 32;     // [2][kVoteRing] vote of tile t at t % kVoteRing: 1 keep, 2 abort

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA schedule: the grid is cut into chunks of chunk_pairs row pairs, longest
  // rows first; inside a chunk the (b, KV head) units follow one another and the
  // G query heads of a pair are adjacent. The CTAs resident at one time then
  // share one or two KV heads, whose K and V stay in L2, while the longest
  // rows still start first. The last chunk may be padded with empty CTAs.
  const int per_unit = p.chunk_pairs * p.G;
  const int per_chunk = p.B * p.Hkv * per_unit;
  const int chunk = static_cast<int>(blockIdx.x) / per_chunk;
  const int in_chunk = static_cast<int>(blockIdx.x) % per_chunk;
  const int unit = in_chunk / per_unit;
  const int b = unit / p.Hkv, hkv = unit % p.Hkv, hq = hkv * p.G + in_chunk % p.G;
  const int bh = b * p.Hq + hq;
  // This CTA's sequence: Lq queries at positions P0 .. P0 + Lq - 1 of Lk keys.
  // A packed batch gives each sequence its own lengths and row offsets into the
  // packed tensors (its pairs are counted from its own last row; the grid covers
  // the longest sequence, and a CTA past its sequence's rows leaves at once).
  int Lq = p.Lq, Lk = p.Lk, q_off = 0, k_off = 0, bt = b;
  if (p.cu_q != nullptr) {  // p.Lq / p.Lk hold the longest sequence's lengths
    q_off = __ldg(p.cu_q + b);
    Lq = __ldg(p.cu_q + b + 1) - q_off;
    k_off = __ldg(p.cu_k + b);
    Lk = __ldg(p.cu_k + b + 1) - k_off;
    bt = 0;
    if (q_off < 0 || Lq < 0 || Lq > p.Lq || q_off + Lq > p.total_q || k_off < 0 || Lk < Lq || Lk > p.Lk ||
        k_off + Lk > p.total_k) {  // nothing of this sequence is touched
      if (threadIdx.x == 0) atomicOr(p.status, kStatusSeqTable);
      return;
    }
  }
  const int P0 = Lk - Lq;
  const int pr = (Lq + 2 * BM - 1) / (2 * BM) - 1 - (chunk * p.chunk_pairs + (in_chunk % per_unit) / p.G);
  if (pr < 0) return;  // padding (uniform across the CTA, before any shared state)
  const int r0 = pr * 2 * BM;  // first row of tile A
  const int last_row = min(r0 + 2 * BM, Lq) - 1;  // among the queries
  const int kb_hi = (P0 + last_row) / BK;         // key tile of the pair's last query
  const int T = kb_hi + 1;

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < NK; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < NV; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&sm_done[i], 128);
      mbar_init(&dec_bar[i], 1);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(mma_final, 1);
    *abort_flag = 0;
    for (int i = 0; i < 2 * kVoteRing; ++i) mbar_init(&vote_bar[i], 1);
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, Lay::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
    prefetch_tensormap(&tm_o);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  const FailState fs{abort_flag, p.status, p.wait_ns};

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_q, 2 * Lay::Q_BYTES);
      for (int x = 0; x < 2; ++x)
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(&tm_q, bar_q, sQ + x * Lay::Q_BYTES + h * (BM * 128), h * 64, hq, q_off + r0 + x * BM, bt);
      int issued = 0, vissued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t % NK;
        const int kb = kb_hi - t;
        if (t >= NK && !mbar_wait(&k_empty[st], ((t / NK) - 1) & 1, fs)) break;
        mbar_arrive_expect_tx(&k_full[st], Lay::KV_BYTES);
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(&tm_k, &k_full[st], sK + st * Lay::KV_BYTES + h * (BK * 128), h * 64, hkv, k_off + kb * BK,
                      bt);
        issued = t + 1;
        if (kPrefetchV) {  // every tile is loaded (load t is tile t): V(t) is fetched ahead into slot t % NV
          const int vs = t % NV;
          if (t >= NV && !mbar_wait(&v_empty[vs], ((t / NV) - 1) & 1, fs)) break;
          mbar_arrive_expect_tx(&v_full[vs], Lay::KV_BYTES);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(&tm_v, &v_full[vs], sV + vs * Lay::KV_BYTES + h * (BK * 128), h * 64, hkv, k_off + kb * BK,
                      bt);
          if (kGate && p.v_tiles != nullptr) atomicAdd(p.v_tiles, 1ull);
          vissued = t + 1;
        }
      }
      mbar_wait_drain(bar_q, 0);
      for (int t = max(0, issued - NK); t < issued; ++t) mbar_wait_drain(&k_full[t % NK], (t / NK) & 1);
      if (kPrefetchV)
        for (int t = max(0, vissued - NV); t < vissued; ++t) mbar_wait_drain(&v_full[t % NV], (t / NV) & 1);
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // operand descriptors, built once and stepped with one add per instruction
      const uint64_t dQk = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dKk = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dVm = sdesc_sw128(smem_u32(sV), BK * 128, 1024);
      int npv[2] = {0, 0};
      auto issue_qk = [&](int x, int t) {
        const int st = t % NK;
        const uint32_t tS = tmem + Lay::COL_S + x * BK;
        const uint64_t qa = sdesc_add(dQk, x * Lay::Q_BYTES), kb = sdesc_add(dKk, st * Lay::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16_ss(tS, sdesc_add(qa, (kk >> 2) * (BM * 128) + (kk & 3) * 32),
                       sdesc_add(kb, (kk >> 2) * (BK * 128) + (kk & 3) * 32), IDESC_QK, kk > 0 ? 1u : 0u);
        umma_commit(&s_full[x]);
      };
      auto issue_pv = [&](int x, int vslot) {
        const uint32_t tP = tmem + Lay::COL_S + x * BK;  // fp16 P over the first half of S
        const uint32_t tO = tmem + Lay::COL_O + x * D;
        const uint64_t vb = sdesc_add(dVm, vslot * Lay::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma_f16_ts(tO, tP + kk * 8, sdesc_add(vb, kk * 2048), IDESC_PV, (npv[x] > 0 || kk > 0) ? 1u : 0u);
        umma_commit(&pv_done[x]);
        ++npv[x];
      };
      bool ok = mbar_wait(bar_q, 0, fs) && mbar_wait(&k_full[0], 0, fs);
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        issue_qk(1, 0);
        umma_commit(&k_empty[0]);
      }
      // V tiles occupy the slots in load order: the n-th loaded tile (a tile
      // some query block of the pair keeps) uses slot n % NV
      int nload = 0;
      for (int t = 0; ok && t < T; ++t) {
        const int vslot = nload % NV;
        // test hook: wait on a barrier only this thread completes (after the
        // loop), so the bounded wait expires and the CTA takes its abort path
        if (t == p.stall_tile && !mbar_wait(mma_final, 0, fs)) break;
        bool v_waited = false;
        for (int x = 0; x < 2 && ok; ++x) {
          if (!mbar_wait(&dec_bar[x], t & 1, fs)) { ok = false; break; }
          const uint32_t dec = *reinterpret_cast<volatile uint32_t*>(&dec_flags[x]);
          if (dec & kDecAbort) { ok = false; break; }
          const bool keep = (dec & kDecPV) != 0;
          if (!mbar_wait(&sm_done[x], t & 1, fs)) { ok = false; break; }  // P_x(t) written (or S_x released)
          if (keep) {
            if (!v_waited && !mbar_wait(&v_full[vslot], (nload / NV) & 1, fs)) { ok = false; break; }
            v_waited = true;
            tc_fence_after();
            issue_pv(x, vslot);
          }
          if (t + 1 < T) {
            if (x == 0 && !mbar_wait(&k_full[(t + 1) % NK], ((t + 1) / NK) & 1, fs)) { ok = false; break; }
            tc_fence_after();
            issue_qk(x, t + 1);
            if (x == 1) umma_commit(&k_empty[(t + 1) % NK]);
          }
        }
        if (!ok) break;
        // V fetched ahead: tile t's load has landed before its slot is handed back,
        // whether or not a PV read it
        if (kPrefetchV && !v_waited) {
          if (!mbar_wait(&v_full[vslot], (nload / NV) & 1, fs)) break;
          v_waited = true;
        }
        if (v_waited) {
          umma_commit(&v_empty[vslot]);  // V(t) read by both PVs
          ++nload;
        }
      }
      umma_commit(mma_final);  // completes once every MMA above has finished
    }
    __syncwarp();
  } else if (warp == 10) {
    // ------------------------------------------------------------ V issuer
    if (kGate && !kPrefetchV && lane == 0) {
      // the vote of warpgroup x on tile t (bit 0 keep, bit 1 abort), once posted.
      // The issuer sleeps in the barrier wait instead of polling, so it takes
      // no issue slots from the softmax warps that share its scheduler (a
      // polling issuer made them ~10% slower on mid-length rows). Slot t %
      // kVoteRing is reused every kVoteRing tiles and a warpgroup runs at most
      // a couple of tiles ahead of the issuer, so the phase parity is never
      // ambiguous.
      auto vote_of = [&](int x, int t) -> uint32_t {
        const int slot = x * kVoteRing + t % kVoteRing;
        if (!mbar_wait(&vote_bar[slot], (t / kVoteRing) & 1, fs)) return 2u;
        return reinterpret_cast<volatile uint32_t*>(vflag)[slot];
      };
      int n = 0;  // V tiles loaded so far; load n goes to slot n % NV
      for (int t = 0; t < T; ++t) {
        uint32_t f = vote_of(0, t);
        if (f & 2u) break;
        if (!(f & 1u)) {
          f = vote_of(1, t);
          if (f & 2u) break;
        }
        if (!(f & 1u)) continue;  // neither tile keeps t: no V(t)
        const int vs = n % NV;
        // the slot's previous load has been read by its PVs
        if (n >= NV && !mbar_wait(&v_empty[vs], ((n / NV) - 1) & 1, fs)) break;
        const int kb = kb_hi - t;
        mbar_arrive_expect_tx(&v_full[vs], Lay::KV_BYTES);
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(&tm_v, &v_full[vs], sV + vs * Lay::KV_BYTES + h * (BK * 128), h * 64, hkv, k_off + kb * BK,
                      bt);
        if (p.v_tiles != nullptr) atomicAdd(p.v_tiles, 1ull);
        ++n;
      }
      // loads the MMA thread may not have waited for (only after a wait gave up)
      for (int i = max(0, n - NV); i < n; ++i) mbar_wait_drain(&v_full[i % NV], (i / NV) & 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax warpgroups
    const int x = warp >> 2;            // my tile: 0 = A, 1 = B
    const int tid = threadIdx.x & 127;  // row within the tile
    const int wq = warp & 3;            // TMEM lane quarter
    const int row0 = r0 + x * BM;
    const int row = row0 + tid;
    const bool row_ok = row < Lq;
    const int pos = P0 + row;  // the query's position: it sees keys 0 .. pos
    const int qi = tid / BQ;
    const int qb = (row0 / BQ) + qi;
    const bool blk_exists = qb < (Lq + BQ - 1) / BQ;
    const int kbf = blk_exists ? (P0 + min((qb + 1) * BQ, Lq) - 1) / BK : -1;
    const float thr = kGate ? p.log2_tau - lg2_approx(static_cast<float>(pos + 1)) : 0.f;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + Lay::COL_S + x * BK + lane_base;
    const uint32_t tO = tmem + Lay::COL_O + x * D + lane_base;
    const float sl2 = p.scale_log2;
    float m_use = -INFINITY, l = 0.f;
    int npv = 0, kept_count = 0;
    bool local_abort = false, all_abort = false;
    uint32_t r[32];
    uint32_t* myvote = vote + x * 8;

    for (int t = 0; t < T; ++t) {
      const int kb = kb_hi - t;
      const bool ok = mbar_wait_warp(&s_full[x], t & 1, fs);
      local_abort |= !ok;
      tc_fence_after();
      const bool diag = kb * BK + BK - 1 > P0 + row0;  // some key of the tile is past some row
      // first pass (row max): all loads of the S row in flight at once, one wait
      float M = -INFINITY;
      {
        uint32_t sv[BK];
#pragma unroll
        for (int ch = 0; ch < BK / 32; ++ch) tmem_ld32_at(tS + ch * 32, sv + ch * 32);
        tmem_ld_wait();
        if (ok) {
          float mp[8];  // eight independent partial maxima (short dependency chains), two columns per step
#pragma unroll
          for (int e = 0; e < 8; ++e) mp[e] = -INFINITY;
          if (!diag) {
#pragma unroll
            for (int j = 0; j < BK; j += 2)
              mp[(j >> 1) & 7] = fmax3(mp[(j >> 1) & 7], __uint_as_float(sv[j]), __uint_as_float(sv[j + 1]));
          } else {
#pragma unroll
            for (int j = 0; j < BK; j += 2)
              mp[(j >> 1) & 7] = fmax3(mp[(j >> 1) & 7], kb * BK + j <= pos ? __uint_as_float(sv[j]) : -INFINITY,
                                       kb * BK + j + 1 <= pos ? __uint_as_float(sv[j + 1]) : -INFINITY);
          }
          M = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7]));
        }
      }
      const bool legal = blk_exists && kb <= kbf;
      bool keep_r;
      if (!legal || !row_ok) keep_r = false;
      else if (kb == kbf || !kGate) keep_r = true;  // first legal tile / full attention
      else keep_r = M * sl2 >= m_use + lg2_approx(l) + thr;  // ratio >= tau/Lq, ties keep
      const unsigned bal = __ballot_sync(0xffffffffu, keep_r);
      if (lane == 0) myvote[(t & 1) * 4 + wq] = (bal ? 1u : 0u) | (local_abort ? 2u : 0u);
      named_bar_sync(1 + x, 128);
      const uint32_t v0 = myvote[(t & 1) * 4 + 0], v1 = myvote[(t & 1) * 4 + 1];
      const uint32_t v2 = myvote[(t & 1) * 4 + 2], v3 = myvote[(t & 1) * 4 + 3];
      const bool any_abort = ((v0 | v1 | v2 | v3) & 2u) != 0;
      const bool bk0 = QPB == 1 ? (((v0 | v1 | v2 | v3) & 1u) != 0) : (((v0 | v1) & 1u) != 0);
      const bool bk1 = QPB == 1 ? false : (((v2 | v3) & 1u) != 0);
      const bool my_keep = qi == 0 ? bk0 : bk1;
      const bool need_pv = bk0 || bk1;
      if (tid == 0) {
        if (kGate && !kPrefetchV) {  // post the vote to the V issuer
          reinterpret_cast<volatile uint32_t*>(vflag)[x * kVoteRing + t % kVoteRing] =
              (need_pv ? 1u : 0u) | (any_abort ? 2u : 0u);
          mbar_arrive(&vote_bar[x * kVoteRing + t % kVoteRing]);  // release: the flag is visible to the waiter
        }
        dec_flags[x] = (need_pv ? kDecPV : 0u) | (any_abort ? kDecAbort : 0u);
        mbar_arrive(&dec_bar[x]);
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
          if (__any_sync(0xffffffffu, need_o)) {  // rare: O holds earlier tiles; wait for their PV first
            if (npv > 0) local_abort |= !mbar_wait_warp(&pv_done[x], (npv - 1) & 1, fs);
            tc_fence_after();
            const float a = need_o ? alpha : 1.f;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
              tmem_ld32(tO + ch * 32, r);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * a);
              tmem_st32(tO + ch * 32, r);
            }
          }
          float rsp[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial row sums
          const bool plain = !diag && row_ok;   // no masking needed for this row and tile
          // second pass over S in halves of 64 columns (two loads in flight, one wait each)
#pragma unroll
          for (int hlf = 0; hlf < BK / 64; ++hlf) {
            uint32_t sh[64];
            tmem_ld32_at(tS + hlf * 64, sh);
            tmem_ld32_at(tS + hlf * 64 + 32, sh + 32);
            tmem_ld_wait();
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
              const int ch = hlf * 2 + c2;
              uint32_t pk[16];
              if (plain) {
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                  const float p0 = ex2_approx(fmaf(__uint_as_float(sh[c2 * 32 + 2 * jj]), sl2, -m_use));
                  const float p1 = ex2_approx(fmaf(__uint_as_float(sh[c2 * 32 + 2 * jj + 1]), sl2, -m_use));
                  pk[jj] = pack_f16x2(p0, p1);
                  rsp[jj & 3] += p0 + p1;  // the normaliser sums the fp32 probabilities
                }
              } else {
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                  const int key = kb * BK + ch * 32 + 2 * jj;
                  const bool l0 = row_ok && key <= pos;
                  const bool l1 = row_ok && key + 1 <= pos;
                  // masked entries go through ex2 as -inf (-> 0): no branch around the inline asm
                  const float p0 = ex2_approx(l0 ? fmaf(__uint_as_float(sh[c2 * 32 + 2 * jj]), sl2, -m_use) : -INFINITY);
                  const float p1 =
                      ex2_approx(l1 ? fmaf(__uint_as_float(sh[c2 * 32 + 2 * jj + 1]), sl2, -m_use) : -INFINITY);
                  pk[jj] = pack_f16x2(p0, p1);
                  rsp[jj & 3] += p0 + p1;
                }
              }
              // P chunk ch covers keys [32ch, 32ch+32) = TMEM columns [16ch, 16ch+16): already read
              tmem_st16(tS + ch * 16, pk);
            }
          }
          l += (rsp[0] + rsp[1]) + (rsp[2] + rsp[3]);
        } else {  // the other query block of this tile keeps it: my rows add nothing
          uint32_t z[16];
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) z[jj] = 0u;
#pragma unroll
          for (int ch = 0; ch < BK / 32; ++ch) tmem_st16(tS + ch * 16, z);
        }
        tmem_st_wait();
        ++npv;
      }
      tc_fence_before();
      mbar_arrive(&sm_done[x]);
    }

    if (!all_abort) {
      // ---------------------------------------------------------- epilogue
      const bool okf = mbar_wait_warp(mma_final, 0, fs);
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const uint32_t sQa = smem_u32(sQ) + x * Lay::Q_BYTES;  // Q_x is free: every QK has completed
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
        const size_t lse_at = p.cu_q != nullptr ? static_cast<size_t>(hq) * p.total_q + q_off + row
                                                : static_cast<size_t>(bh) * Lq + row;
        if (row_ok) p.lse[lse_at] = (m_use + lg2_approx(l)) * 0.69314718055994531f;
      }
      const unsigned okall = __ballot_sync(0xffffffffu, okf);
      if (lane == 0) evote[x * 4 + wq] = okall == 0xffffffffu ? 1u : 0u;
      named_bar_sync(1 + x, 128);
      const bool store = (evote[x * 4 + 0] & evote[x * 4 + 1] & evote[x * 4 + 2] & evote[x * 4 + 3]) != 0;
      // A packed batch's partial tile is stored row by row: a tile store would
      // write the next sequence's rows.
      const bool whole = p.cu_q == nullptr || row0 + BM <= Lq;
      if (whole && tid == 0 && store && row0 < Lq) {
        for (int h = 0; h < D / 64; ++h)
          tma_store_4d(&tm_o, sQ + x * Lay::Q_BYTES + h * (BM * 128), h * 64, hq, q_off + row0, bt);
        tma_store_commit_and_wait();
      }
      if (!whole && store && row_ok) {
        uint4* dst = reinterpret_cast<uint4*>(p.o + (static_cast<size_t>(q_off + row) * p.Hq + hq) * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          uint32_t a0, a1, a2, a3;
          ld_shared_v4(sQa + (c >> 3) * (BM * 128) + sw128_offset(tid, c & 7), a0, a1, a2, a3);
          dst[c] = make_uint4(a0, a1, a2, a3);
        }
      }
      if ((tid % BQ) == 0 && blk_exists && store) atomicAdd(&p.kept_tiles[bh], kept_count);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    if (lane == 0) mbar_wait_drain(mma_final, 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, Lay::TMEM_COLS);
  }
}

// fp16 copy of V for the PV product; values beyond the fp16 range saturate to
// +-65504 and raise kStatusRange in the device status word.
__global__ void __launch_bounds__(256) mala_v_to_f16_kernel(const uint4* __restrict__ v, uint4* __restrict__ v16,
                                                           long long n8, unsigned* status) {
  const long long nthreads = static_cast<long long>(gridDim.x) * blockDim.x;
  bool over = false;
  for (long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; g < n8; g += nthreads) {
    const uint4 a = v[g];
    const uint32_t in[4] = {a.x, a.y, a.z, a.w};
    uint32_t out[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = bf16lo_to_f32(in[e]), hi = bf16hi_to_f32(in[e]);
      over |= fabsf(lo) > 65504.f || fabsf(hi) > 65504.f;
      asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(out[e]) : "f"(hi), "f"(lo));
    }
    v16[g] = make_uint4(out[0], out[1], out[2], out[3]);
  }
  if (over) atomicOr(status, kStatusRange);
}

}  // namespace mala
