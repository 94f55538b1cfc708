// mala_decode.cuh -- MALA decode (one new query per sequence) for sm_100a.
//
// Method (agihunt.info, "MassAlloc Attention: Let Attention Allocate Its Own
// Compute", method and limitations paragraphs): decoding uses the same tau as
// training; every key of the persistent cache is scored; a tile whose largest
// contribution ratio against the running state is below tau/Lq (Lq = Lk,
// every key visible) gets no V load and no PV.
//
// Decode reads the whole K cache once per step, so it is bound by HBM
// bandwidth, not by arithmetic: the dot products run on the CUDA cores and
// the kernel is organised around keeping K and V streaming.
//
// mala_decode_split_kernel: one CTA per (b, KV head, split). The split's key
// tiles run newest -> oldest with a fresh online-softmax state per query
// head; the newest tile of the split is always kept.
//   warps 0-15 compute: for QK, thread t scores key t % BK against a share of
//              the GQA group's query heads; P; PV
//   warp  16   gate warp: lane g runs head g's gate for tile t (and requests
//              V) while the compute warps score tile t + 1
//   warp  17   TMA producer of K tiles through an NK-stage ring
// Scoring a tile first does every product (each lane holds a 16-byte slice of
// a key row and the matching slices of the group's query heads), then reduces
// all of the tile's (key, head) dot products in one butterfly across the lanes
// of a key row, whose exchanges are independent of one another; lane c then
// holds the scores of one key for one or two heads, so exp2 runs once per
// (key, head) and the per-head maxima and sums take a few shuffles. (Reducing
// each key's products on their own, a chain of dependent shuffles per key,
// made scoring the slowest part of a tile: 4.7k -> 3.5k cycles per tile.)
// The gate chain (QK, max, gate, normaliser update) never waits for V: the
// state (m, l) follows from the scores alone. A kept tile's V TMA is issued
// at its gate, its probabilities and rescale factors go to a ring, and its PV
// runs kLag kept tiles later, when V has had time to land. PV maps thread t to
// an output column pair and a quarter of the keys; the slices are summed at
// the end of the split. Each split writes (O_s, LSE_s) per head.
//
// mala_decode_combine_kernel: LSE = log sum_s exp(LSE_s),
// O = sum_s exp(LSE_s - LSE) O_s, one warp per (b, query head).
#pragma once

#include "mala_ptx.cuh"

namespace mala {

constexpr int kDecMaxG = 8;  // query heads per KV head handled by one CTA
constexpr int kDecLag = 2;   // kept tiles between a tile's gate and its PV

struct DecParams {
  int B, Hq, Hkv, Lk, G, nk, n_splits, tiles_per_split;  // paged cache: Lk, nk = the longest sequence's
  float scale_log2;
  float thr;       // log2(tau) - log2(Lk)
  float log2_tau;  // paged cache: the threshold is formed per sequence
  // paged cache (else null): sequence b's key tile kb is page block_table[b * max_pages + kb] of the
  // [num_pages, page = Bk, Hkv, d] pools, its length seqlens[b]
  const int* seqlens;
  const int* block_table;
  int max_pages, num_pages;
  const uint16_t* q;  // [B, Hq, d] bf16
  float* o_part;      // [B, Hq, S, d]
  float* lse_part;    // [B, Hq, S] natural log
  int32_t* kept_tiles;
  uint8_t* keep_map;  // [B, Hq, nk], nullable
  unsigned* status;
  uint64_t wait_ns;  // limit of each bounded wait
  int stall_tile;    // test hook (-1: off): the K producer stalls before this tile
};

// Sum N per-lane values over the L lanes of a group (lane index c = lane % L,
// groups aligned to L lanes) so that afterwards lane c holds the group total
// of value c / (L / N). Each level exchanges half of the values still carried
// (a reduce-scatter butterfly), so N values take log2(N) + log2(L) - ... fewer
// shuffles than N full reductions: N = 4, L = 16 needs 5 instead of 16.
template <int N, int L>
__device__ __forceinline__ float group_reduce_scatter(float (&v)[N], int c) {
  int cnt = N;
#pragma unroll
  for (int o = L / 2; o >= 1; o >>= 1) {
    if (cnt > 1) {
      const bool upper = (c & o) != 0;
      const int half = cnt / 2;
#pragma unroll
      for (int i = 0; i < N / 2; ++i) {
        if (i < half) {
          const float send = upper ? v[i] : v[i + half];
          const float keep = upper ? v[i + half] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      cnt = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
  return v[0];
}

// The same butterfly for N >= L values: afterwards lane c holds the group
// totals of values [c * N / L, (c + 1) * N / L) in v[0 .. N / L). All N / 2
// exchanges of a level are independent, so a whole tile's dot products are
// reduced in log2(L) dependent steps instead of one chain per key.
template <int N, int L>
__device__ __forceinline__ void group_reduce_scatter_all(float (&v)[N], int c) {
  static_assert(N >= L, "at least one value per lane");
  int cnt = N;
#pragma unroll
  for (int o = L / 2; o >= 1; o >>= 1) {
    const bool upper = (c & o) != 0;
    const int half = cnt / 2;
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
      if (i < half) {
        const float send = upper ? v[i] : v[i + half];
        const float keep = upper ? v[i + half] : v[i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    cnt = half;
  }
}

template <int D, int BK, int GP>
struct DecLayout {
  static constexpr int NK = 3;
  static constexpr int NV = kDecLag + 1;
  static constexpr int NP = kDecLag + 1;
  static constexpr int NW = 8;          // compute warps
  static constexpr int NT = NW * 32;    // compute threads
  static constexpr int LPK = D / 8;     // lanes per key row (one 16-byte chunk each)
  static constexpr int KPW = 32 / LPK;  // keys per warp step
  static constexpr int NPART = NW;      // partial O accumulators (one per warp) summed at the end
  static constexpr int T_BYTES = BK * D * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NK * T_BYTES;
  static constexpr int OFF_Q = OFF_V + NV * T_BYTES;        // fp32 [GP][D]
  static constexpr int OFF_ALPHA = OFF_Q + GP * D * 4;        // fp32 [NP][GP]
  static constexpr int OFF_RMAX = OFF_ALPHA + NP * GP * 4;    // fp32 [2 tiles][NW][GP]
  static constexpr int OFF_RSUM = OFF_RMAX + 2 * NW * GP * 4; // fp32 [NW][GP]
  static constexpr int OFF_HEAD = OFF_RSUM + NW * GP * 4;     // keep, m, l per head
  static constexpr int OFF_BAR = OFF_HEAD + 3 * GP * 4;
  static constexpr int N_BARS = 2 * NK + NV;                  // k_full, k_empty, v_full
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr int ALLOC_BYTES = BYTES + 1024;
  static constexpr int ORED_BYTES = NPART * GP * D * 4;       // end-of-split reduction, reuses the K ring
  static_assert(ORED_BYTES <= NK * T_BYTES, "reduction buffer must fit in the K ring");
  static_assert(ALLOC_BYTES <= 232448, "decode shared memory exceeds the per-CTA limit");
};

// kPaged: a paged cache (p.seqlens and p.block_table set); the contiguous
// instantiation keeps every length a kernel parameter.
template <int D, int BK, int GP, bool kGate, bool kPaged>
__global__ void __launch_bounds__(320, 1)
    mala_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                             const DecParams p) {
  using Lay = DecLayout<D, BK, GP>;
  constexpr int NK = Lay::NK, NV = Lay::NV, NP = Lay::NP, TB = Lay::T_BYTES;
  constexpr int NW = Lay::NW, NT = Lay::NT, LPK = Lay::LPK, KPW = Lay::KPW;
  constexpr int KPWT = BK / NW;      // keys per warp per tile
  constexpr int STEPS = KPWT / KPW;  // warp steps per tile
  constexpr int NB = NT + 32;        // threads in the per-tile barriers (compute + gate warp)
  // Batched scoring (a tile's STEPS x GP dot products reduced together) when
  // there are one or two (step, head) values per lane of a key row: lane c
  // then holds VPL values, those of step c / LPS and heads (c % LPS) * VPL ..
  // + VPL - 1 of its key group. Otherwise each step's GP dot products are
  // reduced on their own and every lane keeps its head's score of each step.
  constexpr int NVAL = STEPS * GP;
  constexpr bool kBatch = NVAL >= LPK && NVAL <= 2 * LPK;  // more values per lane would spill
  constexpr int VPL = kBatch ? NVAL / LPK : 1;
  constexpr int LPS = kBatch ? LPK / STEPS : 1;
  static_assert(D == 128 || D == 64, "head dim");
  static_assert(STEPS >= 1 && KPWT % KPW == 0, "tile shape");
  static_assert(GP <= LPK && LPK % GP == 0, "heads spread evenly over the lanes of a key row");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  float* sq = reinterpret_cast<float*>(smem + Lay::OFF_Q);
  float* sAlpha = reinterpret_cast<float*>(smem + Lay::OFF_ALPHA);
  float* sRmax = reinterpret_cast<float*>(smem + Lay::OFF_RMAX);
  float* sRsum = reinterpret_cast<float*>(smem + Lay::OFF_RSUM);
  float* sKeep = reinterpret_cast<float*>(smem + Lay::OFF_HEAD);
  float* sM = sKeep + GP;  // exponent offset per head (log2 units)
  float* sL = sM + GP;     // running normaliser per head
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + NK;
  uint64_t* v_full = bars + 2 * NK;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(misc + 0);
  uint32_t* sflag = misc + 1;  // bit 0: some head keeps the tile; bit 1: abort
  int* sPage = reinterpret_cast<int*>(misc + 4);  // [8] paged cache: page of tile t at t & 7, set by the producer

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int nbk = p.B * p.Hkv;
  const int bk = blockIdx.x % nbk;
  const int sp_idx = static_cast<int>(blockIdx.x / nbk);
  const int b = bk / p.Hkv, hkv = bk % p.Hkv;
  const int G = p.G;
  const int hq0 = hkv * G;
  // this sequence's keys: Lk of them in nk tiles (a paged cache gives each its own)
  int Lk = p.Lk, nk = p.nk, tps = p.tiles_per_split;
  bool bad = false;
  if (kPaged) {
    Lk = __ldg(p.seqlens + b);
    bad = Lk < 1 || Lk > p.Lk;
    if (bad) Lk = 1;
    nk = (Lk + BK - 1) / BK;
    tps = (nk + p.n_splits - 1) / p.n_splits;
  }
  const float thr = kPaged ? p.log2_tau - log2f(static_cast<float>(Lk)) : p.thr;  // log2(tau / Lq), Lq = Lk
  const int t0 = bad ? nk : min(sp_idx * tps, nk);
  const int t1 = bad ? nk : min(t0 + tps, nk);
  const int T = t1 - t0;  // tiles kb = t1-1 ... t0
  const FailState fs{abort_flag, p.status, p.wait_ns};
  // paged cache: the page of key tile kb, checked (an id outside the pool is
  // reported and read as zeros: a TMA load outside the tensor fills)
  auto page_of = [&](int kb) {
    const int pg = __ldg(p.block_table + static_cast<size_t>(b) * p.max_pages + kb);
    if (pg >= 0 && pg < p.num_pages) return pg;
    atomicOr(p.status, kStatusSeqTable);
    return p.num_pages;
  };
  if (bad && sp_idx == 0 && tid == 0) atomicOr(p.status, kStatusSeqTable);

  if (T <= 0) {  // empty split: contributes nothing to the merge
    for (int i = tid; i < G * D; i += blockDim.x) {
      const int g = i / D, c = i % D;
      p.o_part[((static_cast<size_t>(b) * p.Hq + hq0 + g) * p.n_splits + sp_idx) * D + c] = 0.f;
    }
    if (tid < G) p.lse_part[(static_cast<size_t>(b) * p.Hq + hq0 + tid) * p.n_splits + sp_idx] = -INFINITY;
    return;
  }

  if (tid == 0) {
    for (int i = 0; i < NK; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], NT); }
    for (int i = 0; i < NV; ++i) mbar_init(&v_full[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < GP * D; i += blockDim.x) {
    const int g = i / D, c = i % D;
    float x = 0.f;
    if (g < G) x = __uint_as_float(static_cast<uint32_t>(p.q[(static_cast<size_t>(b) * p.Hq + hq0 + g) * D + c]) << 16);
    sq[g * D + c] = x;
  }
  if (tid < GP) {
    sM[tid] = -INFINITY;
    sL[tid] = 0.f;
    sKeep[tid] = 0.f;  // padded heads (G < GP) never keep
  }
  for (int i = tid; i < NW * GP; i += blockDim.x) sRsum[i] = 0.f;
  __syncthreads();

  if (warp == NW + 1) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      int pg_next = kPaged ? page_of(t1 - 1) : 0;  // page ids are read a tile ahead
      for (int t = 0; t < T; ++t) {
        const int st = t % NK;
        const int pg = pg_next;
        if (kPaged && t + 1 < T) pg_next = page_of(t1 - 2 - t);
        if (t >= NK && !mbar_wait(&k_empty[st], ((t / NK) - 1) & 1, fs)) break;
        // test hook: the phase that completes once tile t itself has been
        // consumed never completes before tile t is loaded, so the wait expires
        if (t == p.stall_tile && !mbar_wait(&k_empty[st], (t / NK) & 1, fs)) break;
        const int krow = kPaged ? 0 : (t1 - 1 - t) * BK, kouter = kPaged ? pg : b;
        if (kPaged) sPage[t & 7] = pg;  // for the gate warp's V request (it trails by < 8 tiles)
        mbar_arrive_expect_tx(&k_full[st], TB);
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(&tm_k, &k_full[st], sK + st * TB + h * (BK * 128), h * 64, hkv, krow, kouter);
        issued = t + 1;
      }
      for (int t = max(0, issued - NK); t < issued; ++t) mbar_wait_drain(&k_full[t % NK], (t / NK) & 1);
    }
    __syncwarp();
    return;  // the other warps synchronise with named barriers 1 (compute + gate) and 2 (compute)
  }

  if (warp == NW) {
    // ------------------------------------------------------------ gate warp
    // Lane g < G gates head g for tile t while the compute warps score tile t+1.
    int my_cnt = 0, nkept = 0;
    bool aborted = false;
    for (int t = 0; t < T; ++t) {
      const int kb = t1 - 1 - t;
      named_bar_sync(1, NB);  // A: maxima of tile t and sums of the previous kept tile are in place
      bool keep = false;
      if (lane < G) {
        const int g = lane;
        const float* rm = sRmax + (t & 1) * NW * GP;
        float M = rm[g], sum = sRsum[g];
        for (int w = 1; w < NW; ++w) {
          M = fmaxf(M, rm[w * GP + g]);
          sum += sRsum[w * GP + g];
        }
        float l = sL[g] + sum, mu = sM[g];
        keep = (t == 0) || !kGate || (M * p.scale_log2 >= mu + lg2_approx(l) + thr);
        float alpha = 1.f;
        if (keep) {
          const float mnew = fmaxf(mu, M * p.scale_log2);
          if (mnew > mu + 8.f) {  // lazy rescale: move the offset only when the max grew by > 2^8
            alpha = ex2_approx(mu - mnew);
            l *= alpha;
            mu = mnew;
          }
        }
        sL[g] = l;
        sM[g] = mu;
        sKeep[g] = keep ? 1.f : 0.f;
        sAlpha[(nkept % NP) * GP + g] = alpha;
        my_cnt += keep ? 1 : 0;
        if (p.keep_map) p.keep_map[(static_cast<size_t>(b) * p.Hq + hq0 + g) * p.nk + kb] = keep ? 1 : 0;
      } else if (lane < GP) {
        sAlpha[(nkept % NP) * GP + lane] = 1.f;
      }
      const bool any = __ballot_sync(0xffffffffu, keep) != 0u;
      if (lane == 0) {
        const bool ab = abort_raised(fs);
        if (any && !ab) {  // V is requested only now that a head keeps the tile
          const int vs = nkept % NV;
          const int vrow = kPaged ? 0 : kb * BK, vouter = kPaged ? sPage[t & 7] : b;
          fence_proxy_async_smem();
          mbar_arrive_expect_tx(&v_full[vs], TB);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(&tm_v, &v_full[vs], sV + vs * TB + h * (BK * 128), h * 64, hkv, vrow, vouter);
        }
        *sflag = (any ? 1u : 0u) | (ab ? 2u : 0u);
        aborted = ab;
      }
      aborted = __shfl_sync(0xffffffffu, aborted ? 1 : 0, 0) != 0;
      if (any) ++nkept;
      named_bar_sync(1, NB);  // B: the decision of tile t is visible
      if (aborted) break;
    }
    named_bar_sync(1, NB);  // C: the last probabilities and sums are written
    if (!aborted && lane < G) {
      float sum = 0.f;
      for (int w = 0; w < NW; ++w) sum += sRsum[w * GP + lane];
      sL[lane] += sum;  // fold the last kept tile into the normaliser
    }
    named_bar_sync(1, NB);  // D: the compute warps have summed their partials
    if (!aborted && !abort_raised(fs) && lane < G) {
      const float l = sL[lane];
      p.lse_part[(static_cast<size_t>(b) * p.Hq + hq0 + lane) * p.n_splits + sp_idx] =
          l > 0.f ? (sM[lane] + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
      atomicAdd(&p.kept_tiles[b * p.Hq + hq0 + lane], my_cnt);
    }
    if (lane == 0)
      for (int i = max(0, nkept - NV); i < nkept; ++i) mbar_wait_drain(&v_full[i % NV], (i / NV) & 1);
    return;
  }

  // ---------------------------------------------------------- compute warps
  // Lane (kg, c): key group kg = lane / LPK, 16-byte chunk c = lane % LPK of a
  // key row. In step s the warp handles keys warp*KPWT + s*KPW + kg. q slices
  // live in registers; a dot product is reduced across the LPK lanes of a row.
  const float c2 = p.scale_log2;
  const int kg = lane / LPK, c = lane % LPK;
  constexpr int LPH = LPK / GP;  // lanes of a key row that end up holding the same head
  const int hh = c / LPH;        // the head whose scores this lane holds after the reduction
  const bool owner = kg == 0 && (c % LPH) == 0;  // writes head hh's per-warp statistics
  const int s2_me = kBatch ? c / LPS : 0;        // batched: my step
  const int g0 = kBatch ? (c % LPS) * VPL : 0;   // batched: my first head
  const bool bowner = kg == 0 && s2_me == 0;     // batched: writes heads g0 .. g0 + VPL - 1
  // q slice and output accumulators as packed fp32 pairs (elements e, e+1)
  uint64_t qr[GP][4];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) qr[g][e2] = f2_pack(sq[g * D + c * 8 + 2 * e2], sq[g * D + c * 8 + 2 * e2 + 1]);
  uint64_t acc[GP][4];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) acc[g][e2] = 0ull;  // (+0, +0)
  constexpr int NR = kBatch ? VPL : STEPS;  // probabilities a lane holds per tile
  float ring[NP][NR];  // probabilities of pending kept tiles
#pragma unroll
  for (int i = 0; i < NP; ++i)
#pragma unroll
    for (int st = 0; st < NR; ++st) ring[i][st] = 0.f;
  int pend = 0, nkept = 0, ndone = 0;
  const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
  const uint32_t chunk_atom = (c >> 3) * (BK * 128), chunk_in = c & 7;
  bool aborted = false;

  auto row_addr = [&](uint32_t base, int j) { return base + chunk_atom + j * 128 + ((chunk_in ^ (j & 7)) << 4); };

  float sc_cur[NR], sc_nxt[NR];  // scores (batched: my step's key, heads g0 ..; else head hh, every step)
  auto score = [&](int t, float (&sc)[NR]) {
    const int st = t % NK;
    const int kb = t1 - 1 - t;
    const bool okk = mbar_wait_warp(&k_full[st], (t / NK) & 1, fs);
    if constexpr (kBatch) {
      // every product of the tile first, then one reduction of all of them
      float part[NVAL];  // [step][head]
#pragma unroll
      for (int s2 = 0; s2 < STEPS; ++s2) {
        const int j = warp * KPWT + s2 * KPW + kg;
        uint32_t a[4] = {0u, 0u, 0u, 0u};
        if (okk) ld_shared_v4(row_addr(sKa + st * TB, j), a[0], a[1], a[2], a[3]);
        uint64_t kf[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) kf[e2] = bf16x2_to_f2(a[e2]);
#pragma unroll
        for (int g = 0; g < GP; ++g) {
          uint64_t s2v = f2_fma(kf[0], qr[g][0], 0ull);  // even / odd elements summed separately
#pragma unroll
          for (int e2 = 1; e2 < 4; ++e2) s2v = f2_fma(kf[e2], qr[g][e2], s2v);
          float lo, hi;
          f2_unpack(s2v, lo, hi);
          part[s2 * GP + g] = lo + hi;
        }
      }
      mbar_arrive(&k_empty[st]);  // my reads of this K stage are done
      group_reduce_scatter_all<NVAL, LPK>(part, c);
      const int j = warp * KPWT + s2_me * KPW + kg;
      const bool live = kb * BK + j < Lk;
      float mx[VPL];
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        sc[i] = live ? part[i] : -INFINITY;
        mx[i] = sc[i];
      }
      // max over the warp's keys: the other steps' lanes, then the other key groups
#pragma unroll
      for (int off = LPS; off < 32; off <<= 1)
#pragma unroll
        for (int i = 0; i < VPL; ++i) mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], off));
      if (bowner)
#pragma unroll
        for (int i = 0; i < VPL; ++i) sRmax[((t & 1) * NW + warp) * GP + g0 + i] = mx[i];
    } else {
      float mx = -INFINITY;  // max over my keys of my head's scores
#pragma unroll
      for (int s2 = 0; s2 < STEPS; ++s2) {
        const int j = warp * KPWT + s2 * KPW + kg;
        float part[GP];
#pragma unroll
        for (int g = 0; g < GP; ++g) part[g] = 0.f;
        if (okk) {
          uint32_t a[4];
          ld_shared_v4(row_addr(sKa + st * TB, j), a[0], a[1], a[2], a[3]);
          uint64_t kf[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) kf[e2] = bf16x2_to_f2(a[e2]);
#pragma unroll
          for (int g = 0; g < GP; ++g) {
            uint64_t s2v = f2_fma(kf[0], qr[g][0], 0ull);  // even / odd elements summed separately
#pragma unroll
            for (int e2 = 1; e2 < 4; ++e2) s2v = f2_fma(kf[e2], qr[g][e2], s2v);
            float lo, hi;
            f2_unpack(s2v, lo, hi);
            part[g] = lo + hi;
          }
        }
        const float mine = group_reduce_scatter<GP, LPK>(part, c);  // score of key j for my head hh
        const bool live = kb * BK + j < Lk;
        if (live) mx = fmaxf(mx, mine);
        sc[s2] = live ? mine : -INFINITY;
      }
      mbar_arrive(&k_empty[st]);  // my reads of this K stage are done
#pragma unroll
      for (int off = LPK; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      if (owner) sRmax[((t & 1) * NW + warp) * GP + hh] = mx;
    }
    if (!okk) raise_abort(fs);
  };

  auto run_pv = [&](const float (&pr)[NR]) {  // PV of the oldest pending kept tile
    const int n = ndone++;
    const int vs = n % NV, ps = n % NP;
    const bool okv = mbar_wait_warp(&v_full[vs], (n / NV) & 1, fs);
    if (!okv) { aborted = true; return; }
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      const float al = sAlpha[ps * GP + g];
      const uint64_t al2 = f2_pack(al, al);
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) acc[g][e2] = f2_mul(acc[g][e2], al2);
    }
#pragma unroll
    for (int s2 = 0; s2 < STEPS; ++s2) {
      const int j = warp * KPWT + s2 * KPW + kg;
      uint32_t a[4];
      ld_shared_v4(row_addr(sVa + vs * TB, j), a[0], a[1], a[2], a[3]);
      uint64_t vf[4];
#pragma unroll
      for (int e2 = 0; e2 < 4; ++e2) vf[e2] = bf16x2_to_f2(a[e2]);
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        // P of key j for head g, from the lane that holds it
        const float pg = kBatch ? __shfl_sync(0xffffffffu, pr[g % VPL], kg * LPK + s2 * LPS + g / VPL)
                                : __shfl_sync(0xffffffffu, pr[kBatch ? 0 : s2], kg * LPK + g * LPH);
        const uint64_t pg2 = f2_pack(pg, pg);
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) acc[g][e2] = f2_fma(pg2, vf[e2], acc[g][e2]);
      }
    }
  };

  score(0, sc_cur);
  for (int t = 0; t < T; ++t) {
    named_bar_sync(1, NB);               // A: maxima of tile t are in place
    if (t + 1 < T) score(t + 1, sc_nxt);  // overlaps the gate of tile t
    named_bar_sync(1, NB);               // B: the decision of tile t is visible
    const uint32_t flag = *reinterpret_cast<volatile uint32_t*>(sflag);
    if (flag & 2u) { aborted = true; break; }
    if (flag & 1u) {  // probabilities of tile t for kept heads, and their per-warp sums
      float pv[NR];
      if constexpr (kBatch) {
        float ls[VPL];
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
          const bool on = sKeep[g0 + i] != 0.f;
          pv[i] = ex2_approx(on ? fmaf(sc_cur[i], c2, -sM[g0 + i]) : -INFINITY);  // no branch around the asm
          ls[i] = pv[i];
        }
#pragma unroll
        for (int off = LPS; off < 32; off <<= 1)
#pragma unroll
          for (int i = 0; i < VPL; ++i) ls[i] += __shfl_xor_sync(0xffffffffu, ls[i], off);
        if (bowner)
#pragma unroll
          for (int i = 0; i < VPL; ++i) sRsum[warp * GP + g0 + i] = ls[i];
      } else {
        const bool on = sKeep[hh] != 0.f;
        const float mu = sM[hh];
        float lsum = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < NR; ++s2) {
          pv[s2] = ex2_approx(on ? fmaf(sc_cur[s2], c2, -mu) : -INFINITY);  // no branch around the asm
          lsum += pv[s2];
        }
#pragma unroll
        for (int off = LPK; off < 32; off <<= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
        if (owner) sRsum[warp * GP + hh] = lsum;
      }
#pragma unroll
      for (int i = 0; i + 1 < NP; ++i)
#pragma unroll
        for (int s2 = 0; s2 < NR; ++s2) ring[i][s2] = ring[i + 1][s2];
#pragma unroll
      for (int s2 = 0; s2 < NR; ++s2) ring[NP - 1][s2] = pv[s2];
      ++pend;
      ++nkept;
      if (pend > kDecLag) {  // the oldest pending tile sits at ring[0]
        run_pv(ring[0]);
        --pend;
      }
    } else if (kBatch) {
      if (bowner)
#pragma unroll
        for (int i = 0; i < VPL; ++i) sRsum[warp * GP + g0 + i] = 0.f;
    } else {
      if (owner) sRsum[warp * GP + hh] = 0.f;
    }
#pragma unroll
    for (int s2 = 0; s2 < NR; ++s2) sc_cur[s2] = sc_nxt[s2];
  }

  named_bar_sync(1, NB);  // C
  if (!aborted) {  // drain: pending tiles sit at ring[NP - pend .. NP - 1], oldest first
#pragma unroll
    for (int i = 0; i < NP; ++i)
      if (i >= NP - pend && !aborted) run_pv(ring[i]);
  }
  named_bar_sync(2, NT);  // compute warps only (barrier 2): every read of the rings is done
  float* ored = reinterpret_cast<float*>(sK);  // [NW][GP][D], reuses the K ring
  float accf[GP][8];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int e2 = 0; e2 < 4; ++e2) f2_unpack(acc[g][e2], accf[g][2 * e2], accf[g][2 * e2 + 1]);
#pragma unroll
  for (int off = LPK; off < 32; off <<= 1)  // sum the key groups of the warp
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
      for (int e = 0; e < 8; ++e) accf[g][e] += __shfl_xor_sync(0xffffffffu, accf[g][e], off);
  if (kg == 0) {
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
      for (int e = 0; e < 8; ++e) ored[(warp * GP + g) * D + c * 8 + e] = accf[g][e];
  }
  named_bar_sync(1, NB);  // D (with the gate warp, which has folded the last sums into sL)
  if (!aborted && !abort_raised(fs)) {
    for (int i = tid; i < G * D; i += NT) {
      const int g = i / D, cc = i % D;
      float o = 0.f;
#pragma unroll 4
      for (int x = 0; x < Lay::NPART; ++x) o += ored[(x * GP + g) * D + cc];
      const float l = sL[g];
      p.o_part[((static_cast<size_t>(b) * p.Hq + hq0 + g) * p.n_splits + sp_idx) * D + cc] = l > 0.f ? o / l : 0.f;
    }
  }
}

// One warp per (b, query head): merge the split partials by their LSEs.
template <int D>
__global__ void __launch_bounds__(128) mala_decode_combine_kernel(const float* __restrict__ o_part,
                                                                  const float* __restrict__ lse_part,
                                                                  uint16_t* __restrict__ o, float* __restrict__ lse,
                                                                  int rows, int n_splits) {
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const float* lp = lse_part + static_cast<size_t>(row) * n_splits;
  float mx = -INFINITY;
  for (int s = lane; s < n_splits; s += 32) mx = fmaxf(mx, lp[s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float z = 0.f;
  for (int s = lane; s < n_splits; s += 32) z += lp[s] == -INFINITY ? 0.f : __expf(lp[s] - mx);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  const float L = mx + __logf(z);
  constexpr int PER = D / 32;
  float out[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) out[e] = 0.f;
  for (int s = 0; s < n_splits; ++s) {
    const float ls = lp[s];
    if (ls == -INFINITY) continue;
    const float w = __expf(ls - L);
    const float* src = o_part + (static_cast<size_t>(row) * n_splits + s) * D;
#pragma unroll
    for (int e = 0; e < PER; ++e) out[e] = fmaf(w, src[lane * PER + e], out[e]);
  }
#pragma unroll
  for (int e = 0; e < PER; e += 2) {
    const uint32_t pk = pack_bf16x2(out[e], out[e + 1]);
    *reinterpret_cast<uint32_t*>(o + static_cast<size_t>(row) * D + lane * PER + e) = pk;
  }
  if (lane == 0) lse[row] = L;
}

}  // namespace mala
