// mala_decode_exact.cuh -- split-independent MALA decode for sm_100a.
//
// Method (agihunt.info, "MassAlloc Attention: Let Attention Allocate Its Own
// Compute", method paragraphs): the forward gate of one query row (decode,
// Lq = Lk) visits key tiles from the newest to the oldest and keeps tile t iff
// it is the first, or tau = 0, or its largest ratio exp(s - m) / l against the
// state over the tiles kept so far reaches tau / Lq. In log2 units that ratio
// is 2^{M_t} / Z_prev with M_t the tile's largest score and Z_prev the sum of
// 2^s over the kept newer tiles, i.e. a sum of the kept tiles' 2^{L_t}
// (L_t = log2 of the tile's sum of 2^s). So the whole chain of decisions
// depends only on the per-tile pairs (M_t, L_t), and the decisions equal those
// of one sequential pass whatever the split of the tiles over CTAs. Three
// phases (HBM-bound, CUDA cores; no tensor-core shape here):
//   mala_dx_scores_kernel  every score s = scale * log2(e) * <q, k> of every
//                          query head, stored (fp32), and (M_t, L_t) per tile
//                          and head; K is read once, by the G heads of a group
//                          together, a warp per tile (many warps per SM keep the
//                          loads in flight; a TMA-ring version measured slower)
//   mala_dx_scan_kernel    one warp per (b, query head) walks the chain 32
//                          tiles at a time: it assumes the 32 tiles' decisions,
//                          forms every tile's Z_prev with a prefix sum (linear
//                          units relative to the chunk's largest log-sum), and
//                          corrects the first wrong assumption until none is
//                          left (each round fixes at least one tile)
//   mala_dx_pv_kernel      per (b, KV head, split of the tiles): P = 2^{s - m}
//                          on the kept tiles and P V, the split's O and LSE; V
//                          of the tiles some head of the group keeps streams in
//                          by TMA through a ring, and no other V is read
// and mala_decode_combine_kernel merges the splits by their LSEs.
#pragma once

#include "mala_decode.cuh"

namespace mala {

struct DxParams {
  int B, Hq, Hkv, G, Lk, nk, n_splits, tiles_per_split;
  int Lkp;              // nk * Bk: row length of the score buffer
  float scale_log2;     // scale * log2(e)
  float thr;            // log2(tau) - log2(Lk); gate off: tau = 0
  int gate;             // tau > 0
  const uint16_t* q;    // [B, Hq, d] bf16
  const uint16_t* kc;   // [B, Lk, Hkv, d] bf16
  const uint16_t* vc;   // [B, Lk, Hkv, d] bf16
  float* scores;        // [B, Hq, Lkp] log2 units
  float2* tile_ml;      // [B, Hq, nk]: (M_t, L_t)
  uint8_t* keep;        // [B, Hq, nk]: the decisions
  float* o_part;        // [B, Hq, S, d]
  float* lse_part;      // [B, Hq, S] natural log
  int32_t* kept_tiles;  // [B * Hq]
  uint8_t* keep_map;    // [B, Hq, nk], nullable
  void* o_out;          // [B, Hq, d] bf16 (written by the merge)
  float* lse_out;       // [B, Hq]
  unsigned* status;
  uint64_t wait_ns;     // limit of each bounded wait
};

// Shared-memory layout of the PV kernel: an NS-stage ring of
// [D/64][BK][64] bf16 tiles (128-byte swizzle, as the TMA writes them) with
// the tile's scores of the group's heads ([GP][BK] fp32 per stage), a
// [2][GP][BK] fp32 tile and the ring's barriers; the final cross-warp
// reduction reuses the ring. Three stages keep the CTA under half of an SM's
// shared memory, so two CTAs share an SM (measured 11% faster over the whole
// decode than one CTA per SM with four stages).
template <int D, int BK, int GP>
struct DxLayout {
  static constexpr int NS = 3;
  static constexpr int TB = BK * D * 2;
  static constexpr int SB = GP * BK * 4;                  // scores of one stage
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_SC = OFF_RING + NS * TB;       // fp32 [NS][GP][BK]: the stages' scores
  static constexpr int OFF_T = OFF_SC + NS * SB;          // fp32 [2][GP][BK]: P by tile parity
  static constexpr int OFF_O = OFF_RING;                  // fp32 [8][GP][D + 4] (PV reduction, over the ring once it is drained)
  static_assert(8 * GP * (D + 4) * 4 <= NS * TB, "the PV reduction buffer must fit in the ring");
  static constexpr int OFF_LIST = OFF_T + 2 * GP * BK * 4;  // int tiles [LIST], uint8 bits [LIST]
  static constexpr int LIST = 1024;
  static constexpr int OFF_BAR = (OFF_LIST + LIST * 5 + 7) & ~7;
  static constexpr int OFF_MISC = OFF_BAR + 2 * NS * 8;
  static constexpr int BYTES = OFF_MISC + 128;  // abort flag, list count, m and l per head
  static constexpr int ALLOC_BYTES = BYTES + 1024;
  static_assert(ALLOC_BYTES <= 232448, "shared memory exceeds the per-CTA limit");
};

// 16-byte chunk cc of row j of a [D/64][BK][64] bf16 tile with 128-byte swizzle
template <int BK>
__device__ __forceinline__ uint32_t dx_row_chunk(uint32_t base, int j, int cc) {
  return base + (cc >> 3) * (BK * 128) + j * 128 + (((cc & 7) ^ (j & 7)) << 4);
}

// ---------------------------------------------------------------- scores
// One CTA of 8 warps per (b, KV head, 8 key tiles); a warp per tile. Lane
// c = lane % 16 holds D/16 columns of a key row, so a warp reads two 2*D-byte
// rows per step (fully used lines); the G partial dot products are summed over
// the 16 lanes by a reduce-scatter, after which lane c owns head c / (16 / GP).
template <int D, int BK, int GP>
__global__ void __launch_bounds__(256, 2) mala_dx_scores_kernel(const DxParams p) {
  constexpr int CPL = D / 16;  // columns per lane
  constexpr int LPH = 16 / GP; // lanes per head after the reduce-scatter
  __shared__ float sS[8][GP][BK];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_per_bk = (p.nk + 7) / 8;
  const int bk = blockIdx.x / tiles_per_bk;
  const int kb = (blockIdx.x % tiles_per_bk) * 8 + warp;
  const int b = bk / p.Hkv, hkv = bk % p.Hkv;
  const int hq0 = hkv * p.G;
  if (kb >= p.nk) return;  // warp-uniform; no block-wide barrier below
  const int c = lane & 15, half = lane >> 4;
  // my q columns of every head of the group (padded heads are zero)
  float qf[GP][CPL];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int e = 0; e < CPL; ++e)
      qf[g][e] = g < p.G ? bf16lo_to_f32(p.q[(static_cast<size_t>(b) * p.Hq + hq0 + g) * D + c * CPL + e]) : 0.f;
  const uint16_t* krow0 = p.kc + (static_cast<size_t>(b) * p.Lk * p.Hkv + hkv) * D + c * CPL;
  const size_t kstride = static_cast<size_t>(p.Hkv) * D;
  // rows per lane and group; the next group's loads are issued before this one
  // is used. Eight (4 KB in flight per warp, two CTAs per SM at 128 registers)
  // measured 3% faster over the whole decode than four (three CTAs per SM);
  // sixteen (one CTA per SM) and eight at three CTAs per SM (spills) were slower.
  constexpr int UNR = 8;
  uint32_t nxt[UNR][CPL / 2];
  auto load_group = [&](int it0) {
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int j = kb * BK + (it0 + u) * 2 + half;
      if (j < p.Lk) {
        const uint16_t* src = krow0 + static_cast<size_t>(j) * kstride;
        if constexpr (CPL == 8) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
          nxt[u][0] = v.x; nxt[u][1] = v.y; nxt[u][2] = v.z; nxt[u][3] = v.w;
        } else {
          const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
          nxt[u][0] = v.x; nxt[u][1] = v.y;
        }
      } else {
#pragma unroll
        for (int e = 0; e < CPL / 2; ++e) nxt[u][e] = 0u;
      }
    }
  };
  load_group(0);
  for (int it0 = 0; it0 < BK / 2; it0 += UNR) {
    uint32_t raw[UNR][CPL / 2];
#pragma unroll
    for (int u = 0; u < UNR; ++u)
#pragma unroll
      for (int e = 0; e < CPL / 2; ++e) raw[u][e] = nxt[u][e];
    if (it0 + UNR < BK / 2) load_group(it0 + UNR);
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      float part[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < CPL / 2; ++e) {
          a = fmaf(bf16lo_to_f32(raw[u][e]), qf[g][2 * e], a);
          a = fmaf(bf16hi_to_f32(raw[u][e]), qf[g][2 * e + 1], a);
        }
        part[g] = a;
      }
      const float mine = group_reduce_scatter<GP, 16>(part, c);  // head c / LPH, key of my half
      const int jj = (it0 + u) * 2 + half;
      if (c % LPH == 0) {
        const bool live = kb * BK + jj < p.Lk;
        sS[warp][c / LPH][jj] = live ? mine * p.scale_log2 : -INFINITY;
      }
    }
  }
  __syncwarp();
  // per head: M = max, L = M + log2(sum 2^{s - M}); 32 / GP lanes per head
  constexpr int LPT = 32 / GP;  // lanes per head here
  constexpr int KPL = BK / LPT; // keys per lane
  const int h = lane / LPT, r = lane % LPT;
  float mx = -INFINITY;
#pragma unroll
  for (int e = 0; e < KPL; ++e) mx = fmaxf(mx, sS[warp][h][r + e * LPT]);
#pragma unroll
  for (int o = LPT / 2; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sm = 0.f;
  if (mx != -INFINITY) {
#pragma unroll
    for (int e = 0; e < KPL; ++e) sm += ex2_approx(sS[warp][h][r + e * LPT] - mx);
  }
#pragma unroll
  for (int o = LPT / 2; o >= 1; o >>= 1) sm += __shfl_xor_sync(0xffffffffu, sm, o);
  if (r == 0 && h < p.G)
    p.tile_ml[(static_cast<size_t>(b) * p.Hq + hq0 + h) * p.nk + kb] =
        make_float2(mx, mx == -INFINITY ? -INFINITY : mx + lg2_approx(sm));
  // the scores, a tile of each head as whole lines
  for (int g = 0; g < p.G; ++g) {
    float* dst = p.scores + (static_cast<size_t>(b) * p.Hq + hq0 + g) * p.Lkp + static_cast<size_t>(kb) * BK;
    for (int j = lane * 4; j < BK; j += 128)
      *reinterpret_cast<float4*>(dst + j) =
          make_float4(sS[warp][g][j], sS[warp][g][j + 1], sS[warp][g][j + 2], sS[warp][g][j + 3]);
  }
}

// ---------------------------------------------------------------- scan
// One warp per (b, query head): the decisions of tiles t = 0 .. nk - 1 in
// visit order (tile kb = nk - 1 - t), 32 at a time.
__global__ void __launch_bounds__(128) mala_dx_scan_kernel(const DxParams p) {
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.B * p.Hq) return;
  const float2* ml = p.tile_ml + static_cast<size_t>(row) * p.nk;
  uint8_t* kp = p.keep + static_cast<size_t>(row) * p.nk;
  float logZ = -INFINITY;  // log2 of the sum over the kept tiles so far
  int kept = 0;
  for (int t0 = 0; t0 < p.nk; t0 += 32) {
    const int t = t0 + lane;
    const bool valid = t < p.nk;
    const int kb = p.nk - 1 - t;
    const float2 v = valid ? ml[kb] : make_float2(-INFINITY, -INFINITY);
    // linear units relative to R, the largest log-sum in play: every term <= 1,
    // so the rounds below are plain sums and compares
    float R = fmaxf(logZ, v.y);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) R = fmaxf(R, __shfl_xor_sync(0xffffffffu, R, o));
    if (R == -INFINITY) R = 0.f;
    const float zl = logZ == -INFINITY ? 0.f : ex2_approx(logZ - R);  // the kept tiles before this chunk
    const float w = valid ? ex2_approx(v.y - R) : 0.f;                 // my tile's sum
    const float e = valid ? ex2_approx(v.x - p.thr - R) : 0.f;         // 2^{M - thr}: keep iff e >= Z_prev
    bool tent = valid;  // assumed decision
    float incl = 0.f;
    for (int round = 0; round <= 32; ++round) {
      // Z of the assumed kept tiles before me in this chunk (prefix sum)
      incl = tent ? w : 0.f;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      float excl = __shfl_up_sync(0xffffffffu, incl, 1);
      if (lane == 0) excl = 0.f;
      const bool dec = valid && (t == 0 || !p.gate || e >= zl + excl);  // ties keep
      const unsigned mism = __ballot_sync(0xffffffffu, dec != tent);
      if (mism == 0u) break;
      const int f = __ffs(mism) - 1;  // every tile before f was assumed right, so f's decision is right
      if (lane >= f) tent = dec;      // f is now final; later tiles take a fresh guess
    }
    const float zt = zl + __shfl_sync(0xffffffffu, incl, 31);
    if (zt > 0.f) logZ = R + lg2_approx(zt);
    if (valid) {
      kp[kb] = tent ? 1 : 0;
      if (p.keep_map) p.keep_map[static_cast<size_t>(row) * p.nk + kb] = tent ? 1 : 0;
    }
    kept += __popc(__ballot_sync(0xffffffffu, valid && tent));
  }
  if (lane == 0) p.kept_tiles[row] = kept;
}

// ---------------------------------------------------------------- PV
// One CTA per (b, KV head, split). Per head the split's offset m is the
// largest M_t of its kept tiles and its normaliser l = sum over those tiles of
// 2^{L_t - m} (both from the per-tile pairs). Warp 8 lists the tiles some head
// of the group keeps (with a bit per head) and streams their V by TMA through
// the ring, together with the tile's scores of the group's heads (bulk copies
// on the same barrier, so no compute warp waits on a global load); a tile no
// head keeps is never read. Per listed tile the compute warps form
// P = 2^{s - m} (0 for a head that skips the tile) in shared memory, and warp
// w takes keys [BK/8 * w, BK/8 * (w+1)), two per step: lane c of half h
// accumulates D/16 columns of the G heads' P V over its rows.
template <int D, int BK, int GP>
__global__ void __launch_bounds__(288, 2) mala_dx_pv_kernel(const __grid_constant__ CUtensorMap tm_v,
                                                              const DxParams p) {
  using Lay = DxLayout<D, BK, GP>;
  constexpr int NS = Lay::NS, TB = Lay::TB, LIST = Lay::LIST;
  constexpr int CPL = D / 16;
  constexpr int KPW = BK / 8;                   // keys per compute warp and tile
  constexpr int NPT = (GP * BK + 255) / 256;    // P entries per compute thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* sP = reinterpret_cast<float*>(smem + Lay::OFF_T);  // [2][GP][BK]
  const float* sSc = reinterpret_cast<const float*>(smem + Lay::OFF_SC);  // [NS][GP][BK]
  float* sO = reinterpret_cast<float*>(smem + Lay::OFF_O);  // [8][GP][D + 4]
  int* sList = reinterpret_cast<int*>(smem + Lay::OFF_LIST);
  uint8_t* sBits = smem + Lay::OFF_LIST + LIST * 4;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* empty = full + NS;
  int* misc = reinterpret_cast<int*>(smem + Lay::OFF_MISC);
  int* abort_flag = misc;
  int* sCount = misc + 1;
  float* sM = reinterpret_cast<float*>(misc + 2);  // [GP]
  float* sLn = sM + GP;                            // [GP]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int nbk = p.B * p.Hkv;
  const int bk = blockIdx.x % nbk, sp = blockIdx.x / nbk;
  const int b = bk / p.Hkv, hkv = bk % p.Hkv;
  const int hq0 = hkv * p.G;
  const size_t r0 = static_cast<size_t>(b) * p.Hq + hq0;  // row of head 0 of the group
  const int t0 = min(sp * p.tiles_per_split, p.nk), t1 = min(t0 + p.tiles_per_split, p.nk);
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 8); }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp < GP) {  // warp g: the offset and normaliser of head g over this split
    float m = -INFINITY;
    if (warp < p.G)
      for (int kb = t0 + lane; kb < t1; kb += 32)
        if (p.keep[(r0 + warp) * p.nk + kb]) m = fmaxf(m, p.tile_ml[(r0 + warp) * p.nk + kb].x);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    if (warp < p.G && m != -INFINITY)
      for (int kb = t0 + lane; kb < t1; kb += 32)
        if (p.keep[(r0 + warp) * p.nk + kb]) l += ex2_approx(p.tile_ml[(r0 + warp) * p.nk + kb].y - m);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      sM[warp] = m;
      sLn[warp] = l;
    }
  }
  __syncthreads();
  const FailState fs{abort_flag, p.status, p.wait_ns};
  const int c = lane & 15, half = lane >> 4;
  float acc[GP][CPL];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[g][e] = 0.f;
  const uint32_t ring = smem_u32(smem + Lay::OFF_RING);
  int base = 0;    // listed tiles of earlier segments (ring position)
  int issued = 0;  // warp 8, lane 0: V loads issued (an abort stops the issue)
  for (int seg0 = t0; seg0 < t1; seg0 += LIST) {
    const int seg1 = min(seg0 + LIST, t1);
    if (warp == 8) {  // the segment's list of tiles some head keeps, in order
      int n = 0;
      for (int k0 = seg0; k0 < seg1; k0 += 32) {
        const int kb = k0 + lane;
        uint32_t bits = 0;
        if (kb < seg1)
          for (int g = 0; g < p.G; ++g) bits |= p.keep[(r0 + g) * p.nk + kb] ? (1u << g) : 0u;
        const unsigned any = __ballot_sync(0xffffffffu, bits != 0u);
        const int at = n + __popc(any & ((1u << lane) - 1u));
        if (bits) {
          sList[at] = kb;
          sBits[at] = static_cast<uint8_t>(bits);
        }
        n += __popc(any);
      }
      if (lane == 0) *sCount = n;
    }
    __syncthreads();
    const int n = *sCount;
    if (warp == 8) {
      if (lane == 0) {
        for (int i = 0; i < n; ++i) {
          const int ig = base + i, st = ig % NS;
          if (ig >= NS && !mbar_wait(&empty[st], ((ig / NS) - 1) & 1, fs)) break;
          mbar_arrive_expect_tx(&full[st], TB + p.G * BK * 4);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(&tm_v, &full[st], smem + Lay::OFF_RING + st * TB + h * (BK * 128), h * 64, hkv,
                        sList[i] * BK, b);
          // the scores rows start on 512-byte boundaries (rows of Lkp = nk * BK floats, tiles of BK)
          for (int g = 0; g < p.G; ++g)
            bulk_load_1d(smem + Lay::OFF_SC + (st * GP + g) * BK * 4,
                         p.scores + (r0 + g) * p.Lkp + static_cast<size_t>(sList[i]) * BK, BK * 4, &full[st]);
          issued = ig + 1;
        }
      }
    } else {
      for (int i = 0; i < n; ++i) {
        const int ig = base + i, st = ig % NS;
        float* P = sP + (ig & 1) * GP * BK;
        const bool ok = mbar_wait_warp(&full[st], (ig / NS) & 1, fs);  // V and the scores of this tile
        const uint32_t bits = sBits[i];
#pragma unroll
        for (int k = 0; k < NPT; ++k) {
          const int idx = tid + k * 256, g = idx / BK;
          if (idx < GP * BK) {
            const float s = (ok && ((bits >> g) & 1u)) ? sSc[st * GP * BK + idx] : -INFINITY;
            P[idx] = s == -INFINITY ? 0.f : ex2_approx(s - sM[g]);
          }
        }
        named_bar_sync(1, 256);  // P of this tile is in place (and the one two tiles back is read)
        if (ok) {
#pragma unroll
          for (int u = 0; u < KPW / 2; ++u) {
            const int jj = warp * KPW + u * 2 + half;
            uint32_t raw[CPL / 2];
            if constexpr (CPL == 8) {
              ld_shared_v4(dx_row_chunk<BK>(ring + st * TB, jj, c), raw[0], raw[1], raw[2], raw[3]);
            } else {
              uint32_t a0, a1, a2, a3;
              ld_shared_v4(dx_row_chunk<BK>(ring + st * TB, jj, c >> 1), a0, a1, a2, a3);
              raw[0] = (c & 1) ? a2 : a0;
              raw[1] = (c & 1) ? a3 : a1;
            }
#pragma unroll
            for (int g = 0; g < GP; ++g) {
              const float pg = P[g * BK + jj];
#pragma unroll
              for (int e = 0; e < CPL / 2; ++e) {
                acc[g][2 * e] = fmaf(pg, bf16lo_to_f32(raw[e]), acc[g][2 * e]);
                acc[g][2 * e + 1] = fmaf(pg, bf16hi_to_f32(raw[e]), acc[g][2 * e + 1]);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[st]);  // my rows of this V stage are read
      }
    }
    base += n;
    __syncthreads();  // the next segment's list overwrites this one
  }
  if (warp == 8) {  // the last loads have landed before the CTA ends
    if (lane == 0)
      for (int ig = max(0, issued - NS); ig < issued; ++ig) mbar_wait_drain(&full[ig % NS], (ig / NS) & 1);
    return;
  }
  // sum the two halves, then the 8 warps
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], 16);
  named_bar_sync(1, 256);  // every compute warp is done with the ring, which the reduction reuses
  if (half == 0)
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
      for (int e = 0; e < CPL; ++e) sO[(warp * GP + g) * (D + 4) + c * CPL + e] = acc[g][e];
  named_bar_sync(1, 256);
  for (int i = tid; i < GP * D; i += 256) {
    const int g = i / D, col = i % D;
    if (g >= p.G) continue;
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) o += sO[(w * GP + g) * (D + 4) + col];
    const float l = sLn[g];
    const size_t part = (r0 + g) * p.n_splits + sp;
    p.o_part[part * D + col] = l > 0.f ? o / l : 0.f;
    if (col == 0) p.lse_part[part] = l > 0.f ? (sM[g] + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace mala
