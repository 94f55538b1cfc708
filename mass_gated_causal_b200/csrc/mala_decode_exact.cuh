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
//                          together
//   mala_dx_scan_kernel    one warp per (b, query head) walks the chain 32
//                          tiles at a time: it assumes the 32 tiles' decisions,
//                          forms every tile's Z_prev with a log-add-exp scan,
//                          and corrects the first wrong assumption until none
//                          is left (each round fixes at least one tile)
//   mala_dx_pv_kernel      per (b, KV head, split of the tiles): P = 2^{s - m}
//                          on the kept tiles and P V, the split's O and LSE; V
//                          is read only for tiles some head of the group keeps
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
};

// log2(2^a + 2^b), with -inf as the empty sum
__device__ __forceinline__ float lae2(float a, float b) {
  const float hi = fmaxf(a, b), lo = fminf(a, b);
  if (lo == -INFINITY) return hi;
  return hi + lg2_approx(1.f + ex2_approx(lo - hi));
}

// ---------------------------------------------------------------- scores
// One CTA of 8 warps per (b, KV head, 8 key tiles); a warp per tile. Lane
// c = lane % 16 holds D/16 columns of a key row, so a warp reads two 2*D-byte
// rows per step (fully used lines); the G partial dot products are summed over
// the 16 lanes by a reduce-scatter, after which lane c owns head c / (16 / GP).
template <int D, int BK, int GP>
__global__ void __launch_bounds__(256) mala_dx_scores_kernel(const DxParams p) {
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
  constexpr int UNR = 4;
  for (int it0 = 0; it0 < BK / 2; it0 += UNR) {
    uint32_t raw[UNR][CPL / 2];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int j = kb * BK + (it0 + u) * 2 + half;
      if (j < p.Lk) {
        const uint16_t* src = krow0 + static_cast<size_t>(j) * kstride;
        if constexpr (CPL == 8) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
          raw[u][0] = v.x; raw[u][1] = v.y; raw[u][2] = v.z; raw[u][3] = v.w;
        } else {
          const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
          raw[u][0] = v.x; raw[u][1] = v.y;
        }
      } else {
#pragma unroll
        for (int e = 0; e < CPL / 2; ++e) raw[u][e] = 0u;
      }
    }
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
    bool tent = valid;  // assumed decision
    float incl = -INFINITY;
    for (int round = 0; round <= 32; ++round) {
      // Z of the assumed kept tiles before me in this chunk (log-add-exp scan)
      incl = tent ? v.y : -INFINITY;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl = lae2(incl, u);
      }
      float excl = __shfl_up_sync(0xffffffffu, incl, 1);
      if (lane == 0) excl = -INFINITY;
      const float zprev = lae2(logZ, excl);
      const bool dec = valid && (t == 0 || !p.gate || v.x - zprev >= p.thr);  // ties keep
      const unsigned mism = __ballot_sync(0xffffffffu, dec != tent);
      if (mism == 0u) break;
      const int f = __ffs(mism) - 1;  // every tile before f was assumed right, so f's decision is right
      if (lane >= f) tent = dec;      // f is now final; later tiles take a fresh guess
    }
    logZ = lae2(logZ, __shfl_sync(0xffffffffu, incl, 31));
    if (valid) {
      kp[kb] = tent ? 1 : 0;
      if (p.keep_map) p.keep_map[static_cast<size_t>(row) * p.nk + kb] = tent ? 1 : 0;
    }
    kept += __popc(__ballot_sync(0xffffffffu, valid && tent));
  }
  if (lane == 0) p.kept_tiles[row] = kept;
}

// ---------------------------------------------------------------- PV
// One CTA of 8 warps per (b, KV head, split). Per head the split's offset m is
// the largest M_t of its kept tiles and its normaliser l = sum over those tiles
// of 2^{L_t - m} (both from the per-tile pairs). A tile some head keeps is read
// once: its P = 2^{s - m} (0 for a head that skips it) goes to shared memory,
// and warp w takes keys [BK/8 * w, BK/8 * (w+1)), two per step: lane c of half
// h accumulates D/16 columns of the G heads' P V over its rows.
template <int D, int BK, int GP>
__global__ void __launch_bounds__(256) mala_dx_pv_kernel(const DxParams p) {
  constexpr int CPL = D / 16;
  constexpr int KPW = BK / 8;  // keys per warp and tile
  __shared__ float sP[GP][BK];
  __shared__ float sM[GP], sLn[GP];
  __shared__ int sKeep[2][GP];  // by tile parity: a skipped tile's flags may still be read
  __shared__ float sO[8][GP][D + 4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int nbk = p.B * p.Hkv;
  const int bk = blockIdx.x % nbk, sp = blockIdx.x / nbk;
  const int b = bk / p.Hkv, hkv = bk % p.Hkv;
  const int hq0 = hkv * p.G;
  const size_t r0 = static_cast<size_t>(b) * p.Hq + hq0;  // row of head 0 of the group
  const int t0 = min(sp * p.tiles_per_split, p.nk), t1 = min(t0 + p.tiles_per_split, p.nk);
  const int c = lane & 15, half = lane >> 4;
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
  float acc[GP][CPL];
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[g][e] = 0.f;
  const uint16_t* vrow0 = p.vc + (static_cast<size_t>(b) * p.Lk * p.Hkv + hkv) * D + c * CPL;
  const size_t vstride = static_cast<size_t>(p.Hkv) * D;
  for (int kb = t0; kb < t1; ++kb) {
    int* kf = sKeep[kb & 1];
    if (tid < GP) kf[tid] = tid < p.G ? p.keep[(r0 + tid) * p.nk + kb] : 0;
    __syncthreads();  // also: the previous tile's sP has been read
    int any = 0;
#pragma unroll
    for (int g = 0; g < GP; ++g) any |= kf[g];
    if (!any) continue;  // uniform: V of this tile is not read
    // V rows of my steps and the tile's P, loads issued together
    uint32_t raw[KPW / 2][CPL / 2];
#pragma unroll
    for (int u = 0; u < KPW / 2; ++u) {
      const int j = kb * BK + warp * KPW + u * 2 + half;
      if (j < p.Lk) {
        const uint16_t* src = vrow0 + static_cast<size_t>(j) * vstride;
        if constexpr (CPL == 8) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
          raw[u][0] = v.x; raw[u][1] = v.y; raw[u][2] = v.z; raw[u][3] = v.w;
        } else {
          const uint2 v = __ldg(reinterpret_cast<const uint2*>(src));
          raw[u][0] = v.x; raw[u][1] = v.y;
        }
      } else {
#pragma unroll
        for (int e = 0; e < CPL / 2; ++e) raw[u][e] = 0u;
      }
    }
    for (int i = tid; i < GP * BK; i += 256) {
      const int g = i / BK, j = i % BK;
      float pv = 0.f;
      if (kf[g]) pv = ex2_approx(p.scores[(r0 + g) * p.Lkp + static_cast<size_t>(kb) * BK + j] - sM[g]);
      sP[g][j] = pv;  // keys past Lk have s = -inf: 0
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < KPW / 2; ++u) {
      const int jj = warp * KPW + u * 2 + half;
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const float pg = sP[g][jj];
#pragma unroll
        for (int e = 0; e < CPL / 2; ++e) {
          acc[g][2 * e] = fmaf(pg, bf16lo_to_f32(raw[u][e]), acc[g][2 * e]);
          acc[g][2 * e + 1] = fmaf(pg, bf16hi_to_f32(raw[u][e]), acc[g][2 * e + 1]);
        }
      }
    }
  }
  // sum the two halves, then the 8 warps
#pragma unroll
  for (int g = 0; g < GP; ++g)
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], 16);
  __syncthreads();
  if (half == 0)
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
      for (int e = 0; e < CPL; ++e) sO[warp][g][c * CPL + e] = acc[g][e];
  __syncthreads();
  for (int i = tid; i < GP * D; i += 256) {
    const int g = i / D, col = i % D;
    if (g >= p.G) continue;
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) o += sO[w][g][col];
    const float l = sLn[g];
    const size_t part = (r0 + g) * p.n_splits + sp;
    p.o_part[part * D + col] = l > 0.f ? o / l : 0.f;
    if (col == 0) p.lse_part[part] = l > 0.f ? (sM[g] + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
  }
}

}  // namespace mala
