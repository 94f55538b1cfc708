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
// the work is organised around streaming K tiles through shared memory.
//
// mala_decode_split_kernel: one CTA per (b, KV head, split). The split's key
// tiles run newest -> oldest with a fresh online-softmax state per query
// head; the newest tile of the split is always kept.
//   warps 0-3  thread j scores key j of the tile against the G query heads
//              of the GQA group; head gates; P; PV with thread c owning
//              output column c of every head
//   warp  4    TMA producer of K tiles through an NK-stage ring
// V of a tile is requested (by TMA, thread 0) only after the gate has found
// a head that keeps it. Each split writes (O_s, LSE_s) per head.
//
// mala_decode_combine_kernel: LSE = log sum_s exp(LSE_s),
// O = sum_s exp(LSE_s - LSE) O_s, one warp per (b, query head).
#pragma once

#include "mala_ptx.cuh"

namespace mala {

constexpr int kDecMaxG = 8;  // query heads per KV head handled by one CTA

struct DecParams {
  int B, Hq, Hkv, Lk, G, nk, n_splits, tiles_per_split;
  float scale_log2;
  float thr;  // log2(tau) - log2(Lk)
  const uint16_t* q;  // [B, Hq, d] bf16
  float* o_part;      // [B, Hq, S, d]
  float* lse_part;    // [B, Hq, S] natural log
  int32_t* kept_tiles;
  uint8_t* keep_map;  // [B, Hq, nk], nullable
  unsigned* status;
};

template <int D, int BK>
struct DecLayout {
  static constexpr int NK = 4;
  static constexpr int NV = 2;
  static constexpr int T_BYTES = BK * D * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NK * T_BYTES;
  static constexpr int OFF_Q = OFF_V + NV * T_BYTES;          // fp32 [G][D]
  static constexpr int OFF_P = OFF_Q + kDecMaxG * D * 4;        // fp32 [G][BK]
  static constexpr int OFF_RED = OFF_P + kDecMaxG * BK * 4;     // fp32 [4][G]
  static constexpr int OFF_HEAD = OFF_RED + 4 * kDecMaxG * 4;   // per head: keep, m, alpha
  static constexpr int OFF_BAR = OFF_HEAD + 4 * kDecMaxG * 4;
  static constexpr int N_BARS = 2 * NK + NV;                    // k_full, k_empty, v_full
  static constexpr int OFF_MISC = OFF_BAR + N_BARS * 8;
  static constexpr int BYTES = OFF_MISC + 64;
  static constexpr int ALLOC_BYTES = BYTES + 1024;
  static_assert(ALLOC_BYTES <= 232448, "decode shared memory exceeds the per-CTA limit");
};

template <int D, int BK, bool kGate>
__global__ void __launch_bounds__(160, 1)
    mala_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                             const DecParams p) {
  using Lay = DecLayout<D, BK>;
  constexpr int NK = Lay::NK, NV = Lay::NV, TB = Lay::T_BYTES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  float* sq = reinterpret_cast<float*>(smem + Lay::OFF_Q);
  float* sp = reinterpret_cast<float*>(smem + Lay::OFF_P);
  float* sred = reinterpret_cast<float*>(smem + Lay::OFF_RED);
  float* skeep = reinterpret_cast<float*>(smem + Lay::OFF_HEAD);  // 1.0 if head keeps the tile
  float* smuse = skeep + kDecMaxG;                               // exponent offset (log2 units)
  float* salpha = smuse + kDecMaxG;                              // rescale factor of O
  float* sl = salpha + kDecMaxG;                                 // running normaliser
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::OFF_BAR);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + NK;
  uint64_t* v_full = bars + 2 * NK;
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + Lay::OFF_MISC);
  int* abort_flag = reinterpret_cast<int*>(misc + 0);
  uint32_t* sflag = misc + 1;  // bit 0: some head keeps the tile; bit 1: abort

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int nbk = p.B * p.Hkv;
  const int bk = blockIdx.x % nbk;
  const int sp_idx = static_cast<int>(blockIdx.x / nbk);
  const int b = bk / p.Hkv, hkv = bk % p.Hkv;
  const int G = p.G;
  const int hq0 = hkv * G;
  const int t0 = min(sp_idx * p.tiles_per_split, p.nk);
  const int t1 = min(t0 + p.tiles_per_split, p.nk);
  const int T = t1 - t0;  // tiles kb = t1-1 ... t0
  const FailState fs{abort_flag, p.status};

  if (T <= 0) {  // empty split: contributes nothing to the merge
    for (int i = tid; i < G * D; i += blockDim.x) {
      const int g = i / D, c = i % D;
      p.o_part[((static_cast<size_t>(b) * p.Hq + hq0 + g) * p.n_splits + sp_idx) * D + c] = 0.f;
    }
    if (tid < G) p.lse_part[(static_cast<size_t>(b) * p.Hq + hq0 + tid) * p.n_splits + sp_idx] = -INFINITY;
    return;
  }

  if (tid == 0) {
    for (int i = 0; i < NK; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 128); }
    for (int i = 0; i < NV; ++i) mbar_init(&v_full[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = tid; i < G * D; i += blockDim.x) {
    const int g = i / D, c = i % D;
    const uint32_t bits = p.q[(static_cast<size_t>(b) * p.Hq + hq0 + g) * D + c];
    sq[g * D + c] = __uint_as_float(bits << 16);
  }
  if (tid < kDecMaxG) {
    smuse[tid] = -INFINITY;
    sl[tid] = 0.f;
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      for (int t = 0; t < T; ++t) {
        const int st = t % NK;
        if (t >= NK && !mbar_wait(&k_empty[st], ((t / NK) - 1) & 1, fs)) break;
        const int kb = t1 - 1 - t;
        mbar_arrive_expect_tx(&k_full[st], TB);
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(&tm_k, &k_full[st], sK + st * TB + h * (BK * 128), h * 64, hkv, kb * BK, b);
        issued = t + 1;
      }
      for (int t = max(0, issued - NK); t < issued; ++t) mbar_wait_drain(&k_full[t % NK], (t / NK) & 1);
    }
    __syncwarp();
    return;  // the compute warps below use only named barrier 1
  }

  // ---------------------------------------------------------- compute warps
  const float c2 = p.scale_log2;
  float acc[kDecMaxG];  // O[g][tid] (thread tid owns output column tid)
#pragma unroll
  for (int g = 0; g < kDecMaxG; ++g) acc[g] = 0.f;
  int my_cnt = 0;  // tiles kept by head tid (threads tid < G)
  int nv = 0;  // V loads issued (tiles kept by some head)
  const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);

  for (int t = 0; t < T; ++t) {
    const int st = t % NK;
    const int kb = t1 - 1 - t;
    const bool okk = mbar_wait_warp(&k_full[st], (t / NK) & 1, fs);
    // s_g = q_g . k_j for my key j
    float s[kDecMaxG];
#pragma unroll
    for (int g = 0; g < kDecMaxG; ++g) s[g] = 0.f;
    const int key = kb * BK + tid;
    if (okk && tid < BK) {
      const uint32_t rowbase = sKa + st * TB;
#pragma unroll 4
      for (int ch = 0; ch < D / 8; ++ch) {
        uint32_t a0, a1, a2, a3;
        ld_shared_v4(rowbase + (ch >> 3) * (BK * 128) + sw128_offset(tid, ch & 7), a0, a1, a2, a3);
        const float kf[8] = {bf16lo_to_f32(a0), bf16hi_to_f32(a0), bf16lo_to_f32(a1), bf16hi_to_f32(a1),
                             bf16lo_to_f32(a2), bf16hi_to_f32(a2), bf16lo_to_f32(a3), bf16hi_to_f32(a3)};
#pragma unroll
        for (int g = 0; g < kDecMaxG; ++g) {
          if (g < G) {
            const float4 qa = *reinterpret_cast<const float4*>(sq + g * D + ch * 8);
            const float4 qb = *reinterpret_cast<const float4*>(sq + g * D + ch * 8 + 4);
            s[g] = fmaf(kf[0], qa.x, s[g]); s[g] = fmaf(kf[1], qa.y, s[g]);
            s[g] = fmaf(kf[2], qa.z, s[g]); s[g] = fmaf(kf[3], qa.w, s[g]);
            s[g] = fmaf(kf[4], qb.x, s[g]); s[g] = fmaf(kf[5], qb.y, s[g]);
            s[g] = fmaf(kf[6], qb.z, s[g]); s[g] = fmaf(kf[7], qb.w, s[g]);
          }
        }
      }
    }
    mbar_arrive(&k_empty[st]);  // my key row has been read
    const bool live = tid < BK && key < p.Lk;
#pragma unroll
    for (int g = 0; g < kDecMaxG; ++g) {
      float m = live ? s[g] : -INFINITY;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      if (lane == 0 && g < G) sred[warp * kDecMaxG + g] = m;
    }
    if (!okk) raise_abort(fs);
    named_bar_sync(1, 128);
    // ---- gates, one thread per head
    if (tid < G) {
      const int g = tid;
      float M = sred[g];
      for (int w = 1; w < 4; ++w) M = fmaxf(M, sred[w * kDecMaxG + g]);
      const float mu = smuse[g], l = sl[g];
      const bool keep = (t == 0) || !kGate || (M * c2 >= mu + lg2_approx(l) + p.thr);
      float alpha = 1.f;
      if (keep) {
        const float mnew = fmaxf(mu, M * c2);
        if (mnew > mu + 8.f) {
          alpha = ex2_approx(mu - mnew);
          sl[g] = l * alpha;
          smuse[g] = mnew;
        }
      }
      skeep[g] = keep ? 1.f : 0.f;
      salpha[g] = alpha;
      my_cnt += keep ? 1 : 0;
      if (p.keep_map) p.keep_map[(static_cast<size_t>(b) * p.Hq + hq0 + g) * p.nk + kb] = keep ? 1 : 0;
    }
    named_bar_sync(1, 128);
    if (tid == 0) {
      uint32_t any = 0;
      for (int g = 0; g < G; ++g) any |= skeep[g] != 0.f ? 1u : 0u;
      if (abort_raised(fs)) any |= 2u;
      if (any == 1u) {  // request V only now that a head keeps the tile
        const int slot = nv % NV;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&v_full[slot], TB);
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(&tm_v, &v_full[slot], sV + slot * TB + h * (BK * 128), h * 64, hkv, kb * BK, b);
      }
      *sflag = any;
    }
    named_bar_sync(1, 128);
    const uint32_t flag = *reinterpret_cast<volatile uint32_t*>(sflag);
    if (flag & 2u) break;
    if (!(flag & 1u)) continue;
    // ---- P for kept heads, row sums
#pragma unroll
    for (int g = 0; g < kDecMaxG; ++g) {
      if (g < G) {
        const float pv = (live && skeep[g] != 0.f) ? ex2_approx(fmaf(s[g], c2, -smuse[g])) : 0.f;
        if (tid < BK) sp[g * BK + tid] = pv;
        float sum = pv;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) sred[warp * kDecMaxG + g] = sum;
      }
    }
    const int slot = nv % NV;
    const bool okv = mbar_wait_warp(&v_full[slot], (nv / NV) & 1, fs);
    ++nv;
    named_bar_sync(1, 128);
    if (tid < G) sl[tid] += sred[tid] + sred[kDecMaxG + tid] + sred[2 * kDecMaxG + tid] + sred[3 * kDecMaxG + tid];
    // ---- PV: thread tid owns output column tid of every head
    if (okv && tid < D) {
      float a[kDecMaxG];
#pragma unroll
      for (int g = 0; g < kDecMaxG; ++g) a[g] = g < G ? acc[g] * salpha[g] : 0.f;
      const uint32_t vb = sVa + slot * TB + (tid >> 6) * (BK * 128) + ((tid & 7) << 1);
      const uint32_t chunk = (tid & 63) >> 3;
#pragma unroll 4
      for (int j = 0; j < BK; ++j) {
        const uint32_t addr = vb + j * 128 + ((chunk ^ (j & 7)) << 4);
        unsigned short h;
        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(h) : "r"(addr));
        const float vv = __uint_as_float(static_cast<uint32_t>(h) << 16);
#pragma unroll
        for (int g = 0; g < kDecMaxG; ++g)
          if (g < G) a[g] = fmaf(sp[g * BK + j], vv, a[g]);
      }
#pragma unroll
      for (int g = 0; g < kDecMaxG; ++g) acc[g] = a[g];
    }
    named_bar_sync(1, 128);  // P, V slot and head state are reused by the next kept tile
  }

  // ---- partial results of this split
  named_bar_sync(1, 128);
  if (!abort_raised(fs)) {
    if (tid < D) {
#pragma unroll
      for (int g = 0; g < kDecMaxG; ++g)
        if (g < G) {
          const float l = sl[g];
          p.o_part[((static_cast<size_t>(b) * p.Hq + hq0 + g) * p.n_splits + sp_idx) * D + tid] =
              l > 0.f ? acc[g] / l : 0.f;
        }
    }
    if (tid < G) {
      const float l = sl[tid];
      p.lse_part[(static_cast<size_t>(b) * p.Hq + hq0 + tid) * p.n_splits + sp_idx] =
          l > 0.f ? (smuse[tid] + lg2_approx(l)) * 0.69314718055994531f : -INFINITY;
      atomicAdd(&p.kept_tiles[b * p.Hq + hq0 + tid], my_cnt);
    }
  }
  if (tid == 0)
    for (int i = max(0, nv - NV); i < nv; ++i) mbar_wait_drain(&v_full[i % NV], (i / NV) & 1);
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
