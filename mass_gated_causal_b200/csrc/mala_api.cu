// mala_api.cu -- the C ABI declared in include/mala.h.
//
// Host side only: argument validation, TMA tensor-map construction, launch
// configuration. Every step of the computation runs in the kernels included
// below. The driver's cuTensorMapEncodeTiled is reached through
// cudaGetDriverEntryPoint, so the library loads on machines without a GPU
// driver (its symbols can be inspected there) and needs no -lcuda.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>

#include "../../include/mala.h"
#include "mala_bwd.cuh"
#include "mala_decode.cuh"
#include "mala_decode_exact.cuh"
#include "mala_fwd.cuh"

namespace {

__device__ unsigned int g_mala_status;  // per-device status word, see mala_check_status

// Test hooks (mala_test_hooks): bounded-wait limit, stall tile, V-tile counter.
std::atomic<unsigned long long> g_wait_ns{mala::kWaitLimitNs};
std::atomic<int> g_stall_tile{-1};
std::atomic<unsigned long long*> g_v_tiles{nullptr};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor map over a contiguous bf16 BSHD tensor [B, S, H, D] with a
// {64, 1, rows, 1} box and 128-byte swizzle: one box is a [rows x 64] tile of
// one head, 128 bytes per row, the layout the UMMA descriptors expect.
bool make_bshd_map(CUtensorMap* map, const void* base, int B, int S, int H, int D, int rows,
                   CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(S),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2,
                           static_cast<cuuint64_t>(S) * H * D * 2};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over the fp32 dQ accumulator [B, S, H, D] with a {32, 1, 32, 1}
// box and 128-byte swizzle: a [32 rows x 32] fp32 block of one head.
bool make_dq_acc_map(CUtensorMap* map, const void* base, int B, int S, int H, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(S),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 4, static_cast<cuuint64_t>(H) * D * 4,
                           static_cast<cuuint64_t>(S) * H * D * 4};
  cuuint32_t box[4] = {32, 1, 32, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

unsigned* status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_mala_status) != cudaSuccess) return nullptr;
  return static_cast<unsigned*>(p);
}

int check_train_shape(int B, int Hq, int Hkv, int L, int d, float scale, float tau, int Bq, int Bk) {
  if (B < 1 || Hq < 1 || Hkv < 1 || L < 1) return MALA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return MALA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return MALA_ERR_INVALID_ARG;
  if (!(tau >= 0.f) || !std::isfinite(tau)) return MALA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return MALA_ERR_UNSUPPORTED;
  if ((Bq != 64 && Bq != 128) || (Bk != 64 && Bk != 128)) return MALA_ERR_UNSUPPORTED;
  // element counts must fit the int arithmetic of the kernels
  if (static_cast<long long>(B) * L * Hq * d >= (1ll << 40)) return MALA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Hq >= (1ll << 24)) return MALA_ERR_UNSUPPORTED;
  return MALA_OK;
}

template <typename K>
int set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
             ? MALA_OK
             : MALA_ERR_CUDA;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int sm_count() {
  int sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    sms = 148;
  return sms;
}

// Chunk length of the training kernels' CTA schedule: about one wave of CTAs
// per (b, KV head) unit, but at most a quarter (forward) / half (backward) of
// a unit's work so that the longest items still start first.
int fwd_chunk_pairs(int n_pairs, int G) {
  return std::max(1, std::min(sm_count() / G, (n_pairs + 3) / 4));
}
int bwd_chunk_kb(int n_super) { return std::max(1, std::min(sm_count(), (n_super + 1) / 2)); }

// ---------------------------------------------------------------- forward
template <int D, int BQ, int BK, int MODE>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mo,
               const mala::FwdParams& p, cudaStream_t st) {
  using Lay = mala::FwdLayout<D, BK>;
  auto kern = mala::mala_fwd_kernel<D, BQ, BK, MODE>;
  if (set_smem(kern, Lay::ALLOC_BYTES) != MALA_OK) return MALA_ERR_CUDA;
  const unsigned n_chunks = (p.n_pairs + p.chunk_pairs - 1) / p.chunk_pairs;
  const unsigned grid = n_chunks * p.chunk_pairs * p.B * p.Hq;
  kern<<<grid, 352, Lay::ALLOC_BYTES, st>>>(mq, mk, mv, mo, p);
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}

// mode: 0 no gate, 1 gate with V on demand, 2 gate with V fetched ahead
template <int D, int BQ, int BK>
int launch_fwd_gate(int mode, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                    const CUtensorMap& mo, const mala::FwdParams& p, cudaStream_t st) {
  if (mode == 1) return launch_fwd<D, BQ, BK, 1>(mq, mk, mv, mo, p, st);
  if (mode == 2) return launch_fwd<D, BQ, BK, 2>(mq, mk, mv, mo, p, st);
  return launch_fwd<D, BQ, BK, 0>(mq, mk, mv, mo, p, st);
}

template <int D>
int launch_fwd_tiles(int Bq, int Bk, int mode, const CUtensorMap& mq, const CUtensorMap& mk,
                     const CUtensorMap& mv, const CUtensorMap& mo, const mala::FwdParams& p, cudaStream_t st) {
  if (Bq == 128 && Bk == 128) return launch_fwd_gate<D, 128, 128>(mode, mq, mk, mv, mo, p, st);
  if (Bq == 64 && Bk == 64) return launch_fwd_gate<D, 64, 64>(mode, mq, mk, mv, mo, p, st);
  if (Bq == 64 && Bk == 128) return launch_fwd_gate<D, 64, 128>(mode, mq, mk, mv, mo, p, st);
  return launch_fwd_gate<D, 128, 64>(mode, mq, mk, mv, mo, p, st);
}

// --------------------------------------------------------------- backward
template <int D, int BQ, int BK, bool G>
int launch_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
               const CUtensorMap& mdk, const CUtensorMap& mdv, const CUtensorMap& mdq, const mala::BwdParams& p,
               cudaStream_t st) {
  using Lay = mala::BwdLayout<D>;
  auto kern = p.cu != nullptr ? mala::mala_bwd_kernel<D, BQ, BK, G, true> : mala::mala_bwd_kernel<D, BQ, BK, G, false>;
  if (set_smem(kern, Lay::ALLOC_BYTES) != MALA_OK) return MALA_ERR_CUDA;
  const unsigned n_chunks = (p.n_super + p.chunk_kb - 1) / p.chunk_kb;
  const unsigned grid = n_chunks * p.chunk_kb * p.B * p.Hkv;
  kern<<<grid, 448, Lay::ALLOC_BYTES, st>>>(mq, mk, mv, mdo, mdk, mdv, mdq, p);
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}

template <int D, int BQ, int BK>
int launch_bwd_gate(bool gate, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                    const CUtensorMap& mdo, const CUtensorMap& mdk, const CUtensorMap& mdv,
                    const CUtensorMap& mdq, const mala::BwdParams& p, cudaStream_t st) {
  return gate ? launch_bwd<D, BQ, BK, true>(mq, mk, mv, mdo, mdk, mdv, mdq, p, st)
              : launch_bwd<D, BQ, BK, false>(mq, mk, mv, mdo, mdk, mdv, mdq, p, st);
}

template <int D>
int launch_bwd_tiles(int Bq, int Bk, bool gate, const CUtensorMap& mq, const CUtensorMap& mk,
                     const CUtensorMap& mv, const CUtensorMap& mdo, const CUtensorMap& mdk, const CUtensorMap& mdv,
                     const CUtensorMap& mdq, const mala::BwdParams& p, cudaStream_t st) {
  if (Bq == 128 && Bk == 128) return launch_bwd_gate<D, 128, 128>(gate, mq, mk, mv, mdo, mdk, mdv, mdq, p, st);
  if (Bq == 64 && Bk == 64) return launch_bwd_gate<D, 64, 64>(gate, mq, mk, mv, mdo, mdk, mdv, mdq, p, st);
  if (Bq == 64 && Bk == 128) return launch_bwd_gate<D, 64, 128>(gate, mq, mk, mv, mdo, mdk, mdv, mdq, p, st);
  return launch_bwd_gate<D, 128, 64>(gate, mq, mk, mv, mdo, mdk, mdv, mdq, p, st);
}

// ----------------------------------------------------------------- decode
template <int D, int BK, int GP, bool G>
int launch_dec(const CUtensorMap& mk, const CUtensorMap& mv, const mala::DecParams& p, cudaStream_t st) {
  using Lay = mala::DecLayout<D, BK, GP>;
  auto kern = p.block_table != nullptr ? mala::mala_decode_split_kernel<D, BK, GP, G, true>
                                       : mala::mala_decode_split_kernel<D, BK, GP, G, false>;
  if (set_smem(kern, Lay::ALLOC_BYTES) != MALA_OK) return MALA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hkv * p.n_splits;
  kern<<<grid, 320, Lay::ALLOC_BYTES, st>>>(mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}

// GQA group size padded to the next power of two (1, 2, 4, 8).
template <int D, int BK, bool G>
int launch_dec_g(const CUtensorMap& mk, const CUtensorMap& mv, const mala::DecParams& p, cudaStream_t st) {
  if (p.G <= 1) return launch_dec<D, BK, 1, G>(mk, mv, p, st);
  if (p.G <= 2) return launch_dec<D, BK, 2, G>(mk, mv, p, st);
  if (p.G <= 4) return launch_dec<D, BK, 4, G>(mk, mv, p, st);
  return launch_dec<D, BK, 8, G>(mk, mv, p, st);
}

template <int D, int BK>
int launch_dec_gate(bool gate, const CUtensorMap& mk, const CUtensorMap& mv, const mala::DecParams& p,
                    cudaStream_t st) {
  return gate ? launch_dec_g<D, BK, true>(mk, mv, p, st) : launch_dec_g<D, BK, false>(mk, mv, p, st);
}

template <int D, int BK, int GP>
int launch_dx(const CUtensorMap& mv, const mala::DxParams& p, cudaStream_t st) {
  using Lay = mala::DxLayout<D, BK, GP>;
  auto kpv = mala::mala_dx_pv_kernel<D, BK, GP>;
  if (set_smem(kpv, Lay::ALLOC_BYTES) != MALA_OK) return MALA_ERR_CUDA;
  const unsigned g1 = static_cast<unsigned>(p.B) * p.Hkv * ((p.nk + 7) / 8);
  mala::mala_dx_scores_kernel<D, BK, GP><<<g1, 256, 0, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return MALA_ERR_CUDA;
  mala::mala_dx_scan_kernel<<<(p.B * p.Hq + 3) / 4, 128, 0, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return MALA_ERR_CUDA;
  const unsigned g3 = static_cast<unsigned>(p.B) * p.Hkv * p.n_splits;
  kpv<<<g3, 288, Lay::ALLOC_BYTES, st>>>(mv, p);
  if (cudaGetLastError() != cudaSuccess) return MALA_ERR_CUDA;
  mala::mala_decode_combine_kernel<D><<<(p.B * p.Hq + 3) / 4, 128, 0, st>>>(p.o_part, p.lse_part,
                                                                         reinterpret_cast<uint16_t*>(p.o_out),
                                                                         p.lse_out, p.B * p.Hq, p.n_splits);
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}

template <int D, int BK>
int launch_dx_g(const CUtensorMap& mv, const mala::DxParams& p, cudaStream_t st) {
  if (p.G <= 1) return launch_dx<D, BK, 1>(mv, p, st);
  if (p.G <= 2) return launch_dx<D, BK, 2>(mv, p, st);
  if (p.G <= 4) return launch_dx<D, BK, 4>(mv, p, st);
  return launch_dx<D, BK, 8>(mv, p, st);
}


}  // namespace

extern "C" {

const char* mala_status_string(int status) {
  switch (status) {
    case MALA_OK: return "MALA_OK";
    case MALA_ERR_INVALID_ARG: return "MALA_ERR_INVALID_ARG";
    case MALA_ERR_UNSUPPORTED: return "MALA_ERR_UNSUPPORTED";
    case MALA_ERR_WORKSPACE: return "MALA_ERR_WORKSPACE";
    case MALA_ERR_CUDA: return "MALA_ERR_CUDA";
    case MALA_ERR_DEVICE_TIMEOUT: return "MALA_ERR_DEVICE_TIMEOUT";
    case MALA_ERR_RANGE: return "MALA_ERR_RANGE";
    default: return "MALA_ERR_UNKNOWN";
  }
}

int mala_abi_version(void) { return MALA_ABI_VERSION; }

size_t mala_fwd_workspace_size(int B, int Hkv, int L, int d) {
  if (B < 1 || Hkv < 1 || L < 1 || (d != 64 && d != 128)) return 0;
  return align256(static_cast<size_t>(B) * L * Hkv * d * 2);
}

namespace {
// Packed batch: sequence tables and sizes (null cu_q for a dense batch).
struct Packed {
  const int* cu_q = nullptr;
  const int* cu_k = nullptr;
  int total_q = 0, total_k = 0;
};

// Forward of Lq queries at positions Lk - Lq .. Lk - 1 against Lk keys (the
// training forward is Lq == Lk); arguments already checked by the caller. For a
// packed batch, B counts the sequences and Lq / Lk are the longest lengths.
int run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Lq,
            int Lk, int d, float scale, float tau, int Bq, int Bk, void* workspace, size_t workspace_bytes,
            int32_t* kept_tiles, uint8_t* keep_map, void* stream, const Packed& pk = Packed(),
            bool prefetch_v = false) {
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return MALA_ERR_UNSUPPORTED;
  const bool packed = pk.cu_q != nullptr;
  // tensor extents: [B, L, H, d], a packed batch as one sequence of all its rows
  const int tb = packed ? 1 : B, tq = packed ? pk.total_q : Lq, tk = packed ? pk.total_k : Lk;
  const size_t need = mala_fwd_workspace_size(tb, Hkv, tk, d);
  if (!workspace || workspace_bytes < need || !aligned256(workspace)) return MALA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap mq, mk, mv, mo;
  if (!make_bshd_map(&mq, q, tb, tq, Hq, d, 128) || !make_bshd_map(&mk, k, tb, tk, Hkv, d, Bk) ||
      !make_bshd_map(&mv, workspace, tb, tk, Hkv, d, Bk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16) ||
      !make_bshd_map(&mo, o, tb, tq, Hq, d, 128))
    return MALA_ERR_CUDA;
  unsigned* status = status_ptr();
  if (!status) return MALA_ERR_CUDA;
  mala::FwdParams p;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv;
  p.Lq = Lq; p.Lk = Lk; p.P0 = Lk - Lq;
  p.o = static_cast<uint16_t*>(o);
  p.cu_q = pk.cu_q;
  p.cu_k = pk.cu_k;
  p.total_q = pk.total_q;
  p.total_k = pk.total_k;
  p.nq = (Lq + Bq - 1) / Bq;
  p.nk = (Lk + Bk - 1) / Bk;
  p.n_pairs = (Lq + 255) / 256;
  p.chunk_pairs = fwd_chunk_pairs(p.n_pairs, p.G);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.log2_tau = tau > 0.f ? std::log2(tau) : 0.f;
  p.lse = lse;
  p.kept_tiles = kept_tiles;
  p.keep_map = keep_map;
  p.status = status;
  p.v_tiles = g_v_tiles.load();
  p.wait_ns = g_wait_ns.load();
  p.stall_tile = g_stall_tile.load();
  if (cudaMemsetAsync(kept_tiles, 0, sizeof(int32_t) * B * Hq, st) != cudaSuccess) return MALA_ERR_CUDA;
  const long long n8 = static_cast<long long>(tb) * tk * Hkv * d / 8;
  const int cv_grid = static_cast<int>(std::min<long long>((n8 + 255) / 256, 148LL * 16));
  mala::mala_v_to_f16_kernel<<<cv_grid, 256, 0, st>>>(static_cast<const uint4*>(v), static_cast<uint4*>(workspace),
                                                      n8, status);
  if (cudaGetLastError() != cudaSuccess) return MALA_ERR_CUDA;
  const int mode = tau > 0.f ? (prefetch_v ? 2 : 1) : 0;
  if (d == 128) return launch_fwd_tiles<128>(Bq, Bk, mode, mq, mk, mv, mo, p, st);
  return launch_fwd_tiles<64>(Bq, Bk, mode, mq, mk, mv, mo, p, st);
}
}  // namespace

int mala_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int L,
             int d, float scale, float tau, int Bq, int Bk, void* workspace, size_t workspace_bytes,
             int32_t* kept_tiles, uint8_t* keep_map, void* stream) {
  if (!q || !k || !v || !o || !lse || !kept_tiles) return MALA_ERR_INVALID_ARG;
  int rc = check_train_shape(B, Hq, Hkv, L, d, scale, tau, Bq, Bk);
  if (rc != MALA_OK) return rc;
  return run_fwd(q, k, v, o, lse, B, Hq, Hkv, L, L, d, scale, tau, Bq, Bk, workspace, workspace_bytes, kept_tiles,
                 keep_map, stream);
}

int mala_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int L,
                int d, float scale, float tau, int Bq, int Bk, void* workspace, size_t workspace_bytes,
                int32_t* kept_tiles, uint8_t* keep_map, void* stream, unsigned flags) {
  if (!q || !k || !v || !o || !lse || !kept_tiles) return MALA_ERR_INVALID_ARG;
  if (flags & ~MALA_FWD_PREFETCH_V) return MALA_ERR_INVALID_ARG;
  int rc = check_train_shape(B, Hq, Hkv, L, d, scale, tau, Bq, Bk);
  if (rc != MALA_OK) return rc;
  return run_fwd(q, k, v, o, lse, B, Hq, Hkv, L, L, d, scale, tau, Bq, Bk, workspace, workspace_bytes, kept_tiles,
                 keep_map, stream, Packed(), (flags & MALA_FWD_PREFETCH_V) != 0);
}

int mala_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int Lq,
                 int Lk, int d, float scale, float tau, int Bq, int Bk, void* workspace, size_t workspace_bytes,
                 int32_t* kept_tiles, uint8_t* keep_map, void* stream) {
  if (!q || !k || !v || !o || !lse || !kept_tiles) return MALA_ERR_INVALID_ARG;
  if (Lq < 1 || Lk < Lq) return MALA_ERR_INVALID_ARG;
  int rc = check_train_shape(B, Hq, Hkv, Lk, d, scale, tau, Bq, Bk);
  if (rc != MALA_OK) return rc;
  return run_fwd(q, k, v, o, lse, B, Hq, Hkv, Lq, Lk, d, scale, tau, Bq, Bk, workspace, workspace_bytes,
                 kept_tiles, keep_map, stream);
}

int mala_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* cu_seqlens_q,
                    const int32_t* cu_seqlens_k, int num_seqs, int max_seqlen_q, int max_seqlen_k, int total_q,
                    int total_k, int Hq, int Hkv, int d, float scale, float tau, int Bq, int Bk, void* workspace,
                    size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map, void* stream) {
  if (!q || !k || !v || !o || !lse || !kept_tiles || !cu_seqlens_q || !cu_seqlens_k) return MALA_ERR_INVALID_ARG;
  if (num_seqs < 1 || max_seqlen_q < 1 || max_seqlen_k < 1 || total_q < 1 || total_k < 1)
    return MALA_ERR_INVALID_ARG;
  if (max_seqlen_q > total_q || max_seqlen_k > total_k) return MALA_ERR_INVALID_ARG;
  int rc = check_train_shape(1, Hq, Hkv, std::max(total_q, total_k), d, scale, tau, Bq, Bk);
  if (rc != MALA_OK) return rc;
  if (static_cast<long long>(num_seqs) * Hq >= (1ll << 24)) return MALA_ERR_UNSUPPORTED;
  Packed pk;
  pk.cu_q = cu_seqlens_q;
  pk.cu_k = cu_seqlens_k;
  pk.total_q = total_q;
  pk.total_k = total_k;
  return run_fwd(q, k, v, o, lse, num_seqs, Hq, Hkv, max_seqlen_q, max_seqlen_k, d, scale, tau, Bq, Bk, workspace,
                 workspace_bytes, kept_tiles, keep_map, stream, pk);
}

size_t mala_bwd_workspace_size(int B, int Hq, int L, int d) {
  if (B < 1 || Hq < 1 || L < 1 || (d != 64 && d != 128)) return 0;
  return align256(static_cast<size_t>(B) * L * Hq * d * 4) + align256(static_cast<size_t>(B) * Hq * L * 4);
}

namespace {
// Backward; arguments already checked by the caller. For a packed batch, B
// counts the sequences and L is the longest length.
int run_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse, void* dq,
            void* dk, void* dv, int B, int Hq, int Hkv, int L, int d, float scale, float tau, int Bq, int Bk,
            void* workspace, size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map, void* stream,
            const Packed& pk = Packed()) {
  const void* ptrs[] = {q, k, v, o, dO, lse, dq, dk, dv};
  for (const void* x : ptrs)
    if (!aligned16(x)) return MALA_ERR_UNSUPPORTED;
  const bool packed = pk.cu_q != nullptr;
  const int tb = packed ? 1 : B, tl = packed ? pk.total_q : L;  // tensor extents [tb, tl, H, d]
  const size_t need = mala_bwd_workspace_size(tb, Hq, tl, d);
  if (!workspace || workspace_bytes < need || !aligned256(workspace)) return MALA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap mq, mk, mv, mdo, mdk, mdv;
  if (!make_bshd_map(&mq, q, tb, tl, Hq, d, 128) || !make_bshd_map(&mk, k, tb, tl, Hkv, d, 128) ||
      !make_bshd_map(&mv, v, tb, tl, Hkv, d, 128) || !make_bshd_map(&mdo, dO, tb, tl, Hq, d, 128) ||
      !make_bshd_map(&mdk, dk, tb, tl, Hkv, d, 128) || !make_bshd_map(&mdv, dv, tb, tl, Hkv, d, 128))
    return MALA_ERR_CUDA;
  unsigned* status = status_ptr();
  if (!status) return MALA_ERR_CUDA;
  float* dq_acc = static_cast<float*>(workspace);
  CUtensorMap mdq;
  if (!make_dq_acc_map(&mdq, dq_acc, tb, tl, Hq, d)) return MALA_ERR_CUDA;
  float* dvec = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                         align256(static_cast<size_t>(tb) * tl * Hq * d * 4));
  mala::BwdParams p;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.L = L; p.G = Hq / Hkv;
  p.nq = (L + Bq - 1) / Bq;
  p.nk = (L + Bk - 1) / Bk;
  p.n_super = (L + 127) / 128;
  p.chunk_kb = bwd_chunk_kb(p.n_super);
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.log2_tau = tau > 0.f ? std::log2(tau) : 0.f;
  p.lse = lse;
  p.dvec = dvec;
  p.dq_acc = dq_acc;
  p.cu = pk.cu_q;
  p.total = pk.total_q;
  p.dk_out = static_cast<uint16_t*>(dk);
  p.dv_out = static_cast<uint16_t*>(dv);
  p.kept_tiles = kept_tiles;
  p.keep_map = keep_map;
  p.status = status;
  p.wait_ns = g_wait_ns.load();
  p.stall_tile = g_stall_tile.load();

  const long long chunks = static_cast<long long>(tb) * tl * Hq * (d / 8);  // 16-byte chunks of O / dO
  const int pre_grid = static_cast<int>(std::min<long long>((chunks + 255) / 256, 148LL * 16));
  if (d == 128)
    mala::mala_bwd_pre_kernel<128><<<pre_grid, 256, 0, st>>>(static_cast<const uint4*>(o),
        static_cast<const uint4*>(dO), dvec, reinterpret_cast<float4*>(dq_acc), kept_tiles, B * Hq, tb, tl, Hq);
  else
    mala::mala_bwd_pre_kernel<64><<<pre_grid, 256, 0, st>>>(static_cast<const uint4*>(o),
        static_cast<const uint4*>(dO), dvec, reinterpret_cast<float4*>(dq_acc), kept_tiles, B * Hq, tb, tl, Hq);
  if (cudaGetLastError() != cudaSuccess) return MALA_ERR_CUDA;

  const bool gate = tau > 0.f;
  int rc;
  if (d == 128) rc = launch_bwd_tiles<128>(Bq, Bk, gate, mq, mk, mv, mdo, mdk, mdv, mdq, p, st);
  else rc = launch_bwd_tiles<64>(Bq, Bk, gate, mq, mk, mv, mdo, mdk, mdv, mdq, p, st);
  if (rc != MALA_OK) return rc;

  const long long n8 = static_cast<long long>(tb) * tl * Hq * d / 8;
  const int cv_grid = static_cast<int>(std::min<long long>((n8 + 255) / 256, 148LL * 16));
  mala::mala_dq_convert_kernel<<<cv_grid, 256, 0, st>>>(reinterpret_cast<const float4*>(dq_acc),
                                                         static_cast<uint4*>(dq), n8);
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}
}  // namespace

int mala_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
             void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int L, int d, float scale, float tau, int Bq,
             int Bk, void* workspace, size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map,
             void* stream) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv || !kept_tiles) return MALA_ERR_INVALID_ARG;
  int rc = check_train_shape(B, Hq, Hkv, L, d, scale, tau, Bq, Bk);
  if (rc != MALA_OK) return rc;
  return run_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, L, d, scale, tau, Bq, Bk, workspace,
                 workspace_bytes, kept_tiles, keep_map, stream);
}

int mala_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                    void* dq, void* dk, void* dv, const int32_t* cu_seqlens, int num_seqs, int max_seqlen,
                    int total, int Hq, int Hkv, int d, float scale, float tau, int Bq, int Bk, void* workspace,
                    size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map, void* stream) {
  if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv || !kept_tiles || !cu_seqlens)
    return MALA_ERR_INVALID_ARG;
  if (num_seqs < 1 || max_seqlen < 1 || total < 1 || max_seqlen > total) return MALA_ERR_INVALID_ARG;
  int rc = check_train_shape(1, Hq, Hkv, total, d, scale, tau, Bq, Bk);
  if (rc != MALA_OK) return rc;
  if (static_cast<long long>(num_seqs) * Hq >= (1ll << 24)) return MALA_ERR_UNSUPPORTED;
  Packed pk;
  pk.cu_q = pk.cu_k = cu_seqlens;
  pk.total_q = pk.total_k = total;
  return run_bwd(q, k, v, o, dO, lse, dq, dk, dv, num_seqs, Hq, Hkv, max_seqlen, d, scale, tau, Bq, Bk,
                 workspace, workspace_bytes, kept_tiles, keep_map, stream, pk);
}

size_t mala_decode_workspace_size(int B, int Hq, int d, int n_splits) {
  if (B < 1 || Hq < 1 || n_splits < 1 || (d != 64 && d != 128)) return 0;
  const size_t parts = static_cast<size_t>(B) * Hq * n_splits;
  return align256(parts * d * 4) + align256(parts * 4);
}

int mala_decode_default_splits(int B, int Hkv, int Lk, int Bk) {
  if (B < 1 || Hkv < 1 || Lk < 1 || Bk < 1) return 1;
  int sms = 0, dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
    sms = 148;
  const long long nk = (static_cast<long long>(Lk) + Bk - 1) / Bk;
  const long long units = static_cast<long long>(B) * Hkv;
  // One decode CTA fills an SM. Pick the split count whose grid takes between
  // 2 and 8 waves with the fullest last wave, with a small charge per wave
  // (every CTA pays a pipeline ramp and forces its split's newest tile).
  long long best = 1;
  double best_eff = -1.0;
  for (long long s = 1; s <= std::min(nk, 65535LL); ++s) {
    const long long per = (nk + s - 1) / s;
    if ((nk + per - 1) / per != s) continue;  // every split non-empty
    const double waves = static_cast<double>(units * s) / sms;
    if (waves > 8.0) break;
    const double eff = waves / std::ceil(waves);
    const bool enough = waves >= 2.0;
    const double score = eff + (enough ? 1.0 : 0.0) - 0.01 * waves;  // each wave costs a pipeline ramp
    if (score > best_eff + 1e-9) {
      best_eff = score;
      best = s;
    }
  }
  return static_cast<int>(best);
}

namespace {
// Paged KV cache for decode (null block_table: a contiguous cache).
struct Paged {
  const int* seqlens = nullptr;
  const int* block_table = nullptr;
  int max_pages = 0, num_pages = 0;
};

int check_decode_args(const void* q, const void* kc, const void* vc, const void* o, const float* lse, int B,
                      int Hq, int Hkv, int Lk, int d, float scale, float tau, int Bk, int n_splits,
                      const int32_t* kept_tiles) {
  if (!q || !kc || !vc || !o || !lse || !kept_tiles) return MALA_ERR_INVALID_ARG;
  if (B < 1 || Hq < 1 || Hkv < 1 || Lk < 1 || Hq % Hkv != 0 || n_splits < 0) return MALA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale) || !(tau >= 0.f) || !std::isfinite(tau)) return MALA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || (Bk != 64 && Bk != 128)) return MALA_ERR_UNSUPPORTED;
  if (Hq / Hkv > mala::kDecMaxG) return MALA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Lk * Hkv * d >= (1ll << 40)) return MALA_ERR_UNSUPPORTED;
  const void* ptrs[] = {q, kc, vc, o, lse};
  for (const void* x : ptrs)
    if (!aligned16(x)) return MALA_ERR_UNSUPPORTED;
  return MALA_OK;
}

// Split kernel + combine into caller-provided partials (parts_base: o partials,
// then the LSE partials 256 bytes aligned). Lk is the longest sequence's length.
int run_decode(const void* q, const CUtensorMap& mk, const CUtensorMap& mv, void* o, float* lse, int B, int Hq,
               int Hkv, int Lk, int d, float scale, float tau, int Bk, int n_splits, void* parts_base,
               int32_t* kept_tiles, uint8_t* keep_map, cudaStream_t st, const Paged& pg = Paged()) {
  unsigned* status = status_ptr();
  if (!status) return MALA_ERR_CUDA;
  const size_t parts = static_cast<size_t>(B) * Hq * n_splits;
  mala::DecParams p;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.Lk = Lk; p.G = Hq / Hkv;
  p.nk = (Lk + Bk - 1) / Bk;
  p.n_splits = n_splits;
  p.tiles_per_split = (p.nk + n_splits - 1) / n_splits;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.thr = tau > 0.f ? std::log2(tau) - std::log2(static_cast<float>(Lk)) : 0.f;
  p.log2_tau = tau > 0.f ? std::log2(tau) : 0.f;
  p.seqlens = pg.seqlens;
  p.block_table = pg.block_table;
  p.max_pages = pg.max_pages;
  p.num_pages = pg.num_pages;
  p.q = static_cast<const uint16_t*>(q);
  p.o_part = static_cast<float*>(parts_base);
  p.lse_part = reinterpret_cast<float*>(static_cast<char*>(parts_base) + align256(parts * d * 4));
  p.kept_tiles = kept_tiles;
  p.keep_map = keep_map;
  p.status = status;
  p.wait_ns = g_wait_ns.load();
  p.stall_tile = g_stall_tile.load();
  if (cudaMemsetAsync(kept_tiles, 0, sizeof(int32_t) * B * Hq, st) != cudaSuccess) return MALA_ERR_CUDA;
  const bool gate = tau > 0.f;
  int rc;
  if (d == 128 && Bk == 128) rc = launch_dec_gate<128, 128>(gate, mk, mv, p, st);
  else if (d == 64 && Bk == 128) rc = launch_dec_gate<64, 128>(gate, mk, mv, p, st);
  else if (d == 128 && Bk == 64) rc = launch_dec_gate<128, 64>(gate, mk, mv, p, st);
  else rc = launch_dec_gate<64, 64>(gate, mk, mv, p, st);
  if (rc != MALA_OK) return rc;
  const int rows = B * Hq;
  if (d == 128)
    mala::mala_decode_combine_kernel<128><<<(rows + 3) / 4, 128, 0, st>>>(p.o_part, p.lse_part,
                                                                         static_cast<uint16_t*>(o), lse, rows,
                                                                         n_splits);
  else
    mala::mala_decode_combine_kernel<64><<<(rows + 3) / 4, 128, 0, st>>>(p.o_part, p.lse_part,
                                                                        static_cast<uint16_t*>(o), lse, rows,
                                                                        n_splits);
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}
}  // namespace

int mala_decode(const void* q, const void* kcache, const void* vcache, void* o, float* lse, int B, int Hq,
                int Hkv, int Lk, int d, float scale, float tau, int Bk, int n_splits, void* workspace,
                size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map, void* stream) {
  int rc = check_decode_args(q, kcache, vcache, o, lse, B, Hq, Hkv, Lk, d, scale, tau, Bk, n_splits, kept_tiles);
  if (rc != MALA_OK) return rc;
  if (n_splits == 0) n_splits = mala_decode_default_splits(B, Hkv, Lk, Bk);
  if (n_splits > 65535) return MALA_ERR_UNSUPPORTED;
  const size_t need = mala_decode_workspace_size(B, Hq, d, n_splits);
  if (!workspace || workspace_bytes < need || !aligned256(workspace)) return MALA_ERR_WORKSPACE;
  CUtensorMap mk, mv;
  if (!make_bshd_map(&mk, kcache, B, Lk, Hkv, d, Bk) || !make_bshd_map(&mv, vcache, B, Lk, Hkv, d, Bk))
    return MALA_ERR_CUDA;
  return run_decode(q, mk, mv, o, lse, B, Hq, Hkv, Lk, d, scale, tau, Bk, n_splits, workspace, kept_tiles,
                    keep_map, static_cast<cudaStream_t>(stream));
}

int mala_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                      const int32_t* seqlens_k, void* o, float* lse, int B, int Hq, int Hkv, int num_pages,
                      int page_size, int max_pages_per_seq, int d, float scale, float tau, int n_splits,
                      void* workspace, size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map,
                      void* stream) {
  if (!block_table || !seqlens_k || num_pages < 1 || max_pages_per_seq < 1) return MALA_ERR_INVALID_ARG;
  if (page_size != 64 && page_size != 128) return MALA_ERR_UNSUPPORTED;
  const long long max_lk = static_cast<long long>(max_pages_per_seq) * page_size;
  if (max_lk >= (1ll << 31) || static_cast<long long>(num_pages) * page_size >= (1ll << 31))
    return MALA_ERR_UNSUPPORTED;
  int rc = check_decode_args(q, k_pages, v_pages, o, lse, B, Hq, Hkv, static_cast<int>(max_lk), d, scale, tau,
                             page_size, n_splits, kept_tiles);
  if (rc != MALA_OK) return rc;
  if (static_cast<long long>(num_pages) * page_size * Hkv * d >= (1ll << 40)) return MALA_ERR_UNSUPPORTED;
  if (n_splits == 0) n_splits = mala_decode_default_splits(B, Hkv, static_cast<int>(max_lk), page_size);
  if (n_splits > 65535) return MALA_ERR_UNSUPPORTED;
  const size_t need = mala_decode_workspace_size(B, Hq, d, n_splits);
  if (!workspace || workspace_bytes < need || !aligned256(workspace)) return MALA_ERR_WORKSPACE;
  CUtensorMap mk, mv;  // the pools as [num_pages, page, Hkv, d]: one page per tile
  if (!make_bshd_map(&mk, k_pages, num_pages, page_size, Hkv, d, page_size) ||
      !make_bshd_map(&mv, v_pages, num_pages, page_size, Hkv, d, page_size))
    return MALA_ERR_CUDA;
  Paged pg;
  pg.seqlens = seqlens_k;
  pg.block_table = block_table;
  pg.max_pages = max_pages_per_seq;
  pg.num_pages = num_pages;
  return run_decode(q, mk, mv, o, lse, B, Hq, Hkv, static_cast<int>(max_lk), d, scale, tau, page_size, n_splits,
                    workspace, kept_tiles, keep_map, static_cast<cudaStream_t>(stream), pg);
}

namespace {
struct DxWorkspace {
  size_t scores, tile_ml, keep, o_part, lse_part, total;
};

DxWorkspace dx_layout(int B, int Hq, int Lk, int d, int Bk, int n_splits) {
  DxWorkspace w;
  const size_t nk = (static_cast<size_t>(Lk) + Bk - 1) / Bk;
  const size_t rows = static_cast<size_t>(B) * Hq;
  w.scores = 0;
  w.tile_ml = w.scores + align256(rows * nk * Bk * 4);
  w.keep = w.tile_ml + align256(rows * nk * 8);
  w.o_part = w.keep + align256(rows * nk);
  w.lse_part = w.o_part + align256(rows * n_splits * d * 4);
  w.total = w.lse_part + align256(rows * n_splits * 4);
  return w;
}
}  // namespace

size_t mala_decode_exact_workspace_size(int B, int Hq, int Lk, int d, int Bk, int n_splits) {
  if (B < 1 || Hq < 1 || Lk < 1 || n_splits < 1 || (d != 64 && d != 128) || (Bk != 64 && Bk != 128)) return 0;
  return dx_layout(B, Hq, Lk, d, Bk, n_splits).total;
}

int mala_decode_exact(const void* q, const void* kcache, const void* vcache, void* o, float* lse, int B, int Hq,
                      int Hkv, int Lk, int d, float scale, float tau, int Bk, int n_splits, void* workspace,
                      size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map, void* stream) {
  int rc = check_decode_args(q, kcache, vcache, o, lse, B, Hq, Hkv, Lk, d, scale, tau, Bk, n_splits, kept_tiles);
  if (rc != MALA_OK) return rc;
  if (n_splits == 0) n_splits = mala_decode_default_splits(B, Hkv, Lk, Bk);
  if (n_splits > 65535) return MALA_ERR_UNSUPPORTED;
  const DxWorkspace lay = dx_layout(B, Hq, Lk, d, Bk, n_splits);
  if (!workspace || workspace_bytes < lay.total || !aligned256(workspace)) return MALA_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  mala::DxParams p;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv; p.Lk = Lk;
  p.nk = (Lk + Bk - 1) / Bk;
  p.n_splits = n_splits;
  p.tiles_per_split = (p.nk + n_splits - 1) / n_splits;
  p.Lkp = p.nk * Bk;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.gate = tau > 0.f ? 1 : 0;
  p.thr = tau > 0.f ? std::log2(tau) - std::log2(static_cast<float>(Lk)) : 0.f;
  p.q = static_cast<const uint16_t*>(q);
  p.kc = static_cast<const uint16_t*>(kcache);
  p.vc = static_cast<const uint16_t*>(vcache);
  p.scores = reinterpret_cast<float*>(ws + lay.scores);
  p.tile_ml = reinterpret_cast<float2*>(ws + lay.tile_ml);
  p.keep = reinterpret_cast<uint8_t*>(ws + lay.keep);
  p.o_part = reinterpret_cast<float*>(ws + lay.o_part);
  p.lse_part = reinterpret_cast<float*>(ws + lay.lse_part);
  p.kept_tiles = kept_tiles;
  p.keep_map = keep_map;
  p.o_out = o;
  p.lse_out = lse;
  unsigned* status = status_ptr();
  if (!status) return MALA_ERR_CUDA;
  p.status = status;
  p.wait_ns = g_wait_ns.load();
  CUtensorMap mv;
  if (!make_bshd_map(&mv, vcache, B, Lk, Hkv, d, Bk)) return MALA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 128 && Bk == 128) return launch_dx_g<128, 128>(mv, p, st);
  if (d == 64 && Bk == 128) return launch_dx_g<64, 128>(mv, p, st);
  if (d == 128 && Bk == 64) return launch_dx_g<128, 64>(mv, p, st);
  return launch_dx_g<64, 64>(mv, p, st);
}

int mala_test_hooks(unsigned long long wait_limit_ns, int stall_tile, unsigned long long* fwd_v_tiles) {
  if (stall_tile < -1) return MALA_ERR_INVALID_ARG;
  g_wait_ns.store(wait_limit_ns == 0 ? mala::kWaitLimitNs : wait_limit_ns);
  g_stall_tile.store(stall_tile);
  g_v_tiles.store(fwd_v_tiles);
  return MALA_OK;
}

int mala_check_status(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return MALA_ERR_CUDA;
  unsigned int h = 0;
  if (cudaMemcpyFromSymbol(&h, g_mala_status, sizeof(h)) != cudaSuccess) return MALA_ERR_CUDA;
  if (h != 0) {
    const unsigned int zero = 0;
    if (cudaMemcpyToSymbol(g_mala_status, &zero, sizeof(zero)) != cudaSuccess) return MALA_ERR_CUDA;
    if (h & mala::kStatusTimeout) return MALA_ERR_DEVICE_TIMEOUT;
    return (h & mala::kStatusSeqTable) ? MALA_ERR_INVALID_ARG : MALA_ERR_RANGE;
  }
  return MALA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free decode.
//
// mala_decode_noalloc is mala_decode for callers that cannot allocate device
// memory: for example a plugin running inside a host engine that owns all
// device memory and offers it no allocator, or a serving loop that cannot
// afford the device-wide synchronisation a cudaMalloc may bring. Instead of
// a caller-provided workspace it uses the file-scope array below, which every
// GPU that loads this library holds until the process exits. The call itself
// allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
//
// The array's name is only a host-side stand-in in host code; its device
// address is looked up with cudaGetSymbolAddress the first time the entry
// point runs on a device (with that device current) and cached per device,
// together with the unique id of the CUDA context it was looked up in. A
// call that finds another context current (after cudaDeviceReset, say, the
// library's module lives in a new primary context) looks the address up
// again. The first call on a device, and the first after such a reset, should
// therefore come before any stream capture.
//
// All calls share the array and it keeps the last call's contents. Every
// call overwrites all of the split partials it reads (empty splits included),
// so nothing has to be cleared between calls; calls whose execution overlaps
// on the GPU race on the array and must be serialised by the caller.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(8) << 20;  // 8 MiB
__device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
struct ScratchAddr {
  unsigned long long ctx_id = 0;  // 0: nothing cached
  void* ptr = nullptr;
};
ScratchAddr g_scratch_addr[kMaxDevices];

// Unique id of the current CUDA context (driver entry points fetched at run
// time, as for the tensor maps); false if there is none or the driver lacks
// the calls.
bool current_context_id(unsigned long long* id) {
  using GetCurrentFn = CUresult (*)(CUcontext*);
  using GetIdFn = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr)
    return false;
  return get_id(ctx, id) == CUDA_SUCCESS && *id != 0;
}

// Device address of g_decode_scratch on the current device (set-up on first
// use in each context).
void* decode_scratch_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  unsigned long long id = 0;
  ScratchAddr& e = g_scratch_addr[dev];
  if (e.ptr != nullptr && current_context_id(&id) && id == e.ctx_id) return e.ptr;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) return nullptr;
  // the look-up has made the device's context current if it was not; without
  // a context id the address is not cached and is looked up on every call
  e.ctx_id = current_context_id(&id) ? id : 0;
  e.ptr = e.ctx_id != 0 ? p : nullptr;
  return p;
}

}  // namespace

extern "C" {

size_t mala_decode_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

int mala_decode_noalloc(const void* q, const void* kcache, const void* vcache, void* o, float* lse, int B, int Hq,
                        int Hkv, int Lk, int d, float scale, float tau, int Bk, int n_splits, int32_t* kept_tiles,
                        uint8_t* keep_map, void* stream) {
  int rc = check_decode_args(q, kcache, vcache, o, lse, B, Hq, Hkv, Lk, d, scale, tau, Bk, n_splits, kept_tiles);
  if (rc != MALA_OK) return rc;
  if (n_splits == 0) n_splits = mala_decode_default_splits(B, Hkv, Lk, Bk);
  if (n_splits > 65535) return MALA_ERR_UNSUPPORTED;
  const size_t need = mala_decode_workspace_size(B, Hq, d, n_splits);
  if (need == 0 || need > kNoAllocScratchBytes) return MALA_ERR_WORKSPACE;  // beyond the fixed scratch
  void* scratch = decode_scratch_current_device();
  if (scratch == nullptr) return MALA_ERR_CUDA;
  CUtensorMap mk, mv;
  if (!make_bshd_map(&mk, kcache, B, Lk, Hkv, d, Bk) || !make_bshd_map(&mv, vcache, B, Lk, Hkv, d, Bk))
    return MALA_ERR_CUDA;
  return run_decode(q, mk, mv, o, lse, B, Hq, Hkv, Lk, d, scale, tau, Bk, n_splits, scratch, kept_tiles, keep_map,
                    static_cast<cudaStream_t>(stream));
}

}  // extern "C"
