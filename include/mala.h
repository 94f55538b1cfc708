/*
 * mala.h -- C ABI of the B200 (sm_100a) MALA attention library.
 *
 * MALA (MassAlloc Attention) is causal softmax attention that scores every
 * legal causal QK tile but skips a tile's post-score work when the tile's
 * largest per-key contribution ratio falls below tau/Lq, Lq = i + 1 being the
 * number of causally visible keys of query row i (agihunt.info, "MassAlloc
 * Attention: Let Attention Allocate Its Own Compute", method paragraphs;
 * arXiv 2609.32712 abstract on aihot.vn).
 *
 * Conventions shared by every call:
 *   - All tensor arguments are DEVICE pointers to caller-owned, contiguous
 *     memory on the current CUDA device. Every pointer must be 16-byte
 *     aligned. The library never allocates device memory.
 *   - bf16 tensors are passed as void* holding bfloat16 bit patterns.
 *   - Layouts are BSHD: q, o, dO, dq [B, L, Hq, d]; k, v, dk, dv
 *     [B, L, Hkv, d]; lse [B, Hq, L] fp32 in natural-log units.
 *   - Tiles: nq = ceil(L / Bq) query blocks, nk = ceil(L / Bk) key blocks;
 *     tile (qb, kb) is legal iff kb*Bk <= min((qb+1)*Bq, L) - 1.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream). Arguments are validated on
 *     the host before anything is enqueued: on any error return nothing is
 *     written and nothing is launched.
 *   - GQA: query head hq reads KV head hq / (Hq / Hkv).
 *   - Supported: d in {64, 128}; Bq and Bk each in {64, 128} (independently);
 *     any L >= 1 (a ragged last tile is fine); B, Hq, Hkv >= 1 with
 *     Hq % Hkv == 0.
 *   - Device-side waits are bounded. If one expires the kernel records
 *     MALA_ERR_DEVICE_TIMEOUT in a device status word and returns;
 *     mala_check_status() reports it.
 *   - Calls are not reentrant with respect to the same output buffers.
 */
#ifndef MALA_H_
#define MALA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MALA_ABI_VERSION 1

#if defined(__GNUC__)
#define MALA_API __attribute__((visibility("default")))
#else
#define MALA_API
#endif

typedef enum mala_status {
    MALA_OK = 0,
    MALA_ERR_INVALID_ARG = 1,    /* null pointer, Hq % Hkv != 0, L < 1, scale <= 0, tau < 0, NaN;
                                    also a bad device-side sequence or page table (mala_check_status) */
    MALA_ERR_UNSUPPORTED = 2,    /* d, Bq, Bk outside the supported set; pointer not 16-B aligned */
    MALA_ERR_WORKSPACE = 3,      /* workspace missing or smaller than the size query returns */
    MALA_ERR_CUDA = 4,           /* a CUDA runtime / driver call or a launch failed */
    MALA_ERR_DEVICE_TIMEOUT = 5, /* a bounded device-side wait expired (see mala_check_status) */
    MALA_ERR_RANGE = 6           /* a V value lay outside the fp16 range and was clamped (mala_check_status) */
} mala_status_t;

/* Human-readable name of a status code (static string, never NULL). */
MALA_API const char* mala_status_string(int status);

/* MALA_ABI_VERSION of the loaded library. */
MALA_API int mala_abi_version(void);

/*
 * mala_fwd -- MALA forward (training / prefill of a whole sequence).
 *
 * Source: agihunt.info MALA digest, method paragraphs (forward gate against
 * the running online-softmax state, conservative per query block, visit
 * order from the diagonal back, forced first tile, LSE as the saved state).
 *
 * For every (b, hq, qb), key blocks kb run from the last legal one down to 0.
 * Every legal tile is scored, S = scale * Q K^T (bf16 in, fp32 accumulate).
 * With (m_r, l_r) the online-softmax state over previously kept tiles, the
 * tile is kept iff it is the block's first legal tile, or tau == 0, or some
 * row r with a live key satisfies
 *     max_live_j exp(s_rj - m_r) / l_r >= tau / (i_r + 1)      (ties keep).
 * A kept tile updates (m, l) and O for every row of the block; a skipped
 * tile does no V load, no softmax update and no PV: with tau > 0 the V tile
 * is requested only after a query block's vote has kept it. The PV product runs in
 * fp16 on an fp16 copy of V made by the call in `workspace`; V values must lie
 * inside the fp16 range (|v| <= 65504); larger ones are clamped and reported
 * as MALA_ERR_RANGE by mala_check_status.
 *
 *   q        [B, L, Hq, d]  bf16, in
 *   k, v     [B, L, Hkv, d] bf16, in
 *   o        [B, L, Hq, d]  bf16, out: O_i = acc_i / l_i
 *   lse      [B, Hq, L]     fp32, out: LSE_i = m_i + ln l_i (natural log)
 *   scale    > 0 (usually 1/sqrt(d)); tau >= 0 (tau = 0: full attention)
 *   workspace  device scratch of >= mala_fwd_workspace_size(B, Hkv, L, d)
 *              bytes, 256-byte aligned, caller-owned; contents on entry ignored
 *   kept_tiles [B*Hq] int32, out (required): kept tiles per (b, hq); zeroed
 *            by the call on `stream` before the kernel accumulates into it
 *   keep_map   [B, Hq, nq, nk] uint8, out, nullable (test/debug only): 1 for
 *            a kept tile, 0 for a skipped legal tile; entries of illegal
 *            tiles are not written. The method itself never reads it.
 */
MALA_API int mala_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int L, int d, float scale, float tau, int Bq, int Bk, void* workspace,
             size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map, void* stream);

/*
 * mala_fwd_ex -- mala_fwd with option flags (flags = 0 is exactly mala_fwd).
 *
 *   MALA_FWD_PREFETCH_V  fetch the V tile of every legal key tile ahead of
 *            the gate's decision instead of only after a query block has
 *            voted to keep it. The keep/skip decisions, O, LSE, kept_tiles
 *            and keep_map are the same as without the flag; a skipped tile
 *            still gets no softmax update and no PV, but its V tile is read
 *            (the digest's method paragraphs list the V load among the work a
 *            skip saves, so this is a departure from the method's cost model,
 *            offered because no PV then waits for a V load requested after a
 *            vote). Without tau > 0 the flag changes nothing.
 * Errors: as mala_fwd; MALA_ERR_INVALID_ARG also for an unknown flag bit.
 */
#define MALA_FWD_PREFETCH_V 1u
MALA_API int mala_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int L, int d, float scale, float tau, int Bq, int Bk, void* workspace,
             size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map, void* stream, unsigned flags);

/*
 * Workspace bytes mala_fwd needs: the fp16 copy of V [B, L, Hkv, d] the PV
 * product reads (256-byte aligned). Returns 0 for invalid sizes. mala_prefill
 * needs mala_fwd_workspace_size(B, Hkv, Lk, d).
 */
MALA_API size_t mala_fwd_workspace_size(int B, int Hkv, int L, int d);

/*
 * mala_prefill -- MALA forward of Lq new queries against Lk >= Lq keys (a
 * prompt chunk appended to an existing KV cache).
 *
 * Source: agihunt.info MALA digest, method paragraphs (the forward gate, with
 * Lq the number of keys the query sees) and limitations paragraph (the KV
 * cache is kept whole; one tau for training and serving).
 *
 * The new queries sit at the end of the sequence: query row i (0 <= i < Lq)
 * is at position P0 + i with P0 = Lk - Lq, sees keys 0 .. P0 + i and uses the
 * threshold tau / (P0 + i + 1). Query blocks are cut from the first new
 * query (block qb = rows [qb*Bq, min((qb+1)*Bq, Lq))); key blocks from key 0.
 * Tile (qb, kb) is legal iff kb*Bk <= P0 + min((qb+1)*Bq, Lq) - 1, and the
 * block's first legal tile is the one holding that key. Everything else
 * (visit order, forced first tile, the gate, LSE) is as in mala_fwd; with
 * Lq == Lk the call computes exactly what mala_fwd does.
 *
 *   q          [B, Lq, Hq, d]  bf16, in
 *   k, v       [B, Lk, Hkv, d] bf16, in (the cache with the new keys at the end)
 *   o          [B, Lq, Hq, d]  bf16, out
 *   lse        [B, Hq, Lq]     fp32, out (natural log)
 *   Lq >= 1, Lk >= Lq; other arguments as for mala_fwd, with nq = ceil(Lq/Bq),
 *   nk = ceil(Lk/Bk) for keep_map [B, Hq, nq, nk]
 *   workspace  >= mala_fwd_workspace_size(B, Hkv, Lk, d) bytes
 * Errors: MALA_ERR_INVALID_ARG also for Lq < 1 or Lk < Lq.
 */
MALA_API int mala_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Lq, int Lk, int d, float scale, float tau, int Bq, int Bk, void* workspace,
             size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map, void* stream);

/*
 * mala_fwd_varlen -- MALA forward of a packed batch of variable-length
 * sequences (training, or prefill of several prompts against their caches).
 *
 * Source: as mala_fwd / mala_prefill; a packed batch is independent sequences
 * laid end to end (the gate never looks across a sequence).
 *
 * Sequence s (0 <= s < num_seqs) owns query rows cu_seqlens_q[s] ..
 * cu_seqlens_q[s+1] - 1 of q / o and key rows cu_seqlens_k[s] ..
 * cu_seqlens_k[s+1] - 1 of k / v; with Lq_s and Lk_s its lengths (Lk_s >= Lq_s,
 * Lq_s may be 0) it is exactly mala_prefill(Lq = Lq_s, Lk = Lk_s).
 *
 *   q, o       [total_q, Hq, d]  bf16 (in / out)
 *   k, v       [total_k, Hkv, d] bf16, in
 *   lse        [Hq, total_q]     fp32, out (natural log)
 *   cu_seqlens_q, cu_seqlens_k  [num_seqs + 1] int32, DEVICE memory, in:
 *              non-decreasing offsets starting at 0, ending at total_q / total_k
 *   max_seqlen_q, max_seqlen_k  bounds on Lq_s and Lk_s (they size the grid and keep_map)
 *   workspace  >= mala_fwd_workspace_size(1, Hkv, total_k, d) bytes
 *   kept_tiles [num_seqs * Hq] int32, out (required)
 *   keep_map   [num_seqs, Hq, ceil(max_seqlen_q / Bq), ceil(max_seqlen_k / Bk)] uint8,
 *              nullable; per sequence its legal tiles are written, the rest untouched
 * The sequence tables live on the device and are checked there: a sequence
 * whose entries are out of range (offsets outside the tensors, Lk_s < Lq_s, or
 * a length above the stated maximum) is left untouched and mala_check_status
 * returns MALA_ERR_INVALID_ARG.
 */
MALA_API int mala_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
             const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int num_seqs, int max_seqlen_q,
             int max_seqlen_k, int total_q, int total_k, int Hq, int Hkv, int d, float scale, float tau,
             int Bq, int Bk, void* workspace, size_t workspace_bytes, int32_t* kept_tiles,
             uint8_t* keep_map, void* stream);

/*
 * Workspace bytes mala_bwd needs: an fp32 dQ accumulator [B, L, Hq, d] and
 * an fp32 D = rowsum(dO * O) vector [B, Hq, L], each 256-byte aligned.
 * Returns 0 for invalid sizes.
 */
MALA_API size_t mala_bwd_workspace_size(int B, int Hq, int L, int d);

/*
 * mala_bwd -- MALA backward.
 *
 * Source: agihunt.info MALA digest, method paragraphs (backward gate against
 * the final normaliser, nested support without a stored mask, approximate
 * rather than exact gradient).
 *
 * Scores are recomputed on every legal tile. A tile is kept iff tau == 0 or
 * some live (i, j) has exp(s_ij - LSE_i) >= tau / (i + 1); no tile is forced.
 * With D_i = <dO_i, O_i>, a kept tile computes for its live entries
 *   P = exp(s - LSE), dP = dO V^T, dS = P * (dP - D),
 *   dV += P^T dO, dK += scale * dS^T Q, dQ += scale * dS K;
 * a skipped tile does none of these. dK / dV sum over the GQA group.
 *
 *   q, o, dO   [B, L, Hq, d]  bf16, in (o and lse as written by mala_fwd)
 *   k, v       [B, L, Hkv, d] bf16, in
 *   lse        [B, Hq, L]     fp32, in
 *   dq         [B, L, Hq, d]  bf16, out
 *   dk, dv     [B, L, Hkv, d] bf16, out
 *   workspace  device scratch of >= mala_bwd_workspace_size(B, Hq, L, d)
 *              bytes, 256-byte aligned, caller-owned; contents on entry are
 *              ignored (the call clears what it uses)
 *   kept_tiles [B*Hq] int32, out (required): backward-kept tiles per (b, hq)
 *   keep_map   [B, Hq, nq, nk] uint8, out, nullable: as for mala_fwd
 */
MALA_API int mala_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
             const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int L, int d,
             float scale, float tau, int Bq, int Bk, void* workspace, size_t workspace_bytes,
             int32_t* kept_tiles, uint8_t* keep_map, void* stream);

/*
 * mala_bwd_varlen -- MALA backward of a packed training batch (the queries and
 * keys of sequence s are rows cu_seqlens[s] .. cu_seqlens[s+1] - 1).
 *
 * Source: as mala_bwd, per sequence.
 *
 *   q, o, dO, dq  [total, Hq, d]  bf16; k, v, dk, dv [total, Hkv, d] bf16
 *   lse           [Hq, total] fp32, as mala_fwd_varlen writes it
 *   cu_seqlens    [num_seqs + 1] int32, DEVICE memory; max_seqlen bounds every length
 *   workspace     >= mala_bwd_workspace_size(1, Hq, total, d) bytes
 *   kept_tiles    [num_seqs * Hq] int32, out; keep_map [num_seqs, Hq,
 *                 ceil(max_seqlen / Bq), ceil(max_seqlen / Bk)] uint8, nullable
 * Invalid sequence entries are handled as in mala_fwd_varlen.
 */
MALA_API int mala_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dO,
             const float* lse, void* dq, void* dk, void* dv, const int32_t* cu_seqlens, int num_seqs,
             int max_seqlen, int total, int Hq, int Hkv, int d, float scale, float tau, int Bq, int Bk,
             void* workspace, size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map,
             void* stream);

/*
 * Workspace bytes mala_decode needs for n_splits partial results:
 * fp32 O partials [B, Hq, n_splits, d] and fp32 LSE partials
 * [B, Hq, n_splits], each 256-byte aligned. Returns 0 for invalid sizes.
 */
MALA_API size_t mala_decode_workspace_size(int B, int Hq, int d, int n_splits);

/*
 * Deterministic split count mala_decode uses when n_splits == 0: enough
 * (b, KV head, split) work units to fill the GPU's SMs, at least one tile per
 * split. Depends only on its arguments and the current device's SM count.
 */
MALA_API int mala_decode_default_splits(int B, int Hkv, int Lk, int Bk);

/*
 * mala_decode -- one new query per sequence against a KV cache of Lk keys.
 *
 * Source: agihunt.info MALA digest, method and limitations paragraphs (one
 * tau for training and serving, the KV cache kept whole, decode speed limited
 * by cache reads).
 *
 * The query is row i = Lk - 1, so every key is visible and Lq = Lk. The nk =
 * ceil(Lk / Bk) key tiles are cut into contiguous splits of
 * T = ceil(nk / n_splits) tiles (split s covers [s*T, min((s+1)*T, nk))).
 * Each split runs the forward gate with its own fresh state from its newest
 * tile to its oldest, always keeping its newest tile; the partial results
 * are merged by their LSEs: LSE = log sum_s exp(LSE_s),
 * O = sum_s exp(LSE_s - LSE) O_s. V of a tile is loaded only if some query
 * head of the GQA group keeps it.
 *
 *   q          [B, Hq, d]       bf16, in
 *   kcache, vcache [B, Lk, Hkv, d] bf16, in
 *   o          [B, Hq, d]       bf16, out
 *   lse        [B, Hq]          fp32, out (natural log)
 *   n_splits   >= 1, or 0 for mala_decode_default_splits(B, Hkv, Lk, Bk)
 *   workspace  >= mala_decode_workspace_size(B, Hq, d, n_splits used) bytes
 *   kept_tiles [B*Hq] int32, out (required): tiles whose PV ran per (b, hq)
 *   keep_map   [B, Hq, nk] uint8, out, nullable
 */
MALA_API int mala_decode(const void* q, const void* kcache, const void* vcache, void* o, float* lse, int B,
                int Hq, int Hkv, int Lk, int d, float scale, float tau, int Bk, int n_splits,
                void* workspace, size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map,
                void* stream);

/*
 * Workspace bytes mala_decode_exact needs: fp32 scores [B, Hq, nk * Bk], per
 * tile (max, log-sum) pairs [B, Hq, nk], decisions [B, Hq, nk] and the split
 * partials of mala_decode_workspace_size, each 256-byte aligned. 0 for
 * invalid sizes.
 */
MALA_API size_t mala_decode_exact_workspace_size(int B, int Hq, int Lk, int d, int Bk, int n_splits);

/*
 * mala_decode_exact -- decode whose decisions do not depend on the split.
 *
 * Source: agihunt.info MALA digest, method paragraphs (the forward gate: tiles
 * from the newest to the oldest against the state over the kept tiles, the
 * first tile kept).
 *
 * The decisions are those of ONE sequential pass over all nk tiles (exactly
 * mala_decode with n_splits = 1, i.e. the forward's last query row): tile t
 * is kept iff it is the newest, or tau == 0, or 2^{M_t} / Z >= tau / Lk with
 * M_t its largest score and Z the sum of exp over the kept newer tiles (log2
 * units inside). The work runs in three phases: every score and each tile's
 * (max, log-sum) pair (K read once), a per-row scan of the decisions over
 * those pairs, and the PV of the kept tiles split over n_splits ranges of
 * tiles per (b, KV head) with the usual merge by LSE. n_splits only spreads
 * the PV work; it does not change any decision. V is read only for tiles some
 * head of the group keeps; the scores cost 8 extra bytes per key and head
 * (written once, read once).
 *
 * Arguments and layouts as mala_decode; workspace >=
 * mala_decode_exact_workspace_size(B, Hq, Lk, d, Bk, n_splits used) bytes.
 * kept_tiles [B*Hq] and keep_map [B, Hq, nk] (nullable) hold the decisions.
 */
MALA_API int mala_decode_exact(const void* q, const void* kcache, const void* vcache, void* o, float* lse, int B,
             int Hq, int Hkv, int Lk, int d, float scale, float tau, int Bk, int n_splits, void* workspace,
             size_t workspace_bytes, int32_t* kept_tiles, uint8_t* keep_map, void* stream);

/*
 * mala_decode_paged -- mala_decode against a paged KV cache.
 *
 * Source: as mala_decode (the cache is kept whole; decode reads it).
 *
 * The keys of sequence b are rows 0 .. page_size - 1 of pages
 * block_table[b * max_pages_per_seq + 0], [.. + 1], ... of the page pools, cut
 * at seqlens_k[b] (1 <= seqlens_k[b] <= max_pages_per_seq * page_size). A page
 * is one key tile (Bk = page_size). Each sequence is split into n_splits
 * contiguous ranges of ceil(nk_b / n_splits) tiles (nk_b = its page count), so
 * results equal mala_decode of the gathered cache with the same n_splits.
 *
 *   q          [B, Hq, d] bf16, in;  o [B, Hq, d] bf16, out;  lse [B, Hq] fp32, out
 *   k_pages, v_pages  [num_pages, page_size, Hkv, d] bf16, in
 *   block_table [B, max_pages_per_seq] int32, DEVICE memory (entries past a
 *              sequence's pages are not read)
 *   seqlens_k  [B] int32, DEVICE memory
 *   page_size  64 or 128;  n_splits >= 1, or 0 for
 *              mala_decode_default_splits(B, Hkv, max_pages_per_seq * page_size, page_size)
 *   workspace  >= mala_decode_workspace_size(B, Hq, d, n_splits used) bytes
 *   kept_tiles [B*Hq] int32, out; keep_map [B, Hq, max_pages_per_seq] uint8, nullable
 * A length out of range or a page id outside [0, num_pages) is reported by
 * mala_check_status as MALA_ERR_INVALID_ARG (such a page reads as zeros).
 */
MALA_API int mala_decode_paged(const void* q, const void* k_pages, const void* v_pages,
             const int32_t* block_table, const int32_t* seqlens_k, void* o, float* lse, int B, int Hq,
             int Hkv, int num_pages, int page_size, int max_pages_per_seq, int d, float scale, float tau,
             int n_splits, void* workspace, size_t workspace_bytes, int32_t* kept_tiles,
             uint8_t* keep_map, void* stream);

/*
 * mala_decode_noalloc -- mala_decode without a caller-provided workspace.
 *
 * The operator papers have no counterpart to this call: it exists for
 * callers that cannot allocate device memory, for example a plugin inside a
 * host engine that owns all device memory and offers it no allocator, or a
 * serving loop that cannot afford the device-wide synchronisation a
 * cudaMalloc may bring. The call allocates nothing; its split partials live
 * in one fixed, file-scope device array of mala_decode_noalloc_max_bytes()
 * bytes (8 MiB) that every GPU loading the library holds until exit.
 *
 * Arguments, layouts and results are those of mala_decode, minus the
 * workspace. A problem whose partials need more than the fixed array
 * (mala_decode_workspace_size(B, Hq, d, n_splits used) > 8 MiB) returns
 * MALA_ERR_WORKSPACE and launches nothing. The first call on a device looks
 * up the array's device address for that device and caches it with the id of
 * the CUDA context current at the time; a call that finds another context
 * current (after cudaDeviceReset, for instance) looks it up again. Make the
 * first call, and the first after such a reset, before any stream capture.
 * All calls share the array: calls that overlap on the GPU race and must be
 * serialised by the caller.
 */
MALA_API size_t mala_decode_noalloc_max_bytes(void);
MALA_API int mala_decode_noalloc(const void* q, const void* kcache, const void* vcache, void* o, float* lse,
                                 int B, int Hq, int Hkv, int Lk, int d, float scale, float tau, int Bk,
                                 int n_splits, int32_t* kept_tiles, uint8_t* keep_map, void* stream);

/*
 * mala_test_hooks -- switches for tests of the failure path and of the V
 * traffic. Process-wide; they apply to calls enqueued after this one (on any
 * stream) until changed, and are not meant for production use. The pages
 * describe nothing of the kind.
 *
 *   wait_limit_ns  limit of each bounded device-side wait; 0 restores the
 *                  default (2 s)
 *   stall_tile     -1: off. >= 0: the MMA issuer of mala_fwd / mala_prefill /
 *                  mala_fwd_varlen / mala_bwd / mala_bwd_varlen, and the K
 *                  producer of mala_decode / mala_decode_paged /
 *                  mala_decode_noalloc, wait before key tile `stall_tile` on a
 *                  barrier nothing completes, so that the wait expires: the
 *                  kernel then leaves through its abort path and
 *                  mala_check_status returns MALA_ERR_DEVICE_TIMEOUT. Outputs
 *                  of such a call are undefined.
 *   fwd_v_tiles    NULL: off. Else a DEVICE uint64 the forward kernels (gate
 *                  on) increase by one for every V tile they load.
 * Returns MALA_ERR_INVALID_ARG for stall_tile < -1, else MALA_OK.
 */
MALA_API int mala_test_hooks(unsigned long long wait_limit_ns, int stall_tile, unsigned long long* fwd_v_tiles);

/*
 * Synchronises `stream`, then reads and clears the current device's status
 * word. Returns MALA_OK, MALA_ERR_DEVICE_TIMEOUT if any kernel since the last
 * check gave up on a bounded wait, MALA_ERR_RANGE if a forward call met a V
 * value outside the fp16 range, or MALA_ERR_CUDA if the stream reports an
 * error.
 */
MALA_API int mala_check_status(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MALA_H_ */
