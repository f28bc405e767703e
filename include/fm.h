/*
 * fm.h -- C ABI of the B200 (sm_100a) mask-aware attention library.
 *
 * The library implements the single-GPU hot path of FlashMask-3 ("FlashMask-3:
 * Efficient and Expressive Mask-Aware Distributed Attention"):
 *   - a structured attention mask held as four key-indexed vectors of query-row
 *     bounds, LTS/LTE (lower masked stretch) and UTS/UTE (upper masked stretch)
 *     (learnaivisually.com explainer, "four numbers per avenue"; paper abstract,
 *     "four query-axis boundary vectors");
 *   - per-tile classification into fully masked / partly masked / unmasked from
 *     the per-key-tile minimum and maximum of the vectors, with compacted block
 *     lists (explainer, tile paragraph: "using the maximum and minimum along the
 *     key axis", "fully masked tiles are never loaded");
 *   - clip-shift-max localization of the vectors to a context-parallel rank
 *     (explainer, clip-shift-max / Theorem 1 paragraph; abstract,
 *     "zero-communication clip-shift-max");
 *   - exact softmax attention forward and backward restricted to the unmasked
 *     pairs (abstract: mask-aware kernel; explainer: "only partly masked tiles
 *     apply the row-interval test").
 *
 * Conventions (all calls):
 *   - Mask: key column j masks query row i (0-based) iff
 *       LTS[j] <= i < LTE[j]  or  UTS[j] <= i < UTE[j]      (half-open).
 *     Any int32 value is legal; start >= end is an empty stretch.  A NULL vector
 *     pointer stands for its canonical empty value (LTS = LTE = n_q, UTS = UTE = 0).
 *     Vectors are int32 [B, Hm, n_k] contiguous, Hm = 1 (shared by all heads) or H.
 *   - Tensors Q, O, dO, dQ are [B, n_q, H, D] and K, V, dK, dV are [B, n_k, H_kv, D] (H_kv = H
 *     unless fm_attn_args.H_kv says otherwise: grouped-query attention),
 *     contiguous, all of one element type: bf16 (dtype 0; bf16 tensor-core products) or
 *     fp32 (dtype 1, D = 64 only; tf32 tensor-core products, fp32 accumulation).  LSE is
 *     fp32 [B, H, n_q], natural log.
 *   - All pointers passed to compute calls are DEVICE pointers unless a parameter
 *     says "host".  The caller owns every buffer, including workspaces; the
 *     library never allocates, frees or synchronises.  Work is enqueued on
 *     `stream` (NULL = legacy default stream) and runs asynchronously.
 *   - Arguments are validated on the host before any launch; an invalid call
 *     returns an error and enqueues nothing.  FM_ERR_CUDA reports a failed
 *     launch (cudaGetLastError).  Errors found on the device (a bounded wait
 *     that ran out) are latched in a per-device status word read with
 *     fm_get_device_status.
 */
#ifndef FM_H_
#define FM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fm_stream_t; /* identical to cudaStream_t */

typedef enum {
  FM_OK = 0,
  FM_ERR_INVALID_ARG = 1,     /* a size, pointer, alignment or ordering rule is broken */
  FM_ERR_UNSUPPORTED = 2,     /* valid but not implemented (e.g. n_k not a multiple of 4) */
  FM_ERR_WORKSPACE = 3,       /* workspace pointer NULL/misaligned or ws_bytes too small */
  FM_ERR_CUDA = 4,            /* a CUDA runtime/driver call or launch failed */
  FM_ERR_DEVICE_TIMEOUT = 5,  /* a kernel's bounded wait ran out (see fm_get_device_status) */
  FM_ERR_DEVICE_CHECK = 6     /* FM_DEBUG builds only: an index or shared-memory canary check failed on
                                 the device (the access was skipped; see fm_get_device_status) */
} fm_status;

/* Shape of a mask problem.  tile_q and tile_k must be 128. */
typedef struct {
  int32_t B, Hm, n_q, n_k, tile_q, tile_k;
} fm_mask_desc;

/*
 * Tile metadata built by fm_build_mask_meta; every pointer is a DEVICE view
 * into the caller's workspace.  With T_q = ceil(n_q/tile_q), T_k = ceil(n_k/tile_k):
 *   tile_minmax [B, Hm, T_k, 8]  minLTS, maxLTS, minLTE, maxLTE, minUTS, maxUTS,
 *                                minUTE, maxUTE over the key tile's columns
 *   tile_class  [B, Hm, T_q, T_k] uint8: 0 skip (fully masked), 1 partial, 2 full
 *   row_count   [B, Hm, T_q]     number of non-skip key tiles of each query tile
 *   row_entries [B, Hm, T_q, T_k] first row_count entries valid:
 *                                (kt << 1) | is_partial, kt ascending
 *   col_count   [B, Hm, T_k], col_entries [B, Hm, T_k, T_q]: the transpose,
 *                                (qt << 1) | is_partial, qt ascending
 *   fwd_order   [B, Hm, ceil(T_q/2)] int32: query-tile pairs (2p, 2p+1) by descending
 *                                row_count[2p] + row_count[2p+1], ties by ascending p
 *   bwd_order   [B, Hm, T_k] int32: key tiles by descending col_count, ties by
 *                                ascending index
 *   (both the identity order when T_q or T_k exceeds 4096).  The attention kernels
 *   dispatch the CTAs of each (b, h) in these orders, longest first, one (b, h)
 *   after the other (a scheduling aid with no counterpart in the paper; results
 *   do not depend on it).
 * Rule (per query tile rows [r0, r1), key tile min/max as above):
 *   skip    = (maxLTS <= r0 && minLTE >= r1) || (maxUTS <= r0 && minUTE >= r1)
 *   full    = !skip && (minLTS >= r1 || maxLTE <= r0) && (minUTS >= r1 || maxUTE <= r0)
 *   partial = otherwise.
 * Metadata is valid only for the vectors it was built from.
 */
typedef struct {
  fm_mask_desc d;
  int32_t* tile_minmax;
  int32_t* row_count;
  int32_t* row_entries;
  int32_t* col_count;
  int32_t* col_entries;
  uint8_t* tile_class;
  int32_t* fwd_order;
  int32_t* bwd_order;
} fm_mask_meta;

/* Bytes of workspace fm_build_mask_meta needs for `d` (0 if d is invalid). */
size_t fm_mask_meta_workspace_bytes(const fm_mask_desc* d);

/*
 * Per-key-tile min/max of the four vectors, tile classes and block lists
 * (explainer, tile paragraph; the pages' "KV Index Generator" role, run here as
 * its own bandwidth-bound pass).
 *   d         host pointer; B, Hm >= 1; n_q, n_k >= 1; tile_q = tile_k = 128.
 *   lts..ute  device int32 [B, Hm, n_k] or NULL (canonical empty).
 *   ws        device workspace of ws_bytes >= fm_mask_meta_workspace_bytes(d),
 *             256-byte aligned; owned by the caller, must outlive the metadata.
 *   out       host struct filled with the views into ws (valid once the stream
 *             reaches this call's kernels).
 * Errors: FM_ERR_INVALID_ARG (bad desc / NULL out), FM_ERR_WORKSPACE, FM_ERR_CUDA.
 */
fm_status fm_build_mask_meta(const fm_mask_desc* d, const int32_t* lts, const int32_t* lte,
                             const int32_t* uts, const int32_t* ute, void* ws, size_t ws_bytes,
                             fm_mask_meta* out, fm_stream_t stream);

/*
 * Variable-length batches as one packed sequence (the paper's document masks:
 * sequences packed end to end attend only within themselves).  Sequence s holds
 * rows and keys [cu_seqlens[s], cu_seqlens[s+1]); for key j of sequence s:
 *     LTS[j] = cu_seqlens[s+1], LTE[j] = N   (rows after the sequence are masked)
 *     UTS[j] = 0, UTE[j] = j if causal, else cu_seqlens[s]   (rows before it)
 * so the packed call computes, for every sequence, the attention it would get
 * alone (causal or bidirectional), and every tile between two sequences is a
 * skip tile.  Keys past cu_seqlens[n_seq] (padding) are masked for all rows.
 *   cu_seqlens  device int32 [n_seq + 1]: 0 = cu[0] <= cu[1] <= ... <= cu[n_seq] <= N
 *               (the library reads it on the device and does not check it; an unsorted
 *               array gives a mask of some other shape, never an out-of-bounds access).
 *   n_seq       >= 1, <= 2^20;  N >= 1, the packed length (rows = keys = N).
 *   causal      0 or 1.
 *   lts..ute    device int32 [N] each (one [B = 1, Hm = 1, N] mask); the attention calls
 *               want them 16-byte aligned.
 * Errors: FM_ERR_INVALID_ARG, FM_ERR_CUDA.
 */
fm_status fm_varlen_mask(const int32_t* cu_seqlens, int32_t n_seq, int32_t N, int32_t causal, int32_t* lts,
                         int32_t* lte, int32_t* uts, int32_t* ute, fm_stream_t stream);

/*
 * Clip-shift-max localization (explainer, clip-shift-max / Theorem 1 paragraph:
 * "clip each mark to a chunk, shift it into the rank's concatenated numbering,
 * and take the maximum across the rank's chunks").  For R simulated ranks at
 * once: rank r owns C query chunks [chunk_start[r*C+k], +chunk_len[r*C+k]) in
 * strictly increasing, non-overlapping global order, with local offsets
 * o_k = sum_{k'<k} len_k'.  For every vector value v of every key (keys stay global):
 *     v_loc = max(0, max_k clamp(v - start_k + o_k, 0, o_k + len_k)).
 *   B, Hm, N     vector shape [B, Hm, N] (N = global sequence length >= 1)
 *   in[4]        host array of 4 device pointers (LTS, LTE, UTS, UTE), each
 *                [B, Hm, N]; NULL entries are not allowed here.
 *   R, C         ranks and chunks per rank; 1 <= R*C <= 256.
 *   chunk_start, chunk_len   host int32 [R*C]; lengths >= 1, chunks inside [0, N].
 *   out[4]       host array of 4 device pointers, each [R, B, Hm, N] int32.
 * Errors: FM_ERR_INVALID_ARG (ordering, ranges, NULLs), FM_ERR_CUDA.
 */
fm_status fm_localize(int32_t B, int32_t Hm, int32_t N, const int32_t* const in[4], int32_t R, int32_t C,
                      const int32_t* chunk_start, const int32_t* chunk_len, int32_t* const out[4],
                      fm_stream_t stream);

/*
 * KV-chunk pruning for context-parallel ranks (explainer, across-ranks paragraph:
 * the forward all-gather skips key-value chunks that are fully masked).  For
 * each rank r, with n_loc[r] local query rows and the localized vectors
 * fm_localize wrote, and key chunk c = keys [c * chunk_len, min((c+1) * chunk_len, N)):
 *     pairs[r, b, hm, c] = sum over keys j of chunk c of
 *                          n_loc[r] - |([LTS_j, LTE_j) u [UTS_j, UTE_j)) n [0, n_loc[r])|,
 * the number of unmasked (local row, key) pairs.  A chunk with pairs == 0 is
 * pruned: no local query attends to any of its keys, so the rank never needs
 * its K/V.  Summed over chunks it is the rank's attention work (the quantity a
 * sparsity-aware balancer equalises).  Exact integer counts.
 *   B, Hm, N     vector shape per rank [B, Hm, N]
 *   R            ranks, 1 <= R <= 256, R * B * Hm <= 65535
 *   vec[4]       host array of 4 device pointers, each [R, B, Hm, N] int32
 *                (NULL = canonical empty: LTS = LTE = n_loc[r], UTS = UTE = 0)
 *   n_loc        host int32 [R], local query rows of each rank (>= 0)
 *   chunk_len    keys per chunk (>= 1); n_chunks = ceil(N / chunk_len)
 *   pairs        device int64 [R, B, Hm, n_chunks], 8-byte aligned
 * Errors: FM_ERR_INVALID_ARG, FM_ERR_UNSUPPORTED (R * B * Hm > 65535), FM_ERR_CUDA.
 */
fm_status fm_kv_chunk_pairs(int32_t B, int32_t Hm, int32_t N, int32_t R, const int32_t* const vec[4],
                            const int32_t* n_loc, int32_t chunk_len, int64_t* pairs, fm_stream_t stream);

/* Attention problem.  q, k, v are device pointers (bf16, layouts above). */
typedef struct {
  int32_t B, H, n_q, n_k, D;
  int32_t dtype;  /* 0 = bf16, 1 = fp32 (tf32 products; D = 64 only) */
  float scale;    /* softmax scale, e.g. 1/sqrt(D) */
  const void* q;
  const void* k;
  const void* v;
  int32_t H_kv;   /* K/V heads (grouped-query attention): H % H_kv == 0, query head h reads K/V
                     head h / (H / H_kv); 0 means H_kv = H */
  int32_t deterministic;  /* backward only (the forward always is): 0 = the key tiles add their
                             dQ contributions in whatever order they finish; 1 = in a fixed order,
                             so that dQ is bitwise repeatable (see fm_attn_bwd) */
} fm_attn_args;

/*
 * Mask-aware attention forward: for every (b, h, row i) with U_i the unmasked
 * keys, O_i = sum_{j in U_i} softmax_j(scale q_i.k_j) v_j and
 * LSE_i = ln sum_{j in U_i} exp(scale q_i.k_j); a row with U_i empty gets
 * O_i = 0 and LSE_i = -inf.  Only non-skip key tiles (meta row lists) are read;
 * the row-interval test runs on partial tiles only.
 *   a      host struct; H_kv divides H (0 = H; at most 64 query heads per K/V head);
 *          n_q >= 1 any length, n_k >= 1 a multiple of 4 (ragged lengths: the last
 *          tiles are zero-filled past n and the last key tile always runs the interval test);
 *          at most 4096 tiles each way; D in {64, 128}; dtype 0, or 1 with D = 64;
 *          scale > 0 and finite.
 *   meta   host struct from fm_build_mask_meta with d = {B, Hm, n_q, n_k, 128, 128}.
 *   vec[4] host array of the 4 device vector pointers meta was built from
 *          (NULL entries allowed = canonical empty); 16-byte aligned.
 *   o      device [B, n_q, H, D] of the dtype; lse device fp32 [B, H, n_q].
 * Errors: FM_ERR_INVALID_ARG, FM_ERR_UNSUPPORTED, FM_ERR_CUDA.
 */
fm_status fm_attn_fwd(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4], void* o,
                      float* lse, fm_stream_t stream);

/* Bytes of workspace fm_attn_bwd needs (0 if a is invalid). */
size_t fm_attn_bwd_workspace_bytes(const fm_attn_args* a);

/*
 * Mask-aware attention backward (exact gradient of fm_attn_fwd):
 *   D_i = dO_i.O_i, P_ij = exp(scale q_i.k_j - LSE_i) on unmasked pairs (else 0),
 *   dV_j = sum_i P_ij dO_i, dS_ij = P_ij (dO_i.v_j - D_i),
 *   dQ_i = scale sum_j dS_ij k_j, dK_j = scale sum_i dS_ij q_i.
 * Key tiles iterate their meta column lists (non-skip query tiles only).
 *   o, lse   the forward's outputs; dout device [B, n_q, H, D] of the dtype.
 *   dq, dk, dv device outputs of the dtype; dq [B, n_q, H, D], dk / dv [B, n_k, H_kv, D] (the
 *            gradient of a shared K/V head sums over its query heads); every element is written.
 *   The column lists of the query heads sharing a K/V head are held together: (H / H_kv) x
 *   ceil(n_q / 128) <= 4096, else FM_ERR_UNSUPPORTED.
 *   ws       device workspace, ws_bytes >= fm_attn_bwd_workspace_bytes(a), 256-byte
 *            aligned; holds the fp32 dQ accumulator and per-row statistics.
 *   a->deterministic = 1: the contributions of the key tiles to the fp32 dQ accumulator of a
 *            query tile are added in ascending key-tile order (each key tile waits, bounded,
 *            for the ones before it in that tile's row list), so dQ is bitwise the same from
 *            run to run; dK and dV always are.  Key tiles are then dispatched in ascending
 *            order rather than longest first, and the workspace grows by
 *            B * H * ceil(n_k / 128) * ceil(n_q / 128) * 2 + B * H * ceil(n_q / 128) * 4 bytes.
 *            The order relies on CTAs of lower index starting no later than those of higher
 *            index; if one waits longer than the bound the call reports FM_ERR_DEVICE_TIMEOUT
 *            through fm_get_device_status instead of hanging.
 * Errors: FM_ERR_INVALID_ARG, FM_ERR_UNSUPPORTED, FM_ERR_WORKSPACE, FM_ERR_CUDA.
 */
fm_status fm_attn_bwd(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4],
                      const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                      void* ws, size_t ws_bytes, fm_stream_t stream);

/*
 * Size of the fixed device scratch used by fm_attn_bwd_noalloc: 32 MiB, held
 * by every GPU that loads this library for as long as the process lives.
 */
#define FM_BWD_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * fm_attn_bwd without a caller-supplied workspace.  The paper has no
 * counterpart to this entry point; it exists for callers that cannot allocate
 * device memory when they call the backward: for example a plug-in inside an
 * inference or training engine that plans every device buffer up front and
 * exposes no workspace to its kernels, or a latency-critical loop that must not
 * pay cudaMalloc's implicit device synchronisation.  It computes exactly what
 * fm_attn_bwd computes, with the same arguments minus ws / ws_bytes; its
 * scratch (fp32 dQ accumulator, per-row statistics) lives in one fixed device
 * array of FM_BWD_NOALLOC_SCRATCH_BYTES bytes inside the library, and it calls
 * no cudaMalloc, cudaFree or other allocating routine.
 *   - Limit: fm_attn_bwd_workspace_bytes(a) must not exceed
 *     FM_BWD_NOALLOC_SCRATCH_BYTES (for D = 128 about 64K query rows in total,
 *     B * H * n_q); larger problems are rejected with FM_ERR_WORKSPACE before
 *     any launch.
 *   - Every call looks up the array's address on the current device (a
 *     symbol lookup, nothing allocated), so the address never goes stale; the
 *     first lookup on a device may load the library's device code, so make
 *     the first call before any stream capture.
 *   - Every call on a device shares the one array; it keeps the last call's
 *     contents and each call clears what must start at zero.  Calls whose
 *     kernels overlap on the GPU (different streams, no ordering between
 *     them) race on the array and give wrong gradients: order them.
 * Errors: as fm_attn_bwd, plus FM_ERR_CUDA if the address lookup fails.
 */
fm_status fm_attn_bwd_noalloc(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4],
                              const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                              fm_stream_t stream);

/*
 * Reads and clears the current device's status word: FM_OK, or
 * FM_ERR_DEVICE_TIMEOUT if a kernel gave up on a bounded wait since the last
 * call.  Synchronises `stream` (the one call that does).
 */
fm_status fm_get_device_status(fm_stream_t stream);

/* Static description of a status code. */
const char* fm_status_string(fm_status s);

/*
 * Self-test of the bounded-wait path (no counterpart in the paper).  Every wait in
 * the kernels gives up after 2 s, records FM_ERR_DEVICE_TIMEOUT in the per-device
 * status word and lets its kernel return, so a stuck pipeline surfaces as a status
 * instead of a hung GPU.  This call enqueues one kernel whose only wait is on a
 * barrier nothing completes: about 2 s later it has recorded the timeout, which the
 * next fm_get_device_status(stream) returns (and clears).  Nothing faults; the
 * context stays usable.
 * Errors: FM_ERR_CUDA (launch failed).
 */
fm_status fm_selftest_wait_timeout(fm_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FM_H_ */
