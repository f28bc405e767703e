// Tile metadata pass: per-key-tile min/max of the four boundary vectors,
// classification of every (query tile, key tile) pair, compacted row and
// column block lists.  FlashMask-3 explainer (learnaivisually.com), tile
// paragraph: the kernel "sorts every tile of the score matrix as fully masked,
// partly masked or unmasked, using the maximum and minimum along the key axis",
// and a KV Index Generator role "scans the marks and queues the valid blocks".
// Here that role is a separate bandwidth-bound pass whose lists the attention
// kernels consume.
#include <climits>

#include "fm_common.cuh"

namespace fm {
namespace {

constexpr int kTile = 128;
constexpr int kOrderListMax = 4096;  // longest list (tiles each way) the attention kernels take

struct MetaParams {
  const int32_t* vec[4];  // [B, Hm, n_k] or null
  int32_t* minmax;        // [BHm, T_k, 8]
  uint8_t* cls;           // [BHm, T_q, T_k]
  int32_t* row_count;     // [BHm, T_q]
  int32_t* row_entries;   // [BHm, T_q, T_k]
  int32_t* col_count;     // [BHm, T_k]
  int32_t* col_entries;   // [BHm, T_k, T_q]
  int32_t* fwd_order;     // [BHm, ceil(T_q / 2)]
  int32_t* bwd_order;     // [BHm, T_k]
  int32_t* done;          // [BHm] query-tile CTAs finished (the last one sorts the dispatch orders)
  int32_t BHm, n_q, n_k, T_q, T_k;
};

// Last row (exclusive) of the tile starting at row r0: min(r0 + 128, n_q), without overflow.
__device__ __forceinline__ int tile_r1(int r0, int n_q) { return (n_q - r0 > kTile) ? r0 + kTile : n_q; }

// 0 skip, 1 partial, 2 full for query rows [r0, r1) against one key tile's min/max.
__device__ __forceinline__ int classify(const int4 lo, const int4 hi, int r0, int r1) {
  // lo = (minLTS, maxLTS, minLTE, maxLTE), hi = (minUTS, maxUTS, minUTE, maxUTE)
  const bool skip = (lo.y <= r0 && lo.z >= r1) || (hi.y <= r0 && hi.z >= r1);
  const bool clear_l = (lo.x >= r1) || (lo.w <= r0);
  const bool clear_u = (hi.x >= r1) || (hi.w <= r0);
  return skip ? 0 : ((clear_l && clear_u) ? 2 : 1);
}

// One query tile's row list over the key tiles built by a quad of four warps: warp w of the quad
// classifies positions [w c, (w + 1) c) with c = 32 ceil(L / 128), 32 at a time, keeping the
// ballots of "non-skip" and "partial" in shared memory (masks: 2 x L / 32 words for the quad); after the quad's named barrier each warp knows how
// many entries the warps before it keep and writes its own entries (index << 1 | partial) in
// ascending order.  class_of(idx) gives the class; on_class(idx, c) sees every classified position.
constexpr int kMaskWords = 2 * kOrderListMax / 32;
template <typename ClassOf, typename OnClass>
__device__ __forceinline__ int quad_list(int L, int wq, int lane, int bar_id, uint32_t* masks, int* counts,
                                         int32_t* ent, ClassOf class_of, OnClass on_class) {
  const unsigned below = (1u << lane) - 1u;
  const int chunk = 32 * ((L + 127) / 128);
  const int p0 = wq * chunk, p1 = min(p0 + chunk, L);
  int count = 0;
  for (int k0 = p0, it = 0; k0 < p1; k0 += 32, ++it) {
    const int idx = k0 + lane;
    int c = 0;
    if (idx < p1) {
      c = class_of(idx);
      on_class(idx, c);
    }
    const unsigned keep = __ballot_sync(0xffffffffu, c != 0), part = __ballot_sync(0xffffffffu, c == 1);
    if (lane == 0) {
      masks[2 * (p0 / 32 + it)] = keep;
      masks[2 * (p0 / 32 + it) + 1] = part;
    }
    count += __popc(keep);
  }
  if (lane == 0) counts[wq] = count;
  named_bar_sync(bar_id, 128);
  int base = 0;
  for (int w = 0; w < wq; ++w) base += counts[w];
  for (int k0 = p0, it = 0; k0 < p1; k0 += 32, ++it) {
    const unsigned keep = masks[2 * (p0 / 32 + it)], part = masks[2 * (p0 / 32 + it) + 1];
    if ((keep >> lane) & 1u) ent[base + __popc(keep & below)] = ((k0 + lane) << 1) | ((part >> lane) & 1u);
    base += __popc(keep);
  }
  return counts[0] + counts[1] + counts[2] + counts[3];  // (read before the next use of counts)
}

// The tile rule against a fixed key tile as the query tile qt grows: each of its eight terms
// flips at most once, because r0 = 128 qt and r1 = min(r0 + 128, n_q) never decrease.
//   "x <= r0" holds from qt = first_le_r0(x) on;  "y >= r1" holds for qt < count_ge_r1(y).
// So skip is qt in [s(maxLTS), t(minLTE)) or [s(maxUTS), t(minUTE)), and a non-skip tile is
// partial when qt lies in [t(minLTS), s(maxLTE)) or [t(minUTS), s(maxUTE)) (a vector not clear
// of the tile), full otherwise.
__device__ __forceinline__ int first_le_r0(int32_t x, int T_q) {
  if (x <= 0) return 0;
  const int q = x / kTile + (x % kTile != 0 ? 1 : 0);
  return q < T_q ? q : T_q;
}
__device__ __forceinline__ int count_ge_r1(int32_t y, int n_q, int T_q) {
  if (y >= n_q) return T_q;
  if (y < 0) return 0;
  const int q = y / kTile;
  return q < T_q ? q : T_q;
}

// Key-tile pass: one warp per (bhm, key tile), 8 per CTA.  Min and max of the four vectors over
// the tile's 128 columns (four columns per lane and vector, then shuffles), written to minmax;
// then the tile's column list: the query tiles outside the two skip ranges above (at most three
// runs), each entry marked partial or not, written 32 at a time in ascending order.  Also clears
// the per-bhm counter of the query-tile pass.
constexpr int kColsThreads = 256;
__global__ void __launch_bounds__(kColsThreads) meta_cols_kernel(const MetaParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tile = (int64_t)blockIdx.x * (kColsThreads / 32) + warp;  // (bhm, key tile)
  if (tile >= (int64_t)p.BHm * p.T_k) return;  // (whole warps)
  const int bhm = (int)(tile / p.T_k), kt = (int)(tile % p.T_k);
  if (kt == 0 && lane == 0) p.done[bhm] = 0;
  const int32_t dflt[4] = {p.n_q, p.n_q, 0, 0};
  // every load first (sixteen per lane in flight), then the reductions; only the last key tile of a
  // ragged n_k has columns past the end, which take no part
  const int valid = min(kTile, p.n_k - kt * kTile);  // columns of this tile, >= 1
  const int32_t* vb[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) vb[c] = p.vec[c] ? p.vec[c] + (int64_t)bhm * p.n_k + (int64_t)kt * kTile : nullptr;
  int32_t col[4][kTile / 32];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
#pragma unroll
    for (int t = 0; t < kTile / 32; ++t) {
      const int j = t * 32 + lane;
      col[c][t] = !vb[c] ? dflt[c] : (valid == kTile || j < valid) ? __ldg(vb[c] + j) : 0;
    }
  }
  int32_t mn[4], mx[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    mn[c] = INT_MAX;
    mx[c] = INT_MIN;
#pragma unroll
    for (int t = 0; t < kTile / 32; ++t) {
      const bool in = valid == kTile || t * 32 + lane < valid;
      mn[c] = in ? min(mn[c], col[c][t]) : mn[c];
      mx[c] = in ? max(mx[c], col[c][t]) : mx[c];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      mn[c] = min(mn[c], __shfl_xor_sync(0xffffffffu, mn[c], off));
      mx[c] = max(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], off));
    }
  }
  // (minLTS, maxLTS, minLTE, maxLTE, minUTS, maxUTS, minUTE, maxUTE)
  if (lane < 8) {
    const int32_t v[8] = {mn[0], mx[0], mn[1], mx[1], mn[2], mx[2], mn[3], mx[3]};
    int32_t val = v[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) val = (lane == k) ? v[k] : val;  // select without dynamic indexing
    p.minmax[tile * 8 + lane] = val;
  }
  const int T = p.T_q;
  // skip ranges [a0, a1) and [b0, b1), empty ones moved to T, ordered by start
  int a0 = first_le_r0(mx[0], T), a1 = count_ge_r1(mn[1], p.n_q, T);
  int b0 = first_le_r0(mx[2], T), b1 = count_ge_r1(mn[3], p.n_q, T);
  if (a1 <= a0) a0 = a1 = T;
  if (b1 <= b0) b0 = b1 = T;
  if (b0 < a0) {
    const int x0 = a0, x1 = a1;
    a0 = b0;
    a1 = b1;
    b0 = x0;
    b1 = x1;
  }
  // partial ranges [p0, p1) and [u0, u1)
  const int p0 = count_ge_r1(mn[0], p.n_q, T), p1 = first_le_r0(mx[1], T);
  const int u0 = count_ge_r1(mn[2], p.n_q, T), u1 = first_le_r0(mx[3], T);
  // non-skip runs: [0, a0), then [max(a1, b1), T) if the skip ranges touch, else [a1, b0), [b1, T)
  const bool joined = b0 <= a1;
  const int run_lo[3] = {0, joined ? max(a1, b1) : a1, joined ? T : b1};
  const int run_hi[3] = {a0, joined ? T : b0, T};
  int32_t* ent = p.col_entries + tile * p.T_q;
  int n = 0;
#pragma unroll
  for (int r = 0; r < 3; ++r) {
    const int lo_r = run_lo[r], hi_r = run_hi[r];
    for (int q = lo_r + lane; q < hi_r; q += 32) {
      const bool part = (q >= p0 && q < p1) || (q >= u0 && q < u1);
      ent[n + (q - lo_r)] = (q << 1) | (part ? 1 : 0);
    }
    n += max(hi_r - lo_r, 0);
  }
  if (lane == 0) p.col_count[tile] = n;
}

// Dispatch orders (longest first) of one (b, hm), by the CTA that finishes the query-tile pass
// last: the forward's query-tile pairs by the sum of their two row counts, the backward's key
// tiles by column count; ties keep ascending index.  Bitonic sort in shared memory of the keys
// (cost << 16) | (0xFFFF - index), descending; with at most 4096 items and costs below 2^16 the
// keys are distinct, so the order is deterministic.  The two sorts run side by side, each on 512
// threads of the CTA and its own named barrier.
constexpr int kOrderMax = 4096;
constexpr int kRowsThreads = 1024;
__device__ void sort_order(uint32_t* key, const int32_t* cost_a, bool pairs, int n, int n_b, int32_t* out, int tid,
                           int bar_id) {
  constexpr int kT = kRowsThreads / 2;
  int np2 = 1;
  while (np2 < n) np2 <<= 1;
  for (int i = tid; i < np2; i += kT) {
    uint32_t k = 0;  // padding sorts last
    if (i < n) {
      // counts written by other CTAs of this launch: read through L2 (__ldcg), not a stale L1 line
      const uint32_t cost = pairs ? (uint32_t)(__ldcg(cost_a + 2 * i) + (2 * i + 1 < n_b ? __ldcg(cost_a + 2 * i + 1) : 0))
                                  : (uint32_t)__ldcg(cost_a + i);
      k = (cost << 16) | (0xFFFFu - (uint32_t)i);
    }
    key[i] = k;
  }
  named_bar_sync(bar_id, kT);
  for (int len = 2; len <= np2; len <<= 1) {
    for (int j = len >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < np2; i += kT) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint32_t a = key[i], b = key[ixj];
          const bool desc = (i & len) == 0;  // descending runs merge into one descending sequence
          if (desc ? (a < b) : (a > b)) {
            key[i] = b;
            key[ixj] = a;
          }
        }
      }
      named_bar_sync(bar_id, kT);
    }
  }
  for (int i = tid; i < n; i += kT) out[i] = (int32_t)(0xFFFFu - (key[i] & 0xFFFFu));
}

// The same order for n <= 1024 items, one key per thread of the whole CTA (kRowsThreads = 1024),
// padded to 1024 with zero keys (after every real key: those are >= 0xF000).  Bitonic network
// in registers: partners within a warp (j < 32) by shuffle, the 15 exchanges with j >= 32 through
// shared memory, double-buffered so that each takes one barrier.
__device__ void sort_order1024(uint32_t* buf, const int32_t* cost_a, bool pairs, int n, int n_b, int32_t* out) {
  const int i = threadIdx.x;
  uint32_t k = 0;
  if (i < n) {
    // counts written by other CTAs of this launch: read through L2 (__ldcg), not a stale L1 line
    const uint32_t cost = pairs ? (uint32_t)(__ldcg(cost_a + 2 * i) + (2 * i + 1 < n_b ? __ldcg(cost_a + 2 * i + 1) : 0))
                                : (uint32_t)__ldcg(cost_a + i);
    k = (cost << 16) | (0xFFFFu - (uint32_t)i);
  }
  int phase = 0;
  for (int len = 2; len <= kRowsThreads; len <<= 1) {
    const bool desc = (i & len) == 0;  // descending runs merge into one descending sequence
    for (int j = len >> 1; j > 0; j >>= 1) {
      uint32_t other;
      if (j >= 32) {
        buf[phase * kRowsThreads + i] = k;
        __syncthreads();
        other = buf[phase * kRowsThreads + (i ^ j)];
        phase ^= 1;
      } else {
        other = __shfl_xor_sync(0xffffffffu, k, j);
      }
      const bool lower = (i & j) == 0;  // this thread holds the lower index of the pair
      k = (lower == desc) ? max(k, other) : min(k, other);
    }
  }
  if (i < n) out[i] = (int32_t)(0xFFFFu - (k & 0xFFFFu));
}

// Bits 0..3 of x to bytes 0..3 (one bit per byte): the four shifted copies do not overlap.
__device__ __forceinline__ uint32_t spread4(uint32_t x) { return (x * 0x00204081u) & 0x01010101u; }

// Skip and partial ranges of query tiles against one key tile's min/max (the key-tile pass's
// derivation): skip for qt in [x, y) or [z, w) of the first vector, partial (when not skip) for qt
// in [x, y) or [z, w) of the second.
__device__ __forceinline__ void tile_ranges(const int4 lo, const int4 hi, int n_q, int T_q, int4& sk, int4& pr) {
  sk = make_int4(first_le_r0(lo.y, T_q), count_ge_r1(lo.z, n_q, T_q), first_le_r0(hi.y, T_q), count_ge_r1(hi.z, n_q, T_q));
  pr = make_int4(count_ge_r1(lo.x, n_q, T_q), first_le_r0(lo.w, T_q), count_ge_r1(hi.x, n_q, T_q), first_le_r0(hi.w, T_q));
}

// Query-tile pass: 1024 threads, grid (ceil(T_q / kLists), BHm).  Each query tile gets its row of the
// class matrix and its row list over the key tiles.  The CTA that completes a (b, hm) last also
// writes that (b, hm)'s two dispatch orders.  Two forms:
//  * Quad (small launches, where one warp per list would leave most of the GPU idle, and at most
//    kOrderListMax key tiles, the positions its ballot words and the staged copy hold): four warps
//    per query tile (quad_list), applying the tile rule to the key-tile pass's min/max, staged in
//    shared memory as T_k x (LTS, LTE) then T_k x (UTS, UTE);
//  * otherwise four query tiles per warp, 128 per CTA: the staged copy holds, per key tile, its skip
//    and partial ranges of query tiles (tile_ranges) as bit words over the CTA's 128 query tiles
//    (four skip words, then four partial words, each word a [T_k] array); lane l, for key tile
//    k0 + l, reads the four bits of the warp's query tiles from each, and the four rows' class bytes
//    and list entries take a bit test each, with lane-contiguous stores.
constexpr int kTilesPerWarp = 4;
template <bool Quad>
__global__ void __launch_bounds__(kRowsThreads) meta_rows_kernel(const MetaParams p) {
  constexpr int kLists = Quad ? kRowsThreads / 32 / 4 : kRowsThreads / 32 * kTilesPerWarp;  // query tiles per CTA
  static_assert(Quad || (kLists % 32 == 0 && 2 * (kLists / 32) * 4 == 32), "eight bit words (32 B) per key tile");
  extern __shared__ int4 mm_smem[];  // 32 B per key tile (when T_k <= kOrderMax): see above
  uint32_t* words = reinterpret_cast<uint32_t*>(mm_smem);  // (four-lists-per-warp form) [8][T_k]
  __shared__ uint32_t key_f[kOrderMax / 2];
  __shared__ uint32_t key_b[kOrderMax];
  __shared__ uint32_t masks[Quad ? kLists : 1][Quad ? kMaskWords : 1];
  __shared__ int counts[Quad ? kLists : 1][4];
  __shared__ int last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bhm = blockIdx.y;
  const int4* mm_g = reinterpret_cast<const int4*>(p.minmax + (int64_t)bhm * p.T_k * 8);
  const bool staged = p.T_k <= kOrderMax;  // the launch gives 32 B of shared memory per key tile up to 4096
  if (staged) {
    for (int k = threadIdx.x; k < p.T_k; k += blockDim.x) {
      const int4 lo = __ldg(mm_g + 2 * k), hi = __ldg(mm_g + 2 * k + 1);
      if constexpr (Quad) {
        mm_smem[k] = lo;
        mm_smem[p.T_k + k] = hi;
      } else {
        int4 sk, pr;
        tile_ranges(lo, hi, p.n_q, p.T_q, sk, pr);
        const int q0 = blockIdx.x * kLists;
#pragma unroll
        for (int r = 0; r < kLists / 32; ++r) {
          const int base = q0 + 32 * r;
          words[r * p.T_k + k] = interval_bits32(sk.x, sk.y, base) | interval_bits32(sk.z, sk.w, base);
          words[(kLists / 32 + r) * p.T_k + k] = interval_bits32(pr.x, pr.y, base) | interval_bits32(pr.z, pr.w, base);
        }
      }
    }
    __syncthreads();
  }
  if constexpr (Quad) {
    const int quad = warp >> 2, wq = warp & 3, qt = blockIdx.x * kLists + quad;
    if (qt < p.T_q) {
      const int r0 = qt * kTile, r1 = tile_r1(r0, p.n_q);
      uint8_t* cls = p.cls + ((int64_t)bhm * p.T_q + qt) * p.T_k;
      int32_t* ent = p.row_entries + ((int64_t)bhm * p.T_q + qt) * p.T_k;
      // (consecutive lanes read consecutive 16-byte words of the staged copy: no bank conflicts)
      auto class_of = [&](int kt) { return classify(mm_smem[kt], mm_smem[p.T_k + kt], r0, r1); };
      auto store_class = [&](int kt, int c) { cls[kt] = (uint8_t)c; };
      const int n = quad_list(p.T_k, wq, lane, 1 + quad, masks[quad], counts[quad], ent, class_of, store_class);
      if (wq == 0 && lane == 0) p.row_count[(int64_t)bhm * p.T_q + qt] = n;
    }
  } else {
    const int qt0 = (blockIdx.x * (kRowsThreads / 32) + warp) * kTilesPerWarp;  // this warp's first query tile
    const int nq = min(kTilesPerWarp, p.T_q - qt0);                             // (uniform over the warp)
    if (nq > 0) {
      const unsigned below = (1u << lane) - 1u;
      uint8_t* cls = p.cls + ((int64_t)bhm * p.T_q + qt0) * p.T_k;
      int32_t* ent = p.row_entries + ((int64_t)bhm * p.T_q + qt0) * p.T_k;
      int cnt[kTilesPerWarp] = {};
      const bool aligned = (p.T_k & 3) == 0;  // rows of the class matrix start on 4-byte boundaries
      for (int k0 = 0; k0 < p.T_k; k0 += 32) {
        const int kt = k0 + lane;
        uint32_t skipm = 0xFFFFFFFFu, partm = 0u;  // lanes past the last key tile keep nothing
        if (kt < p.T_k) {
          if (staged) {  // this warp's bits of the CTA's words
            const int r = warp / (32 / kTilesPerWarp), sh = (warp % (32 / kTilesPerWarp)) * kTilesPerWarp;
            skipm = words[r * p.T_k + kt] >> sh;
            partm = words[(kLists / 32 + r) * p.T_k + kt] >> sh;
          } else {
            int4 sk, pr;
            tile_ranges(mm_g[2 * kt], mm_g[2 * kt + 1], p.n_q, p.T_q, sk, pr);
            skipm = interval_bits32(sk.x, sk.y, qt0) | interval_bits32(sk.z, sk.w, qt0);
            partm = interval_bits32(pr.x, pr.y, qt0) | interval_bits32(pr.z, pr.w, qt0);
          }
        }
        // class bytes of the four rows for this lane's key tile: byte q = 2 keep - partial
        const uint32_t k4 = ~skipm & 0xFu, p4 = partm & k4;
        const uint32_t w = (spread4(k4) << 1) - spread4(p4);
        if (aligned && k0 + 32 <= p.T_k) {
          // lane l stores row l / 8, key tiles k0 + 4 (l % 8) .. + 3: byte l / 8 of four lanes' words
          const int src = 4 * (lane & 7), qr = lane >> 3;
          const uint32_t s0 = __shfl_sync(0xffffffffu, w, src), s1 = __shfl_sync(0xffffffffu, w, src + 1);
          const uint32_t s2 = __shfl_sync(0xffffffffu, w, src + 2), s3 = __shfl_sync(0xffffffffu, w, src + 3);
          const uint32_t sel = (uint32_t)qr | ((uint32_t)(qr + 4) << 4);
          const uint32_t out = __byte_perm(__byte_perm(s0, s1, sel), __byte_perm(s2, s3, sel), 0x5410);
          if (qr < nq) *reinterpret_cast<uint32_t*>(cls + (int64_t)qr * p.T_k + k0 + src) = out;
        } else if (kt < p.T_k) {
#pragma unroll
          for (int q = 0; q < kTilesPerWarp; ++q)
            if (q < nq) cls[(int64_t)q * p.T_k + kt] = (uint8_t)(w >> (8 * q));
        }
#pragma unroll
        for (int q = 0; q < kTilesPerWarp; ++q) {
          if (q < nq) {
            const bool keep = ((skipm >> q) & 1u) == 0u, part = ((partm >> q) & 1u) != 0u;
            const unsigned bal = __ballot_sync(0xffffffffu, keep);
            if (keep) ent[(int64_t)q * p.T_k + cnt[q] + __popc(bal & below)] = (kt << 1) | (part ? 1 : 0);
            cnt[q] += __popc(bal);
          }
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int q = 0; q < kTilesPerWarp; ++q)
          if (q < nq) p.row_count[(int64_t)bhm * p.T_q + qt0 + q] = cnt[q];
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's counts before its arrival
    last = atomicAdd(p.done + bhm, 1) == (int)gridDim.x - 1;
    if (last) __threadfence();  // every other CTA's counts after it
  }
  __syncthreads();
  if (!last) return;
  const int n_pairs = (p.T_q + 1) / 2;
  int32_t* fo = p.fwd_order + (int64_t)bhm * n_pairs;
  int32_t* bo = p.bwd_order + (int64_t)bhm * p.T_k;
  if (p.T_q > kOrderMax || p.T_k > kOrderMax) {  // sizes the attention kernels do not take
    for (int i = threadIdx.x; i < n_pairs; i += blockDim.x) fo[i] = i;
    for (int i = threadIdx.x; i < p.T_k; i += blockDim.x) bo[i] = i;
    return;
  }
  if (n_pairs <= kRowsThreads && p.T_k <= kRowsThreads) {  // every list length up to 131072 tokens
    sort_order1024(key_b, p.row_count + (int64_t)bhm * p.T_q, true, n_pairs, p.T_q, fo);
    __syncthreads();  // (the buffer is reused)
    sort_order1024(key_b, p.col_count + (int64_t)bhm * p.T_k, false, p.T_k, 0, bo);
    return;
  }
  constexpr int kT = kRowsThreads / 2;
  if (threadIdx.x < kT)
    sort_order(key_f, p.row_count + (int64_t)bhm * p.T_q, true, n_pairs, p.T_q, fo, threadIdx.x, 1);
  else
    sort_order(key_b, p.col_count + (int64_t)bhm * p.T_k, false, p.T_k, 0, bo, threadIdx.x - kT, 2);
}

// Packed variable-length batch -> document-mask vectors, one thread per key: the key's sequence is
// the largest s < n_seq with cu[s] <= j (binary search; empty sequences are passed over).
__global__ void __launch_bounds__(256) varlen_mask_kernel(const int32_t* __restrict__ cu, int n_seq, int N,
                                                          int causal, int32_t* __restrict__ lts,
                                                          int32_t* __restrict__ lte, int32_t* __restrict__ uts,
                                                          int32_t* __restrict__ ute) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= N) return;
  const int j = (int)t;
  int l0 = 0, l1 = N, u1 = 0;  // a padding key past the last sequence: every row masked
  if (j < __ldg(cu + n_seq)) {
    int lo = 0, hi = n_seq - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (__ldg(cu + mid) <= j) lo = mid;
      else hi = mid - 1;
    }
    l0 = __ldg(cu + lo + 1);             // rows after the sequence
    u1 = causal ? j : __ldg(cu + lo);    // rows before the key (causal) or before the sequence
  }
  lts[j] = l0;
  lte[j] = l1;
  uts[j] = 0;
  ute[j] = u1;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct MetaLayout {
  size_t minmax, row_count, row_entries, col_count, col_entries, cls, fwd_order, bwd_order, done, total;
};

bool meta_layout(const fm_mask_desc* d, MetaLayout* L) {
  if (!d || d->B < 1 || d->Hm < 1 || d->n_q < 1 || d->n_k < 1 || d->tile_q != kTile || d->tile_k != kTile)
    return false;
  const size_t BHm = (size_t)d->B * d->Hm;
  const size_t T_q = (d->n_q + kTile - 1) / kTile, T_k = (d->n_k + kTile - 1) / kTile;
  if (T_k >= (1u << 29) || T_q >= (1u << 29)) return false;
  size_t off = 0;
  L->minmax = off;
  off = align256(off + BHm * T_k * 8 * 4);
  L->row_count = off;
  off = align256(off + BHm * T_q * 4);
  L->row_entries = off;
  off = align256(off + BHm * T_q * T_k * 4);
  L->col_count = off;
  off = align256(off + BHm * T_k * 4);
  L->col_entries = off;
  off = align256(off + BHm * T_k * T_q * 4);
  L->cls = off;
  off = align256(off + BHm * T_q * T_k);
  L->fwd_order = off;
  off = align256(off + BHm * ((T_q + 1) / 2) * 4);
  L->bwd_order = off;
  off = align256(off + BHm * T_k * 4);
  L->done = off;
  off = align256(off + BHm * 4);
  L->total = off;
  return true;
}

}  // namespace
}  // namespace fm

extern "C" {

size_t fm_mask_meta_workspace_bytes(const fm_mask_desc* d) {
  fm::MetaLayout L;
  return fm::meta_layout(d, &L) ? L.total : 0;
}

fm_status fm_build_mask_meta(const fm_mask_desc* d, const int32_t* lts, const int32_t* lte, const int32_t* uts,
                             const int32_t* ute, void* ws, size_t ws_bytes, fm_mask_meta* out,
                             fm_stream_t stream) {
  fm::MetaLayout L;
  if (!out || !fm::meta_layout(d, &L)) return FM_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || ws_bytes < L.total) return FM_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  out->d = *d;
  out->tile_minmax = reinterpret_cast<int32_t*>(w + L.minmax);
  out->row_count = reinterpret_cast<int32_t*>(w + L.row_count);
  out->row_entries = reinterpret_cast<int32_t*>(w + L.row_entries);
  out->col_count = reinterpret_cast<int32_t*>(w + L.col_count);
  out->col_entries = reinterpret_cast<int32_t*>(w + L.col_entries);
  out->tile_class = w + L.cls;
  out->fwd_order = reinterpret_cast<int32_t*>(w + L.fwd_order);
  out->bwd_order = reinterpret_cast<int32_t*>(w + L.bwd_order);

  fm::MetaParams p;
  p.vec[0] = lts;
  p.vec[1] = lte;
  p.vec[2] = uts;
  p.vec[3] = ute;
  p.minmax = out->tile_minmax;
  p.cls = out->tile_class;
  p.row_count = out->row_count;
  p.row_entries = out->row_entries;
  p.col_count = out->col_count;
  p.col_entries = out->col_entries;
  p.fwd_order = out->fwd_order;
  p.bwd_order = out->bwd_order;
  p.done = reinterpret_cast<int32_t*>(w + L.done);
  p.BHm = d->B * d->Hm;
  p.n_q = d->n_q;
  p.n_k = d->n_k;
  p.T_q = (d->n_q + fm::kTile - 1) / fm::kTile;
  p.T_k = (d->n_k + fm::kTile - 1) / fm::kTile;
  if (p.BHm > 65535) return FM_ERR_UNSUPPORTED;  // grid.y of the query-tile pass
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // Lists per launch against the warps the GPU holds (148 SMs x 64): in the query-tile pass, a quad of
  // warps per list when fewer warps would leave most of the GPU idle, four lists per warp otherwise.
  constexpr int64_t kWarpsResident = 148 * 64;
  const int64_t tiles_k = (int64_t)p.BHm * p.T_k, tiles_q = (int64_t)p.BHm * p.T_q;
  fm::meta_cols_kernel<<<(unsigned)((tiles_k + 7) / 8), fm::kColsThreads, 0, s>>>(p);
  // the query-tile pass stages the (b, hm)'s min/max in shared memory (32 B per key tile, <= 128 KiB)
  const int rows_smem = p.T_k <= fm::kOrderMax ? p.T_k * 32 : 0;
  if (4 * tiles_q <= 2 * kWarpsResident && p.T_k <= fm::kOrderListMax) {
    if (!fm::smem_opt_in<fm::meta_rows_kernel<true>>(fm::kOrderMax * 32)) return FM_ERR_CUDA;  // + 33 KiB static
    fm::meta_rows_kernel<true><<<dim3((unsigned)((p.T_q + 7) / 8), (unsigned)p.BHm), fm::kRowsThreads, rows_smem, s>>>(p);
  } else {
    constexpr int kPerCta = fm::kRowsThreads / 32 * fm::kTilesPerWarp;
    if (!fm::smem_opt_in<fm::meta_rows_kernel<false>>(fm::kOrderMax * 32)) return FM_ERR_CUDA;
    fm::meta_rows_kernel<false><<<dim3((unsigned)((p.T_q + kPerCta - 1) / kPerCta), (unsigned)p.BHm), fm::kRowsThreads,
                                  rows_smem, s>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? FM_OK : FM_ERR_CUDA;
}

fm_status fm_varlen_mask(const int32_t* cu_seqlens, int32_t n_seq, int32_t N, int32_t causal, int32_t* lts,
                         int32_t* lte, int32_t* uts, int32_t* ute, fm_stream_t stream) {
  if (!cu_seqlens || !lts || !lte || !uts || !ute || n_seq < 1 || n_seq > (1 << 20) || N < 1 ||
      (causal != 0 && causal != 1))
    return FM_ERR_INVALID_ARG;
  const uintptr_t al = reinterpret_cast<uintptr_t>(cu_seqlens) | reinterpret_cast<uintptr_t>(lts) |
                       reinterpret_cast<uintptr_t>(lte) | reinterpret_cast<uintptr_t>(uts) |
                       reinterpret_cast<uintptr_t>(ute);
  if (al & 3) return FM_ERR_INVALID_ARG;
  fm::varlen_mask_kernel<<<(unsigned)(((int64_t)N + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      cu_seqlens, n_seq, N, causal, lts, lte, uts, ute);
  return cudaGetLastError() == cudaSuccess ? FM_OK : FM_ERR_CUDA;
}

}  // extern "C"
