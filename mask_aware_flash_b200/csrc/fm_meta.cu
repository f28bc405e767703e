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

__device__ __forceinline__ int32_t vec_at(const int32_t* v, int64_t idx, int32_t dflt) {
  return v ? __ldg(v + idx) : dflt;
}

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

// One list (a query tile's row over the key tiles, or a key tile's column over the query tiles)
// built by a quad of four warps: warp w of the quad classifies positions [w c, (w + 1) c) with
// c = 32 ceil(L / 128), 32 at a time, keeping the ballots of "non-skip" and "partial" in shared
// memory (masks: 2 x L / 32 words for the quad); after the quad's named barrier each warp knows how
// many entries the warps before it keep and writes its own entries (index << 1 | partial) in
// ascending order.  class_of(idx) gives the class; on_class(idx, c) sees every classified position.
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

// The same list built by one warp alone, in one pass (a running count of kept positions), for
// launches large enough to fill the GPU with one warp per list.
template <typename ClassOf, typename OnClass>
__device__ __forceinline__ int warp_list(int L, int lane, int32_t* ent, ClassOf class_of, OnClass on_class) {
  const unsigned below = (1u << lane) - 1u;
  int count = 0;
  for (int k0 = 0; k0 < L; k0 += 32) {
    const int idx = k0 + lane;
    int c = 0;
    if (idx < L) {
      c = class_of(idx);
      on_class(idx, c);
    }
    const unsigned keep = __ballot_sync(0xffffffffu, c != 0);
    if (c != 0) ent[count + __popc(keep & below)] = (idx << 1) | (c == 1 ? 1 : 0);
    count += __popc(keep);
  }
  return count;
}

// Key-tile pass: W warps (a quad, or one) per (bhm, key tile), 8 / W tiles per CTA.  Min and max of
// the four vectors over the tile's 128 columns (each warp reads its share, one column per lane;
// a quad combines in shared memory), written to minmax, then the tile's column list over all query
// tiles.  Also clears the per-bhm counter of the query-tile pass.
constexpr int kColsThreads = 256;
constexpr int kMaskWords = 2 * kOrderListMax / 32;
template <int W>  // warps per key tile: 4 (a quad) or 1
__global__ void __launch_bounds__(kColsThreads) meta_cols_kernel(const MetaParams p) {
  constexpr int kLists = kColsThreads / 32 / W;  // key tiles per CTA
  __shared__ int4 red[kLists][W][2];
  __shared__ uint32_t masks[W == 4 ? kLists : 1][W == 4 ? kMaskWords : 1];
  __shared__ int counts[kLists][4];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, quad = warp / W, wq = warp % W;
  const int64_t tile = (int64_t)blockIdx.x * kLists + quad;  // (bhm, key tile)
  const bool live = tile < (int64_t)p.BHm * p.T_k;
  const int bhm = live ? (int)(tile / p.T_k) : 0, kt = live ? (int)(tile % p.T_k) : 0;
  if (live && kt == 0 && threadIdx.x == quad * 32 * W) p.done[bhm] = 0;
  const int32_t dflt[4] = {p.n_q, p.n_q, 0, 0};
  int32_t mn[4], mx[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    mn[c] = INT_MAX;
    mx[c] = INT_MIN;
    for (int t = wq * 32 + lane; t < kTile; t += 32 * W) {  // columns of this warp's share
      const int64_t j = (int64_t)kt * kTile + t;
      if (live && j < p.n_k) {
        const int32_t v = vec_at(p.vec[c], (int64_t)bhm * p.n_k + j, dflt[c]);
        mn[c] = min(mn[c], v);
        mx[c] = max(mx[c], v);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      mn[c] = min(mn[c], __shfl_xor_sync(0xffffffffu, mn[c], off));
      mx[c] = max(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], off));
    }
  }
  if (lane == 0) {
    red[quad][wq][0] = make_int4(mn[0], mx[0], mn[1], mx[1]);
    red[quad][wq][1] = make_int4(mn[2], mx[2], mn[3], mx[3]);
  }
  __syncthreads();
  int4 lo = red[quad][0][0], hi = red[quad][0][1];
#pragma unroll
  for (int w = 1; w < W; ++w) {
    const int4 a = red[quad][w][0], b = red[quad][w][1];
    lo = make_int4(min(lo.x, a.x), max(lo.y, a.y), min(lo.z, a.z), max(lo.w, a.w));
    hi = make_int4(min(hi.x, b.x), max(hi.y, b.y), min(hi.z, b.z), max(hi.w, b.w));
  }
  if (!live) return;  // (a whole quad: the barrier below is per quad)
  if (wq == 0 && lane < 8) {
    const int32_t v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    int32_t val = v[0];
#pragma unroll
    for (int k = 1; k < 8; ++k) val = (lane == k) ? v[k] : val;  // select without dynamic indexing
    p.minmax[tile * 8 + lane] = val;
  }
  int32_t* ent = p.col_entries + tile * p.T_q;
  auto class_of = [&](int qt) { return classify(lo, hi, qt * kTile, tile_r1(qt * kTile, p.n_q)); };
  auto none = [](int, int) {};
  int n;
  if constexpr (W == 4)
    n = quad_list(p.T_q, wq, lane, 1 + quad, masks[quad], counts[quad], ent, class_of, none);
  else
    n = warp_list(p.T_q, lane, ent, class_of, none);
  if (wq == 0 && lane == 0) p.col_count[tile] = n;
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

// Query-tile pass: grid (ceil(T_q / (32 / W)), BHm), 1024 threads, W warps per query tile:
// its row of the class matrix and its row list (quad_list over the key tiles, against the key-tile
// pass's min/max staged in shared memory).  The CTA that completes a (b, hm) last also writes that
// (b, hm)'s two dispatch orders.
template <int W>  // warps per query tile: 4 (a quad) or 1
__global__ void __launch_bounds__(kRowsThreads) meta_rows_kernel(const MetaParams p) {
  constexpr int kLists = kRowsThreads / 32 / W;  // query tiles per CTA
  extern __shared__ int4 mm_smem[];  // this (b, hm)'s min/max, 2 x int4 per key tile (when it fits)
  __shared__ uint32_t key_f[kOrderMax / 2];
  __shared__ uint32_t key_b[kOrderMax];
  __shared__ uint32_t masks[W == 4 ? kLists : 1][W == 4 ? kMaskWords : 1];
  __shared__ int counts[kLists][4];
  __shared__ int last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, quad = warp / W, wq = warp % W;
  const int bhm = blockIdx.y, qt = blockIdx.x * kLists + quad;
  const int4* mm_g = reinterpret_cast<const int4*>(p.minmax + (int64_t)bhm * p.T_k * 8);
  const bool staged = p.T_k <= kOrderMax;  // the launch gives 32 B of shared memory per key tile up to 4096
  if (staged) {
    for (int k = threadIdx.x; k < 2 * p.T_k; k += blockDim.x) mm_smem[k] = __ldg(mm_g + k);
    __syncthreads();
  }
  if (qt < p.T_q) {
    const int r0 = qt * kTile, r1 = tile_r1(r0, p.n_q);
    const int4* mm = staged ? mm_smem : mm_g;
    uint8_t* cls = p.cls + ((int64_t)bhm * p.T_q + qt) * p.T_k;
    int32_t* ent = p.row_entries + ((int64_t)bhm * p.T_q + qt) * p.T_k;
    auto class_of = [&](int kt) { return classify(mm[2 * kt], mm[2 * kt + 1], r0, r1); };
    auto store_class = [&](int kt, int c) { cls[kt] = (uint8_t)c; };
    int n;
    if constexpr (W == 4)
      n = quad_list(p.T_k, wq, lane, 1 + quad, masks[quad], counts[quad], ent, class_of, store_class);
    else
      n = warp_list(p.T_k, lane, ent, class_of, store_class);
    if (wq == 0 && lane == 0) p.row_count[(int64_t)bhm * p.T_q + qt] = n;
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
  // Lists per launch against the warps the GPU holds (148 SMs x 64): a quad of warps per list when
  // one warp per list would leave most of the GPU idle, one warp per list otherwise.
  constexpr int64_t kWarpsResident = 148 * 64;
  const int64_t tiles_k = (int64_t)p.BHm * p.T_k, tiles_q = (int64_t)p.BHm * p.T_q;
  if (4 * tiles_k <= 2 * kWarpsResident)
    fm::meta_cols_kernel<4><<<(unsigned)((tiles_k + 1) / 2), fm::kColsThreads, 0, s>>>(p);
  else
    fm::meta_cols_kernel<1><<<(unsigned)((tiles_k + 7) / 8), fm::kColsThreads, 0, s>>>(p);
  // the query-tile pass stages the (b, hm)'s min/max in shared memory (32 B per key tile, <= 128 KiB)
  const int rows_smem = p.T_k <= fm::kOrderMax ? p.T_k * 32 : 0;
  if (4 * tiles_q <= 2 * kWarpsResident) {
    if (!fm::smem_opt_in<fm::meta_rows_kernel<4>>(fm::kOrderMax * 32)) return FM_ERR_CUDA;  // + 33 KiB static
    fm::meta_rows_kernel<4><<<dim3((unsigned)((p.T_q + 7) / 8), (unsigned)p.BHm), fm::kRowsThreads, rows_smem, s>>>(p);
  } else {
    if (!fm::smem_opt_in<fm::meta_rows_kernel<1>>(fm::kOrderMax * 32)) return FM_ERR_CUDA;
    fm::meta_rows_kernel<1><<<dim3((unsigned)((p.T_q + 31) / 32), (unsigned)p.BHm), fm::kRowsThreads, rows_smem, s>>>(p);
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
