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

struct MetaParams {
  const int32_t* vec[4];  // [B, Hm, n_k] or null
  bool vec16;             // every vector row starts 16-byte aligned (n_k % 4 == 0): 16-byte loads
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

// 0 skip, 1 partial, 2 full for query rows [r0, r1) against one key tile's min/max.
__device__ __forceinline__ int classify(const int4 lo, const int4 hi, int64_t r0, int64_t r1) {
  // lo = (minLTS, maxLTS, minLTE, maxLTE), hi = (minUTS, maxUTS, minUTE, maxUTE)
  const bool skip = ((int64_t)lo.y <= r0 && (int64_t)lo.z >= r1) || ((int64_t)hi.y <= r0 && (int64_t)hi.z >= r1);
  const bool clear_l = ((int64_t)lo.x >= r1) || ((int64_t)lo.w <= r0);
  const bool clear_u = ((int64_t)hi.x >= r1) || ((int64_t)hi.w <= r0);
  return skip ? 0 : ((clear_l && clear_u) ? 2 : 1);
}

// Key-tile pass: one warp per (bhm, key tile).  Min and max of the four vectors over the tile's 128
// columns (one 16-byte load per lane and vector when the rows are 16-byte aligned), written to
// minmax, then the tile's column list: every query tile classified against those eight values,
// 32 per step, the non-skip ones compacted in ascending order.  Also clears the per-bhm counter
// of the query-tile pass.
__global__ void __launch_bounds__(256) meta_cols_kernel(const MetaParams p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= p.BHm * p.T_k) return;
  const int bhm = warp / p.T_k, kt = warp % p.T_k;
  if (kt == 0 && lane == 0) p.done[bhm] = 0;
  const int32_t dflt[4] = {p.n_q, p.n_q, 0, 0};
  int32_t mn[4], mx[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    mn[c] = INT_MAX;
    mx[c] = INT_MIN;
  }
  const int64_t base = (int64_t)bhm * p.n_k;
  const int64_t j0 = (int64_t)kt * kTile;
  if (p.vec16) {
    const int64_t j = j0 + 4 * lane;  // n_k % 4 == 0: a group of 4 is either inside or past the end
    if (j < p.n_k) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        int4 v = make_int4(dflt[c], dflt[c], dflt[c], dflt[c]);
        if (p.vec[c]) v = __ldg(reinterpret_cast<const int4*>(p.vec[c] + base + j));
        mn[c] = min(min(v.x, v.y), min(v.z, v.w));
        mx[c] = max(max(v.x, v.y), max(v.z, v.w));
      }
    }
  } else {
    for (int t = lane; t < kTile; t += 32) {
      const int64_t j = j0 + t;
      if (j >= p.n_k) break;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int32_t v = vec_at(p.vec[c], base + j, dflt[c]);
        mn[c] = min(mn[c], v);
        mx[c] = max(mx[c], v);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      mn[c] = min(mn[c], __shfl_xor_sync(0xffffffffu, mn[c], off));
      mx[c] = max(mx[c], __shfl_xor_sync(0xffffffffu, mx[c], off));
    }
  }
  if (lane < 8) {
    const int c = lane >> 1;
    int32_t val = (lane & 1) ? mx[0] : mn[0];
    // select without dynamic register indexing
    val = (c == 1) ? ((lane & 1) ? mx[1] : mn[1]) : val;
    val = (c == 2) ? ((lane & 1) ? mx[2] : mn[2]) : val;
    val = (c == 3) ? ((lane & 1) ? mx[3] : mn[3]) : val;
    p.minmax[((int64_t)bhm * p.T_k + kt) * 8 + lane] = val;
  }
  // column list of this key tile
  const int4 lo = make_int4(mn[0], mx[0], mn[1], mx[1]), hi = make_int4(mn[2], mx[2], mn[3], mx[3]);
  const unsigned below = (1u << lane) - 1u;
  int32_t* ent = p.col_entries + ((int64_t)bhm * p.T_k + kt) * p.T_q;
  int count = 0;
  for (int q0 = 0; q0 < p.T_q; q0 += 32) {
    const int qt = q0 + lane;
    int c = 0;
    if (qt < p.T_q) {
      const int64_t r0 = (int64_t)qt * kTile, r1 = (r0 + kTile < p.n_q) ? r0 + kTile : (int64_t)p.n_q;
      c = classify(lo, hi, r0, r1);
    }
    const unsigned keep = __ballot_sync(0xffffffffu, c != 0);
    if (c != 0) ent[count + __popc(keep & below)] = (qt << 1) | (c == 1 ? 1 : 0);
    count += __popc(keep);
  }
  if (lane == 0) p.col_count[(int64_t)bhm * p.T_k + kt] = count;
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

// Query-tile pass: grid (ceil(T_q / 32), BHm), 1024 threads, one warp per query tile: its row of the
// class matrix and its row list (key tiles scanned 32 at a time against the key-tile pass's min/max).
// The CTA that completes a (b, hm) last also writes that (b, hm)'s two dispatch orders.
__global__ void __launch_bounds__(kRowsThreads) meta_rows_kernel(const MetaParams p) {
  extern __shared__ int4 mm_smem[];  // this (b, hm)'s min/max, 2 x int4 per key tile (when it fits)
  __shared__ uint32_t key_f[kOrderMax / 2];
  __shared__ uint32_t key_b[kOrderMax];
  __shared__ int last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bhm = blockIdx.y, qt = blockIdx.x * (kRowsThreads / 32) + warp;
  const unsigned below = (1u << lane) - 1u;
  const int4* mm_g = reinterpret_cast<const int4*>(p.minmax + (int64_t)bhm * p.T_k * 8);
  const bool staged = p.T_k <= kOrderMax;  // the launch gives 32 B of shared memory per key tile up to 4096
  if (staged) {
    for (int k = threadIdx.x; k < 2 * p.T_k; k += blockDim.x) mm_smem[k] = __ldg(mm_g + k);
    __syncthreads();
  }
  if (qt < p.T_q) {
    const int64_t r0 = (int64_t)qt * kTile, r1 = (r0 + kTile < p.n_q) ? r0 + kTile : (int64_t)p.n_q;
    const int4* mm = staged ? mm_smem : mm_g;
    uint8_t* cls = p.cls + ((int64_t)bhm * p.T_q + qt) * p.T_k;
    int32_t* ent = p.row_entries + ((int64_t)bhm * p.T_q + qt) * p.T_k;
    int count = 0;
    for (int k0 = 0; k0 < p.T_k; k0 += 32) {
      const int kt = k0 + lane;
      int c = 0;
      if (kt < p.T_k) {
        c = classify(mm[2 * kt], mm[2 * kt + 1], r0, r1);
        cls[kt] = (uint8_t)c;
      }
      const unsigned keep = __ballot_sync(0xffffffffu, c != 0);
      if (c != 0) ent[count + __popc(keep & below)] = (kt << 1) | (c == 1 ? 1 : 0);
      count += __popc(keep);
    }
    if (lane == 0) p.row_count[(int64_t)bhm * p.T_q + qt] = count;
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
  uintptr_t al = (uintptr_t)(d->n_k % 4);
  for (int c = 0; c < 4; ++c) al |= reinterpret_cast<uintptr_t>(p.vec[c]) & 15u;
  p.vec16 = al == 0;
  if (p.BHm > 65535) return FM_ERR_UNSUPPORTED;  // grid.y of the query-tile pass
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t warps_k = (int64_t)p.BHm * p.T_k;
  fm::meta_cols_kernel<<<(unsigned)((warps_k + 7) / 8), 256, 0, s>>>(p);
  // the query-tile pass stages the (b, hm)'s min/max in shared memory (32 B per key tile, <= 128 KiB)
  const int rows_smem = p.T_k <= fm::kOrderMax ? p.T_k * 32 : 0;
  if (!fm::smem_opt_in<fm::meta_rows_kernel>(fm::kOrderMax * 32)) return FM_ERR_CUDA;  // + 24 KiB static
  fm::meta_rows_kernel<<<dim3((unsigned)((p.T_q + 31) / 32), (unsigned)p.BHm), fm::kRowsThreads, rows_smem, s>>>(p);
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
