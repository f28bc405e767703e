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
  int32_t* minmax;        // [BHm, T_k, 8]
  uint8_t* cls;           // [BHm, T_q, T_k]
  int32_t* row_count;     // [BHm, T_q]
  int32_t* row_entries;   // [BHm, T_q, T_k]
  int32_t* col_count;     // [BHm, T_k]
  int32_t* col_entries;   // [BHm, T_k, T_q]
  int32_t* fwd_order;     // [BHm, ceil(T_q / 2)]
  int32_t* bwd_order;     // [BHm, T_k]
  int32_t BHm, n_q, n_k, T_q, T_k;
};

__device__ __forceinline__ int32_t vec_at(const int32_t* v, int64_t idx, int32_t dflt) {
  return v ? __ldg(v + idx) : dflt;
}

// One warp per key tile: lanes stride over the tile's 128 columns.
__global__ void __launch_bounds__(256) meta_minmax_kernel(const MetaParams p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= p.BHm * p.T_k) return;
  const int bhm = warp / p.T_k, kt = warp % p.T_k;
  const int32_t dflt[4] = {p.n_q, p.n_q, 0, 0};
  int32_t mn[4], mx[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    mn[c] = INT_MAX;
    mx[c] = INT_MIN;
  }
  const int64_t base = (int64_t)bhm * p.n_k;
  for (int t = lane; t < kTile; t += 32) {
    const int64_t j = (int64_t)kt * kTile + t;
    if (j >= p.n_k) break;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int32_t v = vec_at(p.vec[c], base + j, dflt[c]);
      mn[c] = min(mn[c], v);
      mx[c] = max(mx[c], v);
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
}

// 0 skip, 1 partial, 2 full for query rows [r0, r1) against one key tile's min/max.
__device__ __forceinline__ int classify(const int4 lo, const int4 hi, int64_t r0, int64_t r1) {
  // lo = (minLTS, maxLTS, minLTE, maxLTE), hi = (minUTS, maxUTS, minUTE, maxUTE)
  const bool skip = ((int64_t)lo.y <= r0 && (int64_t)lo.z >= r1) || ((int64_t)hi.y <= r0 && (int64_t)hi.z >= r1);
  const bool clear_l = ((int64_t)lo.x >= r1) || ((int64_t)lo.w <= r0);
  const bool clear_u = ((int64_t)hi.x >= r1) || ((int64_t)hi.w <= r0);
  return skip ? 0 : ((clear_l && clear_u) ? 2 : 1);
}

// Row lists (blockIdx.y == 0): one warp per (bhm, query tile), scanning key
// tiles 32 at a time; column lists (blockIdx.y == 1): one warp per (bhm, key tile).
__global__ void __launch_bounds__(256) meta_lists_kernel(const MetaParams p) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const unsigned below = (1u << lane) - 1u;
  if (blockIdx.y == 0) {
    if (warp >= p.BHm * p.T_q) return;
    const int bhm = warp / p.T_q, qt = warp % p.T_q;
    const int64_t r0 = (int64_t)qt * kTile, r1 = (r0 + kTile < p.n_q) ? r0 + kTile : (int64_t)p.n_q;
    const int4* mm = reinterpret_cast<const int4*>(p.minmax + (int64_t)bhm * p.T_k * 8);
    uint8_t* cls = p.cls + ((int64_t)bhm * p.T_q + qt) * p.T_k;
    int32_t* ent = p.row_entries + ((int64_t)bhm * p.T_q + qt) * p.T_k;
    int count = 0;
    for (int k0 = 0; k0 < p.T_k; k0 += 32) {
      const int kt = k0 + lane;
      int c = 0;
      if (kt < p.T_k) {
        c = classify(__ldg(mm + 2 * kt), __ldg(mm + 2 * kt + 1), r0, r1);
        cls[kt] = (uint8_t)c;
      }
      const unsigned keep = __ballot_sync(0xffffffffu, c != 0);
      if (c != 0) ent[count + __popc(keep & below)] = (kt << 1) | (c == 1 ? 1 : 0);
      count += __popc(keep);
    }
    if (lane == 0) p.row_count[(int64_t)bhm * p.T_q + qt] = count;
  } else {
    if (warp >= p.BHm * p.T_k) return;
    const int bhm = warp / p.T_k, kt = warp % p.T_k;
    const int4* mm = reinterpret_cast<const int4*>(p.minmax + ((int64_t)bhm * p.T_k + kt) * 8);
    const int4 lo = __ldg(mm), hi = __ldg(mm + 1);
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

// Dispatch orders for the attention kernels (longest first).  One CTA per
// (b, hm) and direction: blockIdx.y = 0 orders query-tile pairs by the sum of
// their two row counts, 1 orders key tiles by column count; ties keep
// ascending index.  Bitonic sort in shared memory of the keys
// (cost << 16) | (0xFFFF - index), descending; with at most 4096 items and
// costs below 2^16 the keys are distinct, so the order is deterministic.
constexpr int kOrderMax = 4096;
__global__ void __launch_bounds__(1024) meta_order_kernel(const MetaParams p) {
  __shared__ uint32_t key[kOrderMax];
  const int bhm = blockIdx.x;
  const bool fwd = blockIdx.y == 0;
  const int n = fwd ? (p.T_q + 1) / 2 : p.T_k;
  int32_t* out = fwd ? p.fwd_order + (int64_t)bhm * n : p.bwd_order + (int64_t)bhm * n;
  if (p.T_q > kOrderMax || p.T_k > kOrderMax) {  // sizes the attention kernels do not take
    for (int i = threadIdx.x; i < n; i += blockDim.x) out[i] = i;
    return;
  }
  int np2 = 1;
  while (np2 < n) np2 <<= 1;
  const int32_t* rc = p.row_count + (int64_t)bhm * p.T_q;
  const int32_t* cc = p.col_count + (int64_t)bhm * p.T_k;
  for (int i = threadIdx.x; i < np2; i += blockDim.x) {
    uint32_t k = 0;  // padding sorts last
    if (i < n) {
      const uint32_t cost = fwd ? (uint32_t)(rc[2 * i] + (2 * i + 1 < p.T_q ? rc[2 * i + 1] : 0)) : (uint32_t)cc[i];
      k = (cost << 16) | (0xFFFFu - (uint32_t)i);
    }
    key[i] = k;
  }
  __syncthreads();
  for (int len = 2; len <= np2; len <<= 1) {
    for (int j = len >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < np2; i += blockDim.x) {
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
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < n; i += blockDim.x) out[i] = (int32_t)(0xFFFFu - (key[i] & 0xFFFFu));
}

struct MetaLayout {
  size_t minmax, row_count, row_entries, col_count, col_entries, cls, fwd_order, bwd_order, total;
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
  p.BHm = d->B * d->Hm;
  p.n_q = d->n_q;
  p.n_k = d->n_k;
  p.T_q = (d->n_q + fm::kTile - 1) / fm::kTile;
  p.T_k = (d->n_k + fm::kTile - 1) / fm::kTile;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t warps_mm = (int64_t)p.BHm * p.T_k;
  fm::meta_minmax_kernel<<<(unsigned)((warps_mm + 7) / 8), 256, 0, s>>>(p);
  const int64_t warps_l = (int64_t)p.BHm * (p.T_q > p.T_k ? p.T_q : p.T_k);
  fm::meta_lists_kernel<<<dim3((unsigned)((warps_l + 7) / 8), 2), 256, 0, s>>>(p);
  fm::meta_order_kernel<<<dim3((unsigned)p.BHm, 2), 1024, 0, s>>>(p);
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
