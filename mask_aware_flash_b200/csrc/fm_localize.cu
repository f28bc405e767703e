// Clip-shift-max localization of the four boundary vectors to context-parallel
// ranks.  FlashMask-3 explainer (learnaivisually.com), clip-shift-max paragraph:
// the vectors are indexed by key but hold query-row numbers, so a rank that owns
// some query chunks can "crop the global marks to its own chunks and renumber
// them from its local zero": clip each mark to a chunk, shift it into the rank's
// concatenated numbering, and keep the maximum over the rank's chunks (Theorem 1:
// the local intervals equal the global ones at the corresponding rows).  The
// paper abstract calls this a "provably zero-communication clip-shift-max".
// All ranks are produced by one launch (each input value read once).
#include "fm_common.cuh"

namespace fm {
namespace {

constexpr int kMaxChunks = 256;

struct LocParams {
  const int32_t* in[4];
  int32_t* out[4];
  int32_t start[kMaxChunks];  // global start of chunk (r, k) at r*C + k
  int32_t len[kMaxChunks];
  int32_t off[kMaxChunks];    // local offset of chunk k inside rank r
  int64_t cols;               // B * Hm * N
  int32_t R, C;
};

__global__ void __launch_bounds__(256) localize_kernel(const LocParams p) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= p.cols) return;
  int32_t v[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) v[c] = __ldg(p.in[c] + j);
  for (int r = 0; r < p.R; ++r) {
    int64_t best[4] = {0, 0, 0, 0};
    for (int k = 0; k < p.C; ++k) {
      const int idx = r * p.C + k;
      const int64_t shift = (int64_t)p.off[idx] - p.start[idx];  // clip to chunk, shift to local numbering
      const int64_t hi = (int64_t)p.off[idx] + p.len[idx];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        int64_t x = (int64_t)v[c] + shift;
        x = x < 0 ? 0 : (x > hi ? hi : x);
        best[c] = x > best[c] ? x : best[c];  // max over the rank's chunks
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) p.out[c][(int64_t)r * p.cols + j] = (int32_t)best[c];
  }
}

}  // namespace
}  // namespace fm

extern "C" fm_status fm_localize(int32_t B, int32_t Hm, int32_t N, const int32_t* const in[4], int32_t R,
                                 int32_t C, const int32_t* chunk_start, const int32_t* chunk_len,
                                 int32_t* const out[4], fm_stream_t stream) {
  if (B < 1 || Hm < 1 || N < 1 || R < 1 || C < 1 || (int64_t)R * C > fm::kMaxChunks) return FM_ERR_INVALID_ARG;
  if (!in || !out || !chunk_start || !chunk_len) return FM_ERR_INVALID_ARG;
  fm::LocParams p;
  for (int c = 0; c < 4; ++c) {
    if (!in[c] || !out[c]) return FM_ERR_INVALID_ARG;
    p.in[c] = in[c];
    p.out[c] = out[c];
  }
  for (int r = 0; r < R; ++r) {
    int64_t acc = 0, prev_end = -1;
    for (int k = 0; k < C; ++k) {
      const int idx = r * C + k;
      const int64_t s = chunk_start[idx], L = chunk_len[idx];
      if (L < 1 || s < 0 || s + L > N) return FM_ERR_INVALID_ARG;
      if (s < prev_end) return FM_ERR_INVALID_ARG;  // chunks must increase and not overlap
      prev_end = s + L;
      p.start[idx] = (int32_t)s;
      p.len[idx] = (int32_t)L;
      p.off[idx] = (int32_t)acc;
      acc += L;
    }
  }
  p.cols = (int64_t)B * Hm * N;
  p.R = R;
  p.C = C;
  const unsigned blocks = (unsigned)((p.cols + 255) / 256);
  fm::localize_kernel<<<blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? FM_OK : FM_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// KV-chunk pruning.  For each simulated rank, the number of unmasked (local
// query row, key) pairs whose key falls in each KV chunk; a chunk with none is
// never needed by the rank's queries, so its K/V need not be sent there.  Per
// key the count is the rank's row count minus the length of the union of the
// two localized intervals clipped to [0, n_loc): O(1) per key, summed exactly
// in int64 (one block per (chunk, rank, b, hm)).
// ---------------------------------------------------------------------------
namespace fm {
namespace {

constexpr int kMaxRanks = 256;

struct ChunkParams {
  const int32_t* vec[4];  // [R, B, Hm, N] or null
  int64_t* pairs;         // [R, B, Hm, n_chunks]
  int32_t n_loc[kMaxRanks];
  int64_t cols;           // B * Hm * N
  int32_t BHm, N, chunk_len, n_chunks;
};

__device__ __forceinline__ int64_t unmasked_rows(int64_t n, int64_t lts, int64_t lte, int64_t uts, int64_t ute) {
  const int64_t a0 = lts < 0 ? 0 : (lts > n ? n : lts), a1 = lte < 0 ? 0 : (lte > n ? n : lte);
  const int64_t b0 = uts < 0 ? 0 : (uts > n ? n : uts), b1 = ute < 0 ? 0 : (ute > n ? n : ute);
  const int64_t la = a1 > a0 ? a1 - a0 : 0, lb = b1 > b0 ? b1 - b0 : 0;
  int64_t ov = 0;
  if (la > 0 && lb > 0) {
    const int64_t lo = a0 > b0 ? a0 : b0, hi = a1 < b1 ? a1 : b1;
    ov = hi > lo ? hi - lo : 0;
  }
  return n - (la + lb - ov);
}

__global__ void __launch_bounds__(256) kv_chunk_pairs_kernel(const ChunkParams p) {
  const int c = blockIdx.x;
  const int64_t rbh = blockIdx.y;  // r * BHm + (b * Hm + hm)
  const int r = (int)(rbh / p.BHm);
  const int64_t n = p.n_loc[r];
  const int64_t row = rbh * p.N;  // start of this (r, b, hm) vector
  const int j0 = c * p.chunk_len, j1 = min(j0 + p.chunk_len, p.N);
  int64_t acc = 0;
  for (int j = j0 + (int)threadIdx.x; j < j1; j += blockDim.x) {
    const int64_t lts = p.vec[0] ? __ldg(p.vec[0] + row + j) : n, lte = p.vec[1] ? __ldg(p.vec[1] + row + j) : n;
    const int64_t uts = p.vec[2] ? __ldg(p.vec[2] + row + j) : 0, ute = p.vec[3] ? __ldg(p.vec[3] + row + j) : 0;
    acc += unmasked_rows(n, lts, lte, uts, ute);
  }
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  __shared__ int64_t part[8];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += part[w];
    p.pairs[rbh * p.n_chunks + c] = t;
  }
}

}  // namespace
}  // namespace fm

extern "C" fm_status fm_kv_chunk_pairs(int32_t B, int32_t Hm, int32_t N, int32_t R, const int32_t* const vec[4],
                                       const int32_t* n_loc, int32_t chunk_len, int64_t* pairs,
                                       fm_stream_t stream) {
  if (B < 1 || Hm < 1 || N < 1 || R < 1 || R > fm::kMaxRanks || chunk_len < 1) return FM_ERR_INVALID_ARG;
  if (!vec || !n_loc || !pairs || (reinterpret_cast<uintptr_t>(pairs) & 7)) return FM_ERR_INVALID_ARG;
  if ((int64_t)R * B * Hm > 65535) return FM_ERR_UNSUPPORTED;  // one grid row per (rank, b, hm)
  fm::ChunkParams p;
  for (int c = 0; c < 4; ++c) p.vec[c] = vec[c];
  for (int r = 0; r < R; ++r) {
    if (n_loc[r] < 0) return FM_ERR_INVALID_ARG;
    p.n_loc[r] = n_loc[r];
  }
  p.pairs = pairs;
  p.BHm = B * Hm;
  p.N = N;
  p.chunk_len = chunk_len;
  p.n_chunks = (int32_t)(((int64_t)N + chunk_len - 1) / chunk_len);
  p.cols = (int64_t)B * Hm * N;
  fm::kv_chunk_pairs_kernel<<<dim3((unsigned)p.n_chunks, (unsigned)(R * B * Hm)), 256, 0,
                              reinterpret_cast<cudaStream_t>(stream)>>>(p);
  return cudaGetLastError() == cudaSuccess ? FM_OK : FM_ERR_CUDA;
}
