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
