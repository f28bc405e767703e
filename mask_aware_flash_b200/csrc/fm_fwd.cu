// Mask-aware attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// FlashMask-3 explainer (learnaivisually.com), tile paragraph: tiles are
// "fully masked, partly masked or unmasked"; "fully masked tiles are never
// loaded" and "only partly masked tiles apply the row-interval test".  The
// pages' Hopper kernel (paper abstract: three-role warp specialisation on the
// FlashAttention-3 TMA/WGMMA pipeline) is prior art; this kernel is designed
// for Blackwell:
//   * one CTA per (query tile of 128 rows, head, batch), two CTAs per SM
//     (256 TMEM columns and ~101 KB shared memory each), so the tensor core of
//     an SM alternates between two independent softmax pipelines;
//   * warp 4 (one lane) issues TMA loads of Q once and of K/V plus the tile's
//     four boundary-vector slices (partial tiles only) for each entry of the
//     query tile's block list;
//   * warp 5 (one lane) issues tcgen05.mma: S = Q K^T into TMEM, then
//     O += P V with P read straight from TMEM (bf16, aliased over S);
//   * warps 0-3 (one thread per query row) read S from TMEM, apply the
//     row-interval test on partial tiles, run the online softmax in the log2
//     domain, write P back to TMEM, rescale O in TMEM when the row maximum
//     grows, and finally normalise O and write O and LSE.
// Every mbarrier wait is bounded; on a timeout the CTA records the failure in
// the device status word and unwinds (no wait can hang the GPU).
#include "fm_common.cuh"

namespace fm {
namespace {

constexpr int kTile = 128;
constexpr int kFwdThreads = 192;
constexpr float kNegInf = -__builtin_huge_valf();

struct FwdParams {
  const int32_t* row_count;    // [B, Hm, T_q]
  const int32_t* row_entries;  // [B, Hm, T_q, T_k]
  const int32_t* vec[4];       // [B, Hm, n_k] or null
  __nv_bfloat16* o;            // [B, n_q, H, D]
  float* lse;                  // [B, H, n_q]
  int* status;
  int B, H, Hm, n_q, n_k, T_q, T_k;
  float scale_log2;            // softmax scale * log2(e)
};

template <int D>
struct FwdSmem {
  static constexpr int kTileBytes = kTile * D * 2;  // 128 rows x D bf16 (D/64 swizzle-atom columns)
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + kTileBytes;
  static constexpr int kV = kK + kTileBytes;
  static constexpr int kMask = kV + kTileBytes;     // [2 buffers][4 vectors][128] int32
  static constexpr int kBar = kMask + 2 * 4 * kTile * 4;
  enum { Q_FULL, K_FULL, K_EMPTY, V_FULL, V_EMPTY, S_FULL, P_FULL, O_DONE, DRAIN, M_FULL0, M_FULL1, M_EMPTY0,
         M_EMPTY1, kNumBars };
  static constexpr int kMisc = kBar + kNumBars * 8;  // [0] TMEM base, [1] abort flag
  static constexpr int kBytes = kMisc + 16;
  static constexpr int kAlloc = kBytes + 1024;       // slack for 1024-byte alignment of the base
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 2)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using S = FwdSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.T_q - 1 - (int)blockIdx.x;  // long (late causal) query tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t bhm = (int64_t)b * p.Hm + (p.Hm == 1 ? 0 : h);
  const int cnt = __ldg(p.row_count + bhm * p.T_q + qt);
  const int32_t* entries = p.row_entries + (bhm * p.T_q + qt) * p.T_k;

  const uint32_t bar0 = smem_u32(smem + S::kBar);
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  const uint32_t q_s = smem_u32(smem + S::kQ), k_s = smem_u32(smem + S::kK), v_s = smem_u32(smem + S::kV);
  const int32_t* mask_smem = reinterpret_cast<const int32_t*>(smem + S::kMask);

  if (threadIdx.x == 0) {
    mbar_init(bar(S::Q_FULL), 1);
    mbar_init(bar(S::K_FULL), 1);
    mbar_init(bar(S::K_EMPTY), 1);
    mbar_init(bar(S::V_FULL), 1);
    mbar_init(bar(S::V_EMPTY), 1);
    mbar_init(bar(S::S_FULL), 1);
    mbar_init(bar(S::P_FULL), kTile);
    mbar_init(bar(S::O_DONE), 1);
    mbar_init(bar(S::DRAIN), 1);
    mbar_init(bar(S::M_FULL0), 1);
    mbar_init(bar(S::M_FULL1), 1);
    mbar_init(bar(S::M_EMPTY0), kTile);
    mbar_init(bar(S::M_EMPTY1), kTile);
    *abort_flag = 0;
    misc[2] = 0;  // a flag nothing raises: lets the final drain wait ignore aborts
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(misc), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const uint32_t tS = tmem, tO = tmem + 128;

  if (warp == 4) {
    // ------------------------------------------------------------ load role
    if (lane == 0 && cnt > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      int nvec = 0;
      for (int c = 0; c < 4; ++c) nvec += p.vec[c] ? 1 : 0;
      mbar_arrive_expect_tx(bar(S::Q_FULL), S::kTileBytes);
      for (int c = 0; c < D / 64; ++c) tma_load_4d(q_s + c * 16384, &tm_q, bar(S::Q_FULL), c * 64, h, qt * kTile, b);
      int pm = 0;
      for (int e = 0; e < cnt; ++e) {
        const int ent = ld_nc_i32(entries + e);
        const int kt = ent >> 1;
        if (e > 0 && !mbar_wait(bar(S::K_EMPTY), (e - 1) & 1, abort_flag)) {
          record_failure(p.status, abort_flag, 1);
          break;
        }
        mbar_arrive_expect_tx(bar(S::K_FULL), S::kTileBytes);
        for (int c = 0; c < D / 64; ++c) tma_load_4d(k_s + c * 16384, &tm_k, bar(S::K_FULL), c * 64, h, kt * kTile, b);
        if (ent & 1) {
          const int buf = pm & 1;
          if (pm >= 2 && !mbar_wait(bar(S::M_EMPTY0 + buf), ((pm >> 1) - 1) & 1, abort_flag)) {
            record_failure(p.status, abort_flag, 2);
            break;
          }
          mbar_arrive_expect_tx(bar(S::M_FULL0 + buf), 512u * nvec);
          for (int c = 0; c < 4; ++c)
            if (p.vec[c])
              bulk_load(smem_u32(mask_smem + (buf * 4 + c) * kTile), p.vec[c] + bhm * p.n_k + (int64_t)kt * kTile,
                        512u, bar(S::M_FULL0 + buf));
          ++pm;
        }
        if (e > 0 && !mbar_wait(bar(S::V_EMPTY), (e - 1) & 1, abort_flag)) {
          record_failure(p.status, abort_flag, 3);
          break;
        }
        mbar_arrive_expect_tx(bar(S::V_FULL), S::kTileBytes);
        for (int c = 0; c < D / 64; ++c) tma_load_4d(v_s + c * 16384, &tm_v, bar(S::V_FULL), c * 64, h, kt * kTile, b);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------- MMA role
    if (lane == 0 && cnt > 0) {
      constexpr uint32_t kIdescQK = idesc_bf16(128, 128, false, false);  // S[q][kv]: Q K-major, K K-major
      constexpr uint32_t kIdescPV = idesc_bf16(128, D, false, true);     // O[q][d]:  P (TMEM), V MN-major
      bool ok = mbar_wait(bar(S::Q_FULL), 0, abort_flag);
      for (int e = 0; ok && e < cnt; ++e) {
        if (!mbar_wait(bar(S::K_FULL), e & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const uint32_t off = (k >> 2) * 16384 + (k & 3) * 32;  // swizzle-atom column, 16-element K step
          umma_ss(tS, smem_desc(q_s + off, 16, 1024), smem_desc(k_s + off, 16, 1024), kIdescQK, k > 0 ? 1u : 0u);
        }
        umma_commit(bar(S::S_FULL));
        umma_commit(bar(S::K_EMPTY));
        if (!mbar_wait(bar(S::P_FULL), e & 1, abort_flag) || !mbar_wait(bar(S::V_FULL), e & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k)  // 16 kv rows per step; P columns advance 8 (bf16 pairs)
          umma_ts(tO, tS + k * 8, smem_desc(v_s + k * 2048, 16384, 1024), kIdescPV, (e > 0 || k > 0) ? 1u : 0u);
        umma_commit(bar(S::O_DONE));
        umma_commit(bar(S::V_EMPTY));
      }
      if (!ok) record_failure(p.status, abort_flag, 4);
      // drain: every MMA issued above has finished before TMEM is released
      umma_commit(bar(S::DRAIN));
      mbar_wait(bar(S::DRAIN), 0, reinterpret_cast<const volatile int*>(misc + 2));
    }
  } else {
    // ---------------------------------------------------------- softmax role
    const int r = threadIdx.x;  // row in tile == TMEM lane
    const int64_t i = (int64_t)qt * kTile + r;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    const bool has[4] = {p.vec[0] != nullptr, p.vec[1] != nullptr, p.vec[2] != nullptr, p.vec[3] != nullptr};
    float m_run = kNegInf, l_run = 0.f;
    int pm = 0;
    bool ok = true;
    for (int e = 0; e < cnt; ++e) {
      const int ent = ld_nc_i32(entries + e);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(S::S_FULL), e & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      // row-interval test, partial tiles only
      uint32_t mbits[4] = {0u, 0u, 0u, 0u};
      if (ent & 1) {
        const int buf = pm & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(S::M_FULL0 + buf), (pm >> 1) & 1, abort_flag));
        if (!ok) break;
        const int32_t* mv = mask_smem + buf * 4 * kTile;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t bits = 0u;
#pragma unroll 8
          for (int c = 0; c < 32; ++c) {
            const int col = cc * 32 + c;
            const int32_t lts = has[0] ? mv[col] : p.n_q, lte = has[1] ? mv[kTile + col] : p.n_q;
            const int32_t uts = has[2] ? mv[2 * kTile + col] : 0, ute = has[3] ? mv[3 * kTile + col] : 0;
            const bool msk = (lts <= i && i < lte) || (uts <= i && i < ute);
            bits |= (msk ? 1u : 0u) << c;
          }
          mbits[cc] = bits;
        }
        mbar_arrive(bar(S::M_EMPTY0 + buf));
        ++pm;
      }
      // pass 1: row maximum of the scaled scores (log2 domain)
      float mx = kNegInf;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sr[32];
        tmem_ld32(tS + lane_addr + cc * 32, sr);
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const float t = ((mbits[cc] >> c) & 1u) ? kNegInf : __uint_as_float(sr[c]) * p.scale_log2;
          mx = fmaxf(mx, t);
        }
      }
      const float m_new = fmaxf(m_run, mx);
      const float m_use = (m_new == kNegInf) ? 0.f : m_new;
      const float alpha = ex2(m_run - m_use);
      // pass 2: P = 2^(t - m) as bf16 pairs written over the first 64 S columns
      float rs = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sr[32];
        tmem_ld32(tS + lane_addr + cc * 32, sr);
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float p0 = ((mbits[cc] >> c) & 1u) ? 0.f : ex2(__uint_as_float(sr[c]) * p.scale_log2 - m_use);
          const float p1 = ((mbits[cc] >> (c + 1)) & 1u) ? 0.f : ex2(__uint_as_float(sr[c + 1]) * p.scale_log2 - m_use);
          rs += p0 + p1;
          pk[c >> 1] = pack_bf16(p0, p1);
        }
        tmem_st16(tS + lane_addr + cc * 16, pk);
      }
      l_run = l_run * alpha + rs;
      // rescale O when the running maximum moved (O holds sum over earlier tiles)
      if (__any_sync(0xffffffffu, e > 0 && alpha != 1.f)) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(S::O_DONE), (e - 1) & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t orr[32];
          tmem_ld32(tO + lane_addr + cc * 32, orr);
#pragma unroll
          for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
          tmem_st32(tO + lane_addr + cc * 32, orr);
        }
      }
      m_run = m_new;
      tc_fence_before();
      mbar_arrive(bar(S::P_FULL));
    }
    if (!ok) record_failure(p.status, abort_flag, 5);
    // epilogue: O = O / l, LSE = (m + log2 l) ln 2; empty rows: O = 0, LSE = -inf
    __nv_bfloat16* orow = p.o + (((int64_t)b * p.n_q + i) * p.H + h) * D;
    const bool live = ok && cnt > 0 && l_run > 0.f;
    bool have_o = false;
    if (ok && cnt > 0) {
      have_o = __all_sync(0xffffffffu, mbar_wait(bar(S::O_DONE), (cnt - 1) & 1, abort_flag));
      if (!have_o) record_failure(p.status, abort_flag, 6);
      tc_fence_after();
    }
    const float inv = live ? 1.f / l_run : 0.f;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t orr[32];
      if (have_o) {
        tmem_ld32(tO + lane_addr + cc * 32, orr);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) orr[c] = 0u;
      }
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2)
        pk[c >> 1] = pack_bf16(__uint_as_float(orr[c]) * inv, __uint_as_float(orr[c + 1]) * inv);
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4)
        st_global_v4(orow + cc * 32 + v4 * 8, pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
    }
    p.lse[((int64_t)b * p.H + h) * p.n_q + i] = live ? (m_run + __log2f(l_run)) * 0.69314718055994531f : kNegInf;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D>
fm_status launch_fwd(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4], void* o,
                     float* lse, cudaStream_t stream) {
  using S = FwdSmem<D>;
  CUtensorMap tq, tk, tv;
  if (!encode_tmap_bf16_4d(&tq, a->q, D, a->H, a->n_q, a->B, kTile) ||
      !encode_tmap_bf16_4d(&tk, a->k, D, a->H, a->n_k, a->B, kTile) ||
      !encode_tmap_bf16_4d(&tv, a->v, D, a->H, a->n_k, a->B, kTile))
    return FM_ERR_CUDA;
  FwdParams p;
  p.row_count = meta->row_count;
  p.row_entries = meta->row_entries;
  for (int c = 0; c < 4; ++c) p.vec[c] = vec ? vec[c] : nullptr;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.status = device_status_ptr();
  p.B = a->B;
  p.H = a->H;
  p.Hm = meta->d.Hm;
  p.n_q = a->n_q;
  p.n_k = a->n_k;
  p.T_q = a->n_q / kTile;
  p.T_k = a->n_k / kTile;
  p.scale_log2 = a->scale * 1.4426950408889634f;
  if (cudaFuncSetAttribute(fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kAlloc) != cudaSuccess)
    return FM_ERR_CUDA;
  fwd_kernel<D><<<dim3(p.T_q, p.H, p.B), kFwdThreads, S::kAlloc, stream>>>(tq, tk, tv, p);
  return cudaGetLastError() == cudaSuccess ? FM_OK : FM_ERR_CUDA;
}

}  // namespace

// Shared argument checks of the attention entry points.
fm_status check_attn_args(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4]) {
  if (!a || !meta) return FM_ERR_INVALID_ARG;
  if (a->B < 1 || a->H < 1 || a->n_q < 1 || a->n_k < 1 || a->B > 65535 || a->H > 65535) return FM_ERR_INVALID_ARG;
  if (!(a->scale == a->scale)) return FM_ERR_INVALID_ARG;
  if (a->dtype != 0) return FM_ERR_UNSUPPORTED;
  if (a->D != 64 && a->D != 128) return FM_ERR_UNSUPPORTED;
  if (a->n_q % kTile || a->n_k % kTile) return FM_ERR_UNSUPPORTED;
  if (!a->q || !a->k || !a->v) return FM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a->q) | reinterpret_cast<uintptr_t>(a->k) | reinterpret_cast<uintptr_t>(a->v)) & 15)
    return FM_ERR_INVALID_ARG;
  const fm_mask_desc& d = meta->d;
  if (d.B != a->B || d.n_q != a->n_q || d.n_k != a->n_k || d.tile_q != kTile || d.tile_k != kTile)
    return FM_ERR_INVALID_ARG;
  if (d.Hm != 1 && d.Hm != a->H) return FM_ERR_INVALID_ARG;
  if (!meta->row_count || !meta->row_entries || !meta->col_count || !meta->col_entries) return FM_ERR_INVALID_ARG;
  if (vec)
    for (int c = 0; c < 4; ++c)
      if (reinterpret_cast<uintptr_t>(vec[c]) & 15) return FM_ERR_INVALID_ARG;
  return FM_OK;
}

}  // namespace fm

extern "C" fm_status fm_attn_fwd(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4],
                                 void* o, float* lse, fm_stream_t stream) {
  fm_status st = fm::check_attn_args(a, meta, vec);
  if (st != FM_OK) return st;
  if (!o || !lse || (reinterpret_cast<uintptr_t>(o) & 15) || (reinterpret_cast<uintptr_t>(lse) & 3))
    return FM_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return a->D == 64 ? fm::launch_fwd<64>(a, meta, vec, o, lse, s) : fm::launch_fwd<128>(a, meta, vec, o, lse, s);
}
