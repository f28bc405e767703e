// Mask-aware attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// FlashMask-3 explainer (learnaivisually.com), tile paragraph: tiles are
// "fully masked, partly masked or unmasked"; "fully masked tiles are never
// loaded" and "only partly masked tiles apply the row-interval test".  The
// pages' Hopper kernel (paper abstract: three-role warp specialisation on the
// FlashAttention-3 TMA/WGMMA pipeline) is prior art; this kernel is designed
// for Blackwell:
//   * one CTA per (pair of 128-row query tiles, head, batch), one CTA per SM,
//     512 TMEM columns: S0 | O0 | S1 | O1 (fp32, 128 lanes x 128 columns each);
//   * the two query tiles walk the merged (union) block list of their two row
//     lists and share every K/V tile, which TMA streams through a two-deep ring;
//   * warp 8 (one lane) issues the TMA loads (Q once; per merged entry K, V and,
//     when a partial tile needs it, the tile's slice of the four vectors);
//   * warp 9 (one lane) issues tcgen05.mma in the order
//       PV0(e), S0(e+1), PV1(e), S1(e+1)
//     so the tensor core computes one tile's scores while the other tile's
//     softmax runs (S = Q K^T into TMEM; O += P V with P, bf16, read from TMEM
//     over the first half of the S columns);
//   * warps 0-3 / 4-7 are the softmax of tile 0 / tile 1 (one thread per row):
//     one TMEM read of the 128 scores, the row-interval test on partial tiles
//     only, online softmax in the log2 domain with the running maximum moved
//     only when it grows by more than 8 (O in TMEM is rescaled then), P written
//     back to TMEM, and the epilogue O / l, LSE.
// Every mbarrier wait is bounded; on a timeout the CTA records the failure in
// the device status word and unwinds (no wait can hang the GPU).
#include <climits>

#include "fm_common.cuh"

namespace fm {
namespace {

constexpr int kTile = 128;
constexpr int kFwdThreads = 320;
constexpr int kMaxList = 4096;  // key tiles per query tile held in shared memory (n_k <= 524288)
constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P may reach 2^8 before O is rescaled
constexpr int kPolyEvery = 8;  // one score pair in kPolyEvery takes exp2_poly2 instead of MUFU ex2
constexpr float kLiveSum = 1e-20f;  // a live row's sum is >= ~1; masked scores add ~2^-125 each

struct FwdParams {
  const int32_t* row_count;    // [B, Hm, T_q]
  const int32_t* row_entries;  // [B, Hm, T_q, T_k]
  const int32_t* order;        // [B, Hm, n_pairs] dispatch order (longest first)
  const int32_t* vec[4];       // [B, Hm, n_k] or null
  const float* v32;            // fp32 V [B, n_k, H, D] (fp32 path: loaded transposed by the load warp)
  void* o;                     // [B, n_q, H, D], bf16 or fp32
  float* lse;                  // [B, H, n_q]
  int* status;
  int B, H, Hm, n_q, n_k, T_q, T_k, n_pairs;
  int H_kv, q_per_kv;          // K/V heads; query heads per K/V head (grouped-query attention)
  int group;                   // heads dispatched together
  float scale_log2;            // softmax scale * log2(e), > 0
};

template <int D, bool F32>
struct FwdSmem {
  static constexpr int kElem = F32 ? 4 : 2;
  static constexpr int kTileBytes = kTile * D * kElem;  // 128 rows x D elements (128-byte swizzle-atom columns)
  static constexpr int kQ = 0;                      // Q0, Q1
  static constexpr int kK = kQ + 2 * kTileBytes;    // K ring, 2 slots
  static constexpr int kV = kK + 2 * kTileBytes;    // V ring, 2 slots
  static constexpr int kMask = kV + 2 * kTileBytes; // [2 buffers][4 vectors][128] int32
  static constexpr int kList = kMask + 2 * 4 * kTile * 4;  // two row lists, kMaxList uint16 each
  static constexpr int kBar = kList + 2 * kMaxList * 2;
  enum { Q_FULL, K_FULL0, K_FULL1, K_EMPTY0, K_EMPTY1, V_FULL0, V_FULL1, V_EMPTY0, V_EMPTY1, S_FULL0, S_FULL1,
         P_FULL0, P_FULL1, P_HALF0, P_HALF1, O_DONE0, O_DONE1, M_FULL0, M_FULL1, M_EMPTY0, M_EMPTY1, DRAIN,
         kNumBars };
  static constexpr int kMisc = kBar + kNumBars * 8;  // [0] TMEM base, [1] abort flag, [2] zero
  static constexpr int kCanaryAt = kMisc + 16;        // FM_DEBUG: shared-memory canary words
  static constexpr int kBytes = kCanaryAt + kCanaryBytes;
  static constexpr int kAlloc = kBytes + 1024;       // slack for 1024-byte alignment of the base
};

// Walks the union of two ascending row lists (entries (kt << 1) | partial).
// Yields each key tile once with the class it has for each query tile
// (0 skip, 1 partial, 2 full).  Every role runs its own copy over the same
// shared-memory lists, so all roles see the same sequence.
// A key tile that runs past n_k (ragged length) is always treated as partial:
// its columns beyond n_k hold zero-filled keys that the interval test masks.
struct MergedList {
  const uint16_t* a;
  const uint16_t* b;
  int na, nb, pa, pb;
  int ragged_kt;  // index of the key tile that runs past n_k, or -1
  __device__ __forceinline__ bool next(int& kt, int& c0, int& c1) {
    const int ea = pa < na ? a[pa] : INT_MAX, eb = pb < nb ? b[pb] : INT_MAX;
    const int ka = ea >> 1, kb = eb >> 1;
    kt = min(ka, kb);
    if (kt == (INT_MAX >> 1)) return false;
    const bool rag = kt == ragged_kt;
    c0 = (ka == kt) ? (((ea & 1) || rag) ? 1 : 2) : 0;
    c1 = (kb == kt) ? (((eb & 1) || rag) ? 1 : 2) : 0;
    pa += (ka == kt);
    pb += (kb == kt);
    return true;
  }
};

// fp32 path: kind::tf32 MMAs read both operands K-major, so PV needs V^T
// ([d][key], keys contiguous).  One warp copies a 128-key fp32 V tile (its first
// `valid` keys; zeros after them) from global memory into that layout (128-byte swizzle; four atoms of 32 keys,
// D rows of 128 bytes each), rounding to tf32 on the way: element (d, key) sits
// at (key / 32) * D * 128 + d * 128 + ((((key % 32) / 4) ^ (d % 8)) * 16) + (key % 4) * 4.
template <int D>
__device__ __forceinline__ void load_vt_f32(uint8_t* dst, const float* src, int64_t row_stride, int valid, int lane) {
  constexpr int kQuads = D / 4;
#pragma unroll 4
  for (int e = lane; e < kTile * kQuads; e += 32) {
    const int key = e / kQuads, dq = e % kQuads;
    const float4 x = key < valid ? __ldg(reinterpret_cast<const float4*>(src + key * row_stride) + dq)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);  // past a ragged n_k
    const float xs[4] = {x.x, x.y, x.z, x.w};
    uint8_t* col = dst + (key >> 5) * (D * 128) + (key & 3) * 4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int d = 4 * dq + j;
      *reinterpret_cast<uint32_t*>(col + d * 128 + ((((key & 31) >> 2) ^ (d & 7)) << 4)) = round_tf32(xs[j]);
    }
  }
}

template <int D, bool F32>
__global__ void __launch_bounds__(kFwdThreads, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const FwdParams p) {
  using S = FwdSmem<D, F32>;
  constexpr int kAtomElems = 128 / S::kElem;        // elements per 128-byte swizzle span
  constexpr int kAtoms = D * S::kElem / 128;         // swizzle-atom columns per tile row
  constexpr int kKStep = F32 ? 8 : 16;               // elements per UMMA K step (32 bytes)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_base_1024(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid (group * n_pairs, ceil(H / group), B): the CTAs of a group of heads are dispatched together,
  // rank by rank over the group's heads (rank r takes the pair with the r-th longest list, so the
  // longest start first); the group is sized so that its heads' K/V stay in L2
  const int h = (int)blockIdx.y * p.group + (int)(blockIdx.x % p.group), b = blockIdx.z;
  if (h >= p.H) return;  // partial last group
  const int64_t bhm = (int64_t)b * p.Hm + (p.Hm == 1 ? 0 : h);
  const int pair = __ldg(p.order + bhm * p.n_pairs + blockIdx.x / p.group);
  const int qt0 = 2 * pair, qt1 = 2 * pair + 1;
  const bool has1 = qt1 < p.T_q;
  const int32_t* rows0 = p.row_entries + (bhm * p.T_q + qt0) * p.T_k;
  const int32_t* rows1 = rows0 + p.T_k;
  const int n0_raw = __ldg(p.row_count + bhm * p.T_q + qt0);
  const int n1_raw = has1 ? __ldg(p.row_count + bhm * p.T_q + qt1) : 0;
  // (debug builds: a count beyond the shared-memory list is recorded below and clamped)
  const int n0 = kDebug ? min(max(n0_raw, 0), kMaxList) : n0_raw;
  const int n1 = kDebug ? min(max(n1_raw, 0), kMaxList) : n1_raw;
  const int ragged_kt = (p.n_k % kTile) ? p.T_k - 1 : -1;

  const uint32_t bar0 = smem_u32(smem + S::kBar);
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  const volatile int* never = reinterpret_cast<const volatile int*>(misc + 2);
  const uint32_t q_s = smem_u32(smem + S::kQ), k_s = smem_u32(smem + S::kK), v_s = smem_u32(smem + S::kV);
  const int32_t* mask_smem = reinterpret_cast<const int32_t*>(smem + S::kMask);
  uint16_t* list0 = reinterpret_cast<uint16_t*>(smem + S::kList);
  uint16_t* list1 = list0 + kMaxList;

  if (threadIdx.x == 0) {
    for (int k = 0; k < S::kNumBars; ++k) mbar_init(bar(k), 1);
    mbar_init(bar(S::P_FULL0), kTile);
    mbar_init(bar(S::P_FULL1), kTile);
    mbar_init(bar(S::P_HALF0), kTile);
    mbar_init(bar(S::P_HALF1), kTile);
    mbar_init(bar(S::M_EMPTY0), 2 * kTile);
    mbar_init(bar(S::M_EMPTY1), 2 * kTile);
    *abort_flag = 0;
    misc[2] = 0;  // a flag nothing raises: lets the final drain wait ignore aborts
    canary_write(smem + S::kCanaryAt);
    check_range(n0_raw, 0, kMaxList + 1, p.status, abort_flag, 31);
    check_range(n1_raw, 0, kMaxList + 1, p.status, abort_flag, 32);
    fence_barrier_init();
    if (n0 + n1 > 0) {  // Q first: its latency overlaps the list copy and the TMEM allocation
      fence_proxy_async_smem();
      prefetch_tmap(&tm_q);
      mbar_arrive_expect_tx(bar(S::Q_FULL), (has1 ? 2 : 1) * S::kTileBytes);
      for (int c = 0; c < kAtoms; ++c) {
        tma_load_4d(q_s + c * 16384, &tm_q, bar(S::Q_FULL), c * kAtomElems, h, qt0 * kTile, b);
        if (has1)
          tma_load_4d(q_s + S::kTileBytes + c * 16384, &tm_q, bar(S::Q_FULL), c * kAtomElems, h, qt1 * kTile, b);
      }
    }
  }
  // both row lists into shared memory (coalesced)
  for (int t = threadIdx.x; t < n0; t += kFwdThreads) list0[t] = (uint16_t)__ldg(rows0 + t);
  for (int t = threadIdx.x; t < n1; t += kFwdThreads) list1[t] = (uint16_t)__ldg(rows1 + t);
  if (warp == 9) {
    tmem_alloc(smem_u32(misc), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const bool any = (n0 + n1) > 0;

  if (warp == 8) {
    // ------------------------------------------------------------ load role
    // bf16: lane 0 issues every TMA load.  fp32: the whole warp walks the list
    // (V^T is copied by all 32 lanes), lane 0 still issuing the TMA loads.
    if ((F32 || lane == 0) && any) {
      auto wait_all = [&](uint32_t bb, uint32_t ph) {
        bool r = mbar_wait(bb, ph, abort_flag);
        if constexpr (F32) r = __all_sync(0xffffffffu, r);
        return r;
      };
      if (lane == 0) {  // (Q was issued at the start)
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
      }
      const int hk = h / p.q_per_kv;  // the K/V head of query head h
      int nvec = 0;
      for (int c = 0; c < 4; ++c) nvec += p.vec[c] ? 1 : 0;
      MergedList it{list0, list1, n0, n1, 0, 0, ragged_kt};
      int kt, c0, c1, e = 0, mcount = 0;
      bool ok = true;
      while (it.next(kt, c0, c1)) {
        const int slot = e & 1;
        if (!check_range(kt, 0, p.T_k, p.status, abort_flag, 33)) {  // a list entry past the key tiles
          ok = false;
          break;
        }
        if (e >= 2 && !wait_all(bar(S::K_EMPTY0 + slot), ((e >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(bar(S::K_FULL0 + slot), S::kTileBytes);
          for (int c = 0; c < kAtoms; ++c)
            tma_load_4d(k_s + slot * S::kTileBytes + c * 16384, &tm_k, bar(S::K_FULL0 + slot), c * kAtomElems, hk,
                        kt * kTile, b);
        }
        if (c0 == 1 || c1 == 1) {
          const int mb = mcount & 1;
          if (mcount >= 2 && !wait_all(bar(S::M_EMPTY0 + mb), ((mcount >> 1) - 1) & 1)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            // a ragged last key tile has (n_k - 128 kt) columns, a multiple of 4 (16-byte copies)
            const uint32_t vbytes = 4u * (uint32_t)min(kTile, p.n_k - kt * kTile);
            mbar_arrive_expect_tx(bar(S::M_FULL0 + mb), vbytes * nvec);
            for (int c = 0; c < 4; ++c)
              if (p.vec[c])
                bulk_load(smem_u32(mask_smem + (mb * 4 + c) * kTile), p.vec[c] + bhm * p.n_k + (int64_t)kt * kTile,
                          vbytes, bar(S::M_FULL0 + mb));
          }
          ++mcount;
        }
        if (e >= 2 && !wait_all(bar(S::V_EMPTY0 + slot), ((e >> 1) - 1) & 1)) {
          ok = false;
          break;
        }
        if constexpr (F32) {
          load_vt_f32<D>(smem + S::kV + slot * S::kTileBytes,
                         p.v32 + (((int64_t)b * p.n_k + (int64_t)kt * kTile) * p.H_kv + hk) * D, (int64_t)p.H_kv * D,
                         min(kTile, p.n_k - kt * kTile), lane);
          fence_proxy_async_smem();  // generic-proxy stores, read next by the tensor core
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(S::V_FULL0 + slot));
        } else {
          mbar_arrive_expect_tx(bar(S::V_FULL0 + slot), S::kTileBytes);
          for (int c = 0; c < kAtoms; ++c)
            tma_load_4d(v_s + slot * S::kTileBytes + c * 16384, &tm_v, bar(S::V_FULL0 + slot), c * kAtomElems, hk,
                        kt * kTile, b);
        }
        ++e;
      }
      if (!ok && lane == 0) record_failure(p.status, abort_flag, 1);
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------- MMA role
    if (lane == 0 && any) {
      // S[q][kv]: Q K-major, K K-major; O[q][d]: P from TMEM, V MN-major (bf16) or V^T K-major (tf32,
      // which takes K-major operands only)
      constexpr uint32_t kIdescQK = F32 ? idesc_tf32(128, 128, false, false) : idesc_bf16(128, 128, false, false);
      constexpr uint32_t kIdescPV = F32 ? idesc_tf32(128, D, false, false) : idesc_bf16(128, D, false, true);
      constexpr int kPvSteps = kTile / kKStep;  // UMMA K steps over the 128 kv rows
      MergedList it{list0, list1, n0, n1, 0, 0, ragged_kt};
      int kt, c0, c1, kn, n0c, n1c;
      bool ok = mbar_wait(bar(S::Q_FULL), 0, abort_flag);
      bool has_cur = ok && it.next(kt, c0, c1);
      int np[2] = {0, 0};  // P tiles consumed per query tile (p_full phases)
      bool acc[2] = {false, false};
      // descriptor words: 128-byte swizzle, SBO = 8 rows x 128 B; per k-step only the low word moves
      constexpr uint32_t kHi = desc_hi(1024);
      const uint32_t lo_q = desc_lo(q_s, 16), lo_k = desc_lo(k_s, 16), lo_v = desc_lo(v_s, F32 ? 16 : 16384);
      // k-th PV step (kKStep kv rows): bf16 V rows of 128 B; tf32 V^T atoms of 32 keys x D rows
      auto pv_off = [&](int k) -> uint32_t {
        return F32 ? (((k >> 2) * (D * 128) + (k & 3) * 32) >> 4) : ((k * kKStep * 128) >> 4);
      };
      constexpr uint32_t kTileW = S::kTileBytes >> 4;  // one tile, in 16-byte descriptor units
      auto issue_s = [&](int t, int kslot) {  // S_t = Q_t K^T
        const uint32_t qa = lo_q + t * kTileW, ka = lo_k + kslot * kTileW;
#pragma unroll
        for (int k = 0; k < D / kKStep; ++k) {
          const uint32_t off = ((k >> 2) * 16384 + (k & 3) * 32) >> 4;  // swizzle-atom column, 32-byte K step
          umma_ss_w<F32>(tmem + t * 256, qa + off, kHi, ka + off, kHi, kIdescQK, k > 0 ? 1u : 0u);
        }
        umma_commit(bar(S::S_FULL0 + t));
      };
      if (has_cur) {
        ok = mbar_wait(bar(S::K_FULL0), 0, abort_flag);
        if (ok) {
          tc_fence_after();
          if (c0) issue_s(0, 0);
          if (c1) issue_s(1, 0);
          umma_commit(bar(S::K_EMPTY0));
        }
      }
      for (int e = 0; ok && has_cur; ++e) {
        const bool has_next = it.next(kn, n0c, n1c);
        const int slot = e & 1, nslot = (e + 1) & 1;
        if (has_next && !mbar_wait(bar(S::K_FULL0 + nslot), ((e + 1) >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        if (!mbar_wait(bar(S::V_FULL0 + slot), (e >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const uint32_t tS = tmem + t * 256, tO = tS + 128;
          if (t ? c1 : c0) {  // O_t += P_t V(e): first half of P as soon as it is in TMEM
            if (!mbar_wait(bar(S::P_HALF0 + t), np[t] & 1, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t va = lo_v + slot * kTileW;
#pragma unroll
            for (int k = 0; k < kPvSteps / 2; ++k)  // kKStep kv rows per step; P columns advance 8 per step
              umma_ts_w<F32>(tO, tS + k * 8, va + pv_off(k), kHi, kIdescPV, (acc[t] || k > 0) ? 1u : 0u);
            if (!mbar_wait(bar(S::P_FULL0 + t), np[t] & 1, abort_flag)) {
              ok = false;
              break;
            }
            ++np[t];
            tc_fence_after();
#pragma unroll
            for (int k = kPvSteps / 2; k < kPvSteps; ++k)
              umma_ts_w<F32>(tO, tS + k * 8, va + pv_off(k), kHi, kIdescPV, 1u);
            umma_commit(bar(S::O_DONE0 + t));
            acc[t] = true;
          }
          if (has_next && (t ? n1c : n0c)) {  // S_t = Q_t K(e+1)^T, after PV_t(e) has read P_t
            tc_fence_after();
            issue_s(t, nslot);
          }
        }
        if (!ok) break;
        umma_commit(bar(S::V_EMPTY0 + slot));
        if (has_next) umma_commit(bar(S::K_EMPTY0 + nslot));
        has_cur = has_next;
        kt = kn;
        c0 = n0c;
        c1 = n1c;
      }
      if (!ok) record_failure(p.status, abort_flag, 4);
      // drain: every MMA issued above has finished before TMEM is released
      umma_commit(bar(S::DRAIN));
      mbar_wait(bar(S::DRAIN), 0, never);
    }
  } else {
    // ---------------------------------------------------------- softmax role
    const int t = warp >> 2;                   // query tile of this warpgroup
    const int r = threadIdx.x & 127;           // row in tile == TMEM lane
    const int qt = t ? qt1 : qt0;
    const int i = qt * kTile + r;  // row (n_q < 2^31)
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + t * 256 + lane_addr, tO = tS + 128;
    const uint32_t has = (p.vec[0] ? 1u : 0u) | (p.vec[1] ? 2u : 0u) | (p.vec[2] ? 4u : 0u) | (p.vec[3] ? 8u : 0u);
    float m_run = kNegInf, l_run = 0.f, lq_run = 0.f;
    int j = 0, mcount = 0;
    bool ok = true;
    MergedList it{list0, list1, n0, n1, 0, 0, ragged_kt};
    int kt, c0, c1;
    const bool live_tile = (t == 0) || has1;
    // A warpgroup without a query tile (odd tile count) still walks the list:
    // both warpgroups release every shared mask buffer.
    while (it.next(kt, c0, c1)) {
      const int ct = t ? c1 : c0;
      const bool has_mask = (c0 == 1 || c1 == 1);
      const int mb = mcount & 1;
      if (ct != 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(S::S_FULL0 + t), j & 1, abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t s[128];
        tmem_ld128(tS, s);
        if (ct == 1) {
          // row-interval test (partial tiles only): masked scores -> -inf
          ok = __all_sync(0xffffffffu, mbar_wait(bar(S::M_FULL0 + mb), (mcount >> 1) & 1, abort_flag));
          if (!ok) break;
          // Lane l turns key columns l, l+32, l+64, l+96 into words of "masked rows of this warp";
          // a bit transpose then gives each row's thread one bit per column.  32-column blocks
          // with no masked entry in the warp are skipped.
          const int32_t* mv = mask_smem + mb * 4 * kTile;
          const int32_t w0 = qt * kTile + (warp & 3) * 32;  // this warp's first row
          uint32_t mw[4];
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            const int c = jb * 32 + lane;
            const int32_t lts = (has & 1u) ? mv[c] : p.n_q, lte = (has & 2u) ? mv[kTile + c] : p.n_q;
            const int32_t uts = (has & 4u) ? mv[2 * kTile + c] : 0, ute = (has & 8u) ? mv[3 * kTile + c] : 0;
            mw[jb] = interval_bits32(lts, lte, w0) | interval_bits32(uts, ute, w0);
          }
          bit_transpose32<4>(mw, lane);
          if (kt == ragged_kt) {  // columns past a ragged n_k hold no key: masked in every row
            const int valid = p.n_k - kt * kTile;
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) {
              const int v = valid - jb * 32;  // valid columns of this 32-column block
              mw[jb] |= v >= 32 ? 0u : (v <= 0 ? 0xFFFFFFFFu : ~((1u << v) - 1u));
            }
          }
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            if (__any_sync(0xffffffffu, mw[jb] != 0u)) {
#pragma unroll
              for (int l = 0; l < 32; ++l)
                s[jb * 32 + l] = ((mw[jb] >> l) & 1u) ? __float_as_uint(kNegInf) : s[jb * 32 + l];
            }
          }
        }
        // row maximum: four independent three-input max chains
        float mx[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
#pragma unroll
        for (int c = 0; c < kTile; c += 8) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            mx[u] = fmax3(mx[u], __uint_as_float(s[c + 2 * u]), __uint_as_float(s[c + 2 * u + 1]));
        }
        const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
        // move the running maximum only when it grows by more than the threshold
        const bool move = (m_tile - m_run) > kRescaleThreshold;  // false when both are -inf
        const float m_new = move ? m_tile : m_run;
        const float alpha = move ? ex2(m_run - m_new) : 1.f;
        const float m_use = (m_new == kNegInf) ? 0.f : m_new;
        // P = 2^(s*scale - m) on pairs (f32x2), in two halves of 64 scores: each half is
        // stored (bf16 pairs over the first S columns) and published on its own barrier so
        // the PV product starts on the first half while the second is computed.
        // rs: exact fp32 row sum (LSE); rq: sum of the bf16-rounded P the PV product uses
        // (O is normalised by it, so O stays a convex combination of V rows).
        const uint64_t sc2 = f2pack(p.scale_log2, p.scale_log2), nm2 = f2pack(-m_use, -m_use);
        uint64_t rs2[4] = {0, 0, 0, 0};
        float rq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          // bf16: 32 packed pairs per half; fp32: 64 tf32-rounded values per half
          uint32_t pk[F32 ? 64 : 32];
#pragma unroll
          for (int c = 0; c < kTile / 2; c += 2) {
            const int cs = hh * (kTile / 2) + c;
            const uint64_t x2 = fma2(((uint64_t)s[cs + 1] << 32) | s[cs], sc2, nm2);
            float p0, p1;
            if (((c >> 1) & (kPolyEvery - 1)) == kPolyEvery - 1) {  // this pair on the FMA pipe
              const uint64_t e2 = exp2_poly2(x2);
              p0 = f2lo(e2);
              p1 = f2hi(e2);
            } else {  // MUFU
              p0 = ex2(f2lo(x2));
              p1 = ex2(f2hi(x2));
            }
            const int k = (c >> 1) & 3;
            rs2[k] = add2(rs2[k], f2pack(p0, p1));
            if constexpr (F32) {
              const uint32_t w0 = round_tf32(p0), w1 = round_tf32(p1);
              rq[k] += __uint_as_float(w0) + __uint_as_float(w1);
              pk[c] = w0;
              pk[c + 1] = w1;
            } else {
              const uint32_t w = pack_bf16(p0, p1);
              rq[k] = add_bf16x2_to_f32(w, rq[k]);
              pk[c >> 1] = w;
            }
          }
          if (hh == 0 && __any_sync(0xffffffffu, move && j > 0)) {
            // O holds the sum over earlier tiles: wait for the last PV, rescale it in TMEM
            // before this tile's PV accumulates into it
            ok = __all_sync(0xffffffffu, mbar_wait(bar(S::O_DONE0 + t), (j - 1) & 1, abort_flag));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < D / 16; ++cc) {
              uint32_t orr[16];
              tmem_ld16(tO + cc * 16, orr);
#pragma unroll
              for (int c = 0; c < 16; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
              tmem_st16(tO + cc * 16, orr);
            }
          }
          if constexpr (F32)
            tmem_st64(tS + hh * 64, pk);
          else
            tmem_st32(tS + hh * 32, pk);
          tc_fence_before();
          mbar_arrive(bar((hh ? S::P_FULL0 : S::P_HALF0) + t));
        }
        if (!ok) break;
        const uint64_t rs2a = add2(add2(rs2[0], rs2[1]), add2(rs2[2], rs2[3]));
        const float rs = f2lo(rs2a) + f2hi(rs2a);
        const float rqs = (rq[0] + rq[1]) + (rq[2] + rq[3]);
        l_run = l_run * alpha + rs;
        lq_run = lq_run * alpha + rqs;
        m_run = m_new;
        ++j;
      } else if (has_mask) {
        // keep the two warpgroups in step on the shared mask buffers
        ok = __all_sync(0xffffffffu, mbar_wait(bar(S::M_FULL0 + mb), (mcount >> 1) & 1, abort_flag));
        if (!ok) break;
      }
      if (has_mask) {
        mbar_arrive(bar(S::M_EMPTY0 + mb));
        ++mcount;
      }
    }
    if (!ok) record_failure(p.status, abort_flag, 5);
    // epilogue: O = O / l, LSE = (m + log2 l) ln 2; empty rows: O = 0, LSE = -inf
    if (live_tile) {
      const bool live = ok && j > 0 && l_run > kLiveSum;
      bool have_o = false;
      if (ok && j > 0) {
        have_o = __all_sync(0xffffffffu, mbar_wait(bar(S::O_DONE0 + t), (j - 1) & 1, abort_flag));
        if (!have_o) record_failure(p.status, abort_flag, 6);
        tc_fence_after();
      }
      const float inv = live ? 1.f / lq_run : 0.f;
      // O tile staged in this tile's Q buffer (every S_t product has finished once O_DONE_t has
      // fired; the PV product does not read Q), 128-byte swizzle, then TMA-stored by one thread
      uint8_t* stage = smem + S::kQ + t * S::kTileBytes;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t orr[32];
        if (have_o) {
          tmem_ld32(tO + cc * 32, orr);
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) orr[c] = 0u;
        }
        if constexpr (F32) {  // 32 fp32 = one atom row
          uint8_t* row = stage + cc * 16384 + r * 128;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch)
            *reinterpret_cast<uint4*>(row + ((ch ^ (r & 7)) << 4)) =
                make_uint4(__float_as_uint(__uint_as_float(orr[4 * ch]) * inv),
                           __float_as_uint(__uint_as_float(orr[4 * ch + 1]) * inv),
                           __float_as_uint(__uint_as_float(orr[4 * ch + 2]) * inv),
                           __float_as_uint(__uint_as_float(orr[4 * ch + 3]) * inv));
        } else {  // 32 bf16 = half an atom row
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 32; c += 2)
            pk[c >> 1] = pack_bf16(__uint_as_float(orr[c]) * inv, __uint_as_float(orr[c + 1]) * inv);
          uint8_t* row = stage + (cc >> 1) * 16384 + r * 128;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
            *reinterpret_cast<uint4*>(row + ((((cc & 1) * 4 + ch) ^ (r & 7)) << 4)) =
                make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(2 + t, 128);
      if (r == 0) {
        for (int c = 0; c < kAtoms; ++c)
          tma_store_4d(&tm_o, smem_u32(stage + c * 16384), c * kAtomElems, h, qt * kTile, b);
        bulk_commit_group();
        bulk_wait_group_read0();
      }
      if (i < p.n_q)  // rows past a ragged n_q are computed on zero-filled queries and dropped
        p.lse[((int64_t)b * p.H + h) * p.n_q + (int64_t)i] = live ? (m_run + __log2f(l_run)) * 0.69314718055994531f : kNegInf;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) canary_check(smem + S::kCanaryAt, p.status, abort_flag, 34);
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Head dimension 256 (bf16).  One 128-row query tile per CTA: S (128 fp32 columns) is double
// buffered in TMEM next to O (256 columns), S0 | S1 | O = 512 columns.  Q takes 64 KiB of shared
// memory, so K and V stream through two-slot rings of 64-key halves (32 KiB each): the S product
// of a 128-key tile is two N = 64 UMMA groups (one per K half), its PV product two K = 64 groups
// (one per V half, P read from TMEM).  Warp 4 loads Q, K and the mask slices, warp 5 loads V,
// warp 6 issues the MMAs in the order S(0), S(1), PV(0), S(2), PV(1), S(3), ..., so S(e+1) runs
// while the softmax of tile e does; warps 0-3 are the softmax (one thread per row), with the same
// interval test, online softmax and epilogue as the two-tile kernel.
// ---------------------------------------------------------------------------
constexpr int kFwd256Threads = 224;
constexpr int kHalf = 64;  // keys per K / V half tile

struct Fwd256Smem {
  static constexpr int kQ = 0;                        // 4 atom columns x 128 rows x 128 B
  static constexpr int kHalfBytes = kHalf * 256 * 2;  // 32 KiB: 4 atom columns x 64 rows x 128 B
  static constexpr int kK = kQ + 128 * 256 * 2;       // K ring, 2 halves
  static constexpr int kV = kK + 2 * kHalfBytes;      // V ring, 2 halves
  static constexpr int kMask = kV + 2 * kHalfBytes;   // [2 buffers][4 vectors][128] int32
  static constexpr int kList = kMask + 2 * 4 * kTile * 4;
  static constexpr int kBar = kList + kMaxList * 2;
  enum { Q_FULL, K_FULL0, K_FULL1, K_EMPTY0, K_EMPTY1, V_FULL0, V_FULL1, V_EMPTY0, V_EMPTY1, S_FULL0, S_FULL1,
         P_HALF0, P_HALF1, P_FULL0, P_FULL1, O_DONE, M_FULL0, M_FULL1, M_EMPTY0, M_EMPTY1, DRAIN, kNumBars };
  static constexpr int kMisc = kBar + kNumBars * 8;  // [0] TMEM base, [1] abort flag, [2] zero
  static constexpr int kCanaryAt = kMisc + 16;        // FM_DEBUG: shared-memory canary words
  static constexpr int kBytes = kCanaryAt + kCanaryBytes;
  static constexpr int kAlloc = kBytes + 1024;
};

__global__ void __launch_bounds__(kFwd256Threads, 1)
    fwd_kernel_d256(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const FwdParams p) {
  using S = Fwd256Smem;
  constexpr int D = 256;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_base_1024(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid (group * T_q, ceil(H / group), B); the query tiles of a head in longest-first order (the
  // metadata orders pairs of tiles: pair = order[rank / 2], tile = 2 pair + rank % 2)
  const int h = (int)blockIdx.y * p.group + (int)(blockIdx.x % p.group), b = blockIdx.z;
  if (h >= p.H) return;
  const int64_t bhm = (int64_t)b * p.Hm + (p.Hm == 1 ? 0 : h);
  const int rank = (int)(blockIdx.x / p.group);
  const int qt = 2 * __ldg(p.order + bhm * p.n_pairs + rank / 2) + (rank & 1);
  if (qt >= p.T_q) return;  // odd tile count: the pair's second tile does not exist
  const int32_t* rows = p.row_entries + (bhm * p.T_q + qt) * p.T_k;
  const int n_raw = __ldg(p.row_count + bhm * p.T_q + qt);
  const int n = kDebug ? min(max(n_raw, 0), kMaxList) : n_raw;  // (debug: recorded below, clamped)
  const int ragged_kt = (p.n_k % kTile) ? p.T_k - 1 : -1;

  const uint32_t bar0 = smem_u32(smem + S::kBar);
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  const volatile int* never = reinterpret_cast<const volatile int*>(misc + 2);
  const uint32_t q_s = smem_u32(smem + S::kQ), k_s = smem_u32(smem + S::kK), v_s = smem_u32(smem + S::kV);
  const int32_t* mask_smem = reinterpret_cast<const int32_t*>(smem + S::kMask);
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + S::kList);

  if (threadIdx.x == 0) {
    for (int k = 0; k < S::kNumBars; ++k) mbar_init(bar(k), 1);
    mbar_init(bar(S::P_HALF0), kTile);
    mbar_init(bar(S::P_HALF1), kTile);
    mbar_init(bar(S::P_FULL0), kTile);
    mbar_init(bar(S::P_FULL1), kTile);
    mbar_init(bar(S::M_EMPTY0), kTile);
    mbar_init(bar(S::M_EMPTY1), kTile);
    *abort_flag = 0;
    misc[2] = 0;
    canary_write(smem + S::kCanaryAt);
    check_range(n_raw, 0, kMaxList + 1, p.status, abort_flag, 41);
    fence_barrier_init();
    if (n > 0) {
      fence_proxy_async_smem();
      prefetch_tmap(&tm_q);
      mbar_arrive_expect_tx(bar(S::Q_FULL), 128 * D * 2);
      for (int c = 0; c < 4; ++c) tma_load_4d(q_s + c * 16384, &tm_q, bar(S::Q_FULL), c * 64, h, qt * kTile, b);
    }
  }
  for (int t = threadIdx.x; t < n; t += kFwd256Threads) list[t] = (uint16_t)__ldg(rows + t);
  if (warp == 6) {
    tmem_alloc(smem_u32(misc), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const int hk = h / p.q_per_kv;
  // class of list entry e: 1 partial, 2 full (a ragged last key tile is always partial)
  auto cls_of = [&](int e, int& kt) {
    const int ent = list[e];
    kt = ent >> 1;
    return ((ent & 1) || kt == ragged_kt) ? 1 : 2;
  };

  if (warp == 4) {
    // ------------------------------------------- K and mask-slice loads (lane 0)
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tm_k);
      int nvec = 0;
      for (int c = 0; c < 4; ++c) nvec += p.vec[c] ? 1 : 0;
      bool ok = true;
      int mcount = 0;
      for (int e = 0; ok && e < n; ++e) {
        int kt;
        const int c = cls_of(e, kt);
        if (!check_range(kt, 0, p.T_k, p.status, abort_flag, 42)) {  // a list entry past the key tiles
          ok = false;
          break;
        }
        for (int hh = 0; hh < 2; ++hh) {
          const int u = 2 * e + hh, slot = u & 1;
          if (u >= 2 && !mbar_wait(bar(S::K_EMPTY0 + slot), ((u >> 1) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(S::K_FULL0 + slot), S::kHalfBytes);
          for (int a = 0; a < 4; ++a)
            tma_load_4d(k_s + slot * S::kHalfBytes + a * 8192, &tm_k, bar(S::K_FULL0 + slot), a * 64, hk,
                        kt * kTile + hh * kHalf, b);
        }
        if (ok && c == 1) {
          const int mb = mcount & 1;
          if (mcount >= 2 && !mbar_wait(bar(S::M_EMPTY0 + mb), ((mcount >> 1) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t vbytes = 4u * (uint32_t)min(kTile, p.n_k - kt * kTile);
          mbar_arrive_expect_tx(bar(S::M_FULL0 + mb), vbytes * nvec);
          for (int v = 0; v < 4; ++v)
            if (p.vec[v])
              bulk_load(smem_u32(mask_smem + (mb * 4 + v) * kTile), p.vec[v] + bhm * p.n_k + (int64_t)kt * kTile,
                        vbytes, bar(S::M_FULL0 + mb));
          ++mcount;
        }
      }
      if (!ok) record_failure(p.status, abort_flag, 21);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------- V loads (lane 0)
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tm_v);
      bool ok = true;
      for (int e = 0; ok && e < n; ++e) {
        int kt;
        cls_of(e, kt);
        for (int hh = 0; hh < 2; ++hh) {
          const int u = 2 * e + hh, slot = u & 1;
          if (u >= 2 && !mbar_wait(bar(S::V_EMPTY0 + slot), ((u >> 1) - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(S::V_FULL0 + slot), S::kHalfBytes);
          for (int a = 0; a < 4; ++a)
            tma_load_4d(v_s + slot * S::kHalfBytes + a * 8192, &tm_v, bar(S::V_FULL0 + slot), a * 64, hk,
                        kt * kTile + hh * kHalf, b);
        }
      }
      if (!ok) record_failure(p.status, abort_flag, 22);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ MMA role (lane 0)
    if (lane == 0 && n > 0) {
      constexpr uint32_t kIdS = idesc_bf16(128, kHalf, false, false);  // S half: Q K-major, K K-major
      constexpr uint32_t kIdPV = idesc_bf16(128, D, false, true);      // O += P V: V MN-major, N = 256
      constexpr uint32_t kHi = desc_hi(1024);
      const uint32_t lo_q = desc_lo(q_s, 16), lo_k = desc_lo(k_s, 16), lo_v = desc_lo(v_s, 8192);
      constexpr uint32_t kHalfW = S::kHalfBytes >> 4;
      auto issue_s = [&](int e) -> bool {  // S(e) into buffer e & 1: one N = 64 group per K half
        const uint32_t tS = tmem + (e & 1) * 128;
        for (int hh = 0; hh < 2; ++hh) {
          const int u = 2 * e + hh, slot = u & 1;
          if (!mbar_wait(bar(S::K_FULL0 + slot), (u >> 1) & 1, abort_flag)) return false;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const uint32_t oq = ((k >> 2) * 16384 + (k & 3) * 32) >> 4, ok_ = ((k >> 2) * 8192 + (k & 3) * 32) >> 4;
            umma_ss_w<false>(tS + hh * kHalf, lo_q + oq, kHi, lo_k + slot * kHalfW + ok_, kHi, kIdS, k > 0 ? 1u : 0u);
          }
          umma_commit(bar(S::K_EMPTY0 + slot));
        }
        umma_commit(bar(S::S_FULL0 + (e & 1)));
        return true;
      };
      bool ok = mbar_wait(bar(S::Q_FULL), 0, abort_flag);
      if (ok) ok = issue_s(0);
      if (ok && n > 1) ok = issue_s(1);
      for (int e = 0; ok && e < n; ++e) {
        const int sb = e & 1, ph = (e >> 1) & 1;
        const uint32_t tS = tmem + sb * 128, tO = tmem + 256;
        // O += P(e) V(e): keys [0, 64) as soon as the first half of P is in TMEM, then keys [64, 128)
        for (int hh = 0; ok && hh < 2; ++hh) {
          const int u = 2 * e + hh, slot = u & 1;
          if (!mbar_wait(bar(hh ? S::P_FULL0 + sb : S::P_HALF0 + sb), ph, abort_flag) ||
              !mbar_wait(bar(S::V_FULL0 + slot), (u >> 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < kHalf / 16; ++k)
            umma_ts_w<false>(tO, tS + hh * 32 + k * 8, lo_v + slot * kHalfW + ((k * 16 * 128) >> 4), kHi, kIdPV,
                             (e > 0 || hh > 0 || k > 0) ? 1u : 0u);
          umma_commit(bar(S::V_EMPTY0 + slot));
        }
        if (!ok) break;
        umma_commit(bar(S::O_DONE));
        if (e + 2 < n) ok = issue_s(e + 2);  // after PV(e) has read P(e) from the same columns
      }
      if (!ok) record_failure(p.status, abort_flag, 23);
      umma_commit(bar(S::DRAIN));
      mbar_wait(bar(S::DRAIN), 0, never);
    }
  } else {
    // ------------------------------------------------------ softmax role (warps 0-3)
    const int r = threadIdx.x;  // row in tile == TMEM lane
    const int i = qt * kTile + r;
    const uint32_t lane_addr = (uint32_t)(warp * 32) << 16;
    const uint32_t has = (p.vec[0] ? 1u : 0u) | (p.vec[1] ? 2u : 0u) | (p.vec[2] ? 4u : 0u) | (p.vec[3] ? 8u : 0u);
    const uint32_t tO = tmem + 256 + lane_addr;
    float m_run = kNegInf, l_run = 0.f, lq_run = 0.f;
    int mcount = 0;
    bool ok = true;
    int e = 0;
    for (; e < n; ++e) {
      int kt;
      const int ct = cls_of(e, kt);
      const int sb = e & 1;
      const uint32_t tS = tmem + sb * 128 + lane_addr;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(S::S_FULL0 + sb), (e >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld128(tS, s);
      if (ct == 1) {
        const int mb = mcount & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(bar(S::M_FULL0 + mb), (mcount >> 1) & 1, abort_flag));
        if (!ok) break;
        const int32_t* mv = mask_smem + mb * 4 * kTile;
        const int32_t w0 = qt * kTile + warp * 32;
        uint32_t mw[4];
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
          const int c = jb * 32 + lane;
          const int32_t lts = (has & 1u) ? mv[c] : p.n_q, lte = (has & 2u) ? mv[kTile + c] : p.n_q;
          const int32_t uts = (has & 4u) ? mv[2 * kTile + c] : 0, ute = (has & 8u) ? mv[3 * kTile + c] : 0;
          mw[jb] = interval_bits32(lts, lte, w0) | interval_bits32(uts, ute, w0);
        }
        bit_transpose32<4>(mw, lane);
        if (kt == ragged_kt) {
          const int valid = p.n_k - kt * kTile;
#pragma unroll
          for (int jb = 0; jb < 4; ++jb) {
            const int v = valid - jb * 32;
            mw[jb] |= v >= 32 ? 0u : (v <= 0 ? 0xFFFFFFFFu : ~((1u << v) - 1u));
          }
        }
#pragma unroll
        for (int jb = 0; jb < 4; ++jb) {
          if (__any_sync(0xffffffffu, mw[jb] != 0u)) {
#pragma unroll
            for (int l = 0; l < 32; ++l) s[jb * 32 + l] = ((mw[jb] >> l) & 1u) ? __float_as_uint(kNegInf) : s[jb * 32 + l];
          }
        }
        __syncwarp();
        mbar_arrive(bar(S::M_EMPTY0 + mb));
        ++mcount;
      }
      float mx[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
#pragma unroll
      for (int c = 0; c < kTile; c += 8) {
#pragma unroll
        for (int u = 0; u < 4; ++u) mx[u] = fmax3(mx[u], __uint_as_float(s[c + 2 * u]), __uint_as_float(s[c + 2 * u + 1]));
      }
      const float m_tile = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2;
      const bool move = (m_tile - m_run) > kRescaleThreshold;
      const float m_new = move ? m_tile : m_run;
      const float alpha = move ? ex2(m_run - m_new) : 1.f;
      const float m_use = (m_new == kNegInf) ? 0.f : m_new;
      const uint64_t sc2 = f2pack(p.scale_log2, p.scale_log2), nm2 = f2pack(-m_use, -m_use);
      uint64_t rs2[4] = {0, 0, 0, 0};
      float rq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < kTile / 2; c += 2) {
          const int cs = hh * (kTile / 2) + c;
          const uint64_t x2 = fma2(((uint64_t)s[cs + 1] << 32) | s[cs], sc2, nm2);
          float p0, p1;
          if (((c >> 1) & (kPolyEvery - 1)) == kPolyEvery - 1) {
            const uint64_t e2 = exp2_poly2(x2);
            p0 = f2lo(e2);
            p1 = f2hi(e2);
          } else {
            p0 = ex2(f2lo(x2));
            p1 = ex2(f2hi(x2));
          }
          const int k = (c >> 1) & 3;
          rs2[k] = add2(rs2[k], f2pack(p0, p1));
          const uint32_t w = pack_bf16(p0, p1);
          rq[k] = add_bf16x2_to_f32(w, rq[k]);
          pk[c >> 1] = w;
        }
        if (hh == 0 && __any_sync(0xffffffffu, move && e > 0)) {
          // O holds the sum over earlier tiles: wait for the last PV, rescale O in TMEM
          ok = __all_sync(0xffffffffu, mbar_wait(bar(S::O_DONE), (e - 1) & 1, abort_flag));
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t orr[32];
            tmem_ld32(tO + cc * 32, orr);
#pragma unroll
            for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
            tmem_st32(tO + cc * 32, orr);
          }
        }
        tmem_st32(tS + hh * 32, pk);
        tc_fence_before();
        mbar_arrive(bar((hh ? S::P_FULL0 : S::P_HALF0) + sb));
      }
      if (!ok) break;
      const uint64_t rs2a = add2(add2(rs2[0], rs2[1]), add2(rs2[2], rs2[3]));
      l_run = l_run * alpha + (f2lo(rs2a) + f2hi(rs2a));
      lq_run = lq_run * alpha + ((rq[0] + rq[1]) + (rq[2] + rq[3]));
      m_run = m_new;
    }
    if (!ok) record_failure(p.status, abort_flag, 24);
    // epilogue: O = O / l staged in the Q buffer (every S product has finished once the last PV
    // has), TMA-stored by one thread; LSE = (m + log2 l) ln 2; empty rows: O = 0, LSE = -inf
    const bool live = ok && n > 0 && l_run > kLiveSum;
    bool have_o = false;
    if (ok && n > 0) {
      have_o = __all_sync(0xffffffffu, mbar_wait(bar(S::O_DONE), (n - 1) & 1, abort_flag));
      if (!have_o) record_failure(p.status, abort_flag, 25);
      tc_fence_after();
    }
    const float inv = live ? 1.f / lq_run : 0.f;
    uint8_t* stage = smem + S::kQ;
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t orr[32];
      if (have_o) {
        tmem_ld32(tO + cc * 32, orr);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) orr[c] = 0u;
      }
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) pk[c >> 1] = pack_bf16(__uint_as_float(orr[c]) * inv, __uint_as_float(orr[c + 1]) * inv);
      uint8_t* row = stage + (cc >> 1) * 16384 + r * 128;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch)
        *reinterpret_cast<uint4*>(row + ((((cc & 1) * 4 + ch) ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
    }
    fence_proxy_async_smem();
    named_bar_sync(2, 128);
    if (r == 0) {
      for (int c = 0; c < 4; ++c) tma_store_4d(&tm_o, smem_u32(stage + c * 16384), c * 64, h, qt * kTile, b);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
    if (i < p.n_q)
      p.lse[((int64_t)b * p.H + h) * p.n_q + (int64_t)i] = live ? (m_run + __log2f(l_run)) * 0.69314718055994531f : kNegInf;
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) canary_check(smem + S::kCanaryAt, p.status, abort_flag, 43);
  if (warp == 6) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

fm_status launch_fwd_d256(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4], void* o,
                          float* lse, cudaStream_t stream) {
  using S = Fwd256Smem;
  static_assert(S::kAlloc <= 227 * 1024, "forward (D = 256) shared memory exceeds the per-CTA limit");
  constexpr int D = 256;
  CUtensorMap tq, tk, tv, to;
  const int H_kv = a->H_kv ? a->H_kv : a->H;
  if (!encode_tmap_bf16_4d(&tq, a->q, D, a->H, a->n_q, a->B, kTile) ||
      !encode_tmap_bf16_4d(&tk, a->k, D, H_kv, a->n_k, a->B, kHalf) ||
      !encode_tmap_bf16_4d(&tv, a->v, D, H_kv, a->n_k, a->B, kHalf) ||
      !encode_tmap_bf16_4d(&to, o, D, a->H, a->n_q, a->B, kTile))
    return FM_ERR_CUDA;
  FwdParams p;
  p.row_count = meta->row_count;
  p.row_entries = meta->row_entries;
  p.order = meta->fwd_order;
  for (int c = 0; c < 4; ++c) p.vec[c] = vec ? vec[c] : nullptr;
  p.v32 = nullptr;
  p.o = o;
  p.lse = lse;
  p.status = device_status_ptr();
  p.B = a->B;
  p.H = a->H;
  p.H_kv = H_kv;
  p.q_per_kv = a->H / H_kv;
  p.Hm = meta->d.Hm;
  p.n_q = a->n_q;
  p.n_k = a->n_k;
  p.T_q = (a->n_q + kTile - 1) / kTile;
  p.T_k = (a->n_k + kTile - 1) / kTile;
  p.n_pairs = (p.T_q + 1) / 2;
  p.group = dispatch_group(p.H, 2.0 * a->n_k * D * 2);
  p.scale_log2 = a->scale * 1.4426950408889634f;
  if (!smem_opt_in<fwd_kernel_d256>(S::kAlloc)) return FM_ERR_CUDA;
  const int ranks = 2 * p.n_pairs;  // query tiles rounded up to whole pairs
  fwd_kernel_d256<<<dim3(p.group * ranks, (p.H + p.group - 1) / p.group, p.B), kFwd256Threads, S::kAlloc, stream>>>(
      tq, tk, tv, to, p);
  return cudaGetLastError() == cudaSuccess ? FM_OK : FM_ERR_CUDA;
}

template <int D, bool F32>
fm_status launch_fwd(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4], void* o,
                     float* lse, cudaStream_t stream) {
  using S = FwdSmem<D, F32>;
  static_assert(S::kAlloc <= 227 * 1024, "forward shared memory exceeds the per-CTA limit");
  CUtensorMap tq, tk, tv, to;
  auto enc = F32 ? encode_tmap_f32_4d : encode_tmap_bf16_4d;
  const int H_kv = a->H_kv ? a->H_kv : a->H;
  if (!enc(&tq, a->q, D, a->H, a->n_q, a->B, kTile) || !enc(&tk, a->k, D, H_kv, a->n_k, a->B, kTile) ||
      !enc(&tv, a->v, D, H_kv, a->n_k, a->B, kTile) || !enc(&to, o, D, a->H, a->n_q, a->B, kTile))
    return FM_ERR_CUDA;
  FwdParams p;
  p.row_count = meta->row_count;
  p.row_entries = meta->row_entries;
  p.order = meta->fwd_order;
  for (int c = 0; c < 4; ++c) p.vec[c] = vec ? vec[c] : nullptr;
  p.v32 = F32 ? static_cast<const float*>(a->v) : nullptr;
  p.o = o;
  p.lse = lse;
  p.status = device_status_ptr();
  p.B = a->B;
  p.H = a->H;
  p.H_kv = H_kv;
  p.q_per_kv = a->H / H_kv;
  p.Hm = meta->d.Hm;
  p.n_q = a->n_q;
  p.n_k = a->n_k;
  p.T_q = (a->n_q + kTile - 1) / kTile;
  p.T_k = (a->n_k + kTile - 1) / kTile;
  p.n_pairs = (p.T_q + 1) / 2;
  p.group = dispatch_group(p.H, 2.0 * a->n_k * D * S::kElem);
  p.scale_log2 = a->scale * 1.4426950408889634f;
  if (!smem_opt_in<fwd_kernel<D, F32>>(S::kAlloc)) return FM_ERR_CUDA;
  fwd_kernel<D, F32><<<dim3(p.group * p.n_pairs, (p.H + p.group - 1) / p.group, p.B), kFwdThreads, S::kAlloc, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError() == cudaSuccess ? FM_OK : FM_ERR_CUDA;
}

}  // namespace

// Shared argument checks of the attention entry points.
fm_status check_attn_args(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4]) {
  if (!a || !meta) return FM_ERR_INVALID_ARG;
  if (a->B < 1 || a->H < 1 || a->n_q < 1 || a->n_k < 1 || a->B > 65535 || a->H > 65535) return FM_ERR_INVALID_ARG;
  if (!(a->scale > 0.f) || a->scale > 3.0e38f) return FM_ERR_INVALID_ARG;  // positive and finite
  if (a->dtype != 0 && a->dtype != 1) return FM_ERR_UNSUPPORTED;
  if (a->D != 64 && a->D != 128 && a->D != 256) return FM_ERR_UNSUPPORTED;
  if (a->dtype == 1 && a->D != 64) return FM_ERR_UNSUPPORTED;  // fp32 tiles of D >= 128 exceed shared memory
  if (a->n_k % 4) return FM_ERR_UNSUPPORTED;  // key tiles' bound vectors are staged by 16-byte bulk copies
  if ((a->n_k + kTile - 1) / kTile > kMaxList || (a->n_q + kTile - 1) / kTile > kMaxList)
    return FM_ERR_UNSUPPORTED;  // lists held in smem
  if (!a->q || !a->k || !a->v) return FM_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a->q) | reinterpret_cast<uintptr_t>(a->k) | reinterpret_cast<uintptr_t>(a->v)) & 15)
    return FM_ERR_INVALID_ARG;
  const fm_mask_desc& d = meta->d;
  if (d.B != a->B || d.n_q != a->n_q || d.n_k != a->n_k || d.tile_q != kTile || d.tile_k != kTile)
    return FM_ERR_INVALID_ARG;
  if (d.Hm != 1 && d.Hm != a->H) return FM_ERR_INVALID_ARG;
  const int H_kv = a->H_kv ? a->H_kv : a->H;  // grouped-query attention: H_kv divides H
  if (H_kv < 1 || H_kv > a->H || a->H % H_kv) return FM_ERR_INVALID_ARG;
  if (a->deterministic != 0 && a->deterministic != 1) return FM_ERR_INVALID_ARG;
  if (a->H / H_kv > 64) return FM_ERR_UNSUPPORTED;  // the backward's per-CTA head table
  if (!meta->row_count || !meta->row_entries || !meta->col_count || !meta->col_entries || !meta->fwd_order ||
      !meta->bwd_order)
    return FM_ERR_INVALID_ARG;
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
  if (a->dtype == 1) return fm::launch_fwd<64, true>(a, meta, vec, o, lse, s);
  if (a->D == 256) return fm::launch_fwd_d256(a, meta, vec, o, lse, s);
  return a->D == 64 ? fm::launch_fwd<64, false>(a, meta, vec, o, lse, s)
                    : fm::launch_fwd<128, false>(a, meta, vec, o, lse, s);
}
