// Mask-aware attention backward for sm_100a (tcgen05 + TMEM + TMA).
//
// The pages report the backward only as a measured speed-up (zicq.com summary,
// end-to-end training paragraph: "attention forward and backward computation
// speed increased by 24.5%-44.9%"); they give no design.  This kernel applies
// the same tile classes as the forward (explainer, tile paragraph): each key
// tile walks its column list of non-skip query tiles and applies the
// row-interval test only on partial tiles.
//
// Per key tile of 128 keys (one CTA; with grouped-query attention, per key
// tile and K/V head), per 64-row query sub-tile of its column list:
//   S^T  = K Q^T        (tcgen05, M=128 keys, N=64 queries)      -> TMEM
//   dP^T = V dO^T       (tcgen05)                                -> TMEM
//   P^T  = 2^(S^T scale log2e - LSE2), masked entries 0         (warps 0-7)
//   dS^T = P^T (dP^T - D_i)                                     (warps 0-7)
//   dV  += P^T dO       (P^T read from TMEM)                    -> TMEM
//   dK  += dS^T Q       (dS^T from shared memory)               -> TMEM
//   dQ^T = K^T dS^T     (per sub-tile)                          -> TMEM -> fp32
//        vector reductions into a global accumulator            (warps 8-11)
// Warps 0-3 / 4-7 each take 32 of the 64 queries of a sub-tile; warp 12 issues
// the TMA loads, warp 13 the MMAs.  A preprocess kernel forms D_i = dO_i.O_i
// and the log2-domain LSE (rows padded to whole query tiles) and clears the
// accumulator; a final kernel scales the accumulator into dQ.  The fp32 path
// (kind::tf32) transposes its MN-major operands in shared memory (drain warps).
#include "fm_common.cuh"

namespace fm {
fm_status check_attn_args(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4]);

namespace {

constexpr int kTile = 128;
constexpr int kBQ = 64;  // query rows per backward sub-tile
constexpr int kBwdThreads = 448;  // 2 x compute, 1 x dQ drain warpgroups, load warp, MMA warp
constexpr int kMaxList = 4096;  // query tiles per key tile held in shared memory
constexpr float kNegInf = -__builtin_huge_valf();
constexpr float kPosInf = __builtin_huge_valf();

struct BwdParams {
  const int32_t* col_count;    // [B, Hm, T_k]
  const int32_t* col_entries;  // [B, Hm, T_k, T_q]
  const int32_t* order;        // [B, Hm, T_k] dispatch order (longest first); null = ascending
  const uint16_t* turn;        // fixed-order dQ: [B, Hm, T_k, T_q] position of key tile kt in the
                               // row list of query tile qt; null = unordered adds
  int* dq_sem;                 // fixed-order dQ: [B, H, T_q] key tiles added so far per query tile
  const int32_t* vec[4];       // [B, Hm, n_k] or null
  const float* lse2;           // [B, H, n_q] log2-domain LSE, +inf on empty rows
  const float* dvec;           // [B, H, n_q] D_i = dO_i . O_i
  float* dq_acc;               // [B, H, n_q/64][16][D][4] fp32
  void* dk;                    // [B, n_k, H, D], bf16 or fp32
  void* dv;
  int* status;
  int B, H, Hm, n_q, n_k, T_q, T_k;
  int n_q_pad;                 // n_q rounded up to whole query tiles (row stride of lse2, dvec, dq_acc)
  int H_kv, q_per_kv;          // K/V heads; query heads per K/V head (grouped-query attention)
  int group;                   // heads dispatched together
  int dh0;                     // D = 256: first d column of the half this launch accumulates (0 or 128)
  float scale, scale_log2;
};

template <int D, bool F32>
struct BwdSmem {
  static constexpr int kElem = F32 ? 4 : 2;
  // fp32 tiles are twice as large; D = 256 keeps K and V whole (64 KiB each) beside one Q/dO stage
  static constexpr int kQStages = D == 256 ? 1 : (F32 ? 2 : 3);
  static constexpr int kDSBufs = (F32 || D == 256) ? 1 : 2;
  // bf16: K, 128 keys x 128 d (the d >= D part kept zero: K^T is a 128-row MMA operand for dQ^T).
  // fp32 (D = 64): K [key][d] in the first half, K^T [d][key] (K-major, four 8 KiB atoms) in the second;
  // V follows, so the 64 rows past the last K^T atom that a 128-row operand reads stay in bounds.
  static constexpr int kK = 0;
  static constexpr int kKBytes = kTile * (D > 128 ? D : 128) * kElem;
  static constexpr int kV = kK + kKBytes;
  static constexpr int kQStage = kBQ * D * kElem;    // one 64-row sub-tile of Q (or dO)
  static constexpr int kQ = kV + kTile * D * kElem;  // kQStages x Q
  static constexpr int kDO = kQ + kQStages * kQStage;  // kQStages x dO
  static constexpr int kDSBytes = kTile * kBQ * kElem;  // dS^T: 128 keys x 64 queries
  static constexpr int kDS = kDO + kQStages * kQStage;  // kDSBufs buffers
  static constexpr int kStats = kDS + kDSBufs * kDSBytes;  // kQStages x (64 lse2 + 64 D_i) fp32
  static constexpr int kList = kStats + kQStages * 2 * kBQ * 4;  // column list, uint16
  static constexpr int kTurn = kList + kMaxList * 2;  // fixed-order dQ: turn of each list entry, uint16
  static constexpr int kHeads = kTurn + kMaxList * 2;  // [q_per_kv + 1] list offsets, int32 (<= 65)
  static constexpr int kBar = kHeads + 65 * 4 + 12;      // (8-byte aligned)
  enum { KV_FULL, QDO_FULL0, QDO_FULL1, QDO_FULL2, QDO_EMPTY0, QDO_EMPTY1, QDO_EMPTY2, SDP_FULL, DP_FREE,
         DS_READY, DS_EMPTY0, DS_EMPTY1, DQ_FULL, DQ_EMPTY, ACC_FULL, DRAIN,
         QT_GO0, QT_GO1, QT_READY0, QT_READY1, KT_READY,  // fp32 path: operand transposes
         kNumBars };
  static constexpr int kMisc = kBar + kNumBars * 8;  // [0] TMEM base, [1] abort, [2] zero flag
  static constexpr int kCanaryAt = kMisc + 16;        // FM_DEBUG: shared-memory canary words
  static constexpr int kBytes = kCanaryAt + kCanaryBytes;
  static constexpr int kAlloc = kBytes + 1024;
};

// fp32 path.  kind::tf32 MMAs take K-major operands only, so the products that
// contract over queries (dV, dK) need Q^T and dO^T, and dQ^T needs K^T.  The
// dQ-drain warpgroup makes them in shared memory.  Layout of an fp32 operand
// with 128-byte swizzle: atoms of 32 columns x R rows, element (row, col) at
// (col / 32) * R * 128 + row * 128 + ((((col % 32) / 4) ^ (row % 8)) * 16) + (col % 4) * 4.
__device__ __forceinline__ uint32_t f32_sw128_off(int row, int col, int rows) {
  return (uint32_t)((col >> 5) * rows * 128 + row * 128 + ((((col & 31) >> 2) ^ (row & 7)) << 4) + (col & 3) * 4);
}

// In-place transpose of a 64 x 64 fp32 tile (Q or dO sub-tile [q][d] -> [d][q]) by 128 threads,
// rounding to tf32.  Named barrier 1 separates the reads from the writes.
__device__ __forceinline__ void transpose64_f32(uint8_t* t, int tid) {
  uint32_t v[32];
#pragma unroll
  for (int it = 0; it < 32; ++it) {
    const int e = it * 128 + tid;
    v[it] = *reinterpret_cast<const uint32_t*>(t + f32_sw128_off(e >> 6, e & 63, 64));
  }
  asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
  for (int it = 0; it < 32; ++it) {
    const int e = it * 128 + tid;
    *reinterpret_cast<uint32_t*>(t + f32_sw128_off(e & 63, e >> 6, 64)) = round_tf32(__uint_as_float(v[it]));
  }
}

// The 128 drain threads leave or enter a transpose (which synchronises on named barrier 1)
// together: each votes after its own bounded wait.
__device__ __forceinline__ bool all_drain_threads(bool v) { return named_bar_and(1, 128, v); }

// K [128 keys][64 d] -> K^T [64 d][128 keys], both fp32 with 128-byte swizzle, by 128 threads.
__device__ __forceinline__ void transpose_k_f32(const uint8_t* k, uint8_t* kt, int tid) {
#pragma unroll 8
  for (int it = 0; it < 64; ++it) {
    const int e = it * 128 + tid, key = e >> 6, d = e & 63;
    const float x = *reinterpret_cast<const float*>(k + f32_sw128_off(key, d, kTile));
    *reinterpret_cast<uint32_t*>(kt + f32_sw128_off(d, key, 64)) = round_tf32(x);
  }
}

template <int D, bool F32>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
               const BwdParams p) {
  using S = BwdSmem<D, F32>;
  constexpr int NS = S::kQStages;
  constexpr int NDS = S::kDSBufs;
  constexpr int kAtomElems = 128 / S::kElem;  // elements per 128-byte swizzle span
  constexpr int kAtoms = D * S::kElem / 128;   // swizzle-atom columns of a K / V / Q / dO row
  // d columns this launch accumulates into dK, dV and dQ: all of D, or one half of D = 256 (from p.dh0)
  constexpr int DH = D > 128 ? 128 : D;
  constexpr int kAtomsH = DH * S::kElem / 128;
  constexpr int kKStep = F32 ? 8 : 16;         // elements per UMMA K step (32 bytes)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_base_1024(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid (group * T_k, ceil(H_kv / group), B): one CTA per (key tile, K/V head hk); a group of K/V
  // heads at a time, rank by rank over the group (rank r takes the key tile with the r-th longest
  // column list), the group sized so that its heads' Q, dO and dQ accumulator stay in L2.  With
  // grouped-query attention the q_per_kv query heads hk * q_per_kv + j share this K/V head: their
  // column lists are walked back to back (dK and dV accumulate over all of them); the list of head
  // j starts at entry hstart[j].
  const int hk = (int)blockIdx.y * p.group + (int)(blockIdx.x % p.group), b = blockIdx.z;
  if (hk >= p.H_kv) return;  // partial last group
  const int G = p.q_per_kv, hq0 = hk * G;
  auto bhm_of = [&](int hq) -> int64_t { return (int64_t)b * p.Hm + (p.Hm == 1 ? 0 : hq); };
  const int kt = p.order ? __ldg(p.order + bhm_of(hq0) * p.T_k + blockIdx.x / p.group) : (int)(blockIdx.x / p.group);
  int cnt_raw = 0;  // entries over the group's query heads
  for (int jq = 0; jq < G; ++jq) cnt_raw += __ldg(p.col_count + bhm_of(hq0 + jq) * p.T_k + kt);
  const int cnt = kDebug ? min(max(cnt_raw, 0), kMaxList) : cnt_raw;  // (debug: recorded below, clamped)
  const int nsub = 2 * cnt;  // two 64-row sub-tiles per listed 128-row query tile

  const uint32_t bar0 = smem_u32(smem + S::kBar);
  auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  const volatile int* never = reinterpret_cast<const volatile int*>(misc + 2);
  const uint32_t k_s = smem_u32(smem + S::kK), v_s = smem_u32(smem + S::kV);
  const uint32_t q_s = smem_u32(smem + S::kQ), do_s = smem_u32(smem + S::kDO), ds_s = smem_u32(smem + S::kDS);
  const float* stats = reinterpret_cast<const float*>(smem + S::kStats);
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + S::kList);

  if (threadIdx.x == 0) {
    for (int k = 0; k < S::kNumBars; ++k) mbar_init(bar(k), 1);
    mbar_init(bar(S::DP_FREE), 2 * kTile);
    mbar_init(bar(S::DS_READY), 2 * kTile);
    mbar_init(bar(S::DQ_EMPTY), kTile);
    mbar_init(bar(S::QT_READY0), kTile);
    mbar_init(bar(S::QT_READY1), kTile);
    mbar_init(bar(S::KT_READY), kTile);
    *abort_flag = 0;
    misc[2] = 0;
    canary_write(smem + S::kCanaryAt);
    check_range(cnt_raw, 0, kMaxList + 1, p.status, abort_flag, 51);
    fence_barrier_init();
    {  // K and V first (as soon as the key tile is known): their latency overlaps the list copy and
       // the TMEM allocation.  A CTA with an empty list waits for them before it exits.
      fence_proxy_async_smem();
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(bar(S::KV_FULL), 2 * kTile * D * S::kElem);
      for (int c = 0; c < kAtoms; ++c) {
        tma_load_4d(k_s + c * 16384, &tm_k, bar(S::KV_FULL), c * kAtomElems, hk, kt * kTile, b);
        tma_load_4d(v_s + c * 16384, &tm_v, bar(S::KV_FULL), c * kAtomElems, hk, kt * kTile, b);
      }
    }
  }
  int* hstart = reinterpret_cast<int*>(smem + S::kHeads);  // [G + 1]
  uint16_t* turn = reinterpret_cast<uint16_t*>(smem + S::kTurn);
  {
    // Fixed-order dQ walks each list from the last query tile down, so that the key tiles of a
    // head, which all start their lists at about the same time, reach a shared query tile in
    // ascending order a few adds apart rather than a whole list apart.
    const bool rev = p.turn != nullptr;
    int start = 0;
    for (int jq = 0; jq < G; ++jq) {
      const int64_t bj = bhm_of(hq0 + jq);
      const int cj = __ldg(p.col_count + bj * p.T_k + kt);
      const int32_t* ej = p.col_entries + (bj * p.T_k + kt) * p.T_q;
      if (threadIdx.x == 0) hstart[jq] = start;
      const int cj_room = kDebug ? min(cj, cnt - start) : cj;  // (debug: never past the clamped total)
      for (int t = threadIdx.x; t < cj_room; t += kBwdThreads) {
        const int32_t e = __ldg(ej + (rev ? cj - 1 - t : t));
        list[start + t] = (uint16_t)e;
        if (rev && (!kDebug || (e >> 1) < p.T_q)) turn[start + t] = __ldg(p.turn + (bj * p.T_k + kt) * p.T_q + (e >> 1));
      }
      start += cj;
    }
    if (threadIdx.x == 0) hstart[G] = start;
  }
  if (!F32 && kAtoms * 128 * kTile < S::kKBytes) {  // K^T as a 128-row MMA operand: rows d >= D read zeros
    uint4* z = reinterpret_cast<uint4*>(smem + S::kK + kAtoms * 128 * kTile);
    for (int t = threadIdx.x; t < (S::kKBytes - kAtoms * 128 * kTile) / 16; t += blockDim.x)
      z[t] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 13) {
    tmem_alloc(smem_u32(misc), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  // TMEM columns: S^T / P^T double buffer [0,64) [64,128), dP^T [128,192), dQ^T [192,256), dV, dK;
  // fp32 (D = 64): dS^T [320,384) as the TMEM operand of dK
  const uint32_t tdP = tmem + 128, tdQ = tmem + 192, tdV = tmem + 256, tdK = tmem + 384, tdS = tmem + 320;
  auto sub_q0 = [&](int i) { return (int)(list[i >> 1] >> 1) * kTile + (i & 1) * kBQ; };
  // query head (offset in the group) of sub-tile i; each role advances its own cursor jh
  auto head_of = [&](int i, int& jh) {
    while ((i >> 1) >= hstart[jh + 1]) ++jh;
    return jh;
  };

  if (warp == 12) {
    // ------------------------------------------------------------ load role
    if (lane == 0 && cnt > 0) {
      prefetch_tmap(&tm_q);  // (K and V were issued at the start)
      prefetch_tmap(&tm_do);
      int jh = 0;
      for (int i = 0; i < nsub; ++i) {
        const int st = i % NS, use = i / NS;
        if (use >= 1 && !mbar_wait(bar(S::QDO_EMPTY0 + st), (use - 1) & 1, abort_flag)) {
          record_failure(p.status, abort_flag, 11);
          break;
        }
        const int q0 = sub_q0(i);
        if (!check_range(q0 >> 7, 0, p.T_q, p.status, abort_flag, 52)) break;  // a list entry past the query tiles
        const int hq = hq0 + (G > 1 ? head_of(i, jh) : 0);
        const int64_t bh = (int64_t)b * p.H + hq;
        const uint32_t fb = bar(S::QDO_FULL0 + st);
        mbar_arrive_expect_tx(fb, 2 * S::kQStage + 2 * kBQ * 4);
        for (int c = 0; c < kAtoms; ++c) {
          tma_load_4d(q_s + st * S::kQStage + c * 8192, &tm_q, fb, c * kAtomElems, hq, q0, b);
          tma_load_4d(do_s + st * S::kQStage + c * 8192, &tm_do, fb, c * kAtomElems, hq, q0, b);
        }
        bulk_load(smem_u32(stats + st * 2 * kBQ), p.lse2 + bh * p.n_q_pad + q0, kBQ * 4, fb);
        bulk_load(smem_u32(stats + st * 2 * kBQ + kBQ), p.dvec + bh * p.n_q_pad + q0, kBQ * 4, fb);
      }
    }
  } else if (warp == 13) {
    // ------------------------------------------------------------- MMA role
    if (lane == 0 && cnt > 0) {
      // S^T, dP^T: [key][q]; dV, dK: [key][d] with B MN-major; dQ^T: [d][q] with A and B MN-major
      constexpr uint32_t kIdSdp = F32 ? idesc_tf32(128, kBQ, false, false) : idesc_bf16(128, kBQ, false, false);
      constexpr uint32_t kIdAcc = F32 ? idesc_tf32(128, DH, false, true) : idesc_bf16(128, DH, false, true);
      constexpr uint32_t kIdDq = F32 ? idesc_tf32(128, kBQ, true, true) : idesc_bf16(128, kBQ, true, true);
      // descriptor words (128-byte swizzle, SBO = 8 rows x 128 B); per k-step only the low word moves
      constexpr uint32_t kHi = desc_hi(1024);
      constexpr uint32_t kStageW = S::kQStage >> 4, kDSW = S::kDSBytes >> 4;
      const uint32_t lo_k = desc_lo(k_s, 16), lo_v = desc_lo(v_s, 16);           // K-major A of S^T, dP^T
      const int ah = (p.dh0 / 64);  // first atom column of this launch's d half (0 unless D = 256)
      const uint32_t lo_kt = desc_lo(k_s + ah * 16384, 16384);                     // K^T as MN-major A of dQ^T
      const uint32_t lo_q = desc_lo(q_s, 16), lo_do = desc_lo(do_s, 16);         // K-major B of S^T, dP^T
      const uint32_t lo_qmn = desc_lo(q_s + ah * 8192, 8192), lo_domn = desc_lo(do_s + ah * 8192, 8192);  // B of dK, dV
      const uint32_t lo_ds = desc_lo(ds_s, 16), lo_dsmn = desc_lo(ds_s, 16384);   // dS^T as A of dK / B of dQ^T
      auto issue_s = [&](int i) {  // S^T_i = K Q_i^T
        const uint32_t qa = lo_q + (i % NS) * kStageW, tS = tmem + (i & 1) * 64;
#pragma unroll
        for (int k = 0; k < D / kKStep; ++k) {
          const uint32_t okv = ((k >> 2) * 16384 + (k & 3) * 32) >> 4, oq = ((k >> 2) * 8192 + (k & 3) * 32) >> 4;
          umma_ss_w<F32>(tS, lo_k + okv, kHi, qa + oq, kHi, kIdSdp, k > 0 ? 1u : 0u);
        }
      };
      auto issue_dp = [&](int i) {  // dP^T_i = V dO_i^T
        const uint32_t da = lo_do + (i % NS) * kStageW;
#pragma unroll
        for (int k = 0; k < D / kKStep; ++k) {
          const uint32_t okv = ((k >> 2) * 16384 + (k & 3) * 32) >> 4, oq = ((k >> 2) * 8192 + (k & 3) * 32) >> 4;
          umma_ss_w<F32>(tdP, lo_v + okv, kHi, da + oq, kHi, kIdSdp, k > 0 ? 1u : 0u);
        }
      };
      // fp32: every operand K-major (atoms of 32 columns); Q^T / dO^T replace Q / dO in their stage once
      // S^T and dP^T have read them, K^T sits after K, dS is stored [q][key]
      constexpr uint32_t kIdAccT = idesc_tf32(128, D, false, false), kIdDqT = idesc_tf32(128, kBQ, false, false);
      const uint32_t lo_ktk = desc_lo(k_s + kTile * D * S::kElem, 16);
      auto toff = [](int k) -> uint32_t { return ((k >> 2) * 8192 + (k & 3) * 32) >> 4; };  // 64-row atoms
      bool ok = mbar_wait(bar(S::KV_FULL), 0, abort_flag) && mbar_wait(bar(S::QDO_FULL0), 0, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
        umma_commit(bar(S::SDP_FULL));
        if constexpr (F32) umma_commit(bar(S::QT_GO0));
      }
      // next sub-tile's S^T (other buffer) and dP^T.  With two or more Q/dO stages they are issued
      // before this sub-tile's dV / dK / dQ^T, so they overlap its softmax; with one stage (D = 256) the
      // next Q/dO can only arrive once this sub-tile's dV and dK have read the stage, so they follow.
      auto issue_next = [&](int i) -> bool {
        if (i + 1 >= nsub) return true;
        if (!mbar_wait(bar(S::QDO_FULL0 + (i + 1) % NS), ((i + 1) / NS) & 1, abort_flag)) return false;
        tc_fence_after();
        issue_s(i + 1);
        if (!mbar_wait(bar(S::DP_FREE), i & 1, abort_flag)) return false;
        tc_fence_after();
        issue_dp(i + 1);
        umma_commit(bar(S::SDP_FULL));
        if constexpr (F32) umma_commit(bar(S::QT_GO0 + (i + 1) % NS));
        return true;
      };
      for (int i = 0; ok && i < nsub; ++i) {
        const int st = i % NS, bi = i % NDS;
        if (NS > 1 && !issue_next(i)) {
          ok = false;
          break;
        }
        if (!mbar_wait(bar(S::DS_READY), i & 1, abort_flag)) {
          ok = false;
          break;
        }
        if constexpr (F32) {
          if (!mbar_wait(bar(S::QT_READY0 + st), (i / NS) & 1, abort_flag) ||
              (i == 0 && !mbar_wait(bar(S::KT_READY), 0, abort_flag))) {
            ok = false;
            break;
          }
        }
        tc_fence_after();
        const uint32_t qmn = lo_qmn + st * kStageW, domn = lo_domn + st * kStageW;
        const uint32_t dsa = lo_ds + bi * kDSW, dsb = lo_dsmn + bi * kDSW;
        const uint32_t tP = tmem + (i & 1) * 64;
        if constexpr (F32) {
          // dV += P^T dO^T-operand, dK += dS^T Q^T-operand (A from TMEM, query q in column q)
#pragma unroll
          for (int k = 0; k < kBQ / kKStep; ++k) {
            const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
            umma_ts_w<true>(tdV, tP + k * 8, lo_do + st * kStageW + toff(k), kHi, kIdAccT, acc);
            umma_ts_w<true>(tdK, tdS + k * 8, lo_q + st * kStageW + toff(k), kHi, kIdAccT, acc);
          }
          umma_commit(bar(S::QDO_EMPTY0 + st));
          if (i > 0 && !mbar_wait(bar(S::DQ_EMPTY), (i - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // dQ^T = K^T dS^T: A = K^T (rows d >= 64 read the next atom; those output rows are ignored),
          // B = dS stored [q][key]
#pragma unroll
          for (int k = 0; k < kTile / kKStep; ++k)
            umma_ss_w<true>(tdQ, lo_ktk + toff(k), kHi, lo_ds + toff(k), kHi, kIdDqT, k > 0 ? 1u : 0u);
        } else {
          // dV += P^T dO (P^T in TMEM, 8 columns per K step; dO MN-major): queries [0, 32) of P^T are
          // packed in columns [0, 16) of the buffer, queries [32, 64) in columns [32, 48).
#pragma unroll
          for (int k = 0; k < kBQ / kKStep; ++k)
            umma_ts_w<false>(tdV, tP + (k >> 1) * 32 + (k & 1) * 8, domn + ((k * kKStep * 128) >> 4), kHi, kIdAcc,
                             (i > 0 || k > 0) ? 1u : 0u);
          // dK += dS^T Q (dS^T K-major in smem; Q MN-major)
#pragma unroll
          for (int k = 0; k < kBQ / kKStep; ++k)
            umma_ss_w<false>(tdK, dsa + (((k >> 2) * 16384 + (k & 3) * 32) >> 4), kHi,
                             qmn + ((k * kKStep * 128) >> 4), kHi, kIdAcc, (i > 0 || k > 0) ? 1u : 0u);
          umma_commit(bar(S::QDO_EMPTY0 + st));
          if (i > 0 && !mbar_wait(bar(S::DQ_EMPTY), (i - 1) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // dQ^T = K^T dS^T (K^T: M = d, MN-major; dS^T as B: N = q, MN-major; 16 keys per step)
#pragma unroll
          for (int k = 0; k < kTile / kKStep; ++k)
            umma_ss_w<false>(tdQ, lo_kt + ((k * kKStep * 128) >> 4), kHi, dsb + ((k * kKStep * 128) >> 4), kHi,
                             kIdDq, k > 0 ? 1u : 0u);
        }
        umma_commit(bar(S::DQ_FULL));
        umma_commit(bar(S::DS_EMPTY0 + bi));
        if (NS == 1 && !issue_next(i)) ok = false;
      }
      if (!ok) record_failure(p.status, abort_flag, 12);
      umma_commit(bar(S::ACC_FULL));
      umma_commit(bar(S::DRAIN));
      mbar_wait(bar(S::DRAIN), 0, never);
    }
  } else if (warp < 8) {
    // ---------------------------- P^T / dS^T role (row = key), warps 0-7
    // Warpgroup hf handles queries [32 hf, 32 hf + 32) of every 64-query sub-tile.
    const int hf = warp >> 2;
    const int r = threadIdx.x & 127;
    const int c0 = 32 * hf;
    const int64_t j = (int64_t)kt * kTile + r;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const bool no_key = j >= p.n_k;  // past a ragged n_k: a zero-filled key row, masked for every query
    int32_t lts, lte, uts, ute;
    auto load_bounds = [&](int jq) {  // this key's bounds for query head hq0 + jq
      const int64_t voff = bhm_of(hq0 + jq) * p.n_k + j;
      lts = (p.vec[0] && !no_key) ? __ldg(p.vec[0] + voff) : p.n_q;
      lte = (p.vec[1] && !no_key) ? __ldg(p.vec[1] + voff) : p.n_q;
      uts = (p.vec[2] && !no_key) ? __ldg(p.vec[2] + voff) : 0;
      ute = (p.vec[3] && !no_key) ? __ldg(p.vec[3] + voff) : 0;
    };
    load_bounds(0);
    const bool per_head = G > 1 && p.Hm != 1;  // grouped query heads with masks of their own
    int jh = 0, jv = 0;  // head cursor; head whose bounds are loaded
    bool ok = true;
    for (int i = 0; i < nsub; ++i) {
      if (per_head) {
        const int jq = head_of(i, jh);
        if (jq != jv) {
          load_bounds(jq);
          jv = jq;
        }
      }
      const int st = i % NS, bi = i % NDS, sb = i & 1;  // Q/dO stage, dS^T buffer, S^T buffer
      const int q0 = sub_q0(i) + c0;
      const bool partial = list[i >> 1] & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(S::SDP_FULL), i & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t sd[64];  // [0, 32): S^T row, [32, 64): dP^T row (this warpgroup's queries)
      tmem_ld32x2(tmem + sb * 64 + c0 + lane_addr, tdP + c0 + lane_addr, sd);
      tc_fence_before();
      mbar_arrive(bar(S::DP_FREE));  // dP^T columns may be overwritten by the next sub-tile
      ok = __all_sync(0xffffffffu, mbar_wait(bar(S::QDO_FULL0 + st), (i / NS) & 1, abort_flag));
      if (!ok) break;
      const float4* l2 = reinterpret_cast<const float4*>(stats + st * 2 * kBQ + c0);
      const float4* dd = reinterpret_cast<const float4*>(stats + st * 2 * kBQ + kBQ + c0);
      // row-interval test (partial tiles only) as a mask of this key's masked queries
      const uint32_t mbits =
          no_key ? 0xFFFFFFFFu : (partial ? (interval_bits32(lts, lte, q0) | interval_bits32(uts, ute, q0)) : 0u);
      const uint64_t sc2 = f2pack(p.scale_log2, p.scale_log2);
      uint32_t pk[F32 ? 32 : 16], dk[F32 ? 32 : 16];  // bf16 pairs or tf32-rounded fp32
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        const float4 L = l2[c4], Dd = dd[c4];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int qc = c4 * 4 + 2 * h2;
          const uint64_t nl2 = h2 ? f2pack(-L.z, -L.w) : f2pack(-L.x, -L.y);
          const uint64_t nd2 = h2 ? f2pack(-Dd.z, -Dd.w) : f2pack(-Dd.x, -Dd.y);
          const uint64_t x2 = fma2(((uint64_t)sd[qc + 1] << 32) | sd[qc], sc2, nl2);
          float p0 = ex2(f2lo(x2)), p1 = ex2(f2hi(x2));  // 0 on empty rows (lse2 = +inf)
          p0 = ((mbits >> qc) & 1) ? 0.f : p0;
          p1 = ((mbits >> (qc + 1)) & 1) ? 0.f : p1;
          const uint64_t ds2 = mul2(f2pack(p0, p1), add2(((uint64_t)sd[32 + qc + 1] << 32) | sd[32 + qc], nd2));
          if constexpr (F32) {
            pk[qc] = round_tf32(p0);
            pk[qc + 1] = round_tf32(p1);
            dk[qc] = round_tf32(f2lo(ds2));
            dk[qc + 1] = round_tf32(f2hi(ds2));
          } else {
            pk[qc >> 1] = pack_bf16(p0, p1);
            dk[qc >> 1] = pack_bf16(f2lo(ds2), f2hi(ds2));
          }
        }
      }
      // P^T (bf16 pairs) into 16 columns of this warpgroup's own S^T range (already read)
      if constexpr (F32)
        tmem_st32(tmem + sb * 64 + c0 + lane_addr, pk);
      else
        tmem_st16(tmem + sb * 64 + c0 + lane_addr, pk);
      if (i >= NDS) {  // dS^T buffer bi free: the dK / dQ^T MMAs of sub-tile i-NDS have read it
        ok = __all_sync(0xffffffffu, mbar_wait(bar(S::DS_EMPTY0 + bi), ((i / NDS) - 1) & 1, abort_flag));
        if (!ok) break;
      }
      if constexpr (F32) {
        // dS^T into TMEM (the A operand of dK), and dS [q][key] K-major (the B operand of dQ^T):
        // for one query the warp's 32 keys fill one 128-byte row of atom r / 32
        tmem_st32(tdS + c0 + lane_addr, dk);
        uint8_t* ds_col = smem + S::kDS + (r >> 5) * 8192 + (r & 3) * 4;
#pragma unroll
        for (int qc = 0; qc < 32; ++qc) {
          const int q = c0 + qc;
          *reinterpret_cast<uint32_t*>(ds_col + q * 128 + ((((r & 31) >> 2) ^ (q & 7)) << 4)) = dk[qc];
        }
      } else {
        // dS^T row r, queries [c0, c0+32), 128-byte swizzle (16-byte chunk c of a row at c ^ (r & 7)):
        // four chunks of the row's single atom

        uint8_t* ds_row = smem + S::kDS + bi * S::kDSBytes + r * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int chunk = 4 * hf + c;
          *reinterpret_cast<uint4*>(ds_row + ((chunk ^ (r & 7)) << 4)) =
              make_uint4(dk[4 * c], dk[4 * c + 1], dk[4 * c + 2], dk[4 * c + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(S::DS_READY));
    }
    if (!ok) record_failure(p.status, abort_flag, 13);
  } else {
    // ------------------------------------- dQ drain role (row = d), warps 8-11
    // fp32: also the operand transposes (K^T once; Q^T and dO^T per sub-tile, in place after S^T and
    // dP^T have read the stage)
    const int d = threadIdx.x - 256;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    int jh = 0;
    bool ok = true;
    if constexpr (F32) {
      if (nsub > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(S::KV_FULL), 0, abort_flag));
        if (ok) {
          transpose_k_f32(smem + S::kK, smem + S::kK + kTile * D * S::kElem, d);
          fence_proxy_async_smem();
          mbar_arrive(bar(S::KT_READY));
        }
      }
    }
    for (int i = 0; ok && i < nsub; ++i) {
      const int q0 = sub_q0(i);
      const int64_t bh = (int64_t)b * p.H + hq0 + (G > 1 ? head_of(i, jh) : 0);
      float* acc_bh = p.dq_acc + bh * (int64_t)p.n_q_pad * D + p.dh0 * 4;
      if constexpr (F32) {
        const int st = i % NS;
        ok = all_drain_threads(mbar_wait(bar(S::QT_GO0 + st), (i / NS) & 1, abort_flag));
        if (!ok) break;
        transpose64_f32(smem + S::kQ + st * S::kQStage, d);
        transpose64_f32(smem + S::kDO + st * S::kQStage, d);
        fence_proxy_async_smem();
        mbar_arrive(bar(S::QT_READY0 + st));
      }
      ok = __all_sync(0xffffffffu, mbar_wait(bar(S::DQ_FULL), i & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t a[64];
      tmem_ld64(tdQ + lane_addr, a);
      tc_fence_before();
      mbar_arrive(bar(S::DQ_EMPTY));
      int* sem = p.dq_sem ? p.dq_sem + bh * p.T_q + (q0 >> 7) : nullptr;
      if (sem && (i & 1) == 0) {  // fixed order: wait until the key tiles before this one have added
        ok = all_drain_threads(d != 0 || flag_wait_eq(sem, turn[i >> 1], p.status, abort_flag));
        if (!ok) break;
      }
      if (d < DH && (!kDebug || check_range(q0 >> 7, 0, p.T_q, p.status, abort_flag, 53))) {
        float* blk = acc_bh + (int64_t)q0 * D;  // [16 groups of 4 queries][D][4]
#pragma unroll
        for (int g = 0; g < 16; ++g)
          red_add_v4(blk + (g * D + d) * 4, __uint_as_float(a[4 * g]), __uint_as_float(a[4 * g + 1]),
                     __uint_as_float(a[4 * g + 2]), __uint_as_float(a[4 * g + 3]));
      }
      if (sem && (i & 1) == 1) {  // both sub-tiles added: pass the query tile on to the next key tile
        all_drain_threads(true);
        if (d == 0) st_release_gpu(sem, turn[i >> 1] + 1);
      }
    }
    if (!ok) record_failure(p.status, abort_flag, 14);
  }

  // ---------------------------------------------- epilogue: dV (warps 0-3), dK (warps 4-7)
  // Each warpgroup stages its 128 x D tile (output dtype, 128-byte swizzle) in the Q (dV) or dO (dK)
  // stage buffers, which no load or MMA touches any more, and one of its threads TMA-stores it.
  if (warp < 8) {
    const int r = threadIdx.x & 127;
    const uint32_t lane_addr = (uint32_t)((warp & 3) * 32) << 16;
    const bool is_dk = warp >= 4;
    bool have = false;
    if (cnt > 0) {
      have = __all_sync(0xffffffffu, mbar_wait(bar(S::ACC_FULL), 0, abort_flag));
      tc_fence_after();
    }
    const float mul = is_dk ? p.scale : 1.f;
    const uint32_t tsrc = (is_dk ? tdK : tdV) + lane_addr;
    uint8_t* stage = smem + (is_dk ? S::kDO : S::kQ);
#pragma unroll
    for (int cc = 0; cc < DH / 32; ++cc) {
      uint32_t a[32];
      if (have) {
        tmem_ld32(tsrc + cc * 32, a);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) a[c] = 0u;
      }
      if constexpr (F32) {  // 32 fp32 = one atom row: chunks 0..7 of atom cc
        uint8_t* row = stage + cc * 16384 + r * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4*>(row + ((ch ^ (r & 7)) << 4)) =
              make_uint4(__float_as_uint(__uint_as_float(a[4 * ch]) * mul),
                         __float_as_uint(__uint_as_float(a[4 * ch + 1]) * mul),
                         __float_as_uint(__uint_as_float(a[4 * ch + 2]) * mul),
                         __float_as_uint(__uint_as_float(a[4 * ch + 3]) * mul));
      } else {  // 32 bf16 = half an atom row: chunks 4 (cc & 1) .. +3 of atom cc / 2
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2)
          pk[c >> 1] = pack_bf16(__uint_as_float(a[c]) * mul, __uint_as_float(a[c + 1]) * mul);
        uint8_t* row = stage + (cc >> 1) * 16384 + r * 128;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          *reinterpret_cast<uint4*>(row + ((((cc & 1) * 4 + ch) ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(is_dk ? 3 : 2, 128);
    if (r == 0) {
      for (int c = 0; c < kAtomsH; ++c)
        tma_store_4d(is_dk ? &tm_dk : &tm_dv, smem_u32(stage + c * 16384), p.dh0 + c * kAtomElems, hk, kt * kTile, b);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  }

  if (threadIdx.x == 0 && cnt == 0) mbar_wait(bar(S::KV_FULL), 0, never);  // no copy in flight at exit
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) canary_check(smem + S::kCanaryAt, p.status, abort_flag, 54);
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D_i = dO_i . O_i, log2-domain LSE (+inf for empty rows so that P = 0), and
// a cleared dQ accumulator.  One thread per (b, i, h) row.
template <int D, bool F32>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const void* __restrict__ o, const void* __restrict__ dout,
                                                       const float* __restrict__ lse, float* __restrict__ lse2,
                                                       float* __restrict__ dvec, float* __restrict__ acc, int B,
                                                       int H, int n_q, int n_q_pad, int* __restrict__ dq_sem) {
  const int64_t rows = (int64_t)B * n_q * H;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < rows) {
    const int h = (int)(t % H);
    const int64_t bi = t / H;
    const int i = (int)(bi % n_q), b = (int)(bi / n_q);
    float s = 0.f;
    if constexpr (F32) {
      const float4* po = reinterpret_cast<const float4*>(static_cast<const float*>(o) + t * D);
      const float4* pd = reinterpret_cast<const float4*>(static_cast<const float*>(dout) + t * D);
#pragma unroll 4
      for (int c = 0; c < D / 4; ++c) {
        const float4 a = __ldg(po + c), g = __ldg(pd + c);
        s = fmaf(a.x, g.x, fmaf(a.y, g.y, fmaf(a.z, g.z, fmaf(a.w, g.w, s))));
      }
    } else {
      const uint4* po = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(o) + t * D);
      const uint4* pd = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(dout) + t * D);
#pragma unroll 4
      for (int c = 0; c < D / 8; ++c) {
        const uint4 a = __ldg(po + c), g = __ldg(pd + c);
        const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, gw[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float2 fa = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&aw[u]));
          const float2 fg = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&gw[u]));
          s = fmaf(fa.x, fg.x, s);
          s = fmaf(fa.y, fg.y, s);
        }
      }
    }
    const int64_t out = ((int64_t)b * H + h) * n_q_pad + i;  // rows padded to whole query tiles
    dvec[out] = s;
    const float l = lse[((int64_t)b * H + h) * n_q + i];
    lse2[out] = (l == kNegInf) ? kPosInf : l * 1.4426950408889634f;
  }
  // padding rows past a ragged n_q: P = 0 there (log2 LSE = +inf), D_i = 0
  const int pad = n_q_pad - n_q;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  if (pad > 0)
    for (int64_t k = t; k < (int64_t)B * H * pad; k += stride) {
      const int64_t row = (k / pad) * n_q_pad + n_q + (k % pad);
      lse2[row] = kPosInf;
      dvec[row] = 0.f;
    }
  // clear the accumulator (B*H*n_q_pad*D floats), grid-stride in float4
  float4* a4 = reinterpret_cast<float4*>(acc);
  const int64_t n4 = (int64_t)B * H * n_q_pad * D / 4;
  for (int64_t k = t; k < n4; k += stride) a4[k] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (dq_sem)  // fixed-order dQ: no key tile has added yet
    for (int64_t k = t; k < (int64_t)B * H * (n_q_pad / kTile); k += stride) dq_sem[k] = 0;
}

// Fixed-order dQ: turn[bhm, kt, qt] = position of key tile kt in the row list of query tile qt
// (the number of non-skip key tiles before it), one warp per row list.  Entries of skip pairs
// are never read and stay unwritten.
__global__ void __launch_bounds__(256) bwd_turn_kernel(const int32_t* __restrict__ row_count,
                                                       const int32_t* __restrict__ row_entries,
                                                       uint16_t* __restrict__ turn, int BHm, int T_q, int T_k) {
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= (int64_t)BHm * T_q) return;
  const int64_t bhm = w / T_q;
  const int qt = (int)(w % T_q);
  const int c = __ldg(row_count + w);
  const int32_t* e = row_entries + w * T_k;
  for (int pos = lane; pos < c; pos += 32)
    turn[(bhm * T_k + (__ldg(e + pos) >> 1)) * T_q + qt] = (uint16_t)pos;
}

// dQ[b, i, h, :] = scale * acc for one 64-row block per CTA: the block (16 groups of 4 rows, each
// D x 4 fp32) is read coalesced into shared memory (padded against bank conflicts) a chunk of at
// most 128 d columns at a time, then each thread writes 8 consecutive d of one row.
template <int D, bool F32>
__global__ void __launch_bounds__(256) bwd_dq_kernel(const float* __restrict__ acc, void* __restrict__ dq,
                                                     int B, int H, int n_q, int n_q_pad, float scale) {
  constexpr int DC = D > 128 ? 128 : D;  // d columns per chunk
  __shared__ float4 buf[16 * DC + 2 * DC];  // one float4 of padding per 8
  const int blocks_per_bh = n_q_pad / 64;
  const int64_t bh = blockIdx.x / blocks_per_bh;
  const int qb = blockIdx.x % blocks_per_bh;
  const int b = (int)(bh / H), h = (int)(bh % H);
  const float4* src = reinterpret_cast<const float4*>(acc + (bh * n_q_pad + (int64_t)qb * 64) * D);
#pragma unroll 1
  for (int dc0 = 0; dc0 < D; dc0 += DC) {
    if (dc0 > 0) __syncthreads();  // the previous chunk's reads of buf are done
    for (int k = threadIdx.x; k < 16 * DC; k += blockDim.x) {
      const int g = k / DC, dd = k % DC;
      buf[k + (k >> 3)] = __ldg(src + g * D + dc0 + dd);
    }
    __syncthreads();
    for (int w = threadIdx.x; w < 64 * (DC / 8); w += blockDim.x) {
      const int q = w / (DC / 8), d0 = (w % (DC / 8)) * 8;
      if (qb * 64 + q >= n_q) continue;  // padding rows past a ragged n_q
      const int g = q >> 2, u = q & 3;
      float x[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const int k = g * DC + d0 + c;
        const float4 f = buf[k + (k >> 3)];
        x[c] = (u == 0 ? f.x : u == 1 ? f.y : u == 2 ? f.z : f.w) * scale;
      }
      const int64_t off = (((int64_t)b * n_q + (int64_t)qb * 64 + q) * H + h) * D + dc0 + d0;
      if constexpr (F32) {
        float* row = static_cast<float*>(dq) + off;
        st_global_v4(row, __float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]), __float_as_uint(x[3]));
        st_global_v4(row + 4, __float_as_uint(x[4]), __float_as_uint(x[5]), __float_as_uint(x[6]),
                     __float_as_uint(x[7]));
      } else {
        __nv_bfloat16* row = static_cast<__nv_bfloat16*>(dq) + off;
        st_global_v4(row, pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
      }
    }
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdLayout {
  size_t acc, lse2, dvec, turn, sem, total;
};

// Workspace: fp32 dQ accumulator, log2 LSE and D_i per padded row; for fixed-order dQ also the
// turn table (sized for Hm = H, the larger of the two mask-head counts) and one counter per
// query tile.
BwdLayout bwd_layout(const fm_attn_args* a) {
  BwdLayout L;
  const size_t T_q = ((size_t)a->n_q + kTile - 1) / kTile, T_k = ((size_t)a->n_k + kTile - 1) / kTile;
  const size_t rows = (size_t)a->B * a->H * T_q * kTile;  // padded rows
  L.acc = 0;
  L.lse2 = align256(rows * a->D * 4);
  L.dvec = L.lse2 + align256(rows * 4);
  L.turn = L.sem = L.total = L.dvec + align256(rows * 4);
  if (a->deterministic) {
    L.sem = L.turn + align256((size_t)a->B * a->H * T_k * T_q * 2);
    L.total = L.sem + align256((size_t)a->B * a->H * T_q * 4);
  }
  return L;
}

template <int D, bool F32>
fm_status launch_bwd(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4], const void* o,
                     const float* lse, const void* dout, void* dq, void* dk, void* dv, void* ws, cudaStream_t stream) {
  using S = BwdSmem<D, F32>;
  static_assert(S::kAlloc <= 227 * 1024, "backward shared memory exceeds the per-CTA limit");
  const BwdLayout L = bwd_layout(a);
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* acc = reinterpret_cast<float*>(w + L.acc);
  float* lse2 = reinterpret_cast<float*>(w + L.lse2);
  float* dvec = reinterpret_cast<float*>(w + L.dvec);
  uint16_t* turn = a->deterministic ? reinterpret_cast<uint16_t*>(w + L.turn) : nullptr;
  int* dq_sem = a->deterministic ? reinterpret_cast<int*>(w + L.sem) : nullptr;
  const int H_kv = a->H_kv ? a->H_kv : a->H;
  CUtensorMap tq, tdo, tk, tv, tdk, tdv;
  auto enc = F32 ? encode_tmap_f32_4d : encode_tmap_bf16_4d;
  if (!enc(&tq, a->q, D, a->H, a->n_q, a->B, kBQ) || !enc(&tdo, dout, D, a->H, a->n_q, a->B, kBQ) ||
      !enc(&tk, a->k, D, H_kv, a->n_k, a->B, kTile) || !enc(&tv, a->v, D, H_kv, a->n_k, a->B, kTile) ||
      !enc(&tdk, dk, D, H_kv, a->n_k, a->B, kTile) || !enc(&tdv, dv, D, H_kv, a->n_k, a->B, kTile))
    return FM_ERR_CUDA;
  const int64_t rows = (int64_t)a->B * a->n_q * a->H;
  bwd_prep_kernel<D, F32><<<(unsigned)((rows + 255) / 256), 256, 0, stream>>>(o, dout, lse, lse2, dvec, acc, a->B,
      a->H, a->n_q, (a->n_q + kTile - 1) / kTile * kTile, dq_sem);
  BwdParams p;
  p.col_count = meta->col_count;
  p.col_entries = meta->col_entries;
  p.order = turn ? nullptr : meta->bwd_order;  // fixed order: key tiles in ascending order
  p.turn = turn;
  p.dq_sem = dq_sem;
  for (int c = 0; c < 4; ++c) p.vec[c] = vec ? vec[c] : nullptr;
  p.lse2 = lse2;
  p.dvec = dvec;
  p.dq_acc = acc;
  p.dk = dk;
  p.dv = dv;
  p.status = device_status_ptr();
  p.B = a->B;
  p.H = a->H;
  p.Hm = meta->d.Hm;
  p.n_q = a->n_q;
  p.n_k = a->n_k;
  p.T_q = (a->n_q + kTile - 1) / kTile;
  p.T_k = (a->n_k + kTile - 1) / kTile;
  p.n_q_pad = p.T_q * kTile;
  p.H_kv = H_kv;
  p.q_per_kv = a->H / H_kv;
  // the CTAs of one K/V head re-read the Q, dO and fp32 dQ accumulator of its q_per_kv query heads
  p.group = dispatch_group(H_kv, (double)p.q_per_kv * a->n_q * D * (2 * S::kElem + 4));
  p.scale = a->scale;
  p.scale_log2 = a->scale * 1.4426950408889634f;
  if (!smem_opt_in<bwd_kernel<D, F32>>(S::kAlloc)) return FM_ERR_CUDA;
  if (turn) {
    const int64_t warps = (int64_t)a->B * meta->d.Hm * p.T_q;
    bwd_turn_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, stream>>>(meta->row_count, meta->row_entries, turn,
                                                                    a->B * meta->d.Hm, p.T_q, p.T_k);
  }
  // D = 256: dK, dV and dQ are accumulated one 128-column half per launch (TMEM holds 256 columns of
  // dK and dV at most); both launches form S^T and dP^T over all 256 columns
  for (p.dh0 = 0; p.dh0 < D; p.dh0 += (D > 128 ? 128 : D))
    bwd_kernel<D, F32><<<dim3(p.group * p.T_k, (p.H_kv + p.group - 1) / p.group, p.B), kBwdThreads, S::kAlloc, stream>>>(
        tq, tdo, tk, tv, tdk, tdv, p);
  bwd_dq_kernel<D, F32><<<(unsigned)((int64_t)a->B * a->H * (p.n_q_pad / 64)), 256, 0, stream>>>(
      acc, dq, a->B, a->H, a->n_q, p.n_q_pad, a->scale);
  return cudaGetLastError() == cudaSuccess ? FM_OK : FM_ERR_CUDA;
}

}  // namespace

// The backward's checks: the attention checks, plus room in shared memory for the column lists of
// all query heads that share a K/V head (q_per_kv x T_q entries at most).
fm_status check_bwd_args(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4]) {
  const fm_status st = check_attn_args(a, meta, vec);
  if (st != FM_OK) return st;
  if (a->D == 256 && a->deterministic) return FM_ERR_UNSUPPORTED;  // fixed-order dQ: D in {64, 128}
  const int H_kv = a->H_kv ? a->H_kv : a->H;
  if ((int64_t)(a->H / H_kv) * ((a->n_q + 127) / 128) > kMaxList) return FM_ERR_UNSUPPORTED;
  return FM_OK;
}

}  // namespace fm

extern "C" {

size_t fm_attn_bwd_workspace_bytes(const fm_attn_args* a) {
  if (!a || a->B < 1 || a->H < 1 || a->n_q < 1 || (a->D != 64 && a->D != 128 && a->D != 256)) return 0;
  return fm::bwd_layout(a).total;
}

fm_status fm_attn_bwd(const fm_attn_args* a, const fm_mask_meta* meta, const int32_t* const vec[4], const void* o,
                      const float* lse, const void* dout, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                      fm_stream_t stream) {
  fm_status st = fm::check_bwd_args(a, meta, vec);
  if (st != FM_OK) return st;
  const uintptr_t al = reinterpret_cast<uintptr_t>(o) | reinterpret_cast<uintptr_t>(dout) |
                       reinterpret_cast<uintptr_t>(dq) | reinterpret_cast<uintptr_t>(dk) |
                       reinterpret_cast<uintptr_t>(dv);
  if (!o || !lse || !dout || !dq || !dk || !dv || (al & 15) || (reinterpret_cast<uintptr_t>(lse) & 3))
    return FM_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255) || ws_bytes < fm_attn_bwd_workspace_bytes(a))
    return FM_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (a->dtype == 1) return fm::launch_bwd<64, true>(a, meta, vec, o, lse, dout, dq, dk, dv, ws, s);
  if (a->D == 256) return fm::launch_bwd<256, false>(a, meta, vec, o, lse, dout, dq, dk, dv, ws, s);
  return a->D == 64 ? fm::launch_bwd<64, false>(a, meta, vec, o, lse, dout, dq, dk, dv, ws, s)
                    : fm::launch_bwd<128, false>(a, meta, vec, o, lse, dout, dq, dk, dv, ws, s);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free backward: the same kernels with their scratch in a fixed
// device array owned by the library (see fm_attn_bwd_noalloc in fm.h).
// ---------------------------------------------------------------------------
static __device__ __align__(256) uint8_t g_bwd_noalloc_scratch[FM_BWD_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of the scratch array on the current device.  Looked up on every call (a symbol
// lookup, no allocation): a cached address would go stale after cudaDeviceReset or a new primary
// context, and the kernels would then write through it.
void* noalloc_scratch() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_bwd_noalloc_scratch) != cudaSuccess) return nullptr;
  return p;
}
}  // namespace

extern "C" fm_status fm_attn_bwd_noalloc(const fm_attn_args* a, const fm_mask_meta* meta,
                                         const int32_t* const vec[4], const void* o, const float* lse,
                                         const void* dout, void* dq, void* dk, void* dv, fm_stream_t stream) {
  fm_status st = fm::check_bwd_args(a, meta, vec);
  if (st != FM_OK) return st;
  if (fm_attn_bwd_workspace_bytes(a) > FM_BWD_NOALLOC_SCRATCH_BYTES) return FM_ERR_WORKSPACE;
  void* ws = noalloc_scratch();
  if (!ws) return FM_ERR_CUDA;
  return fm_attn_bwd(a, meta, vec, o, lse, dout, dq, dk, dv, ws, FM_BWD_NOALLOC_SCRATCH_BYTES, stream);
}
