// MALA backward (Algorithm 2, "Offline Sparse Probability", and Appendix A.1
// "Fused backward execution" of the MassAlloc Attention paper) on sm_100a.
//
// Key-major: one CTA per (batch, KV head, key block j) accumulates dK_j and
// dV_j in TMEM over every query head of the group and every query block i
// ascending from the diagonal whose tile (i, j) the forward retained. For a
// visited tile the score tile S^T = K_j Q_i^T is recomputed and tested
// against the saved log-normaliser: the tile is skipped iff for every legal
// (q, k) s_qk - z_q < log tau - log L_q. A retained tile loads dO_i and runs
//   P^T = exp(S^T - z), dV += P^T dO, dP^T = V dO^T, dS^T = P^T (dP^T - D),
//   dK += dS^T Q, dQ_i += dS K
// with dQ accumulated in fp32 by bulk reduce-add into a blocked workspace.
//
// Roles (192 threads): warps 0-3 compute (thread t owns key row t for
// S^T, P^T, dP^T, dS^T, dK, dV and query row t for the dQ part), warp 4
// TMA producer, warp 5 tcgen05 issuer.
// TMEM: X = cols [0,128) holds S^T, later the tile's dQ part; Y = [128,256)
// holds dP^T; dK = [256,384); dV = [384,512).
// Shared memory: K_j, V_j, Q_i, dO_i, P^T and dS^T tiles (bf16, 128-byte
// swizzle); the P^T tile doubles as the fp32 staging buffer of the dQ
// reduction once dV has consumed it.
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

namespace mala {

namespace {

constexpr int kB = 128;                       // B_q = B_k
constexpr int kD = 128;
constexpr int kThreads = 192;
constexpr uint32_t kTile = kB * kD * 2;       // 32 KB bf16 tile
constexpr uint32_t kChunk = 16384;            // one 64-column swizzle chunk of 128 rows
constexpr float kLog2e = 1.4426950408889634f;

enum Bar {
  kKVFull, kQFull, kQEmpty, kSFull, kXFree, kDecFull, kDecEmpty, kDoFull, kDoEmpty,
  kPtFull, kPtFree, kDpFull, kDsFull, kDsFree, kDqFull, kDone, kNumBars
};

struct Smem {
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kTile;
  static constexpr uint32_t kQ = kV + kTile;
  static constexpr uint32_t kDO = kQ + kTile;
  static constexpr uint32_t kPT = kDO + kTile;
  static constexpr uint32_t kDS = kPT + kTile;
  static constexpr uint32_t kStats = kDS + kTile;          // zl2[128], t2[128], D[128]
  static constexpr uint32_t kBars = kStats + 3 * 128 * 4;
  static constexpr uint32_t kMisc = kBars + kNumBars * 8;
  static constexpr uint32_t kEnd = kMisc + 64;
  static constexpr uint32_t kAlloc = kEnd + 1024;
};
static_assert(Smem::kAlloc > 116 * 1024, "backward CTA must exclude a second resident CTA per SM");
static_assert(Smem::kAlloc <= 232448, "backward CTA exceeds shared memory");

__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}

// Write one 128-element bf16 row (given as 64 packed pairs) into a K-major
// SW128 tile (two 64-column chunks) at row r.
__device__ __forceinline__ void store_row_sw128(uint32_t tile, int r, const uint32_t (&pk)[64]) {
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const uint32_t chunk = tile + (u >> 3) * kChunk + r * 128;
    st_shared_v4(chunk + (((u & 7) ^ (r & 7)) << 4), pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
  }
}

__global__ void __launch_bounds__(kThreads, 1) mala_bwd_tc_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem + Smem::kK;
  uint8_t* sV = smem + Smem::kV;
  uint8_t* sQ = smem + Smem::kQ;
  uint8_t* sDO = smem + Smem::kDO;
  uint8_t* sPT = smem + Smem::kPT;
  uint8_t* sDS = smem + Smem::kDS;
  float* sZl2 = reinterpret_cast<float*>(smem + Smem::kStats);
  float* sT2 = sZl2 + 128;
  float* sDv = sZl2 + 256;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::kBars);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + Smem::kMisc);
  // misc[0] TMEM base, misc[1] abort, misc[2..4] progress (producer, MMA,
  // compute), misc[5] decision, misc[6] tile head, misc[7] tile query block
  // (-1 = no more tiles)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // work item: (b, hk, j), smaller j (more query blocks) first
  const int BK = p.B * p.Hkv;
  const int j = static_cast<int>(blockIdx.x) / BK;
  const int bk = static_cast<int>(blockIdx.x) % BK;
  const int b = bk / p.Hkv;
  const int hk = bk % p.Hkv;
  const int G = p.group_size[hk];

  if (tid == 0) {
    for (int x = 0; x < kNumBars; ++x) {
      uint32_t cnt = 1;
      if (x == kXFree || x == kPtFull || x == kDsFull) cnt = 128;
      if (x == kQEmpty || x == kDecEmpty) cnt = 2;
      mbar_init(&bars[x], cnt);
    }
    for (int x = 1; x < 16; ++x) misc[x] = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(const_cast<uint32_t*>(misc), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const uint32_t tX = tmem, tY = tmem + 128, tDK = tmem + 256, tDV = tmem + 384;

  if (warp == 4) {
    // ===================== producer =====================
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      tma_prefetch_desc(&p.tm_do);
      mbar_expect_tx(&bars[kKVFull], 2 * kTile);
      for (int c = 0; c < 2; ++c) {
        tma_load_4d(sK + c * kChunk, &p.tm_k, &bars[kKVFull], c * 64, hk, j * kB, b);
        tma_load_4d(sV + c * kChunk, &p.tm_v, &bars[kKVFull], c * 64, hk, j * kB, b);
      }
      misc[2] = 0x10000u;
      bool ok = true;
      int n = 0, kc = 0;
      for (int g = 0; ok && g < G; ++g) {
        const int h = p.group_heads[hk][g];
        const int64_t bh = static_cast<int64_t>(b) * p.Hq + h;
        for (int i = j; ok && i < p.nQB; ++i) {
          if (p.fwd_mask && !((p.fwd_mask[(bh * p.nQB + i) * p.mask_words + (j >> 5)] >> (j & 31)) & 1u))
            continue;
          if (!mbar_wait(&bars[kQEmpty], (n & 1) ^ 1, abort_flag, p.err, wait_tag(1, kQEmpty, n))) { ok = false; break; }
          misc[6] = static_cast<uint32_t>(h);
          misc[7] = static_cast<uint32_t>(i);
          mbar_expect_tx(&bars[kQFull], kTile + 3 * 512);
          for (int c = 0; c < 2; ++c)
            tma_load_4d(sQ + c * kChunk, &p.tm_q, &bars[kQFull], c * 64, h, i * kB, b);
          const int64_t row0 = bh * p.Npad + static_cast<int64_t>(i) * kB;
          bulk_load(sZl2, p.zl2 + row0, 512, &bars[kQFull]);
          bulk_load(sT2, p.t2 + row0, 512, &bars[kQFull]);
          bulk_load(sDv, p.Dv + row0, 512, &bars[kQFull]);
          misc[2] = 0x20000u | n;
          if (!mbar_wait(&bars[kDecFull], n & 1, abort_flag, p.err, wait_tag(1, kDecFull, n))) { ok = false; break; }
          const uint32_t keep = misc[5];
          mbar_arrive(&bars[kDecEmpty]);
          if (keep) {
            if (!mbar_wait(&bars[kDoEmpty], (kc & 1) ^ 1, abort_flag, p.err, wait_tag(1, kDoEmpty, kc))) { ok = false; break; }
            mbar_expect_tx(&bars[kDoFull], kTile);
            for (int c = 0; c < 2; ++c)
              tma_load_4d(sDO + c * kChunk, &p.tm_do, &bars[kDoFull], c * 64, h, i * kB, b);
            ++kc;
          }
          ++n;
          misc[2] = 0x30000u | n;
        }
      }
      // end marker: one more "tile" with query block -1
      if (ok && mbar_wait(&bars[kQEmpty], (n & 1) ^ 1, abort_flag, p.err, wait_tag(1, kQEmpty, n))) {
        misc[7] = 0xFFFFFFFFu;
        mbar_arrive(&bars[kQFull]);
      } else {
        drain_pause_ns(50000);
      }
    }
  } else if (warp == 5) {
    // ===================== tcgen05 issuer =====================
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);   // A, B K-major
      constexpr uint32_t id_kmn = idesc_bf16_f32(128, 128, false, true);   // B MN-major
      constexpr uint32_t id_mnmn = idesc_bf16_f32(128, 128, true, true);   // A, B MN-major
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), aDO = smem_u32(sDO);
      const uint32_t aPT = smem_u32(sPT), aDS = smem_u32(sDS);
      bool ok = mbar_wait(&bars[kKVFull], 0, abort_flag, p.err, wait_tag(2, kKVFull, 0));
      int n = 0, kc = 0;
      while (ok) {
        if (!mbar_wait(&bars[kQFull], n & 1, abort_flag, p.err, wait_tag(2, kQFull, n))) { ok = false; break; }
        if (misc[7] == 0xFFFFFFFFu) break;
        if (!mbar_wait(&bars[kXFree], (n & 1) ^ 1, abort_flag, p.err, wait_tag(2, kXFree, n))) { ok = false; break; }
        tc_fence_after();
        // S^T = K_j Q_i^T (K = d)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
          umma_bf16_ss(tX, sdesc_sw128(aK + off, 16, 1024), sdesc_sw128(aQ + off, 16, 1024), id_kk, kk > 0);
        }
        umma_commit(&bars[kSFull]);
        misc[3] = 0x10000u | n;
        if (!mbar_wait(&bars[kDecFull], n & 1, abort_flag, p.err, wait_tag(2, kDecFull, n))) { ok = false; break; }
        const uint32_t keep = misc[5];
        mbar_arrive(&bars[kDecEmpty]);
        if (!keep) {
          umma_commit(&bars[kQEmpty]);
          ++n;
          continue;
        }
        if (!mbar_wait(&bars[kDoFull], kc & 1, abort_flag, p.err, wait_tag(2, kDoFull, kc))) { ok = false; break; }
        if (!mbar_wait(&bars[kPtFull], kc & 1, abort_flag, p.err, wait_tag(2, kPtFull, kc))) { ok = false; break; }
        tc_fence_after();
        // dV += P^T dO (K = queries; dO as MN-major B)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t offa = (kk >> 2) * kChunk + (kk & 3) * 32;
          umma_bf16_ss(tDV, sdesc_sw128(aPT + offa, 16, 1024), sdesc_sw128(aDO + kk * 2048, kChunk, 1024), id_kmn,
                       (kc > 0 || kk > 0) ? 1u : 0u);
        }
        // dP^T = V_j dO^T (K = d)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
          umma_bf16_ss(tY, sdesc_sw128(aV + off, 16, 1024), sdesc_sw128(aDO + off, 16, 1024), id_kk, kk > 0);
        }
        umma_commit(&bars[kDpFull]);
        umma_commit(&bars[kDoEmpty]);
        umma_commit(&bars[kPtFree]);
        misc[3] = 0x20000u | n;
        if (!mbar_wait(&bars[kDsFull], kc & 1, abort_flag, p.err, wait_tag(2, kDsFull, kc))) { ok = false; break; }
        tc_fence_after();
        // dK += dS^T Q_i (K = queries; Q as MN-major B)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t offa = (kk >> 2) * kChunk + (kk & 3) * 32;
          umma_bf16_ss(tDK, sdesc_sw128(aDS + offa, 16, 1024), sdesc_sw128(aQ + kk * 2048, kChunk, 1024), id_kmn,
                       (kc > 0 || kk > 0) ? 1u : 0u);
        }
        // dQ part = dS K_j (K = keys; dS^T tile read as MN-major A, K_j as MN-major B)
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          umma_bf16_ss(tX, sdesc_sw128(aDS + kk * 2048, kChunk, 1024), sdesc_sw128(aK + kk * 2048, kChunk, 1024),
                       id_mnmn, kk > 0);
        }
        umma_commit(&bars[kDqFull]);
        umma_commit(&bars[kQEmpty]);
        umma_commit(&bars[kDsFree]);
        misc[3] = 0x30000u | n;
        ++kc;
        ++n;
      }
      umma_commit(&bars[kDone]);
      mbar_wait(&bars[kDone], 0, abort_flag, p.err, wait_tag(2, kDone, 0));
    }
  } else {
    // ===================== compute warpgroup =====================
    const int t = tid;                          // key row (S^T, dK, dV) / query row (dQ part)
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t aPT = smem_u32(sPT), aDS = smem_u32(sDS);
    int n = 0, kc = 0, visited = 0, kept = 0;
    int64_t slots = 0;
    while (true) {
      const bool okq = __all_sync(0xffffffffu, mbar_wait(&bars[kQFull], n & 1, abort_flag, p.err, wait_tag(0, kQFull, n)));
      const uint32_t qi = misc[7];
      if (bar_or(1, 128, !okq || *abort_flag != 0) || qi == 0xFFFFFFFFu) break;
      const int i = static_cast<int>(qi);
      const int h = static_cast<int>(misc[6]);
      uint32_t sr[4][32];
      const bool oks = __all_sync(0xffffffffu, mbar_wait(&bars[kSFull], n & 1, abort_flag, p.err, wait_tag(0, kSFull, n)));
      if (oks) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(tX + lane_addr + c * 32, sr[c]);
          tmem_ld_wait(sr[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int x = 0; x < 32; ++x) sr[c][x] = 0u;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(sr[c]);
      // legal entries: query column c >= key row t on the diagonal tile; padded
      // query rows carry t2 = zl2 = +inf and never count
      const int lim = (i == j) ? t : 0;         // first legal column
      bool vote = false;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int col = c * 32 + x;
          const float s2 = __uint_as_float(sr[c][x]) * kLog2e;
          vote |= (col >= lim) && (s2 >= sT2[col]);
        }
      const bool keep = bar_or(1, 128, vote);
      misc[4] = 0x10000u | n;
      if (tid == 0) {
        if (mbar_wait(&bars[kDecEmpty], (n & 1) ^ 1, abort_flag, p.err, wait_tag(0, kDecEmpty, n))) {
          misc[5] = keep ? 1u : 0u;
          mbar_arrive(&bars[kDecFull]);
        }
        ++visited;
        if (keep) {
          ++kept;
          slots += static_cast<int64_t>(kB) * min(kB, p.N - i * kB);
          if (p.bwd_mask)
            atomicOr(&p.bwd_mask[((static_cast<int64_t>(b) * p.Hq + h) * p.nQB + i) * p.mask_words + (j >> 5)],
                     1u << (j & 31));
        }
      }
      if (!keep) {
        tc_fence_before();
        mbar_arrive(&bars[kXFree]);
        if (tid == 0) mbar_arrive(&bars[kQEmpty]);
        ++n;
        continue;
      }

      // P^T = exp2(S^T log2e - z log2e) on legal entries (fp32 kept for dS)
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const int col = c * 32 + x;
          const float pv = (col >= lim) ? ex2_approx(fmaf(__uint_as_float(sr[c][x]), kLog2e, -sZl2[col])) : 0.0f;
          sr[c][x] = __float_as_uint(pv);
        }
      mbar_wait(&bars[kPtFree], (kc & 1) ^ 1, abort_flag, p.err, wait_tag(0, kPtFree, kc));
      {
        uint32_t pk[64];
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int x = 0; x < 32; x += 2)
            pk[c * 16 + (x >> 1)] = pack_bf16x2(__uint_as_float(sr[c][x]), __uint_as_float(sr[c][x + 1]));
        store_row_sw128(aPT, t, pk);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bars[kPtFull]);

      // dS^T = P^T (dP^T - D)
      const bool okd = __all_sync(0xffffffffu, mbar_wait(&bars[kDpFull], kc & 1, abort_flag, p.err, wait_tag(0, kDpFull, kc)));
      mbar_wait(&bars[kDsFree], (kc & 1) ^ 1, abort_flag, p.err, wait_tag(0, kDsFree, kc));
      {
        uint32_t pk[64];
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t dp[32];
          if (okd) {
            tmem_ld32(tY + lane_addr + c * 32, dp);
            tmem_ld_wait(dp);
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) dp[x] = 0u;
          }
          reg_fence(dp);
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const int col = c * 32 + x;
            const float d0 = __uint_as_float(sr[c][x]) * (__uint_as_float(dp[x]) - sDv[col]);
            const float d1 = __uint_as_float(sr[c][x + 1]) * (__uint_as_float(dp[x + 1]) - sDv[col + 1]);
            pk[c * 16 + (x >> 1)] = pack_bf16x2(d0, d1);
          }
        }
        store_row_sw128(aDS, t, pk);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[kDsFull]);
      if (tid == 0) mbar_arrive(&bars[kQEmpty]);

      // dQ part (query row t) -> fp32 staging in the P^T tile -> bulk add into dQ_acc
      const bool okq2 = __all_sync(0xffffffffu, mbar_wait(&bars[kDqFull], kc & 1, abort_flag, p.err, wait_tag(0, kDqFull, kc)));
      tc_fence_after();
      float* stage = reinterpret_cast<float*>(sPT);
      float* dst = p.dq_acc + (((static_cast<int64_t>(b) * p.Hq + h) * p.nQB + i) * 4) * (kB * 32);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t dq[32];
        if (okq2) {
          tmem_ld32(tX + lane_addr + c * 32, dq);
          tmem_ld_wait(dq);
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) dq[x] = 0u;
        }
        reg_fence(dq);
        if (c >= 2) {
          // staging half c & 1 is reused: its previous bulk add must have read it
          if (tid == 0) bulk_wait_read<1>();
          named_bar_sync(1, 128);
        }
        float* row = stage + (c & 1) * (kB * 32) + t * 32;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int u = (k + t) & 7;             // rotate to spread banks
          *reinterpret_cast<uint4*>(row + 4 * u) = make_uint4(dq[4 * u], dq[4 * u + 1], dq[4 * u + 2], dq[4 * u + 3]);
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (tid == 0) {
          bulk_reduce_add_f32(dst + c * (kB * 32), stage + (c & 1) * (kB * 32), kB * 32 * 4);
          bulk_commit_group();
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[kXFree]);
      // the P^T tile is free again once the bulk adds have read the staging
      if (tid == 0) bulk_wait_read<0>();
      named_bar_sync(1, 128);
      ++kc;
      ++n;
    }

    // dK_j, dV_j (key row t) -> bf16
    if (tid == 0) bulk_wait_all<0>();
    const bool okdone = __all_sync(0xffffffffu, mbar_wait(&bars[kDone], 0, abort_flag, p.err, wait_tag(0, kDone, 0)));
    const int krow = j * kB + t;
    if (okdone && !*abort_flag) {
      tc_fence_after();
      const bool any_kept = kc > 0;           // dK/dV TMEM untouched when nothing was retained
      __nv_bfloat16* dkr = reinterpret_cast<__nv_bfloat16*>(p.dk) + b * p.dk_sb + static_cast<int64_t>(krow) * p.dk_sn + hk * p.dk_sh;
      __nv_bfloat16* dvr = reinterpret_cast<__nv_bfloat16*>(p.dv) + b * p.dv_sb + static_cast<int64_t>(krow) * p.dv_sn + hk * p.dv_sh;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t base = which == 0 ? tDK : tDV;
        __nv_bfloat16* outr = which == 0 ? dkr : dvr;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(base + lane_addr + c * 32, r);
          tmem_ld_wait(r);
          reg_fence(r);
          if (krow < p.N) {
            uint32_t pk[16];
#pragma unroll
            for (int x = 0; x < 32; x += 2)
              pk[x >> 1] = any_kept ? pack_bf16x2(__uint_as_float(r[x]), __uint_as_float(r[x + 1])) : 0u;
            uint4* d4 = reinterpret_cast<uint4*>(outr + c * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u) d4[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          }
        }
      }
      if (tid == 0 && p.stats) {
        atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[0]), static_cast<unsigned long long>(visited));
        atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[1]), static_cast<unsigned long long>(kept));
        atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[2]), static_cast<unsigned long long>(slots));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// D = rowsum(dO o O), zl2 = z log2e, t2 = (z + log tau - log(q + 1)) log2e,
// padded rows: zl2 = t2 = +inf, D = 0; zero the block's dQ accumulator.
__global__ void __launch_bounds__(128) mala_bwd_pre_kernel(const __grid_constant__ BwdAuxParams p) {
  const int blk = blockIdx.x;                  // (b, h, i)
  const int i = blk % p.nQB;
  const int bh = blk / p.nQB;
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int t = threadIdx.x;
  const int q = i * kB + t;
  const int64_t row = static_cast<int64_t>(bh) * p.Npad + q;
  if (q < p.N) {
    const uint4* o4 = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.o) + b * p.o_sb +
                                                     static_cast<int64_t>(q) * p.o_sn + h * p.o_sh);
    const uint4* g4 = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.dout) + b * p.do_sb +
                                                     static_cast<int64_t>(q) * p.do_sn + h * p.do_sh);
    float acc = 0.0f;
#pragma unroll
    for (int u = 0; u < kD / 8; ++u) {
      const uint4 a = o4[u], g = g4[u];
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 af = __bfloat1622float2(a2[e]);
        const float2 gf = __bfloat1622float2(g2[e]);
        acc = fmaf(af.x, gf.x, acc);
        acc = fmaf(af.y, gf.y, acc);
      }
    }
    const float z = p.lse[static_cast<int64_t>(bh) * p.N + q];
    p.Dv[row] = acc;
    p.zl2[row] = z * kLog2e;
    p.t2[row] = (z + p.log_tau - logf(static_cast<float>(q + 1))) * kLog2e;
  } else {
    p.Dv[row] = 0.0f;
    p.zl2[row] = INFINITY;
    p.t2[row] = INFINITY;
  }
  float4* acc4 = reinterpret_cast<float4*>(p.dq_acc + (static_cast<int64_t>(bh) * p.nQB + i) * (kB * kD));
  for (int e = t; e < kB * kD / 4; e += 128) acc4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dQ (bf16, [B, N, Hq, d]) from the blocked fp32 accumulator
// [B, Hq, nQB, 4 column groups, 128 rows, 32].
__global__ void __launch_bounds__(128) mala_bwd_dq_kernel(const __grid_constant__ BwdAuxParams p) {
  const int blk = blockIdx.x;
  const int i = blk % p.nQB;
  const int bh = blk / p.nQB;
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int t = threadIdx.x;
  const int q = i * kB + t;
  if (q >= p.N) return;
  const float* src = p.dq_acc + (static_cast<int64_t>(bh) * p.nQB + i) * (kB * kD);
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.dq) + b * p.dq_sb + static_cast<int64_t>(q) * p.dq_sn + h * p.dq_sh;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float4* s4 = reinterpret_cast<const float4*>(src + (c * kB + t) * 32);
    uint32_t pk[16];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const float4 v = s4[u];
      pk[2 * u] = pack_bf16x2(v.x, v.y);
      pk[2 * u + 1] = pack_bf16x2(v.z, v.w);
    }
    uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
    for (int u = 0; u < 4; ++u) d4[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
  }
}

}  // namespace

size_t bwd_smem_bytes() { return Smem::kAlloc; }

cudaError_t launch_bwd(const BwdParams& p, const BwdAuxParams& aux, cudaStream_t stream) {
  const unsigned blocks_q = static_cast<unsigned>(aux.B) * aux.Hq * aux.nQB;
  mala_bwd_pre_kernel<<<blocks_q, 128, 0, stream>>>(aux);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(mala_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(Smem::kAlloc));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hkv * p.nKB;
  mala_bwd_tc_kernel<<<grid, kThreads, Smem::kAlloc, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  mala_bwd_dq_kernel<<<blocks_q, 128, 0, stream>>>(aux);
  return cudaGetLastError();
}

}  // namespace mala
