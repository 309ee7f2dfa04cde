// MALA backward (Algorithm 2, "Offline Sparse Probability", and Appendix A.1
// "Fused backward execution" of the MassAlloc Attention paper) on sm_100a.
//
// Key-major: one CTA per (batch or packed sequence, KV head, key block j)
// accumulates dK_j and dV_j in TMEM over every query head of the group and
// every query block i ascending from the first one that sees key block j
// (query q at position q + N_k - N_q) whose tile (i, j) the forward retained. For a
// visited tile the score tile S^T = K_j Q_i^T is recomputed and tested
// against the saved log-normaliser: the tile is skipped iff for every legal
// (q, k) s_qk - z_q < log tau - log L_q. A retained tile loads dO_i and runs
//   P^T = exp(S^T - z), dV += P^T dO, dP^T = V dO^T, dS^T = P^T (dP^T - D),
//   dK += dS^T Q, dQ_i += dS K
// with dQ accumulated in fp32 by vector reductions into a blocked workspace.
//
// Roles (320 threads): warps 0-7 compute in two warpgroups that split the
// 128 query columns of a tile (lane t of TMEM is key row t for S^T, P^T,
// dP^T, dS^T and query row t for the dQ part), warp 8 TMA producer (in
// order, blocking waits: Q of the next tiles, dO one tile ahead), warp 9
// tcgen05 issuer.
// TMEM: X = cols [0,128): S^T(n), then P^T(n) as packed bf16 in [0,64),
// read by the dV MMA straight from TMEM; Y = [128,256): dP^T(n), then the
// tile's dQ part; dK = [256,384); dV = [384,512).
// Shared memory: K_j, V_j, two Q_i stages (with their row statistics), dO_i
// and the dS^T tile.
//
// Issue order of the tensor pipe for a retained tile n:
//   dV(n), dP^T(n) -> Y, S^T(n+1) -> X, dK(n), dQ(n) -> Y
// while the compute warps run the test and P^T of tile n+1 and drain dQ(n).
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

namespace mala {

namespace {

constexpr int kB = 128;                       // B_q = B_k
constexpr int kD = 128;
constexpr int kThreads = 320;
constexpr uint32_t kTile = kB * kD * 2;       // 32 KB bf16 tile
constexpr uint32_t kChunk = 16384;            // one 64-column swizzle chunk of 128 rows
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kEndMarker = 0xFFFFFFFFu;

enum Bar {
  kKVFull, kQFull, kQEmpty = kQFull + 2, kSFull = kQEmpty + 2, kXRead, kDecFull, kDecEmpty,
  kDoFull, kDoEmpty, kPtFull, kDvDone, kYFree, kDpFull, kDsFull, kDqFull, kDone, kNumBars
};

struct Smem {
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kTile;
  static constexpr uint32_t kQ = kV + kTile;                // 2 stages
  static constexpr uint32_t kDO = kQ + 2 * kTile;
  static constexpr uint32_t kDS = kDO + kTile;
  static constexpr uint32_t kStage = kDS + kTile;           // dQ staging: 16 KB per compute warpgroup
  static constexpr uint32_t kStats = kStage + kTile;        // [2 stages][-z log2e, D][128]
  static constexpr uint32_t kBars = kStats + 2 * 2 * 128 * 4;
  static constexpr uint32_t kMisc = kBars + kNumBars * 8;
  static constexpr uint32_t kEnd = kMisc + 64;
  // the dynamic shared memory base is 1024-byte aligned (checked at entry),
  // as the 128-byte swizzled TMA tiles require
  static constexpr uint32_t kAlloc = kEnd;
};
static_assert(Smem::kAlloc > 116 * 1024, "backward CTA must exclude a second resident CTA per SM");
static_assert(Smem::kAlloc <= 232448, "backward CTA exceeds shared memory");

__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}

__global__ void __launch_bounds__(kThreads, 1) mala_bwd_tc_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    // every thread sees the same address: a uniform exit before any barrier
    if (threadIdx.x == 0) atomicCAS(p.err, 0, kErrSmemAlign);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sK = smem + Smem::kK;
  uint8_t* sV = smem + Smem::kV;
  uint8_t* sQ = smem + Smem::kQ;
  uint8_t* sDO = smem + Smem::kDO;
  uint8_t* sDS = smem + Smem::kDS;
  uint8_t* sStage = smem + Smem::kStage;
  float* sStats = reinterpret_cast<float*>(smem + Smem::kStats);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::kBars);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + Smem::kMisc);
  // misc[0] TMEM base, misc[1] abort, misc[2..4] progress (producer, MMA,
  // compute), misc[5] decision, misc[6..7] head of the tile in Q stage 0/1,
  // misc[8..9] its query block (kEndMarker = no more tiles)
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // work item: (b, hk, j), smaller j (more query blocks) first; b is the
  // batch index, or the sequence of a packed call (qrow0 / krow0 its first
  // query / key row, tb its batch coordinate in the tensor maps)
  const int BK = p.B * p.Hkv;
  const int j = static_cast<int>(blockIdx.x) / BK;
  const int bk = static_cast<int>(blockIdx.x) % BK;
  const int b = bk / p.Hkv;
  const int hk = bk % p.Hkv;
  const int G = p.group_size[hk];
  int Nq = p.N, Nk = p.Nk, qrow0 = 0, krow0 = 0, tb = b;
  if (p.seq.n != 0) {
    qrow0 = p.seq.q0[b];
    krow0 = p.seq.k0[b];
    Nq = p.seq.q0[b + 1] - qrow0;
    Nk = p.seq.k0[b + 1] - krow0;
    tb = 0;
    if (j * kB >= Nk) return;       // a shorter sequence: no key block j (uniform exit)
  }
  const int q_off = Nk - Nq;        // query q sits at position q + q_off
  const int nQBs = (Nq + kB - 1) / kB;

  if (tid == 0) {
    for (int x = 0; x < kNumBars; ++x) {
      uint32_t cnt = 1;
      if (x == kXRead || x == kPtFull || x == kDsFull || x == kYFree) cnt = 8;   // one per compute warp
      if (x == kQEmpty || x == kQEmpty + 1 || x == kDecEmpty) cnt = 2;
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

  if (warp == 8) {
    // ===================== producer (in order) =====================
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      tma_prefetch_desc(&p.tm_do);
      mbar_expect_tx(&bars[kKVFull], 2 * kTile);
      for (int c = 0; c < 2; ++c) {
        tma_load_4d(sK + c * kChunk, &p.tm_k, &bars[kKVFull], c * 64, hk, krow0 + j * kB, tb);
        tma_load_4d(sV + c * kChunk, &p.tm_v, &bars[kKVFull], c * 64, hk, krow0 + j * kB, tb);
      }
      // scan state of the next visited tile (group head g, query block i);
      // the first query block with a row at or after key block j's first key
      // (query q sits at position q + q_off)
      const int i_first = max(0, j * kB - q_off) / kB;
      int sg = 0, si = i_first;
      auto next_tile = [&](int& h_out, int& i_out) -> bool {
        while (sg < G) {
          const int h = p.group_heads[hk][sg];
          while (si < nQBs) {
            const int i = si++;
            if (!p.fwd_mask ||
                ((p.fwd_mask[qblock_index(p.seq, p.Hq, p.nQB, b, h, i) * p.mask_words + (j >> 5)] >> (j & 31)) & 1u)) {
              h_out = h;
              i_out = i;
              return true;
            }
          }
          ++sg;
          si = i_first;
        }
        return false;
      };
      // (head, query block) of tile n at [n & 3]: Q of tile n + 2 is loaded
      // only after the decision on tile n was read
      int info_h[4] = {0, 0, 0, 0}, info_i[4] = {0, 0, 0, 0};
      // Q of tile n and its row statistics into stage n & 1; the end marker
      // instead when there is no tile n
      auto load_q = [&](int n) -> bool {
        const int st = n & 1;
        int h = 0, i = 0;
        if (!next_tile(h, i)) {
          misc[8 + st] = kEndMarker;
          mbar_arrive(&bars[kQFull + st]);
          return false;
        }
        info_h[n & 3] = h;
        info_i[n & 3] = i;
        misc[6 + st] = static_cast<uint32_t>(h);
        misc[8 + st] = static_cast<uint32_t>(i);
        mbar_expect_tx(&bars[kQFull + st], kTile + 2 * 512);
        for (int c = 0; c < 2; ++c)
          tma_load_4d(sQ + st * kTile + c * kChunk, &p.tm_q, &bars[kQFull + st], c * 64, h, qrow0 + i * kB, tb);
        const int64_t row0 = qblock_index(p.seq, p.Hq, p.nQB, b, h, i) * kB;
        float* sst = sStats + st * 256;
        bulk_load(sst, p.nzl2 + row0, 512, &bars[kQFull + st]);
        bulk_load(sst + 128, p.Dv + row0, 512, &bars[kQFull + st]);
        return true;
      };
      // In order, with blocking waits. dO of tile n + 1 is loaded one tile
      // ahead, before tile n + 1 is decided, into the single dO buffer as
      // soon as tile n has finished with it (after dP^T(n) for a retained
      // tile n, once its own load has landed for a skipped one), so that
      // its latency stays off the path to dV. Per tile n: read its
      // decision, refill the dO buffer, then refill tile n's Q stage with
      // tile n + 2 once tile n released it. Every wait is for the next event
      // this role needs, so the thread sleeps in the barrier wait instead
      // of polling.
      auto load_do = [&](int n) {
        mbar_expect_tx(&bars[kDoFull], kTile);
        for (int c = 0; c < 2; ++c)
          tma_load_4d(sDO + c * kChunk, &p.tm_do, &bars[kDoFull], c * 64, info_h[n & 3],
                      qrow0 + info_i[n & 3] * kB, tb);
      };
      int n_total = -1;                         // number of tiles, once known
      for (int n = 0; n < 2 && n_total < 0; ++n)
        if (!load_q(n)) n_total = n;
      if (n_total != 0) load_do(0);
      int kept_seen = 0;                        // retained tiles before tile n
      bool ok = true;
      for (int n = 0; n_total < 0 || n < n_total; ++n) {
        ok = mbar_wait(&bars[kDecFull], n & 1, abort_flag, p.err, wait_tag(1, kDecFull, n), p.wait_ns);
        if (!ok) break;
        const uint32_t keep = misc[5];
        mbar_arrive(&bars[kDecEmpty]);
        // tile n + 1 exists iff Q(n + 1) was not the end marker
        if (n_total < 0 || n + 1 < n_total) {
          if (keep)   // the MMAs of tile n release the buffer after dP^T(n)
            ok = mbar_wait(&bars[kDoEmpty], kept_seen & 1, abort_flag, p.err, wait_tag(1, kDoEmpty, n), p.wait_ns);
          else        // nothing reads it: wait for tile n's own load to land
            ok = mbar_wait(&bars[kDoFull], n & 1, abort_flag, p.err, wait_tag(1, kDoFull, n), p.wait_ns);
          if (!ok) break;
          load_do(n + 1);
        }
        if (keep) ++kept_seen;
        if (n_total < 0) {
          ok = mbar_wait(&bars[kQEmpty + (n & 1)], (n >> 1) & 1, abort_flag, p.err, wait_tag(1, kQEmpty + (n & 1), n), p.wait_ns);
          if (!ok) break;
          if (!load_q(n + 2)) n_total = n + 2;
        }
        misc[2] = (static_cast<uint32_t>(n) << 16) | (static_cast<uint32_t>(kept_seen) & 0xffff);
      }
      // the last tile's dO load (no tile reads it when that tile was
      // skipped) must land before the CTA's shared memory is released
      if (ok && n_total > 0)
        ok = mbar_wait(&bars[kDoFull], (n_total - 1) & 1, abort_flag, p.err, wait_tag(1, kDoFull, n_total - 1), p.wait_ns);
      if (!ok) drain_pause_ns(50000);   // let copies already issued land
    }
  } else if (warp == 9) {
    // ===================== tcgen05 issuer =====================
    if (lane == 0) {
      constexpr uint32_t id_kk = idesc_bf16_f32(128, 128, false, false);   // A, B K-major
      constexpr uint32_t id_kmn = idesc_bf16_f32(128, 128, false, true);   // B MN-major
      constexpr uint32_t id_mnmn = idesc_bf16_f32(128, 128, true, true);   // A, B MN-major
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), aDO = smem_u32(sDO);
      const uint32_t aDS = smem_u32(sDS);
      auto issue_s = [&](int n) {
        const uint32_t q = aQ + (n & 1) * kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
          umma_bf16_ss(tX, sdesc_sw128(aK + off, 16, 1024), sdesc_sw128(q + off, 16, 1024), id_kk, kk > 0);
        }
        umma_commit(&bars[kSFull]);
      };
      bool ok = mbar_wait(&bars[kKVFull], 0, abort_flag, p.err, wait_tag(2, kKVFull, 0), p.wait_ns);
      int n = 0, kc = 0, sk = 0;
      bool have_next = false;
      if (ok) ok = mbar_wait(&bars[kQFull], 0, abort_flag, p.err, wait_tag(2, kQFull, 0), p.wait_ns);
      if (ok && misc[8] != kEndMarker) {
        tc_fence_after();
        issue_s(0);
        have_next = true;
      }
      while (ok && have_next) {
        if (!mbar_wait(&bars[kDecFull], n & 1, abort_flag, p.err, wait_tag(2, kDecFull, n), p.wait_ns)) { ok = false; break; }
        const uint32_t keep = misc[5];
        mbar_arrive(&bars[kDecEmpty]);
        const int st = n & 1, stn = (n + 1) & 1;
        if (keep) {
          if (!mbar_wait(&bars[kPtFull], kc & 1, abort_flag, p.err, wait_tag(2, kPtFull, kc), p.wait_ns)) { ok = false; break; }
          if (!mbar_wait(&bars[kDoFull], n & 1, abort_flag, p.err, wait_tag(2, kDoFull, n), p.wait_ns)) { ok = false; break; }
          tc_fence_after();
          // dV += P^T dO: A = P^T from TMEM (8 columns per 16 queries), B = dO MN-major
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16_ts(tDV, tX + kk * 8, sdesc_sw128(aDO + kk * 2048, kChunk, 1024), id_kmn,
                         (kc > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&bars[kDvDone]);
          // dP^T = V_j dO^T into Y once the previous dQ part has left it
          if (!mbar_wait(&bars[kYFree], (kc & 1) ^ 1, abort_flag, p.err, wait_tag(2, kYFree, kc), p.wait_ns)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
            umma_bf16_ss(tY, sdesc_sw128(aV + off, 16, 1024), sdesc_sw128(aDO + off, 16, 1024), id_kk, kk > 0);
          }
          umma_commit(&bars[kDpFull]);
          umma_commit(&bars[kDoEmpty]);
          // S^T of the next tile into X once dV has read P^T from it
          if (!mbar_wait(&bars[kQFull + stn], ((n + 1) >> 1) & 1, abort_flag, p.err, wait_tag(2, kQFull + stn, n + 1), p.wait_ns)) { ok = false; break; }
          have_next = misc[8 + stn] != kEndMarker;
          if (have_next) {
            if (!mbar_wait(&bars[kDvDone], kc & 1, abort_flag, p.err, wait_tag(2, kDvDone, kc), p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            issue_s(n + 1);
          }
          // dK += dS^T Q_i and the dQ part = dS K_j into Y
          if (!mbar_wait(&bars[kDsFull], kc & 1, abort_flag, p.err, wait_tag(2, kDsFull, kc), p.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t q = aQ + st * kTile;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t offa = (kk >> 2) * kChunk + (kk & 3) * 32;
            umma_bf16_ss(tDK, sdesc_sw128(aDS + offa, 16, 1024), sdesc_sw128(q + kk * 2048, kChunk, 1024), id_kmn,
                         (kc > 0 || kk > 0) ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16_ss(tY, sdesc_sw128(aDS + kk * 2048, kChunk, 1024), sdesc_sw128(aK + kk * 2048, kChunk, 1024),
                         id_mnmn, kk > 0);
          umma_commit(&bars[kDqFull]);
          umma_commit(&bars[kQEmpty + st]);
          ++kc;
        } else {
          umma_commit(&bars[kQEmpty + st]);
          if (!mbar_wait(&bars[kQFull + stn], ((n + 1) >> 1) & 1, abort_flag, p.err, wait_tag(2, kQFull + stn, n + 1), p.wait_ns)) { ok = false; break; }
          have_next = misc[8 + stn] != kEndMarker;
          if (have_next) {
            if (!mbar_wait(&bars[kXRead], sk & 1, abort_flag, p.err, wait_tag(2, kXRead, sk), p.wait_ns)) { ok = false; break; }
            tc_fence_after();
            issue_s(n + 1);
          }
          ++sk;
        }
        misc[3] = (static_cast<uint32_t>(n) << 16) | (static_cast<uint32_t>(kc) & 0xffff);
        ++n;
      }
      // every MMA issued above must have finished before TMEM is read or
      // freed: wait for that regardless of the abort flag (MMAs always
      // complete), bounded in time
      umma_commit(&bars[kDone]);
      mbar_wait_drain(&bars[kDone], 0);
    }
  } else {
    // ===================== compute warpgroups =====================
    // warps 0-3 take query columns [0, 64), warps 4-7 columns [64, 128);
    // (warp, lane) owns TMEM lane r = 32 (warp % 4) + lane: key row r of
    // S^T, P^T, dP^T, dS^T and query row r of the dQ part
    const int r = ((warp & 3) << 5) | lane;
    const int half = warp >> 2;
    const int c0 = half * 64;                   // first query column of this half
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t aDS = smem_u32(sDS);
    int n = 0, kc = 0, sk = 0, visited = 0, kept = 0;
    int64_t slots = 0;
    bool pending = false;                       // a dQ part waits in Y
    int pend_h = 0, pend_i = 0;

    // dQ part of the previous retained tile (query row r, this half's 64
    // columns): TMEM -> registers (Y is then free) -> this warpgroup's 16 KB
    // staging buffer in the accumulator's blocked layout [.., 32 column
    // quads, 128 rows, 4] -> one asynchronous bulk fp32 reduction per 32
    // columns (16 KB contiguous in the accumulator), issued by one thread of
    // the warpgroup, in place of one vector reduction per thread and 16
    // bytes. Before a warpgroup refills its buffer, its leader waits until
    // the previous bulk reduction has read it.
    const bool wg_leader = (warp & 3) == 0 && lane == 0;
    auto drain = [&]() {
      const bool okq = __all_sync(0xffffffffu, mbar_wait(&bars[kDqFull], (kc - 1) & 1, abort_flag, p.err,
                                                          wait_tag(0, kDqFull, kc - 1), p.wait_ns));
      uint32_t q0[32], q1[32];
      if (okq) {
        tc_fence_after();
        tmem_ld32(tY + lane_addr + c0, q0);
        tmem_ld32(tY + lane_addr + c0 + 32, q1);
        tmem_ld_wait(q0);
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) q0[x] = q1[x] = 0u;
      }
      reg_fence(q0);
      reg_fence(q1);
      tc_fence_before();
      warp_arrive(&bars[kYFree]);
      float* dst = p.dq_acc + qblock_index(p.seq, p.Hq, p.nQB, b, pend_h, pend_i) * (kB * kD);
      uint8_t* stg = sStage + half * 16384;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const uint32_t* q = c ? q1 : q0;
        // the previous reduction from this half has finished reading it
        if (wg_leader) bulk_wait_read<0>();
        named_bar_sync(2 + half, 128);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          st_shared_v4(smem_u32(stg) + (u * kB + r) * 16, q[4 * u], q[4 * u + 1], q[4 * u + 2], q[4 * u + 3]);
        fence_proxy_async_smem();
        named_bar_sync(2 + half, 128);
        if (wg_leader) {
          // quads [16 half + 8c, + 8): 32 columns, 16 KB contiguous
          bulk_reduce_add_f32(dst + (16 * half + 8 * c) * (kB * 4), stg, 16384);
          bulk_commit_group();
        }
      }
      pending = false;
    };

    while (true) {
      const int st = n & 1;
      const bool okq = __all_sync(0xffffffffu, mbar_wait(&bars[kQFull + st], (n >> 1) & 1, abort_flag, p.err,
                                                         wait_tag(0, kQFull + st, n), p.wait_ns));
      const uint32_t qi = misc[8 + st];
      if (bar_or(1, 256, !okq || *abort_flag != 0) || qi == kEndMarker) break;
      const int i = static_cast<int>(qi);
      const int h = static_cast<int>(misc[6 + st]);
      const float4* nz_4 = reinterpret_cast<const float4*>(sStats + st * 256 + c0);
      const float4* dv_4 = reinterpret_cast<const float4*>(sStats + st * 256 + 128 + c0);
      // test over this half of the S^T row, in log2 units: retain iff some
      // legal entry has u + log2 L_q >= log2 tau, with u = s log2 e - z log2 e
      // (also the exponent of P^T) and L_q = position + 1 of the entry's
      // query column. Illegal entries (keys after the query's position, and
      // key rows past N_k) only occur in tiles whose last key lies beyond the
      // block's first query position; there they are set to -inf once, which
      // makes u = -inf: they drop out of the test and their P^T is exactly 0.
      // Padded query columns carry -z log2 e = -inf and drop out the same way.
      const bool oks = __all_sync(0xffffffffu, mbar_wait(&bars[kSFull], n & 1, abort_flag, p.err, wait_tag(0, kSFull, n), p.wait_ns));
      uint32_t sr[2][32];
      if (oks) {
        tc_fence_after();
        tmem_ld32(tX + lane_addr + c0, sr[0]);
        tmem_ld32(tX + lane_addr + c0 + 32, sr[1]);
        tmem_ld_wait(sr[0]);
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) sr[0][x] = sr[1][x] = 0u;
      }
      reg_fence(sr[0]);
      reg_fence(sr[1]);
      if (j * kB + kB - 1 > i * kB + q_off) {
        // query column c0 + x is at position i * 128 + c0 + x + q_off and
        // sees key j * 128 + r iff that is >= it: x >= lim
        const int lim = (j * kB + r) - (i * kB + q_off) - c0;
#pragma unroll
        for (int x = 0; x < 64; ++x)
          if (x < lim) sr[x >> 5][x & 31] = __float_as_uint(-INFINITY);
      }
      // u kept in sr as the exponent of P^T. L_q of this half's columns lies
      // in [L0, L0 + 63], so with M = max u the row retains when
      // M + log2 L0 >= log2 tau and skips when M + log2(L0 + 63) < log2 tau;
      // only between the two bounds is each entry tested on its own. A row
      // without a legal entry (M = -inf) never retains.
      float mu[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mu[e] = -INFINITY;
#pragma unroll
      for (int x4 = 0; x4 < 16; ++x4) {
        const float4 zv = nz_4[x4];
        const int x = 4 * x4;
        float u[4];
        fma2(u[0], u[1], __uint_as_float(sr[x >> 5][x & 31]), __uint_as_float(sr[x >> 5][(x + 1) & 31]), kLog2e,
             kLog2e, zv.x, zv.y);
        fma2(u[2], u[3], __uint_as_float(sr[x >> 5][(x + 2) & 31]), __uint_as_float(sr[x >> 5][(x + 3) & 31]), kLog2e,
             kLog2e, zv.z, zv.w);
#pragma unroll
        for (int e = 0; e < 4; ++e) sr[x >> 5][(x + e) & 31] = __float_as_uint(u[e]);
        mu[x4 & 7] = max3(mu[x4 & 7], u[0], u[1]);
        mu[x4 & 7] = max3(mu[x4 & 7], u[2], u[3]);
      }
      const float M = fmaxf(fmaxf(fmaxf(mu[0], mu[1]), fmaxf(mu[2], mu[3])),
                            fmaxf(fmaxf(mu[4], mu[5]), fmaxf(mu[6], mu[7])));
      const float L0 = static_cast<float>(i * kB + c0 + q_off + 1);   // L_q of column c0
      bool vote;
      if (!(M > -INFINITY) || M + lg2_approx(L0 + 63.0f) < p.log2_tau) {
        vote = false;
      } else if (M + lg2_approx(L0) >= p.log2_tau) {
        vote = true;
      } else {
        float mx = -INFINITY;
#pragma unroll
        for (int x = 0; x < 64; ++x)
          mx = fmaxf(mx, __uint_as_float(sr[x >> 5][x & 31]) + lg2_approx(L0 + static_cast<float>(x)));
        vote = mx >= p.log2_tau;
      }
      const bool keep = bar_or(1, 256, vote);
      if (tid == 0) {
        misc[4] = (static_cast<uint32_t>(n) << 16) | (static_cast<uint32_t>(kc) & 0xffff);
        if (mbar_wait(&bars[kDecEmpty], (n & 1) ^ 1, abort_flag, p.err, wait_tag(0, kDecEmpty, n), p.wait_ns)) {
          misc[5] = keep ? 1u : 0u;
          mbar_arrive(&bars[kDecFull]);
        }
        ++visited;
        if (keep) {
          ++kept;
          slots += static_cast<int64_t>(kB) * min(kB, Nq - i * kB);
          if (p.bwd_mask)
            atomicOr(&p.bwd_mask[qblock_index(p.seq, p.Hq, p.nQB, b, h, i) * p.mask_words + (j >> 5)],
                     1u << (j & 31));
        }
      }
      if (!keep) {
        tc_fence_before();
        warp_arrive(&bars[kXRead]);
        if (tid == 0) mbar_arrive(&bars[kQEmpty + st]);
        ++sk;
        ++n;
        if (pending) drain();
        continue;
      }

      // P^T = exp2(S^T log2e - z log2e) (0 on illegal entries), as bf16 pairs: kept
      // in registers for dS and written over S^T in X for the dV MMA. Both
      // halves finished reading S^T before the vote, so the packed P^T
      // columns [32 half, 32 half + 32) may overwrite either half's S^T.
      uint32_t pp[32];
#pragma unroll
      for (int x2 = 0; x2 < 32; ++x2)
        pp[x2] = pack_bf16x2(ex2_approx(__uint_as_float(sr[(2 * x2) >> 5][(2 * x2) & 31])),
                             ex2_approx(__uint_as_float(sr[(2 * x2 + 1) >> 5][(2 * x2 + 1) & 31])));
      tmem_st16(tX + lane_addr + half * 32, &pp[0]);
      tmem_st16(tX + lane_addr + half * 32 + 16, &pp[16]);
      tmem_st_wait();
      tc_fence_before();
      warp_arrive(&bars[kPtFull]);

      if (pending) drain();

      // dS^T = P^T (dP^T - D) -> bf16 into this half's chunk of the dS^T tile
      const bool okd = __all_sync(0xffffffffu, mbar_wait(&bars[kDpFull], kc & 1, abort_flag, p.err, wait_tag(0, kDpFull, kc), p.wait_ns));
      uint32_t dp[2][32];
      if (okd) {
        tc_fence_after();
        tmem_ld32(tY + lane_addr + c0, dp[0]);
        tmem_ld32(tY + lane_addr + c0 + 32, dp[1]);
        tmem_ld_wait(dp[0]);
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) dp[0][x] = dp[1][x] = 0u;
      }
      reg_fence(dp[0]);
      reg_fence(dp[1]);
      const uint32_t rowb = aDS + half * kChunk + r * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u) {            // 16-byte unit u: queries c0 + 8u .. + 8
        uint32_t pk[4];
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          const float4 dv = dv_4[2 * u + e2];
          const float dd[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const int x = 8 * u + 4 * e2 + e;
            const uint32_t w = pp[x >> 1];
            float t0, t1, d0, d1;
            sub2(t0, t1, __uint_as_float(dp[x >> 5][x & 31]), __uint_as_float(dp[(x + 1) >> 5][(x + 1) & 31]), dd[e],
                 dd[e + 1]);
            mul2(d0, d1, __uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u), t0, t1);
            pk[2 * e2 + (e >> 1)] = pack_bf16x2(d0, d1);
          }
        }
        st_shared_v4(rowb + ((u ^ (r & 7)) << 4), pk[0], pk[1], pk[2], pk[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      warp_arrive(&bars[kDsFull]);
      if (tid == 0) mbar_arrive(&bars[kQEmpty + st]);
      pending = true;
      pend_h = h;
      pend_i = i;
      ++kc;
      ++n;
    }
    // the drain synchronises each warpgroup on a named barrier, so every
    // compute thread must take the same branch: decide by a vote
    if (!bar_or(1, 256, *abort_flag != 0) && pending) drain();
    // the bulk reductions into the dQ accumulator complete before the CTA
    // exits (the conversion kernel reads the accumulator next)
    if (wg_leader) bulk_wait_all<0>();

    // dK_j, dV_j (key row r, this half's 64 columns) -> bf16
    const bool okdone = __all_sync(0xffffffffu, mbar_wait(&bars[kDone], 0, abort_flag, p.err, wait_tag(0, kDone, 0), p.wait_ns));
    const int krow = j * kB + r;
    if (okdone && !*abort_flag) {
      tc_fence_after();
      const bool any_kept = kc > 0;            // dK/dV TMEM untouched when nothing was retained
      __nv_bfloat16* dkr = reinterpret_cast<__nv_bfloat16*>(p.dk) + tb * p.dk_sb +
                           static_cast<int64_t>(krow0 + krow) * p.dk_sn + hk * p.dk_sh;
      __nv_bfloat16* dvr = reinterpret_cast<__nv_bfloat16*>(p.dv) + tb * p.dv_sb +
                           static_cast<int64_t>(krow0 + krow) * p.dv_sn + hk * p.dv_sh;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t base = which == 0 ? tDK : tDV;
        __nv_bfloat16* outr = which == 0 ? dkr : dvr;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t rr[32];
          tmem_ld32(base + lane_addr + c0 + c * 32, rr);
          tmem_ld_wait(rr);
          reg_fence(rr);
          if (krow < Nk) {
            uint32_t pk[16];
#pragma unroll
            for (int x = 0; x < 32; x += 2)
              pk[x >> 1] = any_kept ? pack_bf16x2(__uint_as_float(rr[x]), __uint_as_float(rr[x + 1])) : 0u;
            uint4* d4 = reinterpret_cast<uint4*>(outr + c0 + c * 32);
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
  // after a timeout, copies issued before the waits gave up land before the
  // CTA's shared memory is released
  if (tid == 0 && *abort_flag) drain_pause_ns(50000);
}

// D = rowsum(dO o O), nzl2 = -z log2e; padded rows: nzl2 = -inf, D = 0; zero
// the block's dQ accumulator.
// Query block of an auxiliary CTA: blk = qblock_index(b, h, i); the
// sequence's first query row, batch coordinate and length.
struct AuxBlock {
  int b, h, i, qrow0, tb, Nq;
};

__device__ __forceinline__ AuxBlock aux_block(const BwdAuxParams& p, int blk) {
  AuxBlock a;
  if (p.seq.n == 0) {
    a.i = blk % p.nQB;
    const int bh = blk / p.nQB;
    a.b = bh / p.Hq;
    a.h = bh % p.Hq;
    a.qrow0 = 0;
    a.tb = a.b;
    a.Nq = p.N;
  } else {
    const int QB = p.seq.qb0[p.seq.n];
    a.h = blk / QB;
    const int gqb = blk % QB;
    int lo = 0, hi = p.seq.n - 1;             // the sequence with qb0[s] <= gqb < qb0[s + 1]
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.seq.qb0[mid] <= gqb) lo = mid; else hi = mid - 1;
    }
    while (p.seq.qb0[lo + 1] <= gqb) ++lo;      // skip sequences without query blocks
    a.b = lo;
    a.i = gqb - p.seq.qb0[lo];
    a.qrow0 = p.seq.q0[lo];
    a.tb = 0;
    a.Nq = p.seq.q0[lo + 1] - a.qrow0;
  }
  return a;
}

__global__ void __launch_bounds__(128) mala_bwd_pre_kernel(const __grid_constant__ BwdAuxParams p) {
  const int blk = blockIdx.x;                  // qblock_index(b, h, i)
  const AuxBlock ab = aux_block(p, blk);
  const int b = ab.tb, h = ab.h, i = ab.i;
  const int t = threadIdx.x;
  const int q = i * kB + t;
  const int64_t row = static_cast<int64_t>(blk) * kB + t;
  if (q < ab.Nq) {
    const int64_t qr = ab.qrow0 + q;
    const uint4* o4 = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.o) + b * p.o_sb +
                                                     qr * p.o_sn + h * p.o_sh);
    const uint4* g4 = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.dout) + b * p.do_sb +
                                                     qr * p.do_sn + h * p.do_sh);
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
    // lse: [B, H_q, N_q], or [H_q, total_q] for packed sequences
    const float z = p.seq.n == 0 ? p.lse[(static_cast<int64_t>(ab.b) * p.Hq + h) * p.N + q]
                                 : p.lse[static_cast<int64_t>(h) * p.seq.q0[p.seq.n] + qr];
    p.Dv[row] = acc;
    p.nzl2[row] = -z * kLog2e;
  } else {
    p.Dv[row] = 0.0f;
    p.nzl2[row] = -INFINITY;
  }
  float4* acc4 = reinterpret_cast<float4*>(p.dq_acc + static_cast<int64_t>(blk) * (kB * kD));
  for (int e = t; e < kB * kD / 4; e += 128) acc4[e] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dQ (bf16, [B, N, Hq, d]) from the blocked fp32 accumulator
// [B, Hq, nQB, 32 column quads, 128 rows, 4].
__global__ void __launch_bounds__(128) mala_bwd_dq_kernel(const __grid_constant__ BwdAuxParams p) {
  const int blk = blockIdx.x;                  // qblock_index(b, h, i)
  const AuxBlock ab = aux_block(p, blk);
  const int t = threadIdx.x;
  const int q = ab.i * kB + t;
  if (q >= ab.Nq) return;
  const float4* src = reinterpret_cast<const float4*>(p.dq_acc + static_cast<int64_t>(blk) * (kB * kD)) + t;
  __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.dq) + ab.tb * p.dq_sb +
                       static_cast<int64_t>(ab.qrow0 + q) * p.dq_sn + ab.h * p.dq_sh;
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int u = 0; u < 16; ++u) {
    const float4 v0 = src[(2 * u) * kB];
    const float4 v1 = src[(2 * u + 1) * kB];
    d4[u] = make_uint4(pack_bf16x2(v0.x, v0.y), pack_bf16x2(v0.z, v0.w), pack_bf16x2(v1.x, v1.y),
                       pack_bf16x2(v1.z, v1.w));
  }
}

}  // namespace

size_t bwd_smem_bytes() { return Smem::kAlloc; }

cudaError_t launch_bwd(const BwdParams& p, const BwdAuxParams& aux, cudaStream_t stream) {
  const unsigned blocks_q = aux.seq.n == 0 ? static_cast<unsigned>(aux.B) * aux.Hq * aux.nQB
                                           : static_cast<unsigned>(aux.Hq) * aux.seq.qb0[aux.seq.n];
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
