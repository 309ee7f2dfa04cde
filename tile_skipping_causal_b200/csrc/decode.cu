// MALA single-token decoding with split-KV (cost paragraph after "Offline
// Sparse Probability" and Appendix A.1 "Fused decoding execution" of the
// MassAlloc Attention paper).
//
// One CTA per (batch, KV head, split). The query rows of the KV head's
// group (G <= 16 heads, one row each, at position N_k - 1 so L_0 = N_k) are
// scored against every key tile of the split, tiles visited in descending
// order, each split with its own running maximum and normalisation sum.
// Decisions are per query head; a tile's V is read iff some head retains
// it, and PV only accumulates the retaining heads' rows.
//
// This is a streaming (HBM-bound) kernel: the G-row contraction is too thin
// for tcgen05 (M >= 64), so scores and PV use warp-level mma.sync on
// operands staged by TMA in 128-byte-swizzled shared memory.
//
// Roles (160 threads):
//   warps 0-3  compute. QK^T: warp w scores keys [32w, 32w+32) of the tile
//              for all rows; row maxima meet in shared memory; every warp
//              then evaluates the same per-head decisions. PV: warp w owns
//              output columns [32w, 32w+32) over all 128 keys.
//   warp 4     TMA producer, polling: K tiles as far ahead as the K ring
//              allows (independent of decisions), V tiles as decisions to
//              retain arrive.
// PV is deferred: a retained tile's P (bf16) and reference maxima wait in
// one of two slots until the slot is needed again or the split ends, so the
// V load issued after the vote overlaps the scoring of later tiles.
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

namespace mala {

namespace {

constexpr int kBK = 128;
constexpr int kD = 128;
constexpr int kNSK = 4;                 // K ring stages
constexpr int kNSV = 2;                 // V / P slots
constexpr int kND = 4;                  // decision ring
constexpr int kThreads = 160;
constexpr uint32_t kTileBytes = kBK * kD * 2;
constexpr int kPStride = 136;           // bf16 per P row (128 + 8 padding)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

enum Bar {
  kKFull = 0,                     // kNSK
  kKEmpty = kKFull + kNSK,        // kNSK, 4 arrivals (one per compute warp)
  kVFull = kKEmpty + kNSK,        // kNSV
  kSlotFree = kVFull + kNSV,      // kNSV, 4 arrivals
  kDecFull = kSlotFree + kNSV,    // kND
  kDecEmpty = kDecFull + kND,     // kND
  kNumBars = kDecEmpty + kND
};

struct Smem {
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kNSK * kTileBytes;
  static constexpr uint32_t kP = kV + kNSV * kTileBytes;                 // [kNSV][16][kPStride] bf16
  static constexpr uint32_t kPendM = kP + kNSV * 16 * kPStride * 2;      // [kNSV][16] float
  static constexpr uint32_t kPMax = kPendM + kNSV * 16 * 4;              // [2][4][16] float
  static constexpr uint32_t kPSum = kPMax + 2 * 4 * 16 * 4;              // [2][4][16] float
  static constexpr uint32_t kBars = kPSum + 2 * 4 * 16 * 4;
  static constexpr uint32_t kMisc = kBars + kNumBars * 8;               // misc words
  static constexpr uint32_t kEnd = kMisc + 64;
  static constexpr uint32_t kAlloc = kEnd + 1024;
};
static_assert(Smem::kAlloc <= 232448, "decode CTA exceeds shared memory");

__global__ void __launch_bounds__(kThreads, 1) mala_decode_split_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem + Smem::kK;
  uint8_t* sV = smem + Smem::kV;
  __nv_bfloat16* sP = reinterpret_cast<__nv_bfloat16*>(smem + Smem::kP);
  float* sPendM = reinterpret_cast<float*>(smem + Smem::kPendM);
  float* sPMax = reinterpret_cast<float*>(smem + Smem::kPMax);
  float* sPSum = reinterpret_cast<float*>(smem + Smem::kPSum);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::kBars);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + Smem::kMisc);
  // misc[1] abort flag, misc[2..4] progress markers (producer / warp 0 /
  // unused), misc[8..8+kND) decision ring
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const int P = p.num_splits;
  const int split = static_cast<int>(blockIdx.x) % P;
  const int bk = static_cast<int>(blockIdx.x) / P;
  const int hk = bk % p.Hkv;
  const int b = bk / p.Hkv;
  const int G = p.group_size[hk];
  const int t0 = static_cast<int>((static_cast<int64_t>(split) * p.nKB) / P);
  const int t1 = static_cast<int>((static_cast<int64_t>(split + 1) * p.nKB) / P);
  const int T = t1 - t0;                 // tiles of this split, visited t1-1 ... t0

  if (tid == 0) {
    for (int x = 0; x < kNumBars; ++x) {
      uint32_t cnt = 1;
      if ((x >= kKEmpty && x < kKEmpty + kNSK) || (x >= kSlotFree && x < kSlotFree + kNSV)) cnt = 4;
      mbar_init(&bars[x], cnt);
    }
    for (int x = 1; x < 16; ++x) misc[x] = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ===================== TMA producer (polling) =====================
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      int next_k = 0, next_d = 0, v_issued = 0, v_req = 0;
      int vq[kND + kNSV];                // tiles waiting for a V load (ring)
      uint64_t idle_since = global_timer_ns();
      bool ok = true;
      while (ok && (next_k < T || next_d < T || v_issued < v_req)) {
        bool progress = false;
        if (next_k < T) {
          const int s = next_k % kNSK;
          if (mbar_test(&bars[kKEmpty + s], ((next_k / kNSK) & 1) ^ 1)) {
            mbar_expect_tx(&bars[kKFull + s], kTileBytes);
            const int j = t1 - 1 - next_k;
            for (int c = 0; c < 2; ++c)
              tma_load_4d(sK + s * kTileBytes + c * 16384, &p.tm_k, &bars[kKFull + s], c * 64, hk,
                          j * kBK, b);
            ++next_k;
            progress = true;
          }
        }
        if (next_d < T) {
          const int s = next_d % kND;
          if (mbar_test(&bars[kDecFull + s], (next_d / kND) & 1)) {
            const uint32_t keep = misc[8 + s];
            mbar_arrive(&bars[kDecEmpty + s]);
            if (keep) vq[v_req++ % (kND + kNSV)] = next_d;
            ++next_d;
            progress = true;
          }
        }
        if (v_issued < v_req) {
          const int s = v_issued % kNSV;
          if (mbar_test(&bars[kSlotFree + s], ((v_issued / kNSV) & 1) ^ 1)) {
            const int t = vq[v_issued % (kND + kNSV)];
            const int j = t1 - 1 - t;
            mbar_expect_tx(&bars[kVFull + s], kTileBytes);
            for (int c = 0; c < 2; ++c)
              tma_load_4d(sV + s * kTileBytes + c * 16384, &p.tm_v, &bars[kVFull + s], c * 64, hk,
                          j * kBK, b);
            ++v_issued;
            progress = true;
          }
        }
        misc[2] = (static_cast<uint32_t>(next_k) << 20) | (static_cast<uint32_t>(next_d) << 10) | v_issued;
        if (progress) {
          idle_since = global_timer_ns();
        } else if (*abort_flag) {
          ok = false;
        } else if (global_timer_ns() - idle_since > kWaitLimitNs) {
          *abort_flag = 1;
          if (atomicCAS(p.err, 0, kErrTimeout) == 0) {
            p.err[1] = wait_tag(1, 0xff, next_d);
            p.err[2] = static_cast<int>(blockIdx.x);
            for (int x = 0; x < 3; ++x) p.err[4 + x] = misc[2 + x];
          }
          ok = false;
        }
      }
      if (!ok) drain_pause_ns(50000);
    }
  } else {
    // ===================== compute warps =====================
    const int g = lane >> 2;             // fragment row (and row + 8)
    const int tq = lane & 3;             // fragment column pair
    const int row_lo = g, row_hi = g + 8;
    const bool has_lo = row_lo < G, has_hi = row_hi < G;
    const int h_lo = has_lo ? p.group_heads[hk][row_lo] : 0;
    const int h_hi = has_hi ? p.group_heads[hk][row_hi] : 0;
    const float thr2 = p.log2_tau - log2f(static_cast<float>(p.Nk));   // log2(tau / L_0)

    // query A fragments for the 8 k-steps over d = 128
    uint32_t qa[8][4];
    {
      const uint32_t* qlo = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const __nv_bfloat16*>(p.q) + b * p.q_sb + h_lo * p.q_sh);
      const uint32_t* qhi = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const __nv_bfloat16*>(p.q) + b * p.q_sb + h_hi * p.q_sh);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        qa[kk][0] = has_lo ? qlo[(16 * kk + 2 * tq) >> 1] : 0u;
        qa[kk][1] = has_hi ? qhi[(16 * kk + 2 * tq) >> 1] : 0u;
        qa[kk][2] = has_lo ? qlo[(16 * kk + 8 + 2 * tq) >> 1] : 0u;
        qa[kk][3] = has_hi ? qhi[(16 * kk + 8 + 2 * tq) >> 1] : 0u;
      }
    }

    float m2_lo = -INFINITY, m2_hi = -INFINITY;   // reference maxima (log2 units)
    float l_lo = 0.0f, l_hi = 0.0f;               // normalisation sums
    float om_lo = -INFINITY, om_hi = -INFINITY;   // reference of the O accumulator rows
    float o[4][4];
#pragma unroll
    for (int nb = 0; nb < 4; ++nb)
#pragma unroll
      for (int x = 0; x < 4; ++x) o[nb][x] = 0.0f;
    int kc = 0, pv_done = 0;                     // retained tiles, PVs executed
    bool prev_any = false;
    uint32_t mw_lo = 0, mw_hi = 0;               // keep-mask word being built per row
    int kept_heads = 0;
    const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);

    auto fold_sums = [&](int par) {
      float a = 0.0f, c = 0.0f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        a += sPSum[(par * 4 + w) * 16 + row_lo];
        c += sPSum[(par * 4 + w) * 16 + row_hi];
      }
      l_lo += a;
      l_hi += c;
    };

    // O += P(slot) V(slot) for the oldest retained tile
    auto do_pv = [&]() -> bool {
      const int s = pv_done % kNSV;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[kVFull + s], (pv_done / kNSV) & 1, abort_flag,
                                                         p.err, wait_tag(0, kVFull + s, pv_done)));
      if (ok) {
        const float pm_lo = sPendM[s * 16 + row_lo], pm_hi = sPendM[s * 16 + row_hi];
        const float f_lo = (pm_lo == om_lo) ? 1.0f : ex2_approx(om_lo - pm_lo);
        const float f_hi = (pm_hi == om_hi) ? 1.0f : ex2_approx(om_hi - pm_hi);
        om_lo = pm_lo;
        om_hi = pm_hi;
#pragma unroll
        for (int nb = 0; nb < 4; ++nb) {
          o[nb][0] *= f_lo; o[nb][1] *= f_lo;
          o[nb][2] *= f_hi; o[nb][3] *= f_hi;
        }
        const uint32_t* prow_lo = reinterpret_cast<const uint32_t*>(sP + (s * 16 + row_lo) * kPStride);
        const uint32_t* prow_hi = reinterpret_cast<const uint32_t*>(sP + (s * 16 + row_hi) * kPStride);
        const uint32_t vbase = sVa + s * kTileBytes;
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a0 = prow_lo[(16 * kk + 2 * tq) >> 1];
          const uint32_t a1 = prow_hi[(16 * kk + 2 * tq) >> 1];
          const uint32_t a2 = prow_lo[(16 * kk + 8 + 2 * tq) >> 1];
          const uint32_t a3 = prow_hi[(16 * kk + 8 + 2 * tq) >> 1];
#pragma unroll
          for (int nb = 0; nb < 4; nb += 2) {
            // matrices: (keys 16kk+[0,8) | +8, cols 32w+8nb) then (cols +8)
            const int key = 16 * kk + ((mi & 1) << 3) + rr;
            const int col = 32 * warp + 8 * (nb + (mi >> 1));
            uint32_t b0, b1, b2, b3;
            ldsm_x4_trans(sw128_addr(vbase, key, col), b0, b1, b2, b3);
            mma_bf16_16816(o[nb], a0, a1, a2, a3, b0, b1);
            mma_bf16_16816(o[nb + 1], a0, a1, a2, a3, b2, b3);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kSlotFree + s]);
      ++pv_done;
      return ok;
    };

    for (int t = 0; t < T; ++t) {
      const int j = t1 - 1 - t;
      const int ks = t % kNSK;
      const bool okk = __all_sync(0xffffffffu, mbar_wait(&bars[kKFull + ks], (t / kNSK) & 1, abort_flag, p.err,
                                                         wait_tag(0, kKFull + ks, t)));
      float sacc[4][4];
#pragma unroll
      for (int nb = 0; nb < 4; ++nb)
#pragma unroll
        for (int x = 0; x < 4; ++x) sacc[nb][x] = 0.0f;
      if (okk) {
        const uint32_t kbase = sKa + ks * kTileBytes;
        const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
          for (int nb = 0; nb < 4; nb += 2) {
            // matrices: (keys 32w+8nb+[0,8), d 16kk | +8), then keys +8
            const int key = 32 * warp + 8 * (nb + (mi >> 1)) + rr;
            const int d0 = 16 * kk + ((mi & 1) << 3);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(sw128_addr(kbase, key, d0), b0, b1, b2, b3);
            mma_bf16_16816(sacc[nb], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
            mma_bf16_16816(sacc[nb + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
          }
        }
      }
      // keys past the cache end (last tile only) do not exist
      float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
      for (int nb = 0; nb < 4; ++nb) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int key = j * kBK + 32 * warp + 8 * nb + 2 * tq + x;
          if (key >= p.Nk) {
            sacc[nb][x] = -INFINITY;
            sacc[nb][2 + x] = -INFINITY;
          }
          mx_lo = fmaxf(mx_lo, sacc[nb][x]);
          mx_hi = fmaxf(mx_hi, sacc[nb][2 + x]);
        }
      }
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
      if (tq == 0) {
        sPMax[((t & 1) * 4 + warp) * 16 + row_lo] = mx_lo;
        sPMax[((t & 1) * 4 + warp) * 16 + row_hi] = mx_hi;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kKEmpty + ks]);
      // one barrier per tile; the OR of the abort flag keeps every warp's exit in step
      if (bar_or(1, 128, *abort_flag != 0)) break;

      // previous tile's sums, this tile's maxima, per-head decisions
      if (prev_any) fold_sums((t - 1) & 1);
      float tm_lo = -INFINITY, tm_hi = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        tm_lo = fmaxf(tm_lo, sPMax[((t & 1) * 4 + w) * 16 + row_lo]);
        tm_hi = fmaxf(tm_hi, sPMax[((t & 1) * 4 + w) * 16 + row_hi]);
      }
      const float tm2_lo = tm_lo * kLog2e, tm2_hi = tm_hi * kLog2e;
      const bool keep_lo = has_lo && (l_lo == 0.0f || tm2_lo - (m2_lo + lg2_approx(l_lo)) >= thr2);
      const bool keep_hi = has_hi && (l_hi == 0.0f || tm2_hi - (m2_hi + lg2_approx(l_hi)) >= thr2);
      const bool any = __any_sync(0xffffffffu, keep_lo || keep_hi);
      if (warp == 0 && tq == 0) {
        if (keep_lo) { mw_lo |= 1u << (j & 31); ++kept_heads; }
        if (keep_hi) { mw_hi |= 1u << (j & 31); ++kept_heads; }
        if ((j & 31) == 0 || t == T - 1) {
          if (p.keep_mask) {
            if (has_lo && mw_lo) atomicOr(&p.keep_mask[(static_cast<int64_t>(b) * p.Hq + h_lo) * p.mask_words + (j >> 5)], mw_lo);
            if (has_hi && mw_hi) atomicOr(&p.keep_mask[(static_cast<int64_t>(b) * p.Hq + h_hi) * p.mask_words + (j >> 5)], mw_hi);
          }
          mw_lo = mw_hi = 0;
        }
      }
      // publish the decision to the producer
      if (warp == 0 && lane == 0) {
        const int s = t % kND;
        if (mbar_wait(&bars[kDecEmpty + s], ((t / kND) & 1) ^ 1, abort_flag, p.err, wait_tag(0, kDecEmpty + s, t))) {
          misc[8 + s] = any ? 1u : 0u;
          mbar_arrive(&bars[kDecFull + s]);
        }
        misc[3] = 0x10000u | t;
      }
      prev_any = any;
      if (!any) continue;

      // online-softmax reference update of the retaining rows
      if (keep_lo) {
        if (l_lo == 0.0f) m2_lo = tm2_lo;
        else if (tm2_lo > m2_lo + kRescaleThreshold) { l_lo *= ex2_approx(m2_lo - tm2_lo); m2_lo = tm2_lo; }
      }
      if (keep_hi) {
        if (l_hi == 0.0f) m2_hi = tm2_hi;
        else if (tm2_hi > m2_hi + kRescaleThreshold) { l_hi *= ex2_approx(m2_hi - tm2_hi); m2_hi = tm2_hi; }
      }
      // P = 2^(s log2e - m2) for retaining rows, 0 otherwise
      float ps_lo = 0.0f, ps_hi = 0.0f;
      uint32_t pk_lo[4], pk_hi[4];
#pragma unroll
      for (int nb = 0; nb < 4; ++nb) {
        const float a0 = keep_lo ? ex2_approx(fmaf(sacc[nb][0], kLog2e, -m2_lo)) : 0.0f;
        const float a1 = keep_lo ? ex2_approx(fmaf(sacc[nb][1], kLog2e, -m2_lo)) : 0.0f;
        const float c0 = keep_hi ? ex2_approx(fmaf(sacc[nb][2], kLog2e, -m2_hi)) : 0.0f;
        const float c1 = keep_hi ? ex2_approx(fmaf(sacc[nb][3], kLog2e, -m2_hi)) : 0.0f;
        ps_lo += a0 + a1;
        ps_hi += c0 + c1;
        pk_lo[nb] = pack_bf16x2(a0, a1);
        pk_hi[nb] = pack_bf16x2(c0, c1);
      }
      ps_lo += __shfl_xor_sync(0xffffffffu, ps_lo, 1);
      ps_lo += __shfl_xor_sync(0xffffffffu, ps_lo, 2);
      ps_hi += __shfl_xor_sync(0xffffffffu, ps_hi, 1);
      ps_hi += __shfl_xor_sync(0xffffffffu, ps_hi, 2);
      if (tq == 0) {
        sPSum[((t & 1) * 4 + warp) * 16 + row_lo] = ps_lo;
        sPSum[((t & 1) * 4 + warp) * 16 + row_hi] = ps_hi;
      }
      // a free P/V slot: run the oldest pending PV when both are taken
      if (kc - pv_done == kNSV) do_pv();
      const int s = kc % kNSV;
      mbar_wait(&bars[kSlotFree + s], ((kc / kNSV) & 1) ^ 1, abort_flag, p.err, wait_tag(0, kSlotFree + s, kc));
      {
        uint32_t* prow_lo = reinterpret_cast<uint32_t*>(sP + (s * 16 + row_lo) * kPStride);
        uint32_t* prow_hi = reinterpret_cast<uint32_t*>(sP + (s * 16 + row_hi) * kPStride);
#pragma unroll
        for (int nb = 0; nb < 4; ++nb) {
          prow_lo[(32 * warp + 8 * nb + 2 * tq) >> 1] = pk_lo[nb];
          prow_hi[(32 * warp + 8 * nb + 2 * tq) >> 1] = pk_hi[nb];
        }
        if (warp == 0 && tq == 0) {
          sPendM[s * 16 + row_lo] = has_lo ? m2_lo : 0.0f;
          sPendM[s * 16 + row_hi] = has_hi ? m2_hi : 0.0f;
        }
      }
      ++kc;
    }

    // drain the deferred PVs; the last barrier makes every warp's P and sums visible
    if (!bar_or(1, 128, *abort_flag != 0)) {
      while (pv_done < kc) do_pv();
      if (prev_any) fold_sums((T - 1) & 1);
      // outputs: rows < G of this warp's 32 columns
      const float inv_lo = l_lo > 0.0f ? 1.0f / l_lo : 0.0f;
      const float inv_hi = l_hi > 0.0f ? 1.0f / l_hi : 0.0f;
      const float z_lo = (m2_lo + log2f(l_lo)) * kLn2;
      const float z_hi = (m2_hi + log2f(l_hi)) * kLn2;
      if (P == 1) {
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.o);
#pragma unroll
        for (int nb = 0; nb < 4; ++nb) {
          const int col = 32 * warp + 8 * nb + 2 * tq;
          if (has_lo)
            *reinterpret_cast<uint32_t*>(out + b * p.o_sb + h_lo * p.o_sh + col) =
                pack_bf16x2(o[nb][0] * inv_lo, o[nb][1] * inv_lo);
          if (has_hi)
            *reinterpret_cast<uint32_t*>(out + b * p.o_sb + h_hi * p.o_sh + col) =
                pack_bf16x2(o[nb][2] * inv_hi, o[nb][3] * inv_hi);
        }
        if (warp == 0 && tq == 0) {
          if (has_lo) p.lse[b * p.Hq + h_lo] = z_lo;
          if (has_hi) p.lse[b * p.Hq + h_hi] = z_hi;
        }
      } else {
#pragma unroll
        for (int nb = 0; nb < 4; ++nb) {
          const int col = 32 * warp + 8 * nb + 2 * tq;
          if (has_lo) {
            float2* dst = reinterpret_cast<float2*>(p.part_o + ((static_cast<int64_t>(b) * p.Hq + h_lo) * P + split) * kD + col);
            *dst = make_float2(o[nb][0] * inv_lo, o[nb][1] * inv_lo);
          }
          if (has_hi) {
            float2* dst = reinterpret_cast<float2*>(p.part_o + ((static_cast<int64_t>(b) * p.Hq + h_hi) * P + split) * kD + col);
            *dst = make_float2(o[nb][2] * inv_hi, o[nb][3] * inv_hi);
          }
        }
        if (warp == 0 && tq == 0) {
          if (has_lo) p.part_lse[(static_cast<int64_t>(b) * p.Hq + h_lo) * P + split] = z_lo;
          if (has_hi) p.part_lse[(static_cast<int64_t>(b) * p.Hq + h_hi) * P + split] = z_hi;
        }
      }
      if (p.stats && warp == 0) {
        int kh = kept_heads;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kh += __shfl_xor_sync(0xffffffffu, kh, off);
        if (lane == 0) {
          atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[0]), static_cast<unsigned long long>(T));
          atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[1]), static_cast<unsigned long long>(kc));
          atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[2]), static_cast<unsigned long long>(kh));
        }
      }
    }
  }
  __syncthreads();
}

// z = log sum_p exp(z_p), O = sum_p exp(z_p - z) O_p, one CTA per (b, head)
__global__ void __launch_bounds__(128) mala_decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  const int bh = blockIdx.x;
  const int b = bh / p.Hq, h = bh % p.Hq;
  const int P = p.num_splits;
  const float* lz = p.part_lse + static_cast<int64_t>(bh) * P;
  float zmax = -INFINITY;
  for (int s = 0; s < P; ++s) zmax = fmaxf(zmax, lz[s]);
  float den = 0.0f;
  for (int s = 0; s < P; ++s) den += expf(lz[s] - zmax);
  const float z = zmax + logf(den);
  const int c = threadIdx.x;
  float acc = 0.0f;
  for (int s = 0; s < P; ++s) acc += expf(lz[s] - z) * p.part_o[(static_cast<int64_t>(bh) * P + s) * kD + c];
  reinterpret_cast<__nv_bfloat16*>(p.o)[b * p.o_sb + h * p.o_sh + c] = __float2bfloat16_rn(acc);
  if (c == 0) p.lse[bh] = z;
}

}  // namespace

size_t decode_smem_bytes() { return Smem::kAlloc; }

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hkv * p.num_splits;
  if (grid == 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(mala_decode_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(Smem::kAlloc));
  if (e != cudaSuccess) return e;
  mala_decode_split_kernel<<<grid, kThreads, Smem::kAlloc, stream>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.num_splits == 1) return e;
  mala_decode_combine_kernel<<<p.B * p.Hq, kD, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mala
