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
// Roles (32 (W + 1) threads; W = 4 compute warps):
//   warps 0..W-1  compute. QK^T: warp w scores keys [w 128/W, (w+1) 128/W)
//              of the tile for all rows; row maxima meet in shared memory;
//              every warp then evaluates the same per-head decisions. PV:
//              warp w owns output columns [w 128/W, (w+1) 128/W) over all
//              128 keys. Warp 0 also issues each retained tile's V load, as
//              soon as its V/P slot is free.
//   warp W     TMA producer for K, in order: tiles as far ahead as the K
//              ring allows (independent of decisions), blocking on the ring.
// PV is deferred: a retained tile's P (bf16) and reference maxima wait in
// one of two slots until the slot is needed again or the split ends, so the
// V load issued after the decision overlaps the scoring of later tiles.
//
// Residency: a bf16 CTA (4-tile K ring) fills an SM's shared memory. An
// e4m3 tile has half the bytes but the same fragment work, so one CTA per
// SM leaves the SM waiting on its per-tile chain; an e4m3 CTA instead keeps
// a 2-tile K ring (76 KB of shared memory, 128 registers per thread) and
// three CTAs share an SM, each streaming its own split.
//
// FP8 (e4m3) caches: tiles arrive as 128-byte rows, and the mma.sync B
// fragments are built straight from them, converting in registers (exactly:
// every e4m3 value is an f16):
//   QK: the head dimension is visited in a permuted order, the same for the
//       query fragments and K, chosen so that a thread's 32 values of a key
//       row are 32 contiguous bytes (two 16-byte loads);
//   PV: the output columns are permuted within each warp's 32, so that one
//       4-byte load of a value row covers the thread's column in all four
//       n-blocks; byte permutes pair consecutive keys for the fragments.
// Both access patterns are free of bank conflicts under the 128-byte
// swizzle. Scores and PV run as f16 mma.sync with the query and P in f16;
// the cache scales are applied in fp32 (to the scores, and to O at the end).
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

#ifndef MALA_DECODE_BF16_WARPS
#define MALA_DECODE_BF16_WARPS 4
#endif
#ifndef MALA_DECODE_FP8_WARPS
#define MALA_DECODE_FP8_WARPS 4
#endif
#ifndef MALA_DECODE_FP8_RING
#define MALA_DECODE_FP8_RING 2
#endif
#ifndef MALA_DECODE_FP8_CTAS
#define MALA_DECODE_FP8_CTAS 3
#endif

namespace mala {

namespace {

constexpr int kBK = 128;
constexpr int kD = 128;
constexpr int kNSKMax = 8;              // K ring stages at most (4 bf16 tiles, 2 e4m3 tiles)
constexpr int kNSV = 2;                 // V / P slots
constexpr uint32_t kTileBytes = kBK * kD * 2;   // bf16 tile
constexpr int kPStride = 136;           // bf16 per P row (128 + 8 padding)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;

enum Bar {
  kKFull = 0,                     // kNSKMax
  kKEmpty = kKFull + kNSKMax,     // kNSKMax, 4 arrivals (one per compute warp)
  kVFull = kKEmpty + kNSKMax,     // kNSV
  kSlotFree = kVFull + kNSV,      // kNSV, 4 arrivals
  kNumBars = kSlotFree + kNSV
};

template <bool FP8>
struct Smem {
  static constexpr int kCW = FP8 ? MALA_DECODE_FP8_WARPS : MALA_DECODE_BF16_WARPS;   // compute warps
  static constexpr int kMinCtas = FP8 ? MALA_DECODE_FP8_CTAS : 1;       // resident CTAs per SM
  static constexpr int kThreads = 32 * (kCW + 1);                       // + the producer warp
  static constexpr int kKPW = kBK / kCW;      // keys (scores) and value columns (PV) per compute warp
  static constexpr int kNBW = kKPW / 8;       // mma n-blocks per compute warp
  static constexpr int kNSK = FP8 ? MALA_DECODE_FP8_RING : 4;          // K ring stages
  static constexpr uint32_t kRing = FP8 ? kBK * kD : kTileBytes;        // bytes of a K / V ring tile
  static constexpr uint32_t kK = 0;
  static constexpr uint32_t kV = kK + kNSK * kRing;
  static constexpr uint32_t kP = kV + kNSV * kRing;                     // [kNSV][16][kPStride] bf16 / f16
  static constexpr uint32_t kPendM = kP + kNSV * 16 * kPStride * 2;      // [kNSV][16] float
  static constexpr uint32_t kPMax = kPendM + kNSV * 16 * 4;              // [2][16][kCW] float
  static constexpr uint32_t kPSum = kPMax + 2 * kCW * 16 * 4;            // [2][16][kCW] float
  static constexpr uint32_t kBars = kPSum + 2 * kCW * 16 * 4;
  static constexpr uint32_t kMisc = kBars + kNumBars * 8;               // misc words
  static constexpr uint32_t kEnd = kMisc + 64;
  static constexpr uint32_t kAlloc = kEnd + 1024;
};
static_assert(Smem<false>::kAlloc <= 232448 && Smem<true>::kAlloc <= 232448, "decode CTA exceeds shared memory");
static_assert(Smem<false>::kPMax % 16 == 0 && Smem<true>::kPMax % 16 == 0, "per-warp row data read as float4");
static_assert(Smem<false>::kNSK <= kNSKMax && Smem<true>::kNSK <= kNSKMax, "K ring exceeds its barriers");

template <bool FP8>
__global__ void __launch_bounds__(Smem<FP8>::kThreads, Smem<FP8>::kMinCtas) mala_decode_split_kernel(const __grid_constant__ DecodeParams p) {
  using Smem = mala::Smem<FP8>;
  constexpr uint32_t kRing = Smem::kRing;
  constexpr int kNSK = Smem::kNSK;
  constexpr int kCW = Smem::kCW, kKPW = Smem::kKPW, kNBW = Smem::kNBW;
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
  // misc[1] abort flag
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
      if ((x >= kKEmpty && x < kKEmpty + kNSKMax) || (x >= kSlotFree && x < kSlotFree + kNSV)) cnt = kCW;
      mbar_init(&bars[x], cnt);
    }
    for (int x = 1; x < 16; ++x) misc[x] = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kCW) {
    // ===================== K producer =====================
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_k);
      for (int t = 0; t < T; ++t) {
        const int s = t % kNSK;
        if (!mbar_wait(&bars[kKEmpty + s], ((t / kNSK) & 1) ^ 1, abort_flag, p.err, wait_tag(1, kKEmpty + s, t), p.wait_ns)) {
          drain_pause_ns(50000);         // copies already issued land before the CTA exits
          break;
        }
        mbar_expect_tx(&bars[kKFull + s], kRing);
        const int j = t1 - 1 - t;
        for (int c = 0; c < (FP8 ? 1 : 2); ++c)
          tma_load_4d(sK + s * kRing + c * 16384, &p.tm_k, &bars[kKFull + s], c * 64, hk, j * kBK, b);
      }
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
    if (warp == 0 && lane == 0) tma_prefetch_desc(&p.tm_v);
    // log2(e) times the scale of the raw scores (FP8 caches: the key scale)
    const float sl2 = FP8 ? kLog2e * p.k_scale : kLog2e;

    // query A fragments for the 8 k-steps over d = 128; FP8 caches: k-step
    // kk, fragment column 2tq + e (+ 8) holds d = 32tq + 4kk + e (+ 2)
    uint32_t qa[8][4];
    {
      const uint32_t* qlo = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const __nv_bfloat16*>(p.q) + b * p.q_sb + h_lo * p.q_sh);
      const uint32_t* qhi = reinterpret_cast<const uint32_t*>(
          reinterpret_cast<const __nv_bfloat16*>(p.q) + b * p.q_sb + h_hi * p.q_sh);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int w0 = FP8 ? 16 * tq + 2 * kk : (16 * kk + 2 * tq) >> 1;
        const int w1 = FP8 ? w0 + 1 : w0 + 4;
        qa[kk][0] = has_lo ? qlo[w0] : 0u;
        qa[kk][1] = has_hi ? qhi[w0] : 0u;
        qa[kk][2] = has_lo ? qlo[w1] : 0u;
        qa[kk][3] = has_hi ? qhi[w1] : 0u;
        if constexpr (FP8) {
#pragma unroll
          for (int x = 0; x < 4; ++x) qa[kk][x] = bf16x2_to_f16x2(qa[kk][x]);
        }
      }
    }

    float m2_lo = -INFINITY, m2_hi = -INFINITY;   // reference maxima (log2 units)
    float l_lo = 0.0f, l_hi = 0.0f;               // normalisation sums
    float om_lo = -INFINITY, om_hi = -INFINITY;   // reference of the O accumulator rows
    float o[kNBW][4];
#pragma unroll
    for (int nb = 0; nb < kNBW; ++nb)
#pragma unroll
      for (int x = 0; x < 4; ++x) o[nb][x] = 0.0f;
    int kc = 0, pv_done = 0;                     // retained tiles, PVs executed
    bool prev_any = false;
    uint32_t mw_lo = 0, mw_hi = 0;               // keep-mask word being built per row
    int kept_heads = 0;
    const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);

    // per-warp row values [par][row][warp]: combined with float4 reads
    auto row_max = [&](const float* base, int par, int row) {
      const float4* v = reinterpret_cast<const float4*>(base + (par * 16 + row) * kCW);
      float m = -INFINITY;
#pragma unroll
      for (int w4 = 0; w4 < kCW / 4; ++w4) {
        const float4 x = v[w4];
        m = fmaxf(m, fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
      }
      return m;
    };
    auto row_sum = [&](const float* base, int par, int row) {
      const float4* v = reinterpret_cast<const float4*>(base + (par * 16 + row) * kCW);
      float a = 0.0f;
#pragma unroll
      for (int w4 = 0; w4 < kCW / 4; ++w4) {
        const float4 x = v[w4];
        a += (x.x + x.y) + (x.z + x.w);
      }
      return a;
    };
    auto fold_sums = [&](int par) {
      const float a = row_sum(sPSum, par, row_lo), c = row_sum(sPSum, par, row_hi);
      l_lo += a;
      l_hi += c;
    };

    // O += P(slot) V(slot) for the oldest retained tile
    auto do_pv = [&]() -> bool {
      const int s = pv_done % kNSV;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[kVFull + s], (pv_done / kNSV) & 1, abort_flag,
                                                         p.err, wait_tag(0, kVFull + s, pv_done), p.wait_ns));
      if (ok) {
        const float pm_lo = sPendM[s * 16 + row_lo], pm_hi = sPendM[s * 16 + row_hi];
        const float f_lo = (pm_lo == om_lo) ? 1.0f : ex2_approx(om_lo - pm_lo);
        const float f_hi = (pm_hi == om_hi) ? 1.0f : ex2_approx(om_hi - pm_hi);
        om_lo = pm_lo;
        om_hi = pm_hi;
#pragma unroll
        for (int nb = 0; nb < kNBW; ++nb) {
          o[nb][0] *= f_lo; o[nb][1] *= f_lo;
          o[nb][2] *= f_hi; o[nb][3] *= f_hi;
        }
        const uint32_t vbase = sVa + s * kRing;
        const int mi = lane >> 3, rr = lane & 7;
        // A fragments of P: matrices (rows 0-7 | 8-15) x (keys 16kk + [0, 8) | + 8)
        const uint32_t pa = smem_u32(sP) + ((s * 16 + ((mi & 1) << 3) + rr) * kPStride + 8 * (mi >> 1)) * 2;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          uint32_t a0, a1, a2, a3;
          ldsm_x4(pa + 32 * kk, a0, a1, a2, a3);
          if constexpr (FP8) {
            // n-block nb, fragment column g is value column kKPW w + kNBW g + nb:
            // bytes [kKPW w + kNBW g, + kNBW) of the rows of keys 16kk + 2tq
            // (+1, +8, +9), paired across consecutive keys
            const int cb = kKPW * warp + kNBW * g;
            uint32_t r[4];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
              const uint32_t a = sw128_addr_b8(vbase, 16 * kk + 2 * tq + (x & 1) + 8 * (x >> 1), cb >> 4) + (cb & 15);
              r[x] = kNBW == 4 ? ld_shared_u32(a) : ld_shared_u16(a);
            }
            uint32_t b0[kNBW], b1[kNBW];
            e4m3x4_to_f16x4(__byte_perm(r[0], r[1], 0x5140), b0[0], b0[1]);
            e4m3x4_to_f16x4(__byte_perm(r[2], r[3], 0x5140), b1[0], b1[1]);
            if constexpr (kNBW == 4) {
              e4m3x4_to_f16x4(__byte_perm(r[0], r[1], 0x7362), b0[2], b0[3]);
              e4m3x4_to_f16x4(__byte_perm(r[2], r[3], 0x7362), b1[2], b1[3]);
            }
#pragma unroll
            for (int nb = 0; nb < kNBW; ++nb) mma_f16_16816(o[nb], a0, a1, a2, a3, b0[nb], b1[nb]);
          } else {
#pragma unroll
            for (int nb = 0; nb < kNBW; nb += 2) {
              // matrices: (keys 16kk+[0,8) | +8, cols 32w+8nb) then (cols +8)
              const int key = 16 * kk + ((mi & 1) << 3) + rr;
              const int col = kKPW * warp + 8 * (nb + (mi >> 1));
              uint32_t b0, b1, b2, b3;
              ldsm_x4_trans(sw128_addr(vbase, key, col), b0, b1, b2, b3);
              mma_bf16_16816(o[nb], a0, a1, a2, a3, b0, b1);
              mma_bf16_16816(o[nb + 1], a0, a1, a2, a3, b2, b3);
            }
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
                                                         wait_tag(0, kKFull + ks, t), p.wait_ns));
      float sacc[kNBW][4];
#pragma unroll
      for (int nb = 0; nb < kNBW; ++nb)
#pragma unroll
        for (int x = 0; x < 4; ++x) sacc[nb][x] = 0.0f;
      if (okk) {
        const uint32_t kbase = sKa + ks * kRing;
        if constexpr (FP8) {
          // n-block nb, fragment column g is key kKPW w + 8nb + g; k-step kk
          // takes bytes 4kk .. 4kk + 3 of its bytes [32tq, 32tq + 32)
#pragma unroll
          for (int nb = 0; nb < kNBW; ++nb) {
            const int key = kKPW * warp + 8 * nb + g;
            uint32_t w[8];
            ld_shared_v4(sw128_addr_b8(kbase, key, 2 * tq), w[0], w[1], w[2], w[3]);
            ld_shared_v4(sw128_addr_b8(kbase, key, 2 * tq + 1), w[4], w[5], w[6], w[7]);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              uint32_t b0, b1;
              e4m3x4_to_f16x4(w[kk], b0, b1);
              mma_f16_16816(sacc[nb], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
            }
          }
        } else {
          const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
            for (int nb = 0; nb < kNBW; nb += 2) {
              // matrices: (keys kKPW w+8nb+[0,8), d 16kk | +8), then keys +8
              const int key = kKPW * warp + 8 * (nb + (mi >> 1)) + rr;
              const int d0 = 16 * kk + ((mi & 1) << 3);
              uint32_t b0, b1, b2, b3;
              ldsm_x4(sw128_addr(kbase, key, d0), b0, b1, b2, b3);
              mma_bf16_16816(sacc[nb], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
              mma_bf16_16816(sacc[nb + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
            }
          }
        }
      }
      // keys past the cache end (last tile only) do not exist
      if (j * kBK + kBK > p.Nk) {
#pragma unroll
        for (int nb = 0; nb < kNBW; ++nb)
#pragma unroll
          for (int x = 0; x < 2; ++x)
            if (j * kBK + kKPW * warp + 8 * nb + 2 * tq + x >= p.Nk) {
              sacc[nb][x] = -INFINITY;
              sacc[nb][2 + x] = -INFINITY;
            }
      }
      float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
      for (int nb = 0; nb < kNBW; ++nb) {
        mx_lo = fmaxf(mx_lo, fmaxf(sacc[nb][0], sacc[nb][1]));
        mx_hi = fmaxf(mx_hi, fmaxf(sacc[nb][2], sacc[nb][3]));
      }
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
      if (tq == 0) {
        // FP8 caches: the scores so far lack the key scale (> 0, so it
        // commutes with the maximum); it enters here and in sl2 below
        sPMax[((t & 1) * 16 + row_lo) * kCW + warp] = FP8 ? mx_lo * p.k_scale : mx_lo;
        sPMax[((t & 1) * 16 + row_hi) * kCW + warp] = FP8 ? mx_hi * p.k_scale : mx_hi;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kKEmpty + ks]);
      // one barrier per tile; the OR of the abort flag keeps every warp's exit in step
      if (bar_or(1, 32 * kCW, *abort_flag != 0)) break;

      // previous tile's sums, this tile's maxima, per-head decisions
      if (prev_any) fold_sums((t - 1) & 1);
      const float tm_lo = row_max(sPMax, t & 1, row_lo), tm_hi = row_max(sPMax, t & 1, row_hi);
      const float tm2_lo = tm_lo * kLog2e, tm2_hi = tm_hi * kLog2e;
      bool keep_lo = has_lo && (l_lo == 0.0f || tm2_lo - (m2_lo + lg2_approx(l_lo)) >= thr2);
      bool keep_hi = has_hi && (l_hi == 0.0f || tm2_hi - (m2_hi + lg2_approx(l_hi)) >= thr2);
      const bool any = __any_sync(0xffffffffu, keep_lo || keep_hi);   // over all 16 rows
      if (p.group_vote) {
        // group-joint voting: the group's rows decide together, like the
        // rows of one query block; every head accumulates a retained tile
        keep_lo = has_lo && any;
        keep_hi = has_hi && any;
      }
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
      uint32_t pk_lo[kNBW], pk_hi[kNBW];
#pragma unroll
      for (int nb = 0; nb < kNBW; ++nb) {
        const float a0 = keep_lo ? ex2_approx(fmaf(sacc[nb][0], sl2, -m2_lo)) : 0.0f;
        const float a1 = keep_lo ? ex2_approx(fmaf(sacc[nb][1], sl2, -m2_lo)) : 0.0f;
        const float c0 = keep_hi ? ex2_approx(fmaf(sacc[nb][2], sl2, -m2_hi)) : 0.0f;
        const float c1 = keep_hi ? ex2_approx(fmaf(sacc[nb][3], sl2, -m2_hi)) : 0.0f;
        ps_lo += a0 + a1;
        ps_hi += c0 + c1;
        pk_lo[nb] = FP8 ? pack_f16x2(a0, a1) : pack_bf16x2(a0, a1);
        pk_hi[nb] = FP8 ? pack_f16x2(c0, c1) : pack_bf16x2(c0, c1);
      }
      ps_lo += __shfl_xor_sync(0xffffffffu, ps_lo, 1);
      ps_lo += __shfl_xor_sync(0xffffffffu, ps_lo, 2);
      ps_hi += __shfl_xor_sync(0xffffffffu, ps_hi, 1);
      ps_hi += __shfl_xor_sync(0xffffffffu, ps_hi, 2);
      if (tq == 0) {
        sPSum[((t & 1) * 16 + row_lo) * kCW + warp] = ps_lo;
        sPSum[((t & 1) * 16 + row_hi) * kCW + warp] = ps_hi;
      }
      // a free P/V slot: run the oldest pending PV when both are taken
      if (kc - pv_done == kNSV) do_pv();
      const int s = kc % kNSV;
      const bool slot_ok = mbar_wait(&bars[kSlotFree + s], ((kc / kNSV) & 1) ^ 1, abort_flag, p.err,
                                     wait_tag(0, kSlotFree + s, kc), p.wait_ns);
      if (warp == 0 && lane == 0 && slot_ok) {
        // every warp has finished the slot's previous PV: load this tile's V
        mbar_expect_tx(&bars[kVFull + s], kRing);
        for (int c = 0; c < (FP8 ? 1 : 2); ++c)
          tma_load_4d(sV + s * kRing + c * 16384, &p.tm_v, &bars[kVFull + s], c * 64, hk, j * kBK, b);
      }
      {
        uint32_t* prow_lo = reinterpret_cast<uint32_t*>(sP + (s * 16 + row_lo) * kPStride);
        uint32_t* prow_hi = reinterpret_cast<uint32_t*>(sP + (s * 16 + row_hi) * kPStride);
#pragma unroll
        for (int nb = 0; nb < kNBW; ++nb) {
          prow_lo[(kKPW * warp + 8 * nb + 2 * tq) >> 1] = pk_lo[nb];
          prow_hi[(kKPW * warp + 8 * nb + 2 * tq) >> 1] = pk_hi[nb];
        }
        if (warp == 0 && tq == 0) {
          sPendM[s * 16 + row_lo] = has_lo ? m2_lo : 0.0f;
          sPendM[s * 16 + row_hi] = has_hi ? m2_hi : 0.0f;
        }
      }
      ++kc;
    }

    // drain the deferred PVs; the last barrier makes every warp's P and sums visible
    if (!bar_or(1, 32 * kCW, *abort_flag != 0)) {
      while (pv_done < kc) do_pv();
      if (prev_any) fold_sums((T - 1) & 1);
      // outputs: rows < G of this warp's 32 columns
      // FP8 caches: the value scale folds into the normalisation
      const float vs = FP8 ? p.v_scale : 1.0f;
      const float inv_lo = l_lo > 0.0f ? vs / l_lo : 0.0f;
      const float inv_hi = l_hi > 0.0f ? vs / l_hi : 0.0f;
      const float z_lo = (m2_lo + log2f(l_lo)) * kLn2;
      const float z_hi = (m2_hi + log2f(l_hi)) * kLn2;
      // column pairs (c, c + 1) this thread writes, c = col[i], with rows lo
      // (vl) and hi (vh): bf16 caches: n-block i, c = kKPW w + 8i + 2tq. FP8
      // caches (n-block nb, fragment column n is kKPW w + kNBW n + nb): the
      // thread's columns are kKPW w + 2 kNBW tq + e, e < 2 kNBW, from
      // o[e % kNBW][e / kNBW]
      int col[kNBW];
      float vl[kNBW][2], vh[kNBW][2];
#pragma unroll
      for (int i = 0; i < kNBW; ++i) {
        const int nb = FP8 ? (2 * i) % kNBW : i, x = FP8 ? (2 * i) / kNBW : 0;
        col[i] = FP8 ? kKPW * warp + 2 * kNBW * tq + 2 * i : kKPW * warp + 8 * i + 2 * tq;
        vl[i][0] = FP8 ? o[nb][x] : o[nb][0];
        vl[i][1] = FP8 ? o[nb + 1][x] : o[nb][1];
        vh[i][0] = FP8 ? o[nb][2 + x] : o[nb][2];
        vh[i][1] = FP8 ? o[nb + 1][2 + x] : o[nb][3];
      }
      if (P == 1) {
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.o);
#pragma unroll
        for (int i = 0; i < kNBW; ++i) {
          if (has_lo)
            *reinterpret_cast<uint32_t*>(out + b * p.o_sb + h_lo * p.o_sh + col[i]) =
                pack_bf16x2(vl[i][0] * inv_lo, vl[i][1] * inv_lo);
          if (has_hi)
            *reinterpret_cast<uint32_t*>(out + b * p.o_sb + h_hi * p.o_sh + col[i]) =
                pack_bf16x2(vh[i][0] * inv_hi, vh[i][1] * inv_hi);
        }
        if (warp == 0 && tq == 0) {
          if (has_lo) p.lse[b * p.Hq + h_lo] = z_lo;
          if (has_hi) p.lse[b * p.Hq + h_hi] = z_hi;
        }
      } else {
#pragma unroll
        for (int i = 0; i < kNBW; ++i) {
          if (has_lo) {
            float2* dst = reinterpret_cast<float2*>(p.part_o + ((static_cast<int64_t>(b) * p.Hq + h_lo) * P + split) * kD + col[i]);
            *dst = make_float2(vl[i][0] * inv_lo, vl[i][1] * inv_lo);
          }
          if (has_hi) {
            float2* dst = reinterpret_cast<float2*>(p.part_o + ((static_cast<int64_t>(b) * p.Hq + h_hi) * P + split) * kD + col[i]);
            *dst = make_float2(vh[i][0] * inv_hi, vh[i][1] * inv_hi);
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
  // after a timeout, copies issued before the waits gave up land before the
  // CTA's shared memory is released
  if (tid == 0 && *abort_flag) drain_pause_ns(50000);
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


cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hkv * p.num_splits;
  if (grid == 0) return cudaSuccess;
  cudaError_t e;
  if (p.kv_fp8) {
    e = cudaFuncSetAttribute(mala_decode_split_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(Smem<true>::kAlloc));
    if (e != cudaSuccess) return e;
    mala_decode_split_kernel<true><<<grid, Smem<true>::kThreads, Smem<true>::kAlloc, stream>>>(p);
  } else {
    e = cudaFuncSetAttribute(mala_decode_split_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(Smem<false>::kAlloc));
    if (e != cudaSuccess) return e;
    mala_decode_split_kernel<false><<<grid, Smem<false>::kThreads, Smem<false>::kAlloc, stream>>>(p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess || p.num_splits == 1) return e;
  mala_decode_combine_kernel<<<p.B * p.Hq, kD, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mala
