// MALA forward (Algorithm 1, "Online Sparse Softmax") on sm_100a tensor cores.
//
// One CTA owns one query block I_i of 128 rows of one (batch, query head).
// Key blocks are visited in descending order from the diagonal (Appendix
// A.1, "Fused forward execution"); every legal tile is scored, and only a
// retained tile loads V and runs the online-softmax update and PV.
//
// Warp roles (192 threads):
//   warps 0-3  "softmax": thread t owns query row t (= TMEM lane t). Reads
//              S from TMEM, applies the causal mask, computes the row max,
//              votes on the skip test, and for retained tiles computes
//              P = exp(S - m) into shared memory and updates m, l.
//   warp 4     TMA producer: Q once, K tiles two ahead, V only after the
//              vote retained the tile.
//   warp 5     tcgen05 issuer: S_t = Q K_t^T into one of two TMEM S buffers
//              (two tiles ahead of the vote), O += P V_t for retained tiles.
// TMEM: S0 = cols [0,128), S1 = [128,256), O = [256, 256 + D).
//
// Numerics: scores are accumulated in fp32 from bf16 operands. The online
// state is kept in base 2: m2 is a reference maximum (in log2 units) and l
// the sum of 2^(s*log2e - m2) over retained keys, so log Z = (m2 + log2 l)
// * ln 2 exactly as m + log l in the paper's notation. The reference is only
// moved up when a retained tile's maximum exceeds it by more than 8 (a factor
// 256), so O is rescaled rarely; P stays below 256, well inside bf16/fp32
// range. The skip test compares in log2 units, which is the natural-log test
// multiplied by log2 e.
#include "kernels.h"
#include "ptx.cuh"

namespace mala {

namespace {

constexpr int kBQ = 128;
constexpr int kBK = 128;
constexpr int kThreads = 192;
constexpr uint32_t kChunkBytes = 128 * 128;     // 128 rows x 64 bf16 (one swizzle column)
constexpr uint32_t kPBytes = kBQ * kBK * 2;     // P tile, bf16
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;       // log2 units

enum Bar {
  kQFull = 0,
  kKFull = 1,     // 2
  kKEmpty = 3,    // 2
  kVFull = 5,     // 2
  kVEmpty = 7,    // 2
  kSFull = 9,     // 2
  kSEmpty = 11,   // 2
  kDecFull = 13,  // 2
  kDecEmpty = 15, // 2
  kPFull = 17,    // 2
  kPEmpty = 19,   // 2
  kMmaDone = 21,
  kNumBars = 22
};

template <int D>
struct Layout {
  static constexpr uint32_t kTile = kBQ * D * 2;   // Q / K / V tile bytes
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTile;       // 2 stages
  static constexpr uint32_t kV = kK + 2 * kTile;   // 2 stages
  static constexpr uint32_t kP = kV + 2 * kTile;   // 2 buffers
  static constexpr uint32_t kBars = kP + 2 * kPBytes;
  static constexpr uint32_t kMisc = kBars + kNumBars * 8;
  static constexpr uint32_t kEnd = kMisc + 64;
  static constexpr uint32_t kAlloc = kEnd + 1024;  // slack for 1024-byte alignment
};

// Ties every later use of r[] to after the preceding tcgen05.wait.
__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}

// Each CTA allocates all 512 TMEM columns, so at most one CTA may be resident
// per SM: the shared-memory footprint alone must rule out a second one.
static_assert(Layout<64>::kAlloc > 116 * 1024 && Layout<128>::kAlloc > 116 * 1024,
              "forward CTA must exclude a second resident CTA per SM");
static_assert(Layout<128>::kAlloc <= 232448, "forward CTA exceeds shared memory");

template <int D>
__global__ void __launch_bounds__(kThreads, 1) mala_fwd_tc_kernel(const __grid_constant__ FwdTcParams p) {
  using L = Layout<D>;
  constexpr int NCH = D / 64;       // 128-byte chunks per row of Q/K/V
  constexpr int KSTEPS = D / 16;    // QK^T k-steps
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sK = smem + L::kK;
  uint8_t* sV = smem + L::kV;
  uint8_t* sP = smem + L::kP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + L::kMisc);
  // misc[0] TMEM base, misc[1] abort flag, misc[2..4] progress markers of the
  // producer / MMA / softmax roles (kept for timeout diagnosis), misc[5..6]
  // decisions of tiles t & 1
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- work item: query blocks with more key tiles first
  const int BH = p.B * p.Hq;
  const int i = p.nQB - 1 - static_cast<int>(blockIdx.x) / BH;
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int b = bh / p.Hq;
  const int h = bh % p.Hq;
  const int hk = p.kv_of_q[h];
  const int q0 = i * kBQ;
  const int last_row = min(q0 + kBQ - 1, p.N - 1);
  const int j_diag = min(last_row / kBK, p.nKB - 1);
  const int T = j_diag + 1;         // tile t visits key block j = j_diag - t

  if (tid == 0) {
    for (int x = 0; x < kNumBars; ++x) {
      uint32_t cnt = 1;
      if (x == kSEmpty || x == kSEmpty + 1 || x == kPFull || x == kPFull + 1) cnt = kBQ;
      if (x == kDecEmpty || x == kDecEmpty + 1) cnt = 2;
      mbar_init(&bars[x], cnt);
    }
    misc[1] = 0;
    misc[2] = misc[3] = misc[4] = 0;
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
  const uint32_t tmem_o = tmem + 256;

  if (warp == 4) {
    // ===================== TMA producer =====================
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_expect_tx(&bars[kQFull], L::kTile);
      for (int c = 0; c < NCH; ++c)
        tma_load_4d(sQ + c * kChunkBytes, &p.tm_q, &bars[kQFull], c * 64, h, q0, b);
      misc[2] = 0x10000u;
      auto load_k = [&](int t) -> bool {
        const int s = t & 1;
        if (!mbar_wait(&bars[kKEmpty + s], ((t >> 1) & 1) ^ 1, abort_flag, p.err, wait_tag(1, kKEmpty + s, t))) return false;
        mbar_expect_tx(&bars[kKFull + s], L::kTile);
        for (int c = 0; c < NCH; ++c)
          tma_load_4d(sK + s * L::kTile + c * kChunkBytes, &p.tm_k, &bars[kKFull + s], c * 64, hk,
                      (j_diag - t) * kBK, b);
        misc[2] = 0x20000u | t;
        return true;
      };
      bool ok = load_k(0);
      if (ok && T > 1) ok = load_k(1);
      int kc = 0;
      for (int t = 0; ok && t < T; ++t) {
        const int s = t & 1;
        if (!mbar_wait(&bars[kDecFull + s], (t >> 1) & 1, abort_flag, p.err, wait_tag(1, kDecFull + s, t))) { ok = false; break; }
        const uint32_t keep = misc[5 + s];
        mbar_arrive(&bars[kDecEmpty + s]);
        misc[2] = 0x30000u | t;
        if (keep) {
          const int vs = kc & 1;
          if (!mbar_wait(&bars[kVEmpty + vs], ((kc >> 1) & 1) ^ 1, abort_flag, p.err, wait_tag(1, kVEmpty + vs, kc))) { ok = false; break; }
          mbar_expect_tx(&bars[kVFull + vs], L::kTile);
          for (int c = 0; c < NCH; ++c)
            tma_load_4d(sV + vs * L::kTile + c * kChunkBytes, &p.tm_v, &bars[kVFull + vs], c * 64,
                        hk, (j_diag - t) * kBK, b);
          ++kc;
        }
        if (t + 2 < T && !load_k(t + 2)) { ok = false; break; }
      }
      if (!ok) drain_pause_ns(50000);   // let copies already issued land
    }
  } else if (warp == 5) {
    // ===================== tcgen05 issuer =====================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV), sPa = smem_u32(sP);
      auto issue_qk = [&](int t) -> bool {
        const int s = t & 1;
        if (!mbar_wait(&bars[kKFull + s], (t >> 1) & 1, abort_flag, p.err, wait_tag(2, kKFull + s, t))) return false;
        if (!mbar_wait(&bars[kSEmpty + s], ((t >> 1) & 1) ^ 1, abort_flag, p.err, wait_tag(2, kSEmpty + s, t))) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          const uint64_t a = sdesc_sw128(sQa + off, 16, 1024);
          const uint64_t bd = sdesc_sw128(sKa + s * L::kTile + off, 16, 1024);
          umma_bf16_ss(tmem + s * 128, a, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars[kSFull + s]);
        umma_commit(&bars[kKEmpty + s]);
        misc[3] = 0x20000u | t;
        return true;
      };
      bool ok = mbar_wait(&bars[kQFull], 0, abort_flag, p.err, wait_tag(2, kQFull, 0));
      if (ok) misc[3] = 0x10000u;
      if (ok) ok = issue_qk(0);
      if (ok && T > 1) ok = issue_qk(1);
      int kc = 0;
      for (int t = 0; ok && t < T; ++t) {
        const int s = t & 1;
        if (!mbar_wait(&bars[kDecFull + s], (t >> 1) & 1, abort_flag, p.err, wait_tag(2, kDecFull + s, t))) { ok = false; break; }
        const uint32_t keep = misc[5 + s];
        mbar_arrive(&bars[kDecEmpty + s]);
        if (t + 2 < T && !issue_qk(t + 2)) { ok = false; break; }
        if (keep) {
          const int ps = kc & 1;
          if (!mbar_wait(&bars[kPFull + ps], (kc >> 1) & 1, abort_flag, p.err, wait_tag(2, kPFull + ps, kc))) { ok = false; break; }
          if (!mbar_wait(&bars[kVFull + ps], (kc >> 1) & 1, abort_flag, p.err, wait_tag(2, kVFull + ps, kc))) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t a = sdesc_sw128(sPa + ps * kPBytes + (kk >> 2) * kChunkBytes + (kk & 3) * 32,
                                           16, 1024);
            const uint64_t bd = sdesc_sw128(sVa + ps * L::kTile + kk * 2048, kChunkBytes, 1024);
            umma_bf16_ss(tmem_o, a, bd, idesc_pv, (kc > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars[kPEmpty + ps]);
          umma_commit(&bars[kVEmpty + ps]);
          misc[3] = 0x40000u | t;
          ++kc;
        }
      }
      // make sure every MMA issued above has finished before TMEM is freed
      umma_commit(&bars[kMmaDone]);
      mbar_wait(&bars[kMmaDone], 0, abort_flag, p.err, wait_tag(2, kMmaDone, 0));
    }
  } else {
    // ===================== softmax warpgroup =====================
    const int r = tid;                       // row within the block = TMEM lane
    const int q = q0 + r;
    const bool valid = q < p.N;
    const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
    const float thr2 = p.log2_tau - log2f(static_cast<float>(q + 1));   // log2(tau / L_q)
    float m2 = -INFINITY;                    // reference maximum, log2 units
    float l = 0.0f;                          // sum of 2^(s log2e - m2) over retained keys
    int kc = 0;
    uint32_t mask_word = 0;
    int kept_tiles = 0;
    const uint32_t sPa = smem_u32(sP);
    const int mask_base = ((b * p.Hq + h) * p.nQB + i) * p.mask_words;
    if (tid == 0 && p.keep_mask) {
      for (int w = j_diag / 32 + 1; w < p.mask_words; ++w) p.keep_mask[mask_base + w] = 0u;
    }

    for (int t = 0; t < T; ++t) {
      const int j = j_diag - t;
      const int s = t & 1;
      uint32_t sr[4][32];
      // tcgen05.ld is warp-collective: load only if every lane's wait succeeded
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[kSFull + s], (t >> 1) & 1, abort_flag, p.err, wait_tag(0, kSFull + s, t)));
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(tmem + lane_addr + s * 128 + c * 32, sr[c]);
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
      tc_fence_before();
      mbar_arrive(&bars[kSEmpty + s]);
      if (tid == 0) misc[4] = (ok ? 0x10000u : 0x90000u) | t;

      // causal mask: key k = j*128 + c is legal iff k <= q
      const int lim = q - j * kBK;           // largest legal column index
      const bool has_key = valid && lim >= 0;
      float rmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const float v = (c * 32 + x <= lim) ? __uint_as_float(sr[c][x]) : -INFINITY;
          sr[c][x] = __float_as_uint(v);
          rmax = fmaxf(rmax, v);
        }
      const float rmax2 = rmax * kLog2e;
      // retain iff the row's largest contribution ratio reaches tau / L_q;
      // an empty retained set (l = 0) always retains
      const bool vote = has_key && (l == 0.0f || rmax2 - (m2 + lg2_approx(l)) >= thr2);
      const bool keep = bar_or(1, kBQ, vote);
      if (tid == 0) misc[4] = 0x20000u | t;
      // every softmax thread must leave at the same tile: OR the flag through a barrier
      if (bar_or(1, kBQ, *abort_flag != 0)) break;

      if (tid == 0) {
        if (mbar_wait(&bars[kDecEmpty + s], ((t >> 1) & 1) ^ 1, abort_flag, p.err, wait_tag(0, kDecEmpty + s, t))) {
          misc[5 + s] = keep ? 1u : 0u;
          mbar_arrive(&bars[kDecFull + s]);
          misc[4] = 0x30000u | t;
        }
        if (keep) {
          mask_word |= 1u << (j & 31);
          ++kept_tiles;
        }
        if ((j & 31) == 0) {
          if (p.keep_mask) p.keep_mask[mask_base + (j >> 5)] = mask_word;
          mask_word = 0;
        }
      }
      if (!keep) continue;

      // ---- online-softmax update for a retained tile
      float new_m2 = m2;
      bool rescale = false;
      if (has_key) {
        if (l == 0.0f) {
          new_m2 = rmax2;
        } else if (rmax2 > m2 + kRescaleThreshold) {
          new_m2 = rmax2;
          rescale = true;
        }
      }
      const float alpha = rescale ? ex2_approx(m2 - new_m2) : 1.0f;
      l *= alpha;
      // O rows of this warp are rescaled together (TMEM access is warp-collective)
      if (kc > 0 && __any_sync(0xffffffffu, rescale)) {
        {
          // O holds PV of earlier retained tiles: wait for the last one
          mbar_wait(&bars[kPEmpty + ((kc - 1) & 1)], ((kc - 1) >> 1) & 1, abort_flag, p.err, wait_tag(0, kPEmpty + ((kc - 1) & 1), kc));
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem_o + lane_addr + c * 32, o);
            tmem_ld_wait(o);
            reg_fence(o);
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
            tmem_st32(tmem_o + lane_addr + c * 32, o);
          }
          tmem_st_wait();
        }
      }
      m2 = new_m2;

      // P buffer kc & 1 is free once PV(kc - 2) has completed
      mbar_wait(&bars[kPEmpty + (kc & 1)], ((kc >> 1) & 1) ^ 1, abort_flag, p.err, wait_tag(0, kPEmpty + (kc & 1), kc));
      const float neg_m2 = has_key ? -m2 : 0.0f;
      float psum = 0.0f;
      const uint32_t prow = sPa + (kc & 1) * kPBytes + r * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pk[16];
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          float a = has_key ? ex2_approx(fmaf(__uint_as_float(sr[c][x]), kLog2e, neg_m2)) : 0.0f;
          float bb = has_key ? ex2_approx(fmaf(__uint_as_float(sr[c][x + 1]), kLog2e, neg_m2)) : 0.0f;
          psum += a + bb;
          pk[x >> 1] = pack_bf16x2(a, bb);
        }
        // keys [32c, 32c + 32): chunk c / 2, 16-byte units u = (c & 1) * 4 + 0..3
        const uint32_t chunk = prow + (c >> 1) * kChunkBytes;
#pragma unroll
        for (int u4 = 0; u4 < 4; ++u4) {
          const uint32_t u = (c & 1) * 4 + u4;
          st_shared_v4(chunk + ((u ^ (r & 7)) << 4), pk[u4 * 4 + 0], pk[u4 * 4 + 1], pk[u4 * 4 + 2],
                       pk[u4 * 4 + 3]);
        }
      }
      l += psum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bars[kPFull + (kc & 1)]);
      ++kc;
    }

    // ---- epilogue: O = acc / l (bf16), z = (m2 + log2 l) ln 2, mask, stats
    if (!*abort_flag) {
      if (kc > 0) mbar_wait(&bars[kPEmpty + ((kc - 1) & 1)], ((kc - 1) >> 1) & 1, abort_flag, p.err, wait_tag(0, kPEmpty + ((kc - 1) & 1), kc));
      tc_fence_after();
      const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + b * p.o_sb +
                            static_cast<int64_t>(q) * p.o_sn + h * p.o_sh;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem_o + lane_addr + c * 32, o);
        tmem_ld_wait(o);
        reg_fence(o);
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2)
            pk[x >> 1] = pack_bf16x2(__uint_as_float(o[x]) * inv_l, __uint_as_float(o[x + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
      if (valid) p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.N + q] = (m2 + log2f(l)) * kLn2;
      if (tid == 0 && p.stats) {
        const int nvalid = last_row - q0 + 1;
        atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[0]), static_cast<unsigned long long>(T));
        atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[1]),
                  static_cast<unsigned long long>(kept_tiles));
        atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[2]),
                  static_cast<unsigned long long>(kept_tiles) * kBK * nvalid);
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

}  // namespace

size_t fwd_tc_smem_bytes(int head_dim) {
  return head_dim == 64 ? Layout<64>::kAlloc : Layout<128>::kAlloc;
}

cudaError_t launch_fwd_tc(const FwdTcParams& p, int head_dim, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hq * p.nQB;
  if (grid == 0) return cudaSuccess;
  if (head_dim == 128) {
    const int smem = Layout<128>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(mala_fwd_tc_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    mala_fwd_tc_kernel<128><<<grid, kThreads, smem, stream>>>(p);
  } else {
    const int smem = Layout<64>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(mala_fwd_tc_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    mala_fwd_tc_kernel<64><<<grid, kThreads, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace mala
