// MALA forward (Algorithm 1, "Online Sparse Softmax") on sm_100a tensor cores.
//
// One CTA owns one query block I_i of 128 rows of one (batch, query head),
// or of one (packed sequence, query head). Query row q sits at position
// q + N_k - N_q (bottom-right alignment; N_q = N_k for training). Key blocks
// are visited in descending order from the diagonal (Appendix A.1, "Fused
// forward execution"); every legal tile is scored, and only a retained tile
// loads V and runs the online-softmax update and PV.
//
// Warp roles (320 threads):
//   warps 0-7  softmax, two warpgroups: warps 0-3 take key columns [0, 64)
//              of every tile, warps 4-7 columns [64, 128); (warp, lane) owns
//              TMEM lane r = 32 (warp % 4) + lane = query row r. Per tile the
//              groups exchange their row maxima (and the previous retained
//              tile's row sums) through shared memory, both evaluate the same
//              skip test, and for a retained tile each writes its half of
//              P = exp(S - m) as packed bf16 over S in TMEM.
//   warp 8     TMA producer, polling: Q once, K as far ahead as the ring
//              allows (independent of the votes), V only for retained tiles.
//   warp 9     tcgen05 issuer: S_t = Q K_t^T into one of three TMEM S buffers
//              (up to three tiles ahead of the softmax), O += P V_t for retained tiles
//              with P read straight from TMEM.
// TMEM: S buffers at cols [0,128), [128,256), [256,384); O = [384, 384 + D).
//
// Group-joint voting (optional): the G CTAs that hold the same query block
// of the G query heads of one KV head run as one thread-block cluster. After
// its own vote, each CTA writes it into every peer's shared memory and
// arrives on the peer's vote barrier; each then takes the OR of the G votes,
// so the group keeps or skips a tile together (the heads' rows act as the
// rows of one block). Votes alternate between two slots by tile parity.
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
constexpr int kThreads = 320;
constexpr int kNS = 3;                          // TMEM S buffers
constexpr uint32_t kChunkBytes = 128 * 128;     // 128 rows x 64 bf16 (one swizzle column)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;       // log2 units

template <int D>
struct Cfg {
  static constexpr int NK = D == 128 ? 3 : 4;   // K ring stages
  static constexpr int NV = D == 128 ? 2 : 4;   // V ring stages
};

enum Bar {
  kQFull = 0,
  kKFull = 1,            // 4 (ring, up to 4 stages)
  kKEmpty = 5,           // 4
  kVFull = 9,            // 4
  kVEmpty = 13,          // 4
  kSFull = 17,           // 3 (per S buffer)
  kSDone = 20,           // 3 (per S buffer, one arrival per softmax warp): both softmax groups are done
                         // with the buffer's tile (P written if retained, S read if skipped);
                         // one phase per use of the buffer, so its parity cannot alias
  kTileDone = 23,        // 3 (per S buffer, MMA commit once per tile after its PV, or
                         // right away for a skipped tile): every MMA issued up to
                         // that tile has completed; one phase per use of the buffer
  kDecFull = 26,         // 2
  kDecEmpty = 28,        // 2 (producer + MMA)
  kMmaDone = 30,
  kNumBars = 31
};

template <int D>
struct Layout {
  static constexpr uint32_t kTile = kBQ * D * 2;   // Q / K / V tile bytes
  static constexpr uint32_t kQ = 0;
  static constexpr uint32_t kK = kQ + kTile;
  static constexpr uint32_t kV = kK + Cfg<D>::NK * kTile;
  static constexpr uint32_t kX = kV + Cfg<D>::NV * kTile;          // exchange area
  static constexpr uint32_t kXMax = kX;                             // [2 parity][2 groups][128] float
  static constexpr uint32_t kXSum = kX + 2 * 2 * 128 * 4;           // [2 parity][2 groups][128] float
  static constexpr uint32_t kBars = kXSum + 2 * 2 * 128 * 4;
  static constexpr uint32_t kMisc = kBars + kNumBars * 8;
  static constexpr uint32_t kCVote = kMisc + 64;                    // [2 parity][8 ranks] uint32 group votes
  static constexpr uint32_t kCBars = kCVote + 2 * 8 * 4;            // 2 vote barriers (G arrivals each)
  static constexpr uint32_t kEnd = kCBars + 2 * 8;
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
static_assert(Layout<64>::kAlloc <= 232448 && Layout<128>::kAlloc <= 232448, "forward CTA exceeds shared memory");

template <int D>
__global__ void __launch_bounds__(kThreads, 1) mala_fwd_tc_kernel(const __grid_constant__ FwdTcParams p) {
  using L = Layout<D>;
  constexpr int NK = Cfg<D>::NK;
  constexpr int NV = Cfg<D>::NV;
  constexpr int NCH = D / 64;       // 128-byte chunks per row of Q/K/V
  constexpr int KSTEPS = D / 16;    // QK^T k-steps
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sK = smem + L::kK;
  uint8_t* sV = smem + L::kV;
  float* xmax = reinterpret_cast<float*>(smem + L::kXMax);
  float* xsum = reinterpret_cast<float*>(smem + L::kXSum);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  volatile uint32_t* misc = reinterpret_cast<volatile uint32_t*>(smem + L::kMisc);
  volatile uint32_t* cvote = reinterpret_cast<volatile uint32_t*>(smem + L::kCVote);
  uint64_t* cbars = reinterpret_cast<uint64_t*>(smem + L::kCBars);
  // misc[0] TMEM base, misc[1] abort flag, misc[2..4] progress markers of the
  // producer / MMA / softmax roles (kept for timeout diagnosis), misc[5..6]
  // decisions of tiles t & 1
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- work item. b is the batch index, or the sequence of a packed call;
  // qrow0 / krow0 are the sequence's first query / key row and tb its batch
  // coordinate in the tensor maps.
  // Fixed lengths: the grid runs band by band, a band being the G query
  // heads of one KV head of one batch entry (p.head_order lists them
  // together) over all query blocks, blocks with more key tiles first and
  // the G heads of a block side by side. The CTAs resident at any time then
  // stream the K / V tiles of one or two KV heads, which stay in L2, and the
  // heavy-first order inside each band keeps the tail of the grid light.
  int i, b, h, Nq, Nk, qrow0, krow0, tb;
  if (p.seq.n == 0) {
    const int x = static_cast<int>(blockIdx.x);
    const int HQB = p.Hq * p.nQB;
    const int GQB = p.group * p.nQB;
    b = x / HQB;
    const int band = (x % HQB) / GQB;
    const int r = (x % HQB) % GQB;
    i = p.nQB - 1 - r / p.group;
    h = p.head_order[band * p.group + r % p.group];
    Nq = p.N;
    Nk = p.Nk;
    qrow0 = krow0 = 0;
    tb = b;
  } else {
    const int SH = p.seq.n * p.Hq;
    i = p.nQB - 1 - static_cast<int>(blockIdx.x) / SH;
    const int sh = static_cast<int>(blockIdx.x) % SH;
    b = sh / p.Hq;
    h = sh % p.Hq;
    qrow0 = p.seq.q0[b];
    krow0 = p.seq.k0[b];
    Nq = p.seq.q0[b + 1] - qrow0;
    Nk = p.seq.k0[b + 1] - krow0;
    tb = 0;
    if (i * kBQ >= Nq) return;      // a shorter sequence: no query block i (uniform exit)
  }
  const int q_off = Nk - Nq;        // bottom-right alignment: query row q sits at position q + q_off
  const int hk = p.kv_of_q[h];
  const int q0 = i * kBQ;
  const int last_row = min(q0 + kBQ - 1, Nq - 1);
  const int j_diag = min((last_row + q_off) / kBK, (Nk + kBK - 1) / kBK - 1);
  const int T = j_diag + 1;         // tile t visits key block j = j_diag - t

  if (tid == 0) {
    for (int x = 0; x < kNumBars; ++x) {
      uint32_t cnt = 1;
      if (x >= kSDone && x < kSDone + kNS) cnt = 8;   // one per softmax warp
      if (x == kDecEmpty || x == kDecEmpty + 1) cnt = 2;
      mbar_init(&bars[x], cnt);
    }
    if (p.group_vote) {
      mbar_init(&cbars[0], p.group);
      mbar_init(&cbars[1], p.group);
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
  // every CTA of the cluster has initialised its vote barriers before any
  // peer arrives on them
  if (p.group_vote) cluster_sync_all();
  const uint32_t crank = p.group_vote ? cluster_ctarank() : 0u;
  const uint32_t tmem = misc[0];
  const uint32_t tmem_o = tmem + kNS * 128;

  if (warp == 8) {
    // ===================== TMA producer (polling) =====================
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      mbar_expect_tx(&bars[kQFull], L::kTile);
      for (int c = 0; c < NCH; ++c)
        tma_load_4d(sQ + c * kChunkBytes, &p.tm_q, &bars[kQFull], c * 64, h, qrow0 + q0, tb);
      misc[2] = 0x10000u;
      int next_k = 0, next_d = 0, v_issued = 0, v_req = 0;
      int vq[8];                         // retained tiles waiting for their V load
      uint64_t idle_since = global_timer_ns();
      bool ok = true;
      while (ok && (next_k < T || next_d < T || v_issued < v_req)) {
        bool progress = false;
        if (next_k < T) {
          const int s = next_k % NK;
          if (mbar_test(&bars[kKEmpty + s], ((next_k / NK) & 1) ^ 1)) {
            mbar_expect_tx(&bars[kKFull + s], L::kTile);
            for (int c = 0; c < NCH; ++c)
              tma_load_4d(sK + s * L::kTile + c * kChunkBytes, &p.tm_k, &bars[kKFull + s], c * 64, hk,
                          krow0 + (j_diag - next_k) * kBK, tb);
            ++next_k;
            progress = true;
          }
        }
        if (next_d < T && v_req - v_issued < 8) {
          const int s = next_d & 1;
          if (mbar_test(&bars[kDecFull + s], (next_d >> 1) & 1)) {
            const uint32_t keep = misc[5 + s];
            mbar_arrive(&bars[kDecEmpty + s]);
            if (keep) vq[v_req++ & 7] = next_d;
            ++next_d;
            progress = true;
          }
        }
        if (v_issued < v_req) {
          const int s = v_issued % NV;
          if (mbar_test(&bars[kVEmpty + s], ((v_issued / NV) & 1) ^ 1)) {
            const int t = vq[v_issued & 7];
            mbar_expect_tx(&bars[kVFull + s], L::kTile);
            for (int c = 0; c < NCH; ++c)
              tma_load_4d(sV + s * L::kTile + c * kChunkBytes, &p.tm_v, &bars[kVFull + s], c * 64, hk,
                          krow0 + (j_diag - t) * kBK, tb);
            ++v_issued;
            progress = true;
          }
        }
        misc[2] = (static_cast<uint32_t>(next_k) << 20) | (static_cast<uint32_t>(next_d) << 10) |
                  static_cast<uint32_t>(v_issued & 0x3ff);
        if (progress) {
          idle_since = global_timer_ns();
        } else if (*abort_flag) {
          ok = false;
        } else if (global_timer_ns() - idle_since > p.wait_ns) {
          *abort_flag = 1;
          if (atomicCAS(p.err, 0, kErrTimeout) == 0) {
            p.err[1] = wait_tag(1, 0xff, next_d);
            p.err[2] = static_cast<int>(blockIdx.x);
            for (int x = 0; x < 3; ++x) p.err[4 + x] = misc[2 + x];
          }
          ok = false;
        }
      }
      if (!ok) drain_pause_ns(50000);   // let copies already issued land
    }
  } else if (warp == 9) {
    // ===================== tcgen05 issuer =====================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, false, true);
      const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
      auto issue_qk = [&](int t) -> bool {
        const int ks = t % NK;
        if (!mbar_wait(&bars[kKFull + ks], (t / NK) & 1, abort_flag, p.err, wait_tag(2, kKFull + ks, t), p.wait_ns)) return false;
        tc_fence_after();
        const uint32_t sb = tmem + (t % kNS) * 128;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
          umma_bf16_ss(sb, sdesc_sw128(sQa + off, 16, 1024), sdesc_sw128(sKa + ks * L::kTile + off, 16, 1024),
                       idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars[kSFull + (t % kNS)]);
        umma_commit(&bars[kKEmpty + ks]);
        misc[3] = 0x20000u | t;
        return true;
      };
      bool ok = mbar_wait(&bars[kQFull], 0, abort_flag, p.err, wait_tag(2, kQFull, 0), p.wait_ns);
      for (int t = 0; ok && t < kNS && t < T; ++t) ok = issue_qk(t);
      int kc = 0;
      for (int t = 0; ok && t < T; ++t) {
        const int ds = t & 1;
        if (!mbar_wait(&bars[kDecFull + ds], (t >> 1) & 1, abort_flag, p.err, wait_tag(2, kDecFull + ds, t), p.wait_ns)) { ok = false; break; }
        const uint32_t keep = misc[5 + ds];
        mbar_arrive(&bars[kDecEmpty + ds]);
        if (keep) {
          const int vs = kc % NV;
          if (!mbar_wait(&bars[kSDone + t % kNS], (t / kNS) & 1, abort_flag, p.err, wait_tag(2, kSDone + t % kNS, t), p.wait_ns)) { ok = false; break; }
          if (!mbar_wait(&bars[kVFull + vs], (kc / NV) & 1, abort_flag, p.err, wait_tag(2, kVFull + vs, kc), p.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t pb = tmem + (t % kNS) * 128;   // P as packed bf16 pairs over S
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16_ts(tmem_o, pb + kk * 8, sdesc_sw128(sVa + vs * L::kTile + kk * 2048, kChunkBytes, 1024),
                         idesc_pv, (kc > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&bars[kVEmpty + vs]);
          misc[3] = 0x40000u | t;
          ++kc;
        }
        umma_commit(&bars[kTileDone + t % kNS]);
        // S buffer t % 3 takes tile t + 3 once tile t's contents are consumed:
        // both softmax groups are done with it and every MMA reading it (the
        // PV of a retained tile) has completed
        if (t + kNS < T) {
          if (!keep &&
              !mbar_wait(&bars[kSDone + t % kNS], (t / kNS) & 1, abort_flag, p.err, wait_tag(2, kSDone + t % kNS, t), p.wait_ns)) { ok = false; break; }
          if (!mbar_wait(&bars[kTileDone + t % kNS], (t / kNS) & 1, abort_flag, p.err, wait_tag(2, kTileDone + t % kNS, t), p.wait_ns)) { ok = false; break; }
          if (!issue_qk(t + kNS)) { ok = false; break; }
        }
      }
      // every MMA issued above must have finished before TMEM is freed:
      // wait for that regardless of the abort flag (MMAs always complete),
      // bounded in time
      umma_commit(&bars[kMmaDone]);
      mbar_wait_drain(&bars[kMmaDone], 0);
    }
  } else {
    // ===================== softmax warpgroups =====================
    const int r = ((warp & 3) << 5) | lane;     // query row within the block = TMEM lane
    const int g = warp >> 2;                    // column group: key columns [64g, 64g + 64)
    const int c0 = g * 64;
    const int q = q0 + r;
    const bool valid = q < Nq;
    const int qa = q + q_off;                   // the row's position: keys k <= qa are legal
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float thr2 = p.log2_tau - log2f(static_cast<float>(qa + 1));   // log2(tau / L_q)
    float m2 = -INFINITY;                    // reference maximum, log2 units
    float l = 0.0f;                          // sum of 2^(s log2e - m2) over retained keys
    int kc = 0;
    bool prev_kept = false;
    uint32_t mask_word = 0;
    int kept_tiles = 0;
    int pending = -1;                        // group voting: tile whose exchange wait is deferred
    const int mask_base = (p.seq.n == 0 ? (b * p.Hq + h) * p.nQB + i
                                        : h * p.seq.qb0[p.seq.n] + p.seq.qb0[b] + i) * p.mask_words;
    if (tid == 0 && p.keep_mask) {
      for (int w = j_diag / 32 + 1; w < p.mask_words; ++w) p.keep_mask[mask_base + w] = 0u;
    }

    for (int t = 0; t < T; ++t) {
      const int j = j_diag - t;
      const int sb = t % kNS;
      uint32_t sr[2][32];
      // tcgen05.ld is warp-collective: load only if every lane's wait succeeded
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[kSFull + sb], (t / kNS) & 1, abort_flag, p.err,
                                                        wait_tag(0, kSFull + sb, t), p.wait_ns));
      if (ok) {
        tc_fence_after();
        tmem_ld32(tmem + sb * 128 + lane_addr + c0, sr[0]);
        tmem_ld32(tmem + sb * 128 + lane_addr + c0 + 32, sr[1]);
        tmem_ld_wait(sr[0]);
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) sr[0][x] = sr[1][x] = 0u;
      }
      reg_fence(sr[0]);
      reg_fence(sr[1]);

      // causal mask: key k = j*128 + c is legal iff k <= qa; this group's
      // columns are c = c0 + x. Only tiles whose last key lies beyond the
      // block's first row position can hold illegal keys (the diagonal
      // tile, and the one before it when q_off is not a multiple of 128).
      const bool has_key = valid && qa >= j * kBK;
      if (j * kBK + kBK - 1 > q0 + q_off) {
        const int lim = qa - j * kBK - c0;    // largest legal x
#pragma unroll
        for (int x = 0; x < 64; ++x)
          if (x > lim) sr[x >> 5][x & 31] = __float_as_uint(-INFINITY);
      }
      // row maximum of this half: eight independent chains, then a tree
      float mx[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mx[e] = -INFINITY;
#pragma unroll
      for (int x = 0; x < 64; x += 2)
        mx[(x >> 1) & 7] = max3(mx[(x >> 1) & 7], __uint_as_float(sr[x >> 5][x & 31]),
                                __uint_as_float(sr[x >> 5][(x + 1) & 31]));
      const float pmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const int par = t & 1;
      xmax[(par * 2 + g) * 128 + r] = pmax;
      // exchange barrier; the OR of the abort flag keeps both groups' exits in step
      if (bar_or(1, 256, *abort_flag != 0)) break;
      if (tid == 0) misc[4] = 0x10000u | t;
      if (prev_kept) l += xsum[((par ^ 1) * 2 + 0) * 128 + r] + xsum[((par ^ 1) * 2 + 1) * 128 + r];
      const float rmax = fmaxf(xmax[(par * 2 + 0) * 128 + r], xmax[(par * 2 + 1) * 128 + r]);
      const float rmax2 = rmax * kLog2e;
      // retain iff the row's largest contribution ratio reaches tau / L_q;
      // an empty retained set (l = 0) always retains
      const bool vote = has_key && (l == 0.0f || rmax2 - (m2 + lg2_approx(l)) >= thr2);
      bool keep = bar_or(1, 256, vote);
      if (p.group_vote) {
        // group-joint voting. A CTA sends its tile t vote only after its
        // own wait for tile t - 1 has completed, so no arrival for tile
        // t + 2 can land in the phase that still collects tile t, and no
        // peer rewrites a vote slot before this CTA has read it. When this
        // CTA's own vote already retains the tile, the OR is known and the
        // wait moves to the next tile's exchange, off the critical path.
        // The deferred wait only orders this CTA's sends, so only warp 0
        // (whose lanes send) takes it; every thread that reads the vote
        // slots of a tile has done so before the next tile's vote barrier,
        // which precedes the next send.
        if (pending >= 0) {
          if (warp == 0)
            mbar_wait<true>(&cbars[pending & 1], (pending >> 1) & 1, abort_flag, p.err,
                            wait_tag(0, 0x40 + (pending & 1), pending), p.wait_ns);
          pending = -1;
        }
        if (tid < p.group) {          // one lane per peer, in parallel
          const uint32_t slot = smem_u32(const_cast<uint32_t*>(&cvote[par * 8 + crank]));
          st_cluster_u32(mapa_shared(slot, tid), keep ? 1u : 0u);
          mbar_arrive_cluster(mapa_shared(smem_u32(&cbars[par]), tid));
        }
        if (keep) {
          pending = t;
        } else if (mbar_wait<true>(&cbars[par], (t >> 1) & 1, abort_flag, p.err, wait_tag(0, 0x40 + par, t), p.wait_ns)) {
          bool any = false;
          for (int rr = 0; rr < p.group; ++rr) any = any || cvote[par * 8 + rr] != 0u;
          keep = any;
        }
      }

      if (tid == 0) {
        if (mbar_wait(&bars[kDecEmpty + par], ((t >> 1) & 1) ^ 1, abort_flag, p.err, wait_tag(0, kDecEmpty + par, t), p.wait_ns)) {
          misc[5 + par] = keep ? 1u : 0u;
          mbar_arrive(&bars[kDecFull + par]);
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
      if (!keep) {
        tc_fence_before();
        warp_arrive(&bars[kSDone + sb]);
        prev_kept = false;
        continue;
      }

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
      // O rows of this warp are rescaled together (TMEM access is warp-collective);
      // each group rescales its half of the D columns
      if (kc > 0 && __any_sync(0xffffffffu, rescale)) {
        // O holds the PVs of earlier retained tiles: wait until every MMA up
        // to the previous tile has completed (t >= 1 since kc > 0)
        const int tp = t - 1;
        mbar_wait(&bars[kTileDone + tp % kNS], (tp / kNS) & 1, abort_flag, p.err, wait_tag(0, kTileDone + tp % kNS, tp), p.wait_ns);
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t o[32];
          const uint32_t oaddr = tmem_o + lane_addr + g * (D / 2) + c * 32;
          tmem_ld32(oaddr, o);
          tmem_ld_wait(o);
          reg_fence(o);
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] = __float_as_uint(__uint_as_float(o[x]) * alpha);
          tmem_st32(oaddr, o);
        }
        tmem_st_wait();
      }
      m2 = new_m2;

      // P = 2^(s log2e - m2) as packed bf16 pairs over this tile's S buffer:
      // key column c goes to packed column c / 2, so this group writes packed
      // columns [32g, 32g + 32); both groups finished reading S before the vote
      // rows without a legal key (padding) get P = 0 through m2 = +inf
      const float neg_m2 = has_key ? -m2 : -INFINITY;
      float psum[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};   // four pairs of partial sums
      uint32_t pk[32];
#pragma unroll
      for (int x = 0; x < 64; x += 2) {
        float ea, eb;
        fma2(ea, eb, __uint_as_float(sr[x >> 5][x & 31]), __uint_as_float(sr[x >> 5][(x + 1) & 31]), kLog2e, kLog2e,
             neg_m2, neg_m2);
        const float a = ex2_approx(ea);
        const float bb = ex2_approx(eb);
        const int q2 = 2 * ((x >> 1) & 3);
        add2(psum[q2], psum[q2 + 1], psum[q2], psum[q2 + 1], a, bb);
        pk[x >> 1] = pack_bf16x2(a, bb);
      }
      const float ps = ((psum[0] + psum[1]) + (psum[2] + psum[3])) + ((psum[4] + psum[5]) + (psum[6] + psum[7]));
      tmem_st16(tmem + sb * 128 + lane_addr + g * 32, &pk[0]);
      tmem_st16(tmem + sb * 128 + lane_addr + g * 32 + 16, &pk[16]);
      xsum[(par * 2 + g) * 128 + r] = ps;
      tmem_st_wait();
      tc_fence_before();
      warp_arrive(&bars[kSDone + sb]);
      prev_kept = true;
      ++kc;
    }

    // ---- epilogue: O = acc / l (bf16), z = (m2 + log2 l) ln 2, mask, stats
    const bool aborted = bar_or(1, 256, *abort_flag != 0);   // also publishes the last sums
    if (!aborted) {
      if (prev_kept) l += xsum[(((T - 1) & 1) * 2 + 0) * 128 + r] + xsum[(((T - 1) & 1) * 2 + 1) * 128 + r];
      if (kc > 0)
        mbar_wait(&bars[kTileDone + (T - 1) % kNS], ((T - 1) / kNS) & 1, abort_flag, p.err,
                  wait_tag(0, kTileDone + (T - 1) % kNS, T - 1), p.wait_ns);
      tc_fence_after();
      const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) + static_cast<int64_t>(tb) * p.o_sb +
                            static_cast<int64_t>(qrow0 + q) * p.o_sn + h * p.o_sh;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t o[32];
        const int col = g * (D / 2) + c * 32;
        tmem_ld32(tmem_o + lane_addr + col, o);
        tmem_ld_wait(o);
        reg_fence(o);
        if (valid) {
          uint32_t pko[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2)
            pko[x >> 1] = pack_bf16x2(__uint_as_float(o[x]) * inv_l, __uint_as_float(o[x + 1]) * inv_l);
          uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
          for (int u = 0; u < 4; ++u) dst[u] = make_uint4(pko[4 * u], pko[4 * u + 1], pko[4 * u + 2], pko[4 * u + 3]);
        }
      }
      if (valid && g == 0) {
        // [B, H_q, N_q], or [H_q, total_q] for packed sequences
        const int64_t li = p.seq.n == 0 ? (static_cast<int64_t>(b) * p.Hq + h) * p.N + q
                                        : static_cast<int64_t>(h) * p.seq.q0[p.seq.n] + qrow0 + q;
        p.lse[li] = (m2 + log2f(l)) * kLn2;
      }
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
  // after a timeout, copies issued before the waits gave up land before the
  // CTA's shared memory is released
  if (tid == 0 && *abort_flag) drain_pause_ns(50000);
  // no CTA leaves while a peer may still write to its shared memory
  if (p.group_vote) cluster_sync_all();
}

}  // namespace

size_t fwd_tc_smem_bytes(int head_dim) {
  return head_dim == 64 ? Layout<64>::kAlloc : Layout<128>::kAlloc;
}

// Group-joint voting: clusters of G consecutive CTAs, which the work-item
// order makes the G query heads of one KV head on the same query block
// (fixed lengths; packed sequences list a block's heads side by side too).
template <int D>
cudaError_t launch_fwd_tc_clustered(const FwdTcParams& p, unsigned grid, int smem, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(p.group);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mala_fwd_tc_kernel<D>, p);
}

cudaError_t launch_fwd_tc(const FwdTcParams& p, int head_dim, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hq * p.nQB;
  if (grid == 0) return cudaSuccess;
  if (p.group_vote && (p.group < 1 || p.group > 8 || p.Hq % p.group != 0)) return cudaErrorInvalidValue;
  if (head_dim == 128) {
    const int smem = Layout<128>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(mala_fwd_tc_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (p.group_vote) return launch_fwd_tc_clustered<128>(p, grid, smem, stream);
    mala_fwd_tc_kernel<128><<<grid, kThreads, smem, stream>>>(p);
  } else {
    const int smem = Layout<64>::kAlloc;
    cudaError_t e = cudaFuncSetAttribute(mala_fwd_tc_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    if (p.group_vote) return launch_fwd_tc_clustered<64>(p, grid, smem, stream);
    mala_fwd_tc_kernel<64><<<grid, kThreads, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace mala
