/*
 * mala.h - C ABI of the MassAlloc Attention (MALA) operator library for B200.
 *
 * Source of the operation: "MassAlloc Attention: Let Attention Allocate Its
 * Own Compute", method section. Run-in headings cited below:
 *   "Setup"                       problem statement: Q [N_q, d], K/V [N_k, d],
 *                                 1/sqrt(d) folded into Q, natural exp/log,
 *                                 query blocks I_i of B_q rows, key blocks J_j
 *                                 of B_k rows, L_q = |C_q|, threshold tau/L_q;
 *                                 L_q = q + 1 in training, L_0 = N_k in
 *                                 single-token decoding.
 *   "Online Sparse Softmax"       forward skip test (Algorithm 1).
 *   "Offline Sparse Probability"  backward skip test (Algorithm 2).
 *   Appendix A.1                  fused forward / backward / decoding
 *                                 execution and traversal orders.
 * Tensor layout follows the FlashAttention interface on the attention
 * tutorial page ("Hardware paths and kernel contracts"): Q, O, dQ, dO are
 * [B, N_q, H_q, d]; K, V, dK, dV are [B, N_k, H_kv, d]; the last dimension
 * is contiguous and the other strides are passed in elements.
 *
 * Conventions common to every entry point
 *   - All tensor pointers are caller-owned DEVICE memory. The library never
 *     allocates or frees memory; scratch space is the caller's `workspace`
 *     buffer of at least mala_*_workspace_size() bytes (NULL allowed when
 *     that size is 0).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Arguments are checked on the host before anything is
 *     launched; on a non-zero return nothing was launched.
 *   - Scale: the caller folds 1/sqrt(d) into Q; gradients are with respect
 *     to the scaled Q.
 *   - tau >= 0. tau = 0 skips nothing (FullAttn); tau = +inf retains only
 *     the first legal tile of every query block / split.
 *   - Query head h reads key/value head q_to_kv[h] (a HOST array of H_q
 *     entries, copied during the call); NULL means h / (H_q / H_kv).
 *   - keep masks are uint32 bit sets: bit (j % 32) of word j / 32 of the
 *     row for (b, h, i) is set iff tile (i, j) was retained.
 *   - Kernels never trap. A device-side bounded wait that gives up records
 *     MALA_ERR_TIMEOUT, which mala_check_device_error() reports; the wait
 *     limit is 2 s unless the call sets wait_limit_ns.
 */
#ifndef MALA_H_
#define MALA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MALA_API __attribute__((visibility("default")))
#else
#define MALA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
enum {
  MALA_OK = 0,
  MALA_ERR_INVALID_ARG = 1,   /* NULL pointer, bad size/stride/alignment, tau < 0 or NaN */
  MALA_ERR_UNSUPPORTED = 2,   /* valid request this build has no kernel for */
  MALA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
  MALA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  MALA_ERR_TIMEOUT = 5        /* a device-side bounded wait gave up */
};

/* element types of Q, K, V, O (and dO, dQ, dK, dV); MALA_FP8_E4M3 only for
 * the K / V cache of mala_decode (kv_dtype) */
enum { MALA_BF16 = 0, MALA_FP32 = 1, MALA_FP8_E4M3 = 2 };

/* masking mode of mala_fwd */
enum {
  MALA_CAUSAL = 0,  /* N_q <= N_k, bottom-right aligned: query q sits at position
                       p_q = q + N_k - N_q, key k is legal iff k <= p_q, L_q = p_q + 1
                       (N_q = N_k: L_q = q + 1; a chunk of queries appended to a
                       context of N_k - N_q keys otherwise) */
  MALA_DECODE = 1   /* reserved for mala_fwd: single-token decoding uses mala_decode */
};

/*
 * Forward / prefill: Algorithm 1 ("Online Sparse Softmax", Appendix A.1
 * "Fused forward execution"). For every query block, every legal key tile is
 * scored (S_ij = Q_i K_j^T), key blocks visited in descending order from the
 * diagonal. A tile is skipped iff, for every valid row q with a legal key in
 * it, max_k s_qk - (m_q + log l_q) < log tau - log L_q; a row whose retained
 * set is empty always retains. Only retained tiles load V and run the
 * online-softmax update and PV.
 *
 * Outputs: o [B, N_q, H_q, d] (same dtype as q) = softmax renormalised over
 * the retained tiles; lse [B, H_q, N_q] fp32 = z_q = m_q + log l_q (natural
 * log), the state the backward pass consumes; keep_mask (optional, may be
 * NULL) [B, H_q, ceil(N_q/B_q), ceil(ceil(N_k/B_k)/32)] uint32; stats
 * (optional device int64[4], accumulated with atomics, caller zeroes):
 * tiles tested, tiles retained, post-score key slots (B_k per row per
 * retained tile, valid rows only), reserved.
 *
 * Supported: dtype MALA_BF16 with d in {64, 128} and B_q = B_k = 128 (tensor
 * core path); dtype MALA_FP32 or MALA_BF16 with d in {64, 128} and
 * B_q, B_k in {16, 32, 64, 128} (CUDA-core path). mode MALA_CAUSAL only.
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  uint32_t* keep_mask;
  int64_t batch, heads_q, heads_kv, seqlen_q, seqlen_k, head_dim;
  int64_t q_stride[3];          /* batch, sequence, head strides in elements */
  int64_t k_stride[3];
  int64_t v_stride[3];
  int64_t o_stride[3];
  const int32_t* q_to_kv;       /* host array [heads_q] or NULL */
  int32_t block_q, block_k;
  float tau;
  int32_t dtype;
  int32_t mode;
  int64_t* stats;               /* device int64[4] or NULL */
  /* Packed variable-length sequences (NULL = fixed lengths). HOST arrays of
   * batch + 1 ascending offsets, cu_seqlens_q[0] = cu_seqlens_k[0] = 0:
   * sequence s owns query rows [cu_seqlens_q[s], cu_seqlens_q[s+1]) and key
   * rows [cu_seqlens_k[s], cu_seqlens_k[s+1]), each bottom-right aligned on
   * its own (N_q,s <= N_k,s). q, o are then [1, total_q, H_q, d] and k, v
   * [1, total_k, H_kv, d] (stride[0] unused); seqlen_q / seqlen_k give the
   * totals; lse is [H_q, total_q]; keep_mask is [H_q, QB, ceil(KB/32)] with
   * QB = sum_s ceil(N_q,s / B_q) (sequence s's blocks after those of the
   * earlier sequences) and KB = max_s ceil(N_k,s / B_k). Tensor-core path
   * only (bf16, 128 x 128 tiles); at most MALA_MAX_SEQS sequences. */
  const int32_t* cu_seqlens_q;
  const int32_t* cu_seqlens_k;
  /* 0 (the default): every query head decides for itself. 1: group-joint
   * voting, one decision per (query block, key tile) for the G = H_q / H_kv
   * query heads of a KV head: their rows of the block are treated like the
   * rows of one query block, so a tile is skipped only when every row of
   * every head passes the skip test, and a retained tile is accumulated by
   * every head. keep_mask bits are then equal across a group, and mala_bwd
   * replays them as usual. Tensor-core path only (bf16, 128 x 128 tiles),
   * the default head map (q_to_kv NULL or h -> h / G) and G <= 8, else
   * MALA_ERR_UNSUPPORTED; other values MALA_ERR_INVALID_ARG. */
  int32_t group_vote;
  /* Limit in nanoseconds of every device-side bounded wait of this call;
   * 0 (the default) means 2 s, far above any legitimate wait. A smaller
   * value exists for tests of the timeout path: a wait that runs out makes
   * the call's kernels stop early, leave their outputs undefined and record
   * MALA_ERR_TIMEOUT for mala_check_device_error(). Negative values:
   * MALA_ERR_INVALID_ARG. */
  int64_t wait_limit_ns;
} mala_fwd_args;

#define MALA_MAX_SEQS 128

MALA_API size_t mala_fwd_workspace_size(const mala_fwd_args* args);
MALA_API int mala_fwd(const mala_fwd_args* args, void* workspace, size_t workspace_bytes,
             void* stream);

/*
 * Backward: Algorithm 2 ("Offline Sparse Probability", Appendix A.1 "Fused
 * backward execution"). Key-major: for every key block j, query blocks are
 * visited ascending from the diagonal; the score tile is recomputed and the
 * tile is skipped iff s_qk - z_q < log tau - log L_q for every legal (q, k)
 * entry, z = lse from mala_fwd. Retained tiles reconstruct P = exp(S - z)
 * and run dV += P^T dO, dP = dO V^T, dS = P * (dP - D) with
 * D_q = sum_d dO_q O_q, dQ += dS K, dK += dS^T Q. dK and dV of a key/value
 * head sum the contributions of every query head mapped to it.
 *
 * keep_mask (input, optional): the forward's mask. When given, only tiles
 * the forward retained are recomputed (mask replay; by the support-nesting
 * argument of the same section this selects the same tiles up to rounding).
 * NULL visits every legal tile. bwd_keep_mask (output, optional): same
 * layout, bits of tiles the backward retained. dq, dk, dv are fully
 * overwritten. Supported: MALA_BF16, d = 128, B_q = B_k = 128, causal with
 * N_q <= N_k bottom-right aligned as for mala_fwd (key rows that no query
 * sees get dK = dV = 0).
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;
  const uint32_t* keep_mask;
  void* dq;
  void* dk;
  void* dv;
  uint32_t* bwd_keep_mask;
  int64_t batch, heads_q, heads_kv, seqlen_q, seqlen_k, head_dim;
  int64_t q_stride[3];
  int64_t k_stride[3];
  int64_t v_stride[3];
  int64_t o_stride[3];
  int64_t do_stride[3];
  int64_t dq_stride[3];
  int64_t dk_stride[3];
  int64_t dv_stride[3];
  const int32_t* q_to_kv;
  int32_t block_q, block_k;
  float tau;
  int32_t dtype;
  int64_t* stats;               /* device int64[4]: tiles tested, retained, slots, reserved */
  /* Packed variable-length sequences, as for mala_fwd (NULL = fixed
   * lengths); dout and dq follow q's packed layout, dk and dv k's; lse and
   * the masks use mala_fwd's packed layouts. */
  const int32_t* cu_seqlens_q;
  const int32_t* cu_seqlens_k;
  /* Limit in nanoseconds of every device-side bounded wait of this call;
   * 0 (the default) means 2 s, far above any legitimate wait. A smaller
   * value exists for tests of the timeout path: a wait that runs out makes
   * the call's kernels stop early, leave their outputs undefined and record
   * MALA_ERR_TIMEOUT for mala_check_device_error(). Negative values:
   * MALA_ERR_INVALID_ARG. */
  int64_t wait_limit_ns;
} mala_bwd_args;

MALA_API size_t mala_bwd_workspace_size(const mala_bwd_args* args);
MALA_API int mala_bwd(const mala_bwd_args* args, void* workspace, size_t workspace_bytes,
             void* stream);

/*
 * Single-token decoding with split-KV (cost paragraph after "Offline Sparse
 * Probability"; Appendix A.1 "Fused decoding execution"). One query per
 * (batch, head) at position N_k - 1, so L_0 = N_k. The T = ceil(N_k/B_k) key
 * tiles are split into P contiguous ranges, split p covering tiles
 * [floor(p*T/P), floor((p+1)*T/P)); each split visits its tiles in
 * descending order with its own running maximum and normalisation sum, and
 * tests every tile against tau / N_k. A tile's V is read iff some query
 * head of the group retains it; PV runs only for the retaining heads (for
 * every head of the group with group_vote = 1). The
 * partial outputs are merged by their log-normalisers:
 * z = log sum_p exp(z_p), O = sum_p exp(z_p - z) O_p.
 *
 * q [B, 1, H_q, d]; k, v [B, N_k, H_kv, d]; o [B, 1, H_q, d]; lse [B, H_q]
 * fp32; keep_mask optional [B, H_q, ceil(T/32)] uint32.
 * num_splits: in 0 = let the library choose, else the requested P
 * (1 <= P <= T); out: the P used (host-side value, known before launch).
 * Supported: q in MALA_BF16, the K / V cache in MALA_BF16 or
 * MALA_FP8_E4M3 (kv_dtype), d = 128, B_k = 128, H_q / H_kv <= 16.
 */
typedef struct {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  uint32_t* keep_mask;
  int64_t batch, heads_q, heads_kv, seqlen_k, head_dim;
  int64_t q_stride[3];
  int64_t k_stride[3];
  int64_t v_stride[3];
  int64_t o_stride[3];
  const int32_t* q_to_kv;
  int32_t block_k;
  float tau;
  int32_t dtype;
  int32_t num_splits;
  int64_t* stats;               /* device int64[4]: tiles tested, V tiles read, head-tiles retained, reserved */
  /* K / V cache element type: MALA_BF16 (0, the default) or MALA_FP8_E4M3
   * (OCP e4m3, one byte per element, head_dim 128, strides in elements as
   * for every tensor). An e4m3 cache holds codes whose values are
   * code * k_scale for K and code * v_scale for V (positive, finite; unused
   * for bf16); q stays bf16. The scores then use the query rounded to f16
   * (exact for |q| >= 2^-14) and P in f16. The NaN codes (0x7F, 0xFF) have
   * no defined result. */
  int32_t kv_dtype;
  float k_scale;
  float v_scale;
  /* 0 (the default): every query head decides for itself ("Online Sparse
   * Softmax" applied per head). 1: group-joint voting, one decision per key
   * tile for all query heads that share a KV head: their rows are treated
   * like the rows of one query block, so a tile is skipped only when every
   * head of the group passes the skip test, and a retained tile is
   * accumulated by every head of the group. keep_mask bits are then equal
   * across a group. Other values: MALA_ERR_INVALID_ARG. */
  int32_t group_vote;
  /* Limit in nanoseconds of every device-side bounded wait of this call;
   * 0 (the default) means 2 s, far above any legitimate wait. A smaller
   * value exists for tests of the timeout path: a wait that runs out makes
   * the call's kernels stop early, leave their outputs undefined and record
   * MALA_ERR_TIMEOUT for mala_check_device_error(). Negative values:
   * MALA_ERR_INVALID_ARG. */
  int64_t wait_limit_ns;
} mala_decode_args;

MALA_API size_t mala_decode_workspace_size(const mala_decode_args* args);
MALA_API int mala_decode(mala_decode_args* args, void* workspace, size_t workspace_bytes,
                void* stream);

/*
 * mala_decode_noalloc: mala_decode for callers that cannot allocate device
 * memory. The paper has no counterpart to this entry point; it exists for
 * code that is handed only its input and output buffers, such as a plugin
 * inside a host framework that owns every device allocation and offers no
 * workspace, or a serving loop that forbids allocation after start-up to
 * keep its memory footprint fixed. Such callers cannot provide the
 * workspace that mala_decode needs for its split partials.
 *
 * Same arguments, semantics and results as mala_decode, but the split
 * partials live in a buffer built into the library: a device array of
 * MALA_DECODE_NOALLOC_SCRATCH_BYTES that every GPU loading the library
 * holds until the process exits. Nothing is allocated or freed by the call.
 *   - The partials take batch * heads_q * (128 + 1) * 4 bytes per split.
 *     num_splits = 0 picks the same split count as mala_decode, lowered
 *     until the partials fit (down to one split, which needs no scratch); an
 *     explicit num_splits whose partials do not fit returns
 *     MALA_ERR_WORKSPACE with the sizes in mala_last_error_message().
 *   - The first call on each device looks up the buffer's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture. The address is kept for the life of the
 *     process: after cudaDeviceReset() on a device, do not call this entry
 *     point on that device again in the same process (the library's device
 *     error block, looked up the same way, has the same limit).
 *   - All calls share the one buffer, which keeps the last call's contents.
 *     Calls whose kernels overlap on the GPU (e.g. on different streams
 *     without ordering) race on it and give wrong results: order them.
 */
#define MALA_DECODE_NOALLOC_SCRATCH_BYTES (4u << 20)
MALA_API int mala_decode_noalloc(mala_decode_args* args, void* stream);

/* Human-readable name of a return code. */
MALA_API const char* mala_status_string(int status);

/* Detail of the last host-side argument error in this thread (never NULL). */
MALA_API const char* mala_last_error_message(void);

/*
 * Synchronise `stream` and report a device-side failure recorded by any
 * kernel of this library since the previous call: MALA_ERR_TIMEOUT if a
 * bounded wait gave up; MALA_ERR_CUDA if the stream reports a CUDA error,
 * or if the backward kernel found its dynamic shared memory base not
 * 1024-byte aligned (its swizzled tiles need it; it then computes nothing);
 * else MALA_OK. Clears the recorded flag.
 */
MALA_API int mala_check_device_error(void* stream);

/* Library version, e.g. "0.1.0". */
MALA_API const char* mala_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MALA_H_ */
