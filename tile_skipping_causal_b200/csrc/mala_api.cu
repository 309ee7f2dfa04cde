// Host side of the C ABI declared in include/mala.h: argument checks, TMA
// descriptor encoding, kernel selection and launches. Nothing here allocates
// device memory; scratch space comes from the caller's workspace.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>

#include "kernels.h"
#include "mala.h"

static_assert(MALA_MAX_SEQS == mala::kMaxSeqs, "packed-sequence limit of the header and the kernels differ");

namespace mala {
// {code, tag, block, parity, progress x3, spare} of the first device-side
// wait that gave up
__device__ int g_device_error[8] = {0, 0, 0, 0, 0, 0, 0, 0};
}  // namespace mala

namespace {

thread_local char g_msg[512] = "";

int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MALA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda directly.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 4-D bf16 view {d, heads, seq, batch} of a [B, N, H, d] tensor with element
// strides (sb, sn, sh), box {64, 1, rows, 1}, 128-byte swizzle.
int make_map_bf16(CUtensorMap* map, const void* ptr, int64_t B, int64_t N, int64_t H, int64_t d,
                  const int64_t* st, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MALA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)(st[2] * 2), (cuuint64_t)(st[1] * 2), (cuuint64_t)(st[0] * 2)};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MALA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MALA_OK;
}

// 4-D byte view {d, heads, seq, batch} of an e4m3 [B, N, H, d] tensor, box
// {128, 1, rows, 1}: one 128-byte row per key, 128-byte swizzle.
int make_map_u8(CUtensorMap* map, const void* ptr, int64_t B, int64_t N, int64_t H, int64_t d,
                const int64_t* st, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MALA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)N, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)st[2], (cuuint64_t)st[1], (cuuint64_t)st[0]};
  cuuint32_t box[4] = {128, 1, (cuuint32_t)rows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MALA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return MALA_OK;
}

// Device address of the error block on the current device (looked up once
// per device; calls from several host threads are serialised here).
int* device_error_ptr() {
  static int* ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, mala::g_device_error) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<int*>(p);
  }
  return ptrs[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Wait limit of a call's kernels: the caller's value, or 2 s for 0.
int wait_limit(int64_t ns, uint64_t* out) {
  if (ns < 0) return fail(MALA_ERR_INVALID_ARG, "wait_limit_ns %lld is negative", (long long)ns);
  *out = ns == 0 ? 2000000000ull : static_cast<uint64_t>(ns);
  return MALA_OK;
}

// Checks one [B, N, H, d] operand: non-NULL, 16-byte aligned, strides
// non-negative multiples of 16 bytes, rows that do not overlap.
int check_tensor(const char* name, const void* p, const int64_t* st, int64_t esize, int64_t d,
                 int64_t H) {
  if (!p) return fail(MALA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(p)) return fail(MALA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  for (int x = 0; x < 3; ++x) {
    if (st[x] < 0 || (st[x] * esize) % 16 != 0)
      return fail(MALA_ERR_INVALID_ARG, "%s stride[%d]=%lld is not a non-negative multiple of 16 bytes",
                  name, x, (long long)st[x]);
  }
  if (st[2] < d) return fail(MALA_ERR_INVALID_ARG, "%s head stride smaller than head_dim", name);
  if (st[1] < st[2] * H && st[1] != 0)
    ;  // sequence stride may interleave heads arbitrarily as long as rows are distinct
  return MALA_OK;
}

int head_map(const int32_t* q_to_kv, int64_t Hq, int64_t Hkv, uint8_t* out) {
  if (Hq > mala::kMaxHeads) return fail(MALA_ERR_UNSUPPORTED, "heads_q > %d", mala::kMaxHeads);
  for (int64_t h = 0; h < Hq; ++h) {
    int64_t v = q_to_kv ? q_to_kv[h] : h / (Hq / Hkv);
    if (v < 0 || v >= Hkv) return fail(MALA_ERR_INVALID_ARG, "q_to_kv[%lld]=%lld out of range", (long long)h, (long long)v);
    out[h] = static_cast<uint8_t>(v);
  }
  return MALA_OK;
}

int check_common(int64_t B, int64_t Hq, int64_t Hkv, int64_t d, float tau, int dtype) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0) return fail(MALA_ERR_INVALID_ARG, "batch and head counts must be positive");
  if (Hq % Hkv != 0) return fail(MALA_ERR_INVALID_ARG, "heads_q %% heads_kv != 0");
  if (isnan(tau) || tau < 0.0f) return fail(MALA_ERR_INVALID_ARG, "tau must be >= 0");
  if (dtype != MALA_BF16 && dtype != MALA_FP32) return fail(MALA_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  if (d != 64 && d != 128) return fail(MALA_ERR_UNSUPPORTED, "head_dim %lld not in {64, 128}", (long long)d);
  return MALA_OK;
}

bool block_ok(int x) { return x == 16 || x == 32 || x == 64 || x == 128; }

}  // namespace

extern "C" {

const char* mala_version(void) { return "0.1.0"; }

const char* mala_status_string(int s) {
  switch (s) {
    case MALA_OK: return "MALA_OK";
    case MALA_ERR_INVALID_ARG: return "MALA_ERR_INVALID_ARG";
    case MALA_ERR_UNSUPPORTED: return "MALA_ERR_UNSUPPORTED";
    case MALA_ERR_WORKSPACE: return "MALA_ERR_WORKSPACE";
    case MALA_ERR_CUDA: return "MALA_ERR_CUDA";
    case MALA_ERR_TIMEOUT: return "MALA_ERR_TIMEOUT";
    default: return "MALA_ERR_UNKNOWN";
  }
}

const char* mala_last_error_message(void) { return g_msg; }

int mala_check_device_error(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int rec[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  e = cudaMemcpyFromSymbol(rec, mala::g_device_error, sizeof(rec));
  if (e != cudaSuccess) return cuda_fail(e, "read device error flag");
  if (rec[0] != 0) {
    int zero[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    cudaMemcpyToSymbol(mala::g_device_error, zero, sizeof(zero));
    if (rec[0] == mala::kErrSmemAlign)
      return fail(MALA_ERR_CUDA, "a kernel found its dynamic shared memory base misaligned; nothing was computed");
    return fail(MALA_ERR_TIMEOUT,
                "a device-side bounded wait gave up (role %d, barrier %d, tile %d, block %d, parity %d; "
                "progress %08x %08x %08x)",
                (rec[1] >> 24) & 0xf, (rec[1] >> 16) & 0xff, rec[1] & 0xffff, rec[2], rec[3], rec[4],
                rec[5], rec[6]);
  }
  return MALA_OK;
}

// Packed variable-length sequences: checks the host offset arrays and fills
// the kernels' sequence table; nQB / nKB receive the per-sequence maxima.
int seq_table(const int32_t* cq, const int32_t* ck, int64_t nseq, int64_t total_q, int64_t total_k,
              mala::SeqTable* t, int* nQB, int* nKB) {
  if (!cq || !ck) return fail(MALA_ERR_INVALID_ARG, "packed sequences need both cu_seqlens_q and cu_seqlens_k");
  if (nseq > mala::kMaxSeqs) return fail(MALA_ERR_UNSUPPORTED, "more than %d packed sequences", mala::kMaxSeqs);
  if (cq[0] != 0 || ck[0] != 0) return fail(MALA_ERR_INVALID_ARG, "cu_seqlens must start at 0");
  if (cq[nseq] != total_q || ck[nseq] != total_k)
    return fail(MALA_ERR_INVALID_ARG, "cu_seqlens must end at seqlen_q / seqlen_k (the packed totals)");
  t->n = static_cast<int>(nseq);
  *nQB = *nKB = 1;
  int qb = 0;
  for (int64_t s = 0; s < nseq; ++s) {
    const int64_t lq = static_cast<int64_t>(cq[s + 1]) - cq[s], lk = static_cast<int64_t>(ck[s + 1]) - ck[s];
    if (lq < 0 || lk < 0) return fail(MALA_ERR_INVALID_ARG, "cu_seqlens must be non-decreasing");
    if (lq > lk)
      return fail(MALA_ERR_UNSUPPORTED, "sequence %lld has more queries than keys (needs N_q <= N_k)", (long long)s);
    t->q0[s] = cq[s];
    t->k0[s] = ck[s];
    t->qb0[s] = qb;
    const int bq = static_cast<int>((lq + 127) / 128), bk = static_cast<int>((lk + 127) / 128);
    qb += bq;
    *nQB = std::max(*nQB, bq);
    *nKB = std::max(*nKB, bk);
  }
  t->q0[nseq] = static_cast<int>(total_q);
  t->k0[nseq] = static_cast<int>(total_k);
  t->qb0[nseq] = qb;
  return MALA_OK;
}

// ------------------------------------------------------------------ forward

size_t mala_fwd_workspace_size(const mala_fwd_args* a) {
  (void)a;
  return 0;
}

int mala_fwd(const mala_fwd_args* a, void* workspace, size_t ws_bytes, void* stream_) {
  (void)workspace;
  (void)ws_bytes;
  g_msg[0] = 0;
  if (!a) return fail(MALA_ERR_INVALID_ARG, "args is NULL");
  int rc = check_common(a->batch, a->heads_q, a->heads_kv, a->head_dim, a->tau, a->dtype);
  if (rc) return rc;
  if (a->wait_limit_ns < 0) return fail(MALA_ERR_INVALID_ARG, "wait_limit_ns %lld is negative", (long long)a->wait_limit_ns);
  if (a->mode != MALA_CAUSAL)
    return fail(MALA_ERR_UNSUPPORTED, "mala_fwd supports MALA_CAUSAL; use mala_decode for decoding");
  if (a->seqlen_q <= 0 || a->seqlen_k <= 0) return fail(MALA_ERR_INVALID_ARG, "sequence lengths must be positive");
  if (a->seqlen_q > a->seqlen_k)
    return fail(MALA_ERR_UNSUPPORTED, "causal mode needs seqlen_q <= seqlen_k (bottom-right alignment)");
  if (a->seqlen_k > (1 << 30)) return fail(MALA_ERR_UNSUPPORTED, "sequence too long");
  if (!block_ok(a->block_q) || !block_ok(a->block_k))
    return fail(MALA_ERR_UNSUPPORTED, "block sizes must be in {16, 32, 64, 128}");
  if (!a->lse) return fail(MALA_ERR_INVALID_ARG, "lse is NULL");
  const int64_t es = a->dtype == MALA_BF16 ? 2 : 4;
  const int64_t d = a->head_dim;
  if ((rc = check_tensor("q", a->q, a->q_stride, es, d, a->heads_q))) return rc;
  if ((rc = check_tensor("k", a->k, a->k_stride, es, d, a->heads_kv))) return rc;
  if ((rc = check_tensor("v", a->v, a->v_stride, es, d, a->heads_kv))) return rc;
  if ((rc = check_tensor("o", a->o, a->o_stride, es, d, a->heads_q))) return rc;
  if ((reinterpret_cast<uintptr_t>(a->lse) & 3u) != 0) return fail(MALA_ERR_INVALID_ARG, "lse misaligned");
  if (a->stats && (reinterpret_cast<uintptr_t>(a->stats) & 7u) != 0)
    return fail(MALA_ERR_INVALID_ARG, "stats misaligned");
  const int64_t N = a->seqlen_q;
  const int64_t Nk = a->seqlen_k;
  int nQB = static_cast<int>((N + a->block_q - 1) / a->block_q);
  int nKB = static_cast<int>((Nk + a->block_k - 1) / a->block_k);
  const bool packed = a->cu_seqlens_q || a->cu_seqlens_k;
  mala::SeqTable seq;
  seq.n = 0;
  if (packed) {
    if (!(a->dtype == MALA_BF16 && a->block_q == 128 && a->block_k == 128))
      return fail(MALA_ERR_UNSUPPORTED, "packed sequences need bf16 and 128 x 128 tiles");
    if ((rc = seq_table(a->cu_seqlens_q, a->cu_seqlens_k, a->batch, N, Nk, &seq, &nQB, &nKB))) return rc;
  }
  const int mask_words = (nKB + 31) / 32;
  if ((double)a->batch * a->heads_q * nQB > 2147483647.0) return fail(MALA_ERR_UNSUPPORTED, "grid too large");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);

  const bool tc = a->dtype == MALA_BF16 && a->block_q == 128 && a->block_k == 128;
  if (a->group_vote != 0 && a->group_vote != 1)
    return fail(MALA_ERR_INVALID_ARG, "group_vote %d is neither 0 nor 1", a->group_vote);
  if (a->group_vote && !tc)
    return fail(MALA_ERR_UNSUPPORTED, "group-joint voting needs the tensor-core path (bf16, 128 x 128 tiles)");
  if (tc) {
    mala::FwdTcParams p;
    memset(&p, 0, sizeof(p));
    if ((rc = head_map(a->q_to_kv, a->heads_q, a->heads_kv, p.kv_of_q))) return rc;
    // query heads in KV-head order (a stable sort by KV head), so that the
    // grid can run the heads that share K / V side by side
    {
      int pos = 0;
      for (int64_t hk = 0; hk < a->heads_kv; ++hk)
        for (int64_t h = 0; h < a->heads_q; ++h)
          if (p.kv_of_q[h] == hk) p.head_order[pos++] = static_cast<uint8_t>(h);
    }
    p.group = static_cast<int>(a->heads_q / a->heads_kv);
    if (a->group_vote) {
      const int G = static_cast<int>(a->heads_q / a->heads_kv);
      if (G > 8) return fail(MALA_ERR_UNSUPPORTED, "group-joint voting supports groups of at most 8 query heads");
      for (int64_t h = 0; h < a->heads_q; ++h)
        if (p.kv_of_q[h] != h / G)
          return fail(MALA_ERR_UNSUPPORTED, "group-joint voting needs the default head map (h -> h / G)");
      p.group_vote = 1;
    }
    // packed sequences: one batch entry of total_q / total_k rows
    const int64_t mb = packed ? 1 : a->batch;
    if ((rc = make_map_bf16(&p.tm_q, a->q, mb, N, a->heads_q, d, a->q_stride, 128))) return rc;
    if ((rc = make_map_bf16(&p.tm_k, a->k, mb, Nk, a->heads_kv, d, a->k_stride, 128))) return rc;
    if ((rc = make_map_bf16(&p.tm_v, a->v, mb, Nk, a->heads_kv, d, a->v_stride, 128))) return rc;
    p.seq = seq;
    if ((rc = wait_limit(a->wait_limit_ns, &p.wait_ns))) return rc;
    p.err = device_error_ptr();
    if (!p.err) return fail(MALA_ERR_CUDA, "cannot resolve the device error word");
    p.o = a->o;
    p.lse = a->lse;
    p.keep_mask = a->keep_mask;
    p.stats = a->stats;
    p.o_sb = a->o_stride[0];
    p.o_sn = a->o_stride[1];
    p.o_sh = a->o_stride[2];
    p.B = static_cast<int>(a->batch);
    p.Hq = static_cast<int>(a->heads_q);
    p.Hkv = static_cast<int>(a->heads_kv);
    p.N = static_cast<int>(N);
    p.Nk = static_cast<int>(Nk);
    p.q_off = static_cast<int>(Nk - N);
    p.nQB = nQB;
    p.nKB = nKB;
    p.mask_words = mask_words;
    p.log2_tau = a->tau == 0.0f ? -INFINITY : log2f(a->tau);
    cudaError_t e = mala::launch_fwd_tc(p, static_cast<int>(d), stream);
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return MALA_OK;
  }
  mala::FwdSimtParams p;
  memset(&p, 0, sizeof(p));
  if ((rc = head_map(a->q_to_kv, a->heads_q, a->heads_kv, p.kv_of_q))) return rc;
  p.q = a->q;
  p.k = a->k;
  p.v = a->v;
  p.o = a->o;
  p.lse = a->lse;
  p.keep_mask = a->keep_mask;
  p.stats = a->stats;
  p.q_sb = a->q_stride[0]; p.q_sn = a->q_stride[1]; p.q_sh = a->q_stride[2];
  p.k_sb = a->k_stride[0]; p.k_sn = a->k_stride[1]; p.k_sh = a->k_stride[2];
  p.v_sb = a->v_stride[0]; p.v_sn = a->v_stride[1]; p.v_sh = a->v_stride[2];
  p.o_sb = a->o_stride[0]; p.o_sn = a->o_stride[1]; p.o_sh = a->o_stride[2];
  p.B = static_cast<int>(a->batch);
  p.Hq = static_cast<int>(a->heads_q);
  p.Hkv = static_cast<int>(a->heads_kv);
  p.N = static_cast<int>(N);
  p.Nk = static_cast<int>(Nk);
  p.q_off = static_cast<int>(Nk - N);
  p.BQ = a->block_q;
  p.BK = a->block_k;
  p.nQB = nQB;
  p.nKB = nKB;
  p.mask_words = mask_words;
  p.log_tau = a->tau == 0.0f ? -INFINITY : logf(a->tau);
  cudaError_t e = mala::launch_fwd_simt(p, static_cast<int>(d), a->dtype == MALA_FP32, stream);
  if (e != cudaSuccess) return cuda_fail(e, "forward launch");
  return MALA_OK;
}

// ------------------------------------------------------------------ backward

namespace {

int bwd_check(const mala_bwd_args* a) {
  int rc = check_common(a->batch, a->heads_q, a->heads_kv, a->head_dim, a->tau, a->dtype);
  if (rc) return rc;
  if (a->wait_limit_ns < 0) return fail(MALA_ERR_INVALID_ARG, "wait_limit_ns %lld is negative", (long long)a->wait_limit_ns);
  if (a->dtype != MALA_BF16) return fail(MALA_ERR_UNSUPPORTED, "backward supports bf16 only");
  if (a->head_dim != 128) return fail(MALA_ERR_UNSUPPORTED, "backward supports head_dim 128 only");
  if (a->block_q != 128 || a->block_k != 128) return fail(MALA_ERR_UNSUPPORTED, "backward supports 128 x 128 tiles only");
  if (a->seqlen_q <= 0 || a->seqlen_k <= 0) return fail(MALA_ERR_INVALID_ARG, "sequence lengths must be positive");
  if (a->seqlen_q > a->seqlen_k)
    return fail(MALA_ERR_UNSUPPORTED, "causal backward needs seqlen_q <= seqlen_k (bottom-right alignment)");
  if (a->seqlen_k > (1 << 30)) return fail(MALA_ERR_UNSUPPORTED, "sequence too long");
  if (a->heads_kv > mala::kMaxKvHeads) return fail(MALA_ERR_UNSUPPORTED, "heads_kv > %d", mala::kMaxKvHeads);
  if (!a->lse) return fail(MALA_ERR_INVALID_ARG, "lse is NULL");
  if (a->cu_seqlens_q || a->cu_seqlens_k) {
    mala::SeqTable t;
    int nQB = 0, nKB = 0;
    if ((rc = seq_table(a->cu_seqlens_q, a->cu_seqlens_k, a->batch, a->seqlen_q, a->seqlen_k, &t, &nQB, &nKB)))
      return rc;
  }
  if ((rc = check_tensor("q", a->q, a->q_stride, 2, 128, a->heads_q))) return rc;
  if ((rc = check_tensor("k", a->k, a->k_stride, 2, 128, a->heads_kv))) return rc;
  if ((rc = check_tensor("v", a->v, a->v_stride, 2, 128, a->heads_kv))) return rc;
  if ((rc = check_tensor("o", a->o, a->o_stride, 2, 128, a->heads_q))) return rc;
  if ((rc = check_tensor("dout", a->dout, a->do_stride, 2, 128, a->heads_q))) return rc;
  if ((rc = check_tensor("dq", a->dq, a->dq_stride, 2, 128, a->heads_q))) return rc;
  if ((rc = check_tensor("dk", a->dk, a->dk_stride, 2, 128, a->heads_kv))) return rc;
  if ((rc = check_tensor("dv", a->dv, a->dv_stride, 2, 128, a->heads_kv))) return rc;
  return MALA_OK;
}

// Rows of the backward workspace: B H_q nQB 128 for fixed lengths, or
// H_q QB 128 for packed sequences (QB = all packed query blocks).
size_t bwd_rows(const mala_bwd_args* a) {
  if (a->cu_seqlens_q) {
    size_t qb = 0;
    for (int64_t s = 0; s < a->batch; ++s) qb += static_cast<size_t>((a->cu_seqlens_q[s + 1] - a->cu_seqlens_q[s] + 127) / 128);
    return static_cast<size_t>(a->heads_q) * qb * 128;
  }
  const size_t npad = static_cast<size_t>((a->seqlen_q + 127) / 128) * 128;
  return static_cast<size_t>(a->batch) * a->heads_q * npad;
}

// workspace: -z log2e, D (one fp32 per row each) then the blocked dQ accumulator
size_t bwd_ws_bytes(const mala_bwd_args* a) {
  const size_t rows = bwd_rows(a);
  return rows * 2 * sizeof(float) + rows * 128 * sizeof(float) + 256;
}

}  // namespace

size_t mala_bwd_workspace_size(const mala_bwd_args* a) {
  if (!a || bwd_check(a) != MALA_OK) return 0;
  return bwd_ws_bytes(a);
}

int mala_bwd(const mala_bwd_args* a, void* workspace, size_t ws_bytes, void* stream_) {
  g_msg[0] = 0;
  if (!a) return fail(MALA_ERR_INVALID_ARG, "args is NULL");
  int rc = bwd_check(a);
  if (rc) return rc;
  const size_t need = bwd_ws_bytes(a);
  if (!workspace || ws_bytes < need) return fail(MALA_ERR_WORKSPACE, "backward workspace of %zu bytes needed", need);
  if (!aligned16(workspace)) return fail(MALA_ERR_INVALID_ARG, "workspace misaligned");
  const int N = static_cast<int>(a->seqlen_q);
  const int Nk = static_cast<int>(a->seqlen_k);
  int nQB = (N + 127) / 128;
  int nKB = (Nk + 127) / 128;
  const int Npad = nQB * 128;
  const size_t rows = bwd_rows(a);
  const bool packed = a->cu_seqlens_q != nullptr;

  mala::BwdParams p;
  memset(&p, 0, sizeof(p));
  if (packed && (rc = seq_table(a->cu_seqlens_q, a->cu_seqlens_k, a->batch, N, Nk, &p.seq, &nQB, &nKB))) return rc;
  uint8_t kv_of_q[mala::kMaxHeads];
  if ((rc = head_map(a->q_to_kv, a->heads_q, a->heads_kv, kv_of_q))) return rc;
  for (int64_t h = 0; h < a->heads_q; ++h) {
    const int hk = kv_of_q[h];
    if (p.group_size[hk] >= mala::kMaxGroup)
      return fail(MALA_ERR_UNSUPPORTED, "more than %d query heads share KV head %d", mala::kMaxGroup, hk);
    p.group_heads[hk][p.group_size[hk]++] = static_cast<uint8_t>(h);
  }
  const int64_t mb = packed ? 1 : a->batch;   // packed sequences: one batch entry of total rows
  if ((rc = make_map_bf16(&p.tm_q, a->q, mb, N, a->heads_q, 128, a->q_stride, 128))) return rc;
  if ((rc = make_map_bf16(&p.tm_k, a->k, mb, Nk, a->heads_kv, 128, a->k_stride, 128))) return rc;
  if ((rc = make_map_bf16(&p.tm_v, a->v, mb, Nk, a->heads_kv, 128, a->v_stride, 128))) return rc;
  if ((rc = make_map_bf16(&p.tm_do, a->dout, mb, N, a->heads_q, 128, a->do_stride, 128))) return rc;
  float* ws = static_cast<float*>(workspace);
  p.nzl2 = ws;
  p.Dv = ws + rows;
  p.dq_acc = ws + 2 * rows;
  p.dk = a->dk;
  p.dv = a->dv;
  p.fwd_mask = a->keep_mask;
  p.bwd_mask = a->bwd_keep_mask;
  p.stats = a->stats;
  p.log2_tau = a->tau == 0.0f ? -INFINITY : log2f(a->tau);
  if ((rc = wait_limit(a->wait_limit_ns, &p.wait_ns))) return rc;
  p.err = device_error_ptr();
  if (!p.err) return fail(MALA_ERR_CUDA, "cannot resolve the device error word");
  p.dk_sb = a->dk_stride[0]; p.dk_sn = a->dk_stride[1]; p.dk_sh = a->dk_stride[2];
  p.dv_sb = a->dv_stride[0]; p.dv_sn = a->dv_stride[1]; p.dv_sh = a->dv_stride[2];
  p.B = static_cast<int>(a->batch);
  p.Hq = static_cast<int>(a->heads_q);
  p.Hkv = static_cast<int>(a->heads_kv);
  p.N = N;
  p.Nk = Nk;
  p.q_off = Nk - N;
  p.Npad = Npad;
  p.nQB = nQB;
  p.nKB = nKB;
  p.mask_words = (nKB + 31) / 32;

  mala::BwdAuxParams x;
  memset(&x, 0, sizeof(x));
  x.o = a->o;
  x.dout = a->dout;
  x.lse = a->lse;
  x.nzl2 = ws;
  x.Dv = ws + rows;
  x.dq_acc = ws + 2 * rows;
  x.dq = a->dq;
  x.o_sb = a->o_stride[0]; x.o_sn = a->o_stride[1]; x.o_sh = a->o_stride[2];
  x.do_sb = a->do_stride[0]; x.do_sn = a->do_stride[1]; x.do_sh = a->do_stride[2];
  x.dq_sb = a->dq_stride[0]; x.dq_sn = a->dq_stride[1]; x.dq_sh = a->dq_stride[2];
  x.B = p.B;
  x.Hq = p.Hq;
  x.N = N;
  x.Npad = Npad;
  x.nQB = nQB;
  x.seq = p.seq;

  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (a->bwd_keep_mask) {
    const size_t mrows = packed ? static_cast<size_t>(a->heads_q) * p.seq.qb0[p.seq.n]
                                : static_cast<size_t>(a->batch) * a->heads_q * nQB;
    cudaError_t e = cudaMemsetAsync(a->bwd_keep_mask, 0, mrows * p.mask_words * 4, stream);
    if (e != cudaSuccess) return cuda_fail(e, "backward mask clear");
  }
  cudaError_t e = mala::launch_bwd(p, x, stream);
  if (e != cudaSuccess) return cuda_fail(e, "backward launch");
  return MALA_OK;
}

// ------------------------------------------------------------------ decode

namespace {

int decode_check(const mala_decode_args* a, int* nKB_out) {
  int rc = check_common(a->batch, a->heads_q, a->heads_kv, a->head_dim, a->tau, a->dtype);
  if (rc) return rc;
  if (a->dtype != MALA_BF16) return fail(MALA_ERR_UNSUPPORTED, "decode supports bf16 only");
  if (a->head_dim != 128) return fail(MALA_ERR_UNSUPPORTED, "decode supports head_dim 128 only");
  if (a->block_k != 128) return fail(MALA_ERR_UNSUPPORTED, "decode supports block_k 128 only");
  if (a->seqlen_k <= 0) return fail(MALA_ERR_INVALID_ARG, "seqlen_k must be positive");
  if (a->seqlen_k > (1 << 30)) return fail(MALA_ERR_UNSUPPORTED, "cache too long");
  if (a->heads_kv > mala::kMaxKvHeads) return fail(MALA_ERR_UNSUPPORTED, "heads_kv > %d", mala::kMaxKvHeads);
  if (!a->lse) return fail(MALA_ERR_INVALID_ARG, "lse is NULL");
  if (a->wait_limit_ns < 0) return fail(MALA_ERR_INVALID_ARG, "wait_limit_ns %lld is negative", (long long)a->wait_limit_ns);
  const int nKB = static_cast<int>((a->seqlen_k + 127) / 128);
  if (a->num_splits < 0 || a->num_splits > nKB)
    return fail(MALA_ERR_INVALID_ARG, "num_splits %d outside [0, %d]", a->num_splits, nKB);
  if (a->kv_dtype != MALA_BF16 && a->kv_dtype != MALA_FP8_E4M3)
    return fail(MALA_ERR_INVALID_ARG, "kv_dtype %d is neither MALA_BF16 nor MALA_FP8_E4M3", a->kv_dtype);
  const bool fp8 = a->kv_dtype == MALA_FP8_E4M3;
  if (a->group_vote != 0 && a->group_vote != 1)
    return fail(MALA_ERR_INVALID_ARG, "group_vote %d is neither 0 nor 1", a->group_vote);
  if (fp8 && !(a->k_scale > 0.0f && a->k_scale < INFINITY && a->v_scale > 0.0f && a->v_scale < INFINITY))
    return fail(MALA_ERR_INVALID_ARG, "e4m3 cache scales must be positive and finite");
  const int64_t kes = fp8 ? 1 : 2;
  if ((rc = check_tensor("q", a->q, a->q_stride, 2, 128, a->heads_q))) return rc;
  if ((rc = check_tensor("k", a->k, a->k_stride, kes, 128, a->heads_kv))) return rc;
  if ((rc = check_tensor("v", a->v, a->v_stride, kes, 128, a->heads_kv))) return rc;
  if ((rc = check_tensor("o", a->o, a->o_stride, 2, 128, a->heads_q))) return rc;
  *nKB_out = nKB;
  return MALA_OK;
}

// K / V cache tensor maps, element type and scales of a decode call.
int decode_cache_maps(const mala_decode_args* a, mala::DecodeParams* p) {
  int rc;
  if (a->kv_dtype == MALA_FP8_E4M3) {
    if ((rc = make_map_u8(&p->tm_k, a->k, a->batch, a->seqlen_k, a->heads_kv, 128, a->k_stride, 128))) return rc;
    if ((rc = make_map_u8(&p->tm_v, a->v, a->batch, a->seqlen_k, a->heads_kv, 128, a->v_stride, 128))) return rc;
    p->kv_fp8 = 1;
    p->k_scale = a->k_scale;
    p->v_scale = a->v_scale;
  } else {
    if ((rc = make_map_bf16(&p->tm_k, a->k, a->batch, a->seqlen_k, a->heads_kv, 128, a->k_stride, 128))) return rc;
    if ((rc = make_map_bf16(&p->tm_v, a->v, a->batch, a->seqlen_k, a->heads_kv, 128, a->v_stride, 128))) return rc;
    p->kv_fp8 = 0;
    p->k_scale = p->v_scale = 1.0f;
  }
  return MALA_OK;
}

// Splits per (batch, KV head): enough CTAs for several waves over the SMs,
// at least 4 key tiles per split.
int choose_splits(int64_t units, int nKB) {
  int sms = 148;
  int dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0) sms = v;
  }
  int64_t want = (8LL * sms + units - 1) / units;
  int64_t cap = nKB / 4 > 0 ? nKB / 4 : 1;
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return static_cast<int>(want);
}

size_t decode_ws_bytes(const mala_decode_args* a, int P) {
  if (P <= 1) return 0;
  return static_cast<size_t>(a->batch) * a->heads_q * P * (128 + 1) * sizeof(float) + 256;
}

// Fills the decode kernel parameters of a checked call and launches it on
// the caller's stream. partials: [B, H_q, P, 128] + [B, H_q, P] fp32 when
// P > 1 (unused otherwise); it needs no clearing, since every split writes
// all of its rows before the merge kernel reads them.
int decode_launch(mala_decode_args* a, int nKB, int P, float* partials, void* stream_) {
  int rc;
  mala::DecodeParams p;
  memset(&p, 0, sizeof(p));
  uint8_t kv_of_q[mala::kMaxHeads];
  if ((rc = head_map(a->q_to_kv, a->heads_q, a->heads_kv, kv_of_q))) return rc;
  for (int64_t h = 0; h < a->heads_q; ++h) {
    const int hk = kv_of_q[h];
    if (p.group_size[hk] >= mala::kMaxGroup)
      return fail(MALA_ERR_UNSUPPORTED, "more than %d query heads share KV head %d", mala::kMaxGroup, hk);
    p.group_heads[hk][p.group_size[hk]++] = static_cast<uint8_t>(h);
  }
  if ((rc = decode_cache_maps(a, &p))) return rc;
  p.group_vote = a->group_vote;
  if ((rc = wait_limit(a->wait_limit_ns, &p.wait_ns))) return rc;
  p.err = device_error_ptr();
  if (!p.err) return fail(MALA_ERR_CUDA, "cannot resolve the device error word");
  p.q = a->q;
  p.o = a->o;
  p.lse = a->lse;
  p.keep_mask = a->keep_mask;
  p.stats = a->stats;
  if (P > 1) {
    p.part_o = partials;
    p.part_lse = partials + static_cast<size_t>(a->batch) * a->heads_q * P * 128;
  }
  p.q_sb = a->q_stride[0];
  p.q_sh = a->q_stride[2];
  p.o_sb = a->o_stride[0];
  p.o_sh = a->o_stride[2];
  p.B = static_cast<int>(a->batch);
  p.Hq = static_cast<int>(a->heads_q);
  p.Hkv = static_cast<int>(a->heads_kv);
  p.Nk = static_cast<int>(a->seqlen_k);
  p.nKB = nKB;
  p.mask_words = (nKB + 31) / 32;
  p.num_splits = P;
  p.log2_tau = a->tau == 0.0f ? -INFINITY : log2f(a->tau);
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (a->keep_mask) {
    cudaError_t e = cudaMemsetAsync(a->keep_mask, 0,
                                    static_cast<size_t>(a->batch) * a->heads_q * p.mask_words * 4, stream);
    if (e != cudaSuccess) return cuda_fail(e, "keep mask clear");
  }
  cudaError_t e = mala::launch_decode(p, stream);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  a->num_splits = P;
  return MALA_OK;
}

}  // namespace

size_t mala_decode_workspace_size(const mala_decode_args* a) {
  if (!a) return 0;
  int nKB = 0;
  if (decode_check(a, &nKB) != MALA_OK) return 0;
  const int P = a->num_splits > 0 ? a->num_splits : choose_splits(a->batch * a->heads_kv, nKB);
  return decode_ws_bytes(a, P);
}

int mala_decode(mala_decode_args* a, void* workspace, size_t ws_bytes, void* stream_) {
  g_msg[0] = 0;
  if (!a) return fail(MALA_ERR_INVALID_ARG, "args is NULL");
  int nKB = 0;
  int rc = decode_check(a, &nKB);
  if (rc) return rc;
  const int P = a->num_splits > 0 ? a->num_splits : choose_splits(a->batch * a->heads_kv, nKB);
  const size_t need = decode_ws_bytes(a, P);
  if (need > 0 && (!workspace || ws_bytes < need))
    return fail(MALA_ERR_WORKSPACE, "decode workspace of %zu bytes needed", need);
  if (need > 0 && !aligned16(workspace)) return fail(MALA_ERR_INVALID_ARG, "workspace misaligned");

  return decode_launch(a, nKB, P, static_cast<float*>(workspace), stream_);
}

}  // extern "C"

// ------------------------------------------------------------------ decode without allocation

namespace {

// Built-in scratch for mala_decode_noalloc: the split-KV partial outputs and
// log-normalisers ([B, H_q, P, 128] + [B, H_q, P] fp32). Every GPU that
// loads the library holds it until the process exits. In host code the name
// only stands for the symbol; its device address comes from
// cudaGetSymbolAddress (see decode_noalloc_scratch below).
static __device__ __align__(256) float g_decode_noalloc_scratch[MALA_DECODE_NOALLOC_SCRATCH_BYTES / sizeof(float)];

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached.
float* decode_noalloc_scratch() {
  static float* ptrs[64] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    ptrs[dev] = static_cast<float*>(p);
  }
  return ptrs[dev];
}

}  // namespace

extern "C" int mala_decode_noalloc(mala_decode_args* a, void* stream_) {
  g_msg[0] = 0;
  if (!a) return fail(MALA_ERR_INVALID_ARG, "args is NULL");
  int nKB = 0;
  int rc = decode_check(a, &nKB);
  if (rc) return rc;
  // bytes of partials per split: one 128-float row and one log-normaliser per (batch, head)
  const size_t per_split = static_cast<size_t>(a->batch) * a->heads_q * (128 + 1) * sizeof(float);
  const size_t cap = MALA_DECODE_NOALLOC_SCRATCH_BYTES;
  int P = a->num_splits;
  if (P > 1 && per_split * P > cap)
    return fail(MALA_ERR_WORKSPACE,
                "num_splits=%d needs %zu bytes of scratch; the built-in buffer holds %zu (use fewer splits)",
                P, per_split * P, cap);
  if (P == 0) {
    P = choose_splits(a->batch * a->heads_kv, nKB);
    while (P > 1 && per_split * P > cap) --P;   // fall back to fewer splits, down to none
  }
  float* scratch = nullptr;
  if (P > 1) {
    scratch = decode_noalloc_scratch();
    if (!scratch) return fail(MALA_ERR_CUDA, "cannot resolve the built-in decode scratch buffer");
  }
  return decode_launch(a, nKB, P, scratch, stream_);
}
