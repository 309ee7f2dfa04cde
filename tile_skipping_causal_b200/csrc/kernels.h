// Internal launch interfaces between the C ABI layer (mala_api.cu) and the
// kernel translation units. Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mala {

constexpr int kMaxHeads = 256;

// Code a kernel writes to the library's device error word when its dynamic
// shared memory base is not 1024-byte aligned (the 128-byte swizzled TMA
// tiles need it); it then returns without computing anything.
constexpr int kErrSmemAlign = 6;

// Forward, tensor-core path (bf16, B_q = B_k = 128).
// Packed variable-length sequences (n = 0: fixed lengths, batch dimension
// used instead). Sequence s owns query rows [q0[s], q0[s+1]) and key rows
// [k0[s], k0[s+1]) of the packed tensors; its query blocks are numbered from
// qb0[s] in the packed mask and workspace layouts.
constexpr int kMaxSeqs = 128;
struct SeqTable {
  int n;
  int q0[kMaxSeqs + 1];
  int k0[kMaxSeqs + 1];
  int qb0[kMaxSeqs + 1];
};

struct FwdTcParams {
  CUtensorMap tm_q;     // [B, N, Hq, D] as 4-D {D, Hq, N, B}, box {64, 1, 128, 1}, 128B swizzle
  CUtensorMap tm_k;     // [B, N, Hkv, D]
  CUtensorMap tm_v;
  void* o;
  float* lse;
  uint32_t* keep_mask;
  int64_t* stats;
  int* err;             // library device error block int[4]
  int64_t o_sb, o_sn, o_sh;
  int B, Hq, Hkv, N;    // N = N_q
  int Nk, q_off;        // N_k >= N_q; query q sits at position q + q_off (q_off = N_k - N_q)
  int nQB, nKB, mask_words;
  float log2_tau;       // log2(tau): -inf for tau = 0, +inf for tau = inf
  uint8_t kv_of_q[kMaxHeads];
  uint8_t head_order[kMaxHeads];   // query heads listed KV head by KV head
  SeqTable seq;         // packed sequences: nQB / nKB / mask_words are then maxima
  int group;            // G = Hq / Hkv
  int group_vote;       // group-joint voting: the G CTAs of a query block's
                        // KV-head group form one cluster (G <= 8)
  uint64_t wait_ns;     // limit of every bounded wait (ns)
};

cudaError_t launch_fwd_tc(const FwdTcParams& p, int head_dim, cudaStream_t stream);
size_t fwd_tc_smem_bytes(int head_dim);

// Forward, CUDA-core path (fp32 or bf16, any supported block sizes).
struct FwdSimtParams {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  uint32_t* keep_mask;
  int64_t* stats;
  int64_t q_sb, q_sn, q_sh, k_sb, k_sn, k_sh, v_sb, v_sn, v_sh, o_sb, o_sn, o_sh;
  int B, Hq, Hkv, N;    // N = N_q
  int Nk, q_off;        // N_k >= N_q; query q sits at position q + q_off
  int BQ, BK;
  int nQB, nKB, mask_words;
  float log_tau;        // natural log of tau (+-inf allowed)
  uint8_t kv_of_q[kMaxHeads];
};

cudaError_t launch_fwd_simt(const FwdSimtParams& p, int head_dim, bool fp32,
                            cudaStream_t stream);

// Split-KV decoding (bf16, d = 128, B_k = 128, group size <= 16).
constexpr int kMaxKvHeads = 64;
constexpr int kMaxGroup = 16;

struct DecodeParams {
  CUtensorMap tm_k;     // [B, Nk, Hkv, 128] as 4-D, box {64, 1, 128, 1}, 128B swizzle
  CUtensorMap tm_v;
  const void* q;        // [B, 1, Hq, 128]
  void* o;              // [B, 1, Hq, 128]
  float* lse;           // [B, Hq]
  uint32_t* keep_mask;  // [B, Hq, mask_words] (zeroed by the host before the launch)
  int64_t* stats;
  int* err;
  float* part_o;        // [B, Hq, P, 128] fp32 (P > 1)
  float* part_lse;      // [B, Hq, P]
  int64_t q_sb, q_sh, o_sb, o_sh;
  int B, Hq, Hkv, Nk, nKB, mask_words, num_splits;
  float log2_tau;
  int kv_fp8;           // K and V cache in e4m3 (tm_k / tm_v are then byte maps)
  float k_scale, v_scale;   // e4m3 cache scales (value = code * scale)
  int group_vote;       // one decision per key tile for the whole query-head group
  uint8_t group_size[kMaxKvHeads];
  uint8_t group_heads[kMaxKvHeads][kMaxGroup];
  uint64_t wait_ns;     // limit of every bounded wait (ns)
};

cudaError_t launch_decode(const DecodeParams& p, cudaStream_t stream);

// Backward (bf16, d = 128, B_q = B_k = 128, N_q <= N_k bottom-right aligned).
struct BwdParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_do;   // 4-D maps, box {64, 1, 128, 1}, 128B swizzle
  const float* nzl2;       // [B, Hq, Npad] -z log2e
  const float* Dv;         // [B, Hq, Npad] rowsum(dO o O)
  float* dq_acc;           // [B, Hq, nQB, 32 column quads, 128 rows, 4] fp32
  void* dk;
  void* dv;
  const uint32_t* fwd_mask;  // [B, Hq, nQB, mask_words] or NULL (visit every legal tile)
  uint32_t* bwd_mask;        // same layout, zeroed by the host, or NULL
  int64_t* stats;
  int* err;
  int64_t dk_sb, dk_sn, dk_sh, dv_sb, dv_sn, dv_sh;
  int B, Hq, Hkv, N, Npad, nQB, nKB, mask_words;   // N = N_q, Npad = nQB * 128
  int Nk, q_off;           // N_k >= N_q; query q sits at position q + q_off
  uint8_t group_size[kMaxKvHeads];
  uint8_t group_heads[kMaxKvHeads][kMaxGroup];
  SeqTable seq;            // packed sequences (B = their number; nQB / nKB maxima)
  uint64_t wait_ns;        // limit of every bounded wait (ns)
  float log2_tau;          // log2(tau): -inf for tau = 0, +inf for tau = inf
};

struct BwdAuxParams {      // pre-pass and dQ conversion
  const void* o;
  const void* dout;
  const float* lse;
  float* nzl2;
  float* Dv;
  float* dq_acc;
  void* dq;
  int64_t o_sb, o_sn, o_sh, do_sb, do_sn, do_sh, dq_sb, dq_sn, dq_sh;
  int B, Hq, N, Npad, nQB;   // N = N_q
  SeqTable seq;              // packed sequences (B = their number)
};

// Index of query block i of (batch or packed sequence b, query head h) in
// the [.., 128 rows] workspace blocks, the dQ accumulator and the mask rows:
// (b H_q + h) nQB + i for fixed lengths, h QB + qb0[b] + i for packed
// sequences (QB = all packed query blocks).
__host__ __device__ inline int64_t qblock_index(const SeqTable& seq, int Hq, int nQB, int b, int h, int i) {
  return seq.n == 0 ? (static_cast<int64_t>(b) * Hq + h) * nQB + i
                    : static_cast<int64_t>(h) * seq.qb0[seq.n] + seq.qb0[b] + i;
}

cudaError_t launch_bwd(const BwdParams& p, const BwdAuxParams& aux, cudaStream_t stream);
size_t bwd_smem_bytes();

}  // namespace mala
