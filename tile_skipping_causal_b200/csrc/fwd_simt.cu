// MALA forward (Algorithm 1, "Online Sparse Softmax") on CUDA cores.
//
// Serves fp32 inputs and block sizes the tensor-core kernel does not take.
// One CTA per (batch, query head, query block), one thread per query row.
// K and V tiles are staged in shared memory as fp32; every thread scores its
// row against the K tile (fp32 FMA), the CTA votes on the skip test with
// __syncthreads_or, and only a retained tile loads V and updates m, l, O.
// Natural exp/log in full fp32 precision.
#include <math.h>

#include "kernels.h"
#include "ptx.cuh"

namespace mala {

namespace {

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

template <typename T, int D>
__global__ void __launch_bounds__(128) mala_fwd_simt_kernel(const FwdSimtParams p) {
  extern __shared__ float sm[];
  const int BQ = p.BQ, BK = p.BK;
  float* sK = sm;                     // [BK][D]
  float* sV = sK + BK * D;            // [BK][D]
  float* sS = sV + BK * D;            // [BQ][BK + 1]
  const int SS = BK + 1;

  const int BH = p.B * p.Hq;
  const int i = p.nQB - 1 - static_cast<int>(blockIdx.x) / BH;
  const int bh = static_cast<int>(blockIdx.x) % BH;
  const int b = bh / p.Hq;
  const int h = bh % p.Hq;
  const int hk = p.kv_of_q[h];
  const int r = threadIdx.x;
  const int q0 = i * BQ;
  const int q = q0 + r;
  const bool valid = q < p.N;
  const int qa = q + p.q_off;                     // position of the row (bottom-right alignment)
  const int last_row = min(q0 + BQ - 1, p.N - 1);
  const int j_diag = min((last_row + p.q_off) / BK, p.nKB - 1);

  const T* Q = reinterpret_cast<const T*>(p.q);
  const T* K = reinterpret_cast<const T*>(p.k);
  const T* V = reinterpret_cast<const T*>(p.v);

  float qr[D];
  float acc[D];
#pragma unroll
  for (int x = 0; x < D; ++x) {
    qr[x] = valid ? to_f32(Q[b * p.q_sb + static_cast<int64_t>(q) * p.q_sn + h * p.q_sh + x]) : 0.0f;
    acc[x] = 0.0f;
  }
  const float thr = p.log_tau - logf(static_cast<float>(qa + 1));   // log(tau / L_q)
  float m = -INFINITY, l = 0.0f;
  uint32_t mask_word = 0;
  int kept_tiles = 0;
  const int mask_base = ((b * p.Hq + h) * p.nQB + i) * p.mask_words;
  if (r == 0 && p.keep_mask)
    for (int w = j_diag / 32 + 1; w < p.mask_words; ++w) p.keep_mask[mask_base + w] = 0u;

  for (int j = j_diag; j >= 0; --j) {
    const int k0 = j * BK;
    __syncthreads();
    for (int e = r; e < BK * D; e += BQ) {
      const int c = e / D, x = e % D, k = k0 + c;
      sK[e] = (k < p.Nk) ? to_f32(K[b * p.k_sb + static_cast<int64_t>(k) * p.k_sn + hk * p.k_sh + x]) : 0.0f;
    }
    __syncthreads();
    const int lim = qa - k0;                      // legal columns: c <= lim
    const bool has_key = valid && lim >= 0;
    float rmax = -INFINITY;
    for (int c = 0; c < BK; ++c) {
      float s = -INFINITY;
      if (has_key && c <= lim) {
        s = 0.0f;
#pragma unroll
        for (int x = 0; x < D; ++x) s = fmaf(qr[x], sK[c * D + x], s);
      }
      sS[r * SS + c] = s;
      rmax = fmaxf(rmax, s);
    }
    const bool vote = has_key && (l == 0.0f || rmax - (m + logf(l)) >= thr);
    const bool keep = __syncthreads_or(vote) != 0;
    if (r == 0) {
      if (keep) { mask_word |= 1u << (j & 31); ++kept_tiles; }
      if ((j & 31) == 0) {
        if (p.keep_mask) p.keep_mask[mask_base + (j >> 5)] = mask_word;
        mask_word = 0;
      }
    }
    if (!keep) continue;
    for (int e = r; e < BK * D; e += BQ) {
      const int c = e / D, x = e % D, k = k0 + c;
      sV[e] = (k < p.Nk) ? to_f32(V[b * p.v_sb + static_cast<int64_t>(k) * p.v_sn + hk * p.v_sh + x]) : 0.0f;
    }
    __syncthreads();
    if (has_key) {
      const float m_new = fmaxf(m, rmax);
      const float alpha = (l > 0.0f) ? expf(m - m_new) : 0.0f;
      l *= alpha;
#pragma unroll
      for (int x = 0; x < D; ++x) acc[x] *= alpha;
      for (int c = 0; c <= min(lim, BK - 1); ++c) {
        const float pr = expf(sS[r * SS + c] - m_new);
        l += pr;
#pragma unroll
        for (int x = 0; x < D; ++x) acc[x] = fmaf(pr, sV[c * D + x], acc[x]);
      }
      m = m_new;
    }
  }

  if (valid) {
    T* O = reinterpret_cast<T*>(p.o) + b * p.o_sb + static_cast<int64_t>(q) * p.o_sn + h * p.o_sh;
    const float inv = 1.0f / l;
#pragma unroll
    for (int x = 0; x < D; ++x) O[x] = from_f32<T>(acc[x] * inv);
    p.lse[(static_cast<int64_t>(b) * p.Hq + h) * p.N + q] = m + logf(l);
  }
  if (r == 0 && p.stats) {
    const int nvalid = last_row - q0 + 1;
    atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[0]), static_cast<unsigned long long>(j_diag + 1));
    atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[1]), static_cast<unsigned long long>(kept_tiles));
    atomicAdd(reinterpret_cast<unsigned long long*>(&p.stats[2]),
              static_cast<unsigned long long>(kept_tiles) * BK * nvalid);
  }
}

template <typename T, int D>
cudaError_t launch(const FwdSimtParams& p, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(p.B) * p.Hq * p.nQB;
  if (grid == 0) return cudaSuccess;
  const size_t smem = (2 * static_cast<size_t>(p.BK) * D + static_cast<size_t>(p.BQ) * (p.BK + 1)) * 4;
  cudaError_t e = cudaFuncSetAttribute(mala_fwd_simt_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  mala_fwd_simt_kernel<T, D><<<grid, p.BQ, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_fwd_simt(const FwdSimtParams& p, int head_dim, bool fp32, cudaStream_t stream) {
  if (fp32) return head_dim == 64 ? launch<float, 64>(p, stream) : launch<float, 128>(p, stream);
  return head_dim == 64 ? launch<__nv_bfloat16, 64>(p, stream) : launch<__nv_bfloat16, 128>(p, stream);
}

}  // namespace mala
