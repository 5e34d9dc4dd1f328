// The linear-attention branch of the Based hybrid ("Simple linear attention
// language models balance the recall-throughput tradeoff", proposed method:
// linear attention whose feature dimension sets the recurrent state, no position
// encoding).  Reading of "linear attention" (a kernel approximation of softmax
// attention, per "Sliding-window beats linear attention", section 1): the
// second-order Taylor kernel of exp,
//     kappa(q, k) = 1 + x + x^2 / 2,  x = scale * q.k,
// with features phi(u) = [1, sqrt(scale) u, scale vec(u u^T) / sqrt(2)]
// (F = 1 + dk + dk^2, the outer product row-major), state S = sum phi(k) v^T
// [F, dv] and z = sum phi(k) [F], and out_t = phi(q_t) S_t / phi(q_t).z_t.
//
// dk = 16 and dv = 64 (F = 273).  Prefill walks each (sequence, head) in
// chunks: the output of a chunk is phi(Q) S (the earlier chunks, from the state)
// plus the causal kappa(Q K^T) V of the chunk itself, normalised by the same
// two terms with v replaced by 1; then S += phi(K)^T V.  The tensor-core kernel
// (swa_based_linear_tc.cu) does this with tcgen05; this file holds the CUDA-core
// form of the same chunked step (fp32 throughout) and the decode step, which
// reads and writes the state in global memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "based_linear.h"
#include "based_linear_decode.cuh"

namespace swa {
namespace {

constexpr int kDK = 16;
constexpr int kDV = 64;
constexpr int kF = 1 + kDK + kDK * kDK;        // 273
constexpr int kCols = kDV + 1;                 // the S columns and the z column
constexpr int kGroups = 4;                     // feature ranges
constexpr int kFPer = (kF + kGroups - 1) / kGroups;   // 69
constexpr int kThreads = 288;                  // 4 x 65 = 260 working threads, 9 warps
constexpr int kChunk = 64;

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p, long long i) { return __bfloat162float(p[i]); }

using lin::feature;

__global__ void __launch_bounds__(kThreads, 1)
    swa_based_linear_fwd_simt_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                                const __nv_bfloat16* __restrict__ v, void* __restrict__ out, float* __restrict__ state,
                                float* __restrict__ zsum, int L, int H, float scale, int out_f32) {
  extern __shared__ float sm[];
  float* qs = sm;                               // [kChunk][kDK]
  float* ks = qs + kChunk * kDK;                // [kChunk][kDK]
  float* vs = ks + kChunk * kDK;                // [kChunk][kCols] (column 64 = 1)
  float* phi = vs + kChunk * kCols;             // [kChunk][kF]: phi(Q), then phi(K)
  float* part = phi + kChunk * kF;              // [kGroups][kChunk][kCols]
  float* amat = part + kGroups * kChunk * kCols;   // [kChunk][kChunk] causal kappa(Q K^T)

  const int b = blockIdx.x / H, h = blockIdx.x % H;
  const int tid = threadIdx.x;
  const bool worker = tid < kGroups * kCols;
  const int c = tid % kCols, g = tid / kCols;
  const int f0 = g * kFPer, f1 = min(kF, f0 + kFPer);
  const float rs = sqrtf(scale), s_over_r2 = scale * 0.70710678118654752f;

  float S[kFPer];
#pragma unroll
  for (int i = 0; i < kFPer; ++i) S[i] = 0.f;

  for (int t0 = 0; t0 < L; t0 += kChunk) {
    const int n = min(kChunk, L - t0);
    // inputs of the chunk (rows past the end are zero and never stored)
    for (int i = tid; i < kChunk * kDK; i += kThreads) {
      const int t = i / kDK, e = i % kDK;
      const long long row = (static_cast<long long>(b) * L + t0 + t) * H + h;
      qs[i] = t < n ? bf16_at(q, row * kDK + e) : 0.f;
      ks[i] = t < n ? bf16_at(k, row * kDK + e) : 0.f;
    }
    for (int i = tid; i < kChunk * kCols; i += kThreads) {
      const int t = i / kCols, e = i % kCols;
      const long long row = (static_cast<long long>(b) * L + t0 + t) * H + h;
      vs[i] = e == kDV ? 1.f : (t < n ? bf16_at(v, row * kDV + e) : 0.f);
    }
    __syncthreads();
    // phi(Q) of the chunk, and the causal kernel matrix of the chunk
    for (int i = tid; i < kChunk * kF; i += kThreads) phi[i] = feature(qs + (i / kF) * kDK, i % kF, rs, s_over_r2);
    for (int i = tid; i < kChunk * kChunk; i += kThreads) {
      const int t = i / kChunk, s = i % kChunk;
      float x = 0.f;
#pragma unroll
      for (int e = 0; e < kDK; ++e) x = fmaf(qs[t * kDK + e], ks[s * kDK + e], x);
      x *= scale;
      amat[i] = s <= t ? 1.f + x + 0.5f * x * x : 0.f;
    }
    __syncthreads();
    // earlier chunks: part[g][t][c] = sum over this thread's features of phi(q_t) S
    if (worker) {
      for (int t = 0; t < kChunk; ++t) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < kFPer; ++i)
          if (f0 + i < f1) acc = fmaf(phi[t * kF + f0 + i], S[i], acc);
        part[(g * kChunk + t) * kCols + c] = acc;
      }
    }
    __syncthreads();
    // this chunk: out = (sum_g part + kappa V) / (the same for the z column)
    if (worker) {
      for (int t = g * (kChunk / kGroups); t < (g + 1) * (kChunk / kGroups); ++t) {
        float acc = part[(0 * kChunk + t) * kCols + c] + part[(1 * kChunk + t) * kCols + c] +
                    part[(2 * kChunk + t) * kCols + c] + part[(3 * kChunk + t) * kCols + c];
        for (int s = 0; s <= t; ++s) acc = fmaf(amat[t * kChunk + s], vs[s * kCols + c], acc);
        part[t * kCols + c] = acc;            // group 0's slice now holds the totals of rows t
      }
    }
    __syncthreads();
    if (worker && c < kDV) {
      for (int t = g * (kChunk / kGroups); t < (g + 1) * (kChunk / kGroups); ++t) {
        if (t >= n) break;
        const float o = part[t * kCols + c] / part[t * kCols + kDV];
        const long long idx = ((static_cast<long long>(b) * L + t0 + t) * H + h) * kDV + c;
        if (out_f32) static_cast<float*>(out)[idx] = o;
        else static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(o);
      }
    }
    __syncthreads();
    // phi(K) over phi(Q), then S += phi(K)^T V
    for (int i = tid; i < kChunk * kF; i += kThreads) phi[i] = feature(ks + (i / kF) * kDK, i % kF, rs, s_over_r2);
    __syncthreads();
    if (worker) {
      for (int s = 0; s < n; ++s) {
        const float vv = vs[s * kCols + c];
#pragma unroll
        for (int i = 0; i < kFPer; ++i)
          if (f0 + i < f1) S[i] = fmaf(phi[s * kF + f0 + i], vv, S[i]);
      }
    }
    __syncthreads();
  }
  if (worker && state != nullptr) {
    const long long bh = static_cast<long long>(b) * H + h;
#pragma unroll
    for (int i = 0; i < kFPer; ++i) {
      if (f0 + i >= f1) break;
      if (c < kDV) state[(bh * kF + f0 + i) * kDV + c] = S[i];
      else if (zsum != nullptr) zsum[bh * kF + f0 + i] = S[i];
    }
  }
}

// One decode step per (sequence, head) (lin::decode_step); 64 registers, so that
// four CTAs share an SM and one CTA's stores overlap another's loads.
__global__ void __launch_bounds__(lin::kDecThreads, 4)
    swa_based_linear_decode_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                                   const __nv_bfloat16* __restrict__ v, float* __restrict__ state,
                                   float* __restrict__ zsum, void* __restrict__ out, float scale, int out_f32) {
  lin::decode_step(blockIdx.x, threadIdx.x, q, k, v, state, zsum, out, scale, out_f32);
}

}  // namespace

int based_linear_features(int dk) { return 1 + dk + dk * dk; }

cudaError_t launch_based_linear_fwd_simt(const BasedLinearArgs& a, cudaStream_t stream) {
  const size_t smem = sizeof(float) * (2 * kChunk * kDK + kChunk * kCols + kChunk * kF +
                                       kGroups * kChunk * kCols + kChunk * kChunk);
  cudaError_t e = cudaFuncSetAttribute(swa_based_linear_fwd_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  swa_based_linear_fwd_simt_kernel<<<a.B * a.H, kThreads, smem, stream>>>(
      static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
      static_cast<const __nv_bfloat16*>(a.v), a.out, a.state, a.zsum, a.L, a.H, a.scale, a.out_f32);
  return cudaGetLastError();
}

cudaError_t launch_based_linear_decode(const void* q, const void* k, const void* v, float* state, float* zsum,
                                       void* out, int B, int H, float scale, bool out_f32, cudaStream_t stream) {
  swa_based_linear_decode_kernel<<<B * H, lin::kDecThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), state, zsum, out, scale, out_f32 ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace swa
