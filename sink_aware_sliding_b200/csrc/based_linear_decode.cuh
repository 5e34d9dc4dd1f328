// The recurrent decode step of the Based linear branch as a block-level device
// function, shared by the standalone decode kernel and the fused hybrid decode.
//
// Taylor-kernel linear attention (see swa_based_linear.cu for the reading of the
// Based page): features phi(u) = [1, sqrt(scale) u, scale vec(u u^T) / sqrt(2)]
// (F = 1 + dk + dk^2), state S = sum phi(k) v^T [F, dv], normaliser z = sum phi(k).
// One step for one (sequence, head): S += phi(k) v^T, z += phi(k),
// out = phi(q) S / phi(q).z.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

namespace swa {
namespace lin {

constexpr int kDK = 16;
constexpr int kDV = 64;
constexpr int kF = 1 + kDK + kDK * kDK;                    // 273
// 256 threads: thread (c4, g) owns columns 4 c4 .. 4 c4 + 3 of S for the features
// f = g, g + 16, ...; its rows are read in two batches of nine 16-byte loads, all in
// flight at once (the step is HBM-bound).
constexpr int kDecThreads = 256;
constexpr int kDecGroups = kDecThreads / (kDV / 4);        // 16
constexpr int kDecRows = (kF + kDecGroups - 1) / kDecGroups;  // 18 rows per group at most

// phi(u) entry f for u (dk values in shared memory).
__device__ __forceinline__ float feature(const float* u, int f, float rs, float s_over_r2) {
  if (f == 0) return 1.0f;
  if (f <= kDK) return rs * u[f - 1];
  const int p = f - 1 - kDK;
  return s_over_r2 * u[p / kDK] * u[p % kDK];
}

// One decode step for (sequence, head) bh, run by all kDecThreads threads of a block.
__device__ __forceinline__ void decode_step(long long bh, int tid, const __nv_bfloat16* __restrict__ q,
                                            const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                                            float* __restrict__ state, float* __restrict__ zsum,
                                            void* __restrict__ out, float scale, int out_f32) {
  __shared__ float qs[kDK], ks[kDK], fq[kF], fk[kF];
  __shared__ float4 part[kDecGroups][kDV / 4];
  __shared__ float zpart[kDecThreads / 32];
  const float rs = sqrtf(scale), s_over_r2 = scale * 0.70710678118654752f;
  if (tid < kDK) {
    qs[tid] = __bfloat162float(q[bh * kDK + tid]);
    ks[tid] = __bfloat162float(k[bh * kDK + tid]);
  }
  const int c4 = tid % (kDV / 4), g = tid / (kDV / 4);
  float4 vv;
  {
    const __nv_bfloat16* pv = v + bh * kDV + 4 * c4;
    vv = make_float4(__bfloat162float(pv[0]), __bfloat162float(pv[1]), __bfloat162float(pv[2]),
                     __bfloat162float(pv[3]));
  }
  __syncthreads();
  for (int f = tid; f < kF; f += kDecThreads) {
    fq[f] = feature(qs, f, rs, s_over_r2);
    fk[f] = feature(ks, f, rs, s_over_r2);
  }
  __syncthreads();
  float4* S4 = reinterpret_cast<float4*>(state + bh * kF * kDV) + c4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int h0 = 0; h0 < kDecRows; h0 += kDecRows / 2) {
    float4 row[kDecRows / 2];
#pragma unroll
    for (int i = 0; i < kDecRows / 2; ++i) {
      const int f = g + kDecGroups * (h0 + i);
      if (f < kF) row[i] = S4[f * (kDV / 4)];
    }
#pragma unroll
    for (int i = 0; i < kDecRows / 2; ++i) {
      const int f = g + kDecGroups * (h0 + i);
      if (f < kF) {
        const float a = fk[f], b = fq[f];
        float4 r = row[i];
        r.x = fmaf(a, vv.x, r.x);
        r.y = fmaf(a, vv.y, r.y);
        r.z = fmaf(a, vv.z, r.z);
        r.w = fmaf(a, vv.w, r.w);
        S4[f * (kDV / 4)] = r;
        acc.x = fmaf(b, r.x, acc.x);
        acc.y = fmaf(b, r.y, acc.y);
        acc.z = fmaf(b, r.z, acc.z);
        acc.w = fmaf(b, r.w, acc.w);
      }
    }
  }
  part[g][c4] = acc;
  // normaliser: z += phi(k), den = phi(q).z
  float zd = 0.f;
  for (int f = tid; f < kF; f += kDecThreads) {
    const float zn = zsum[bh * kF + f] + fk[f];
    zsum[bh * kF + f] = zn;
    zd = fmaf(fq[f], zn, zd);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) zd += __shfl_xor_sync(0xffffffffu, zd, o);
  if ((tid & 31) == 0) zpart[tid >> 5] = zd;
  __syncthreads();
  if (tid < kDV) {
    float den = 0.f;
#pragma unroll
    for (int i = 0; i < kDecThreads / 32; ++i) den += zpart[i];
    float num = 0.f;
    const int cc = tid >> 2, e = tid & 3;
#pragma unroll
    for (int i = 0; i < kDecGroups; ++i) {
      const float4 p = part[i][cc];
      num += e == 0 ? p.x : (e == 1 ? p.y : (e == 2 ? p.z : p.w));
    }
    const long long idx = bh * kDV + tid;
    if (out_f32) static_cast<float*>(out)[idx] = num / den;
    else static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(num / den);
  }
}

}  // namespace lin
}  // namespace swa
