// Rotary position encoding kernels: in-place rotation of prefill queries and
// keys, and the decode step's fused rotate-then-append of the new key into the
// ring cache (the rotation itself is in rope.cuh; the decode kernel rotates its
// query the same way).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "rope.cuh"
#include "swa_internal.h"

namespace swa {
namespace {

// One thread per (token, low-half chunk c): it computes the 8 angles of its
// chunk once and applies them to chunk c and its partner c + d/16 of every
// head of q and of k.  A warp covers 32 / (d/16) tokens, so each head's load
// instruction reads whole 128-byte lines.
__global__ void __launch_bounds__(256)
    swa_rope_qk_kernel(uint4* __restrict__ q, uint4* __restrict__ k, const int32_t* __restrict__ positions,
                       long long T, int Hq, int Hkv, int half_chunks, const __grid_constant__ RopeTable rt) {
  const long long n = T * half_chunks;
  const int vec = 2 * half_chunks;                        // 16-byte chunks per head row
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long t = i / half_chunks;
    const int c = static_cast<int>(i % half_chunks);
    const int p = positions[t];
    float cs[8], sn[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) rope_cos_sin(p, rt.theta[c * 8 + e], cs[e], sn[e]);
    auto rot = [&](uint4* row) {
      uint4 lo = row[c], hi = row[c + half_chunks];
      uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
      uint32_t* h = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
      for (int qd = 0; qd < 4; ++qd) {
        const float xl0 = __uint_as_float(l[qd] << 16), xl1 = __uint_as_float(l[qd] & 0xffff0000u);
        const float xh0 = __uint_as_float(h[qd] << 16), xh1 = __uint_as_float(h[qd] & 0xffff0000u);
        const int e = 2 * qd;
        __nv_bfloat162 a = __floats2bfloat162_rn(fmaf(xl0, cs[e], -xh0 * sn[e]), fmaf(xl1, cs[e + 1], -xh1 * sn[e + 1]));
        __nv_bfloat162 b = __floats2bfloat162_rn(fmaf(xl0, sn[e], xh0 * cs[e]), fmaf(xl1, sn[e + 1], xh1 * cs[e + 1]));
        l[qd] = *reinterpret_cast<uint32_t*>(&a);
        h[qd] = *reinterpret_cast<uint32_t*>(&b);
      }
      row[c] = lo;
      row[c + half_chunks] = hi;
    };
    for (int h = 0; h < Hq; ++h) rot(q + (t * Hq + h) * vec);
    if (k != nullptr)
      for (int h = 0; h < Hkv; ++h) rot(k + (t * Hkv + h) * vec);
  }
}

// One thread per (b, kv head, low-half chunk c): rotate k_new's chunks c and
// c + d/16 at pos[b], then store them (and v_new's two chunks) in ring slot
// pos mod W and, for pos < S, in sink slot pos.
__global__ void __launch_bounds__(256)
    swa_rope_append_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                           const int32_t* __restrict__ pos, uint4* kc, uint4* vc, uint4* sk, uint4* sv,
                           int B, int Hkv, int half_chunks, int W, int S, const __grid_constant__ RopeTable rt) {
  const long long n = static_cast<long long>(B) * Hkv * half_chunks;
  const int vec = 2 * half_chunks;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i % half_chunks);
    const long long bh = i / half_chunks;
    const int b = static_cast<int>(bh / Hkv);
    const int p = pos[b];
    if (p < 0) continue;
    uint4 lo = k[bh * vec + c], hi = k[bh * vec + c + half_chunks];
    rope_rotate_chunks(lo, hi, p, c * 8, rt.theta);
    const uint4 vlo = v[bh * vec + c], vhi = v[bh * vec + c + half_chunks];
    const size_t dst = (static_cast<size_t>(bh) * W + (p % W)) * vec;
    kc[dst + c] = lo;
    kc[dst + c + half_chunks] = hi;
    vc[dst + c] = vlo;
    vc[dst + c + half_chunks] = vhi;
    if (p < S) {
      const size_t ds = (static_cast<size_t>(bh) * S + p) * vec;
      sk[ds + c] = lo;
      sk[ds + c + half_chunks] = hi;
      sv[ds + c] = vlo;
      sv[ds + c + half_chunks] = vhi;
    }
  }
}

}  // namespace

void make_rope_table(double base, int d, RopeTable* t) {
  for (int i = 0; i < 64; ++i) t->theta[i] = i < d / 2 ? std::pow(base, -2.0 * i / d) : 0.0;
}

cudaError_t launch_rope_qk(void* q, void* k, const int32_t* positions, long long T, int Hq, int Hkv,
                           int d, const RopeTable& rt, cudaStream_t stream) {
  const int half_chunks = d / 16;
  const long long n = T * half_chunks;
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = std::min<long long>((n + threads - 1) / threads, 148LL * 32);
  swa_rope_qk_kernel<<<static_cast<int>(blocks), threads, 0, stream>>>(
      static_cast<uint4*>(q), static_cast<uint4*>(k), positions, T, Hq, Hkv, half_chunks, rt);
  return cudaGetLastError();
}

cudaError_t launch_rope_append(const void* k, const void* v, const int32_t* pos, void* kc, void* vc,
                               void* sk, void* sv, int B, int Hkv, int d, int W, int S,
                               const RopeTable& rt, cudaStream_t stream) {
  const int half_chunks = d / 16;
  const long long n = static_cast<long long>(B) * Hkv * half_chunks;
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const long long blocks = std::min<long long>((n + threads - 1) / threads, 148LL * 16);
  swa_rope_append_kernel<<<static_cast<int>(blocks), threads, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), pos, static_cast<uint4*>(kc),
      static_cast<uint4*>(vc), static_cast<uint4*>(sk), static_cast<uint4*>(sv), B, Hkv, half_chunks, W, S,
      rt);
  return cudaGetLastError();
}

}  // namespace swa
