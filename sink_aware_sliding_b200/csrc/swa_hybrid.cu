// One decode step of a Based-style hybrid layer in a single launch ("Simple linear
// attention language models balance the recall-throughput tradeoff", proposed
// method: a short sliding window and a linear attention side by side; abstract:
// generation throughput).  Every generated token needs, per sequence, the window
// branch (append the new key and value to the ring cache, attend over the window
// and the sinks) and the linear branch (its recurrent state step).  Both are
// HBM-bound and small per head, so one grid runs them together: the first
// B * H_l blocks take one (sequence, head) step of the linear branch each (the
// larger share of the bytes, so it starts first), the rest one (sequence, query
// head) of the window branch each.
//
// Window branch (d = 64, window + n_sink <= 512): visible keys of position p are
// the ring positions max(0, p - W + 1) .. p and the sinks j < min(S, p - W + 1)
// ("Sliding-window beats linear attention", sections 1 and 3).  The newest key
// and value are read from the step's inputs, not from the ring: the block that
// owns a KV head (query head h with h mod G == 0) writes them into ring slot
// p mod W (and sink slot p when p < S) during the same step, and no block reads
// those slots in this step (slot p mod W held position p - W, which has left the
// window, and sink slot p is not visible from p).  Scores by one thread per key,
// a block-wide max and sum, then P V with a warp per group of keys reading whole
// 128-byte value rows.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "based_linear_decode.cuh"
#include "ptx.cuh"
#include "swa_internal.h"

namespace swa {
namespace {

constexpr int kHybThreads = lin::kDecThreads;   // 256
constexpr int kHybD = 64;
constexpr int kHybMaxKeys = 2 * kHybThreads;    // two keys per thread in the score step
constexpr int kKeyGroups = kHybThreads / 32;    // warps in the P V step

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Key or value row of visible key number idx (0 = the newest position) of (b, kvh).
__device__ __forceinline__ const __nv_bfloat16* key_row(const HybridArgs& a, const __nv_bfloat16* fresh,
                                                        const __nv_bfloat16* ring, const __nv_bfloat16* sinks,
                                                        int b, int kvh, int p, int n_ring, int idx) {
  const size_t seg = static_cast<size_t>(b) * a.Hkv + kvh;
  if (idx == 0) return fresh + seg * kHybD;
  if (idx < n_ring) return ring + (seg * a.W + static_cast<size_t>((p - idx) % a.W)) * kHybD;
  return sinks + (seg * a.S + static_cast<size_t>(idx - n_ring)) * kHybD;
}

__device__ __forceinline__ float block_reduce(float x, float* red, int tid, bool is_max) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, x, o);
    x = is_max ? fmaxf(x, y) : x + y;
  }
  if ((tid & 31) == 0) red[tid >> 5] = x;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < kHybThreads / 32; ++w) r = is_max ? fmaxf(r, red[w]) : r + red[w];
  __syncthreads();
  return r;
}

__device__ __forceinline__ void window_step(const HybridArgs& a, int bh, int tid) {
  __shared__ float qs[kHybD];
  __shared__ float ps[kHybMaxKeys];
  __shared__ float red[kHybThreads / 32];
  __shared__ float2 opart[kKeyGroups][kHybD / 2];
  const int b = bh / a.Hq, h = bh % a.Hq, kvh = h / a.G;
  const int p = a.pos[b];                        // >= 0 (documented); a negative one touches no memory
  const int n_ring = max(min(p + 1, a.W), 0);
  const int n = n_ring + min(max(p - a.W + 1, 0), a.S);
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);
  if (tid < kHybD) qs[tid] = __bfloat162float(q[static_cast<size_t>(bh) * kHybD + tid]) * a.scale_log2;
  if (p >= 0 && h % a.G == 0 && tid < 2 * (kHybD / 8)) {
    // append: 8 threads copy the key, 8 the value (16 bytes each)
    const bool is_v = tid >= kHybD / 8;
    const int c = tid % (kHybD / 8);
    const size_t seg = static_cast<size_t>(b) * a.Hkv + kvh;
    const uint4 x = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(is_v ? a.v_new : a.k_new) +
                                                   seg * kHybD)[c];
    reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(is_v ? a.vcache : a.kcache) +
                             (seg * a.W + static_cast<size_t>(p % a.W)) * kHybD)[c] = x;
    if (p < a.S)
      reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(is_v ? a.sink_v : a.sink_k) +
                               (seg * a.S + static_cast<size_t>(p)) * kHybD)[c] = x;
  }
  __syncthreads();
  const __nv_bfloat16* kn = static_cast<const __nv_bfloat16*>(a.k_new);
  const __nv_bfloat16* vn = static_cast<const __nv_bfloat16*>(a.v_new);
  const __nv_bfloat16* kc = static_cast<const __nv_bfloat16*>(a.kcache);
  const __nv_bfloat16* vc = static_cast<const __nv_bfloat16*>(a.vcache);
  const __nv_bfloat16* sk = static_cast<const __nv_bfloat16*>(a.sink_k);
  const __nv_bfloat16* sv = static_cast<const __nv_bfloat16*>(a.sink_v);
  // scores (log2 units) of keys tid and tid + 256
  float sc[2];
  float m = -INFINITY;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int idx = tid + kHybThreads * r;
    sc[r] = -INFINITY;
    if (idx < n) {
      const uint4* kr = reinterpret_cast<const uint4*>(key_row(a, kn, kc, sk, b, kvh, p, n_ring, idx));
      float acc = 0.f;
#pragma unroll
      for (int c = 0; c < kHybD / 8; ++c) {
        const uint4 w = kr[c];
        acc = fmaf(qs[8 * c + 0], bf16_lo(w.x), acc);
        acc = fmaf(qs[8 * c + 1], bf16_hi(w.x), acc);
        acc = fmaf(qs[8 * c + 2], bf16_lo(w.y), acc);
        acc = fmaf(qs[8 * c + 3], bf16_hi(w.y), acc);
        acc = fmaf(qs[8 * c + 4], bf16_lo(w.z), acc);
        acc = fmaf(qs[8 * c + 5], bf16_hi(w.z), acc);
        acc = fmaf(qs[8 * c + 6], bf16_lo(w.w), acc);
        acc = fmaf(qs[8 * c + 7], bf16_hi(w.w), acc);
      }
      sc[r] = acc;
      m = fmaxf(m, acc);
    }
  }
  const float M = block_reduce(m, red, tid, true);
  float l = 0.f;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int idx = tid + kHybThreads * r;
    if (idx < n) {
      const float e = ex2_approx(sc[r] - M);
      ps[idx] = e;
      l += e;
    }
  }
  const float Lsum = block_reduce(l, red, tid, false);   // its barriers also publish ps
  // O: warp kg takes keys kg, kg + 8, ...; lane dp the value dims 2 dp, 2 dp + 1
  const int dp = tid & 31, kg = tid >> 5;
  float2 acc = make_float2(0.f, 0.f);
  constexpr int kBatch = 8;                      // value rows in flight per warp
  for (int i0 = kg; i0 < n; i0 += kBatch * kKeyGroups) {
    uint32_t w[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int idx = i0 + u * kKeyGroups;
      w[u] = idx < n ? reinterpret_cast<const uint32_t*>(key_row(a, vn, vc, sv, b, kvh, p, n_ring, idx))[dp] : 0u;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int idx = i0 + u * kKeyGroups;
      const float e = idx < n ? ps[idx] : 0.f;
      acc.x = fmaf(e, bf16_lo(w[u]), acc.x);
      acc.y = fmaf(e, bf16_hi(w[u]), acc.y);
    }
  }
  opart[kg][dp] = acc;
  __syncthreads();
  if (tid < kHybD / 2) {
    float2 o = opart[0][tid];
#pragma unroll
    for (int g = 1; g < kKeyGroups; ++g) {
      o.x += opart[g][tid].x;
      o.y += opart[g][tid].y;
    }
    const float inv = 1.0f / Lsum;
    reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(a.out) + static_cast<size_t>(bh) * kHybD)[tid] =
        __floats2bfloat162_rn(o.x * inv, o.y * inv);
    if (tid == 0 && a.lse != nullptr) a.lse[bh] = (M + log2f(Lsum)) * 0.69314718055994531f;
  }
}

// Five blocks per SM (48 registers, a few bytes spilled): measured 4% faster than
// four (64 registers, no spill); six spill too much and are slower.
__global__ void __launch_bounds__(kHybThreads, 5) swa_hybrid_decode_kernel(const __grid_constant__ HybridArgs a) {
  const int n_lin = a.B * a.H_l;
  if (static_cast<int>(blockIdx.x) < n_lin) {
    lin::decode_step(blockIdx.x, threadIdx.x, static_cast<const __nv_bfloat16*>(a.ql),
                     static_cast<const __nv_bfloat16*>(a.kl), static_cast<const __nv_bfloat16*>(a.vl), a.state, a.zsum,
                     a.out_l, a.scale_l, 0);
  } else {
    window_step(a, static_cast<int>(blockIdx.x) - n_lin, threadIdx.x);
  }
}

}  // namespace

bool hybrid_window_supported(int d, int window, int n_sink) {
  return d == kHybD && window >= 1 && n_sink >= 0 && window + n_sink <= kHybMaxKeys;
}

cudaError_t launch_hybrid_decode(const HybridArgs& a, cudaStream_t stream) {
  const long long blocks = static_cast<long long>(a.B) * a.H_l + static_cast<long long>(a.B) * a.Hq;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  swa_hybrid_decode_kernel<<<static_cast<unsigned>(blocks), kHybThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace swa
