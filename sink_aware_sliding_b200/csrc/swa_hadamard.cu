// Hadamard output projection after attention ("Rethinking Attention Output
// Projection: Structured Hadamard Transforms for Efficient Transformers",
// section 2): z = alpha * (y H) + beta per token, H the orthonormal Sylvester
// Walsh-Hadamard matrix of size n = Hq * d, applied as a fast Walsh-Hadamard
// transform (log2 n butterfly stages of additions and subtractions) instead of
// a dense n x n product.
//
// The transform is a product of independent 2-point butterflies, one per bit of
// the element index, and butterflies on different bits commute, so each bit can
// be transformed wherever the data happens to sit.  A row is spread over NT
// threads holding J chunks of 8 consecutive elements each (one 16-byte bf16 load
// per chunk); element i = (j * NT + t) * 8 + e for chunk j of thread t, so every
// load and store instruction of a warp covers a contiguous span.  The bits of e
// and j are transformed inside the thread, the low five bits of t (the lane)
// with warp shuffles; rows wider than one warp finish the remaining (warp) bits
// after a single shared-memory transpose and write the result from there.  Rows
// of fewer than 256 elements share a warp.  Memory-bound: each element is read
// once and written once; the arithmetic is fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"

namespace swa {
namespace {

template <int LOGN>
struct HadCfg {
  static constexpr int N = 1 << LOGN;
  static constexpr int C = N / 8;                                    // chunks per row
  static constexpr int NT = C <= 32 ? C : (C / 4 > 32 ? C / 4 : 32);  // threads per row
  static constexpr int J = C / NT;                                   // chunks per thread
  static constexpr int CTA = NT >= 128 ? NT : 128;                   // threads per CTA
  static constexpr int ROWS = CTA / NT;                              // rows per CTA
  static constexpr size_t SMEM = NT > 32 ? sizeof(float) * ROWS * N : 0;
};

// 16-byte streaming load: each element is read once, so it skips L1.
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <bool OUT_F32>
__device__ __forceinline__ void store4(void* z, long long idx, float a, float b, float c, float d) {
  if constexpr (OUT_F32) {
    *reinterpret_cast<float4*>(static_cast<float*>(z) + idx) = make_float4(a, b, c, d);
  } else {
    uint2 w;
    w.x = pack_bf16x2(a, b);
    w.y = pack_bf16x2(c, d);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(z) + idx) = w;
  }
}

template <int LOGN, bool OUT_F32>
__global__ void __launch_bounds__(HadCfg<LOGN>::CTA)
    swa_hadamard_kernel(const __nv_bfloat16* __restrict__ y, const float* __restrict__ alpha,
                        const float* __restrict__ beta, void* __restrict__ z, long long n_rows) {
  using Cfg = HadCfg<LOGN>;
  constexpr int N = Cfg::N, NT = Cfg::NT, J = Cfg::J, ROWS = Cfg::ROWS;
  extern __shared__ float xs[];                           // ROWS x N, when NT > 32
  const int tr = threadIdx.x % NT;                        // thread within its row
  const int rr = threadIdx.x / NT;                        // row within the CTA
  const long long row = static_cast<long long>(blockIdx.x) * ROWS + rr;
  const bool live = row < n_rows;
  const float inv_sqrt_n = rsqrtf(static_cast<float>(N));

  float x[J][8];
  {
    uint4 w[J];
#pragma unroll
    for (int j = 0; j < J; ++j) {
      w[j] = make_uint4(0, 0, 0, 0);
      if (live) w[j] = ld_nc_v4(y + row * N + (j * NT + tr) * 8);
    }
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const uint32_t u[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        x[j][2 * i] = __uint_as_float(u[i] << 16);
        x[j][2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
      }
    }
  }
  // bits of e (element within the chunk) and of j (chunk within the thread)
#pragma unroll
  for (int j = 0; j < J; ++j)
#pragma unroll
    for (int s = 1; s < 8; s <<= 1)
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if ((e & s) == 0) {
          const float a = x[j][e], b = x[j][e + s];
          x[j][e] = a + b;
          x[j][e + s] = a - b;
        }
#pragma unroll
  for (int s = 1; s < J; s <<= 1)
#pragma unroll
    for (int j = 0; j < J; ++j)
      if ((j & s) == 0)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float a = x[j][e], b = x[j + s][e];
          x[j][e] = a + b;
          x[j + s][e] = a - b;
        }
  // low bits of t: warp shuffles (a warp holds whole rows when NT < 32)
#pragma unroll
  for (int s = 1; s < (NT < 32 ? NT : 32); s <<= 1) {
    const bool upper = (tr & s) != 0;
#pragma unroll
    for (int j = 0; j < J; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float p = __shfl_xor_sync(0xffffffffu, x[j][e], s);
        x[j][e] = upper ? p - x[j][e] : x[j][e] + p;
      }
  }

  if constexpr (NT <= 32) {
    if (!live) return;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int c0 = (j * NT + tr) * 8;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float4 a = *reinterpret_cast<const float4*>(alpha + c0 + 4 * h);
        const float4 b = *reinterpret_cast<const float4*>(beta + c0 + 4 * h);
        const float* v = &x[j][4 * h];
        store4<OUT_F32>(z, row * N + c0 + 4 * h, fmaf(a.x, v[0] * inv_sqrt_n, b.x),
                        fmaf(a.y, v[1] * inv_sqrt_n, b.y), fmaf(a.z, v[2] * inv_sqrt_n, b.z),
                        fmaf(a.w, v[3] * inv_sqrt_n, b.w));
      }
    }
  } else {
    // warp bits of t: one transpose through shared memory.  Write every chunk at its
    // element position (the two 16-byte halves in an order that keeps the eight
    // lanes of each quarter-warp on distinct banks), then each thread reads the
    // 2^NW quads that differ only in the warp bits, finishes them and stores.
    constexpr int NW = NT == 64 ? 1 : NT == 128 ? 2 : NT == 256 ? 3 : NT == 512 ? 4 : 5;  // warp bits
    constexpr int NWV = 1 << NW;
    constexpr int GPT = 8 * N / (NT * NT);                // quad groups per thread
    static_assert(GPT * NT * NWV * 4 == N, "quad groups must tile the row");
    float* mine = xs + rr * N;
    const int flip = (tr >> 2) & 1;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      float4* c4 = reinterpret_cast<float4*>(mine + (j * NT + tr) * 8);
      const float4 lo = make_float4(x[j][0], x[j][1], x[j][2], x[j][3]);
      const float4 hi = make_float4(x[j][4], x[j][5], x[j][6], x[j][7]);
      c4[flip] = flip ? hi : lo;
      c4[flip ^ 1] = flip ? lo : hi;
    }
    __syncthreads();
    if (!live) return;
#pragma unroll
    for (int k = 0; k < GPT; ++k) {
      const int g = k * NT + tr;
      const int qbase = (g & 63) | ((g >> 6) << (6 + NW));
      float v[NWV][4];
#pragma unroll
      for (int w = 0; w < NWV; ++w) {
        const float4 t = *reinterpret_cast<const float4*>(mine + 4 * (qbase | (w << 6)));
        v[w][0] = t.x; v[w][1] = t.y; v[w][2] = t.z; v[w][3] = t.w;
      }
#pragma unroll
      for (int s = 1; s < NWV; s <<= 1)
#pragma unroll
        for (int w = 0; w < NWV; ++w)
          if ((w & s) == 0)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float a = v[w][c], b = v[w + s][c];
              v[w][c] = a + b;
              v[w + s][c] = a - b;
            }
#pragma unroll
      for (int w = 0; w < NWV; ++w) {
        const int e0 = 4 * (qbase | (w << 6));
        const float4 a = *reinterpret_cast<const float4*>(alpha + e0);
        const float4 b = *reinterpret_cast<const float4*>(beta + e0);
        store4<OUT_F32>(z, row * N + e0, fmaf(a.x, v[w][0] * inv_sqrt_n, b.x),
                        fmaf(a.y, v[w][1] * inv_sqrt_n, b.y), fmaf(a.z, v[w][2] * inv_sqrt_n, b.z),
                        fmaf(a.w, v[w][3] * inv_sqrt_n, b.w));
      }
    }
  }
}

template <int LOGN, bool OUT_F32>
cudaError_t launch_hadamard_impl(const void* y, const float* alpha, const float* beta, void* z,
                                 long long n_rows, cudaStream_t stream) {
  using Cfg = HadCfg<LOGN>;
  const long long blocks = (n_rows + Cfg::ROWS - 1) / Cfg::ROWS;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  auto kern = swa_hadamard_kernel<LOGN, OUT_F32>;
  if (Cfg::SMEM > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Cfg::SMEM));
    if (e != cudaSuccess) return e;
  }
  kern<<<static_cast<unsigned>(blocks), Cfg::CTA, Cfg::SMEM, stream>>>(
      static_cast<const __nv_bfloat16*>(y), alpha, beta, z, n_rows);
  return cudaGetLastError();
}

template <bool OUT_F32>
cudaError_t dispatch(int logn, const void* y, const float* alpha, const float* beta, void* z,
                     long long n_rows, cudaStream_t stream) {
  switch (logn) {
    case 5: return launch_hadamard_impl<5, OUT_F32>(y, alpha, beta, z, n_rows, stream);
    case 6: return launch_hadamard_impl<6, OUT_F32>(y, alpha, beta, z, n_rows, stream);
    case 7: return launch_hadamard_impl<7, OUT_F32>(y, alpha, beta, z, n_rows, stream);
    case 8: return launch_hadamard_impl<8, OUT_F32>(y, alpha, beta, z, n_rows, stream);
    case 9: return launch_hadamard_impl<9, OUT_F32>(y, alpha, beta, z, n_rows, stream);
    case 10: return launch_hadamard_impl<10, OUT_F32>(y, alpha, beta, z, n_rows, stream);
    case 11: return launch_hadamard_impl<11, OUT_F32>(y, alpha, beta, z, n_rows, stream);
    case 12: return launch_hadamard_impl<12, OUT_F32>(y, alpha, beta, z, n_rows, stream);
    case 13: return launch_hadamard_impl<13, OUT_F32>(y, alpha, beta, z, n_rows, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_hadamard(const void* y, const float* alpha, const float* beta, void* z,
                            long long n_rows, int n, bool out_f32, cudaStream_t stream) {
  int logn = 0;
  while ((1 << logn) < n) ++logn;
  return out_f32 ? dispatch<true>(logn, y, alpha, beta, z, n_rows, stream)
                 : dispatch<false>(logn, y, alpha, beta, z, n_rows, stream);
}

}  // namespace swa
