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
// threads holding E = 64 elements each (J = 8 chunks of 8 consecutive elements,
// one 16-byte bf16 load per chunk; element i = (j * NT + t) * 8 + e for chunk j
// of thread t, so every load of a warp covers a contiguous span).  Three passes,
// each transforming the bits that are inside the thread at that point:
//   1. registers as loaded: the bits of e (0..2) and of j (the top bits);
//   2. after a transpose through shared memory: up to five bits of t (3..7),
//      read as 8-byte pairs (elements i, i+1) spaced 8 elements apart;
//   3. after a second pass through shared memory: the remaining R bits of t,
//      read as 2^R chunks of 8 consecutive elements, which are then scaled,
//      shifted and stored with 16-byte stores.
// The exchange goes through shared memory rather than warp shuffles (a shuffle
// stage moves every value once per bit; a shared-memory pass moves it once for
// up to five bits).  The arithmetic runs on packed fp32 pairs (one instruction
// for two butterflies); the pairs lie along bit 0, so only pass 1's bit-0 stage
// is scalar.  The fp32 buffer is padded (4 floats after every 32, 8 after every
// 2^(3+P2)) so pass 2's pair reads and the chunk accesses of passes 1 and 3
// touch distinct banks, and pass 2's offsets are compile-time constants.
// Memory-bound in principle (each element read once and written once; 8 bytes
// of HBM traffic per element for bf16 in and out), issue-bound in practice, so
// the design minimises instructions per element.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "ptx.cuh"
#include "swa_internal.h"

namespace swa {
namespace {


template <int LOGN>
struct HadCfg {
  static constexpr int N = 1 << LOGN;
  static constexpr int E = N < 64 ? N : 64;               // elements per thread
  static constexpr int J = E / 8;                         // chunks per thread
  static constexpr int LOGJ = J == 8 ? 3 : 2;
  static constexpr int NT = N / E;                        // threads per row
  static constexpr int TB = LOGN - 3 - LOGJ;              // bits of t
  static constexpr int P2 = TB < 5 ? TB : 5;              // bits done in pass 2
  static constexpr int R = TB - P2;                       // bits done in pass 3
  static constexpr int CTA = NT >= 256 ? NT : 256;        // threads per CTA
  static constexpr int ROWS = CTA / NT;                   // rows per CTA
  // padded fp32 row in shared memory (floats), a multiple of 4
  static constexpr int XROW = TB > 0 ? ((N + N / 8 + ((8 * N) >> (3 + P2)) + 3) / 4) * 4 : 0;
  static constexpr size_t SMEM = sizeof(float) * ROWS * XROW;
  static_assert(R <= LOGJ, "pass 3 groups must fit a thread");
};

// Padded position of element i in a row's fp32 exchange buffer (strictly
// increasing, so one-to-one; keeps runs of 8 elements aligned to 8 contiguous).
template <int P2>
__device__ __forceinline__ int xpos(int i) {
  return i + 4 * (i >> 5) + 8 * (i >> (3 + P2));
}

// 16-byte streaming load: each element is read once, so it skips L1.
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// Butterflies over the index of M packed pairs (M a power of two).
template <int M>
__device__ __forceinline__ void fwht_pairs(uint64_t (&p)[M]) {
#pragma unroll
  for (int s = 1; s < M; s <<= 1)
#pragma unroll
    for (int a = 0; a < M; ++a)
      if ((a & s) == 0) {
        const uint64_t u = p[a], v = p[a + s];
        p[a] = f2_add(u, v);
        p[a + s] = f2_sub(u, v);
      }
}

// Scale, shift and store n_pairs pairs of consecutive outputs at element e0 of
// the row, given alpha (a) and beta (b) of those elements as packed pairs.
template <bool OUT_F32, int NP>
__device__ __forceinline__ void store_pairs(const uint64_t* v, const uint64_t* a, const uint64_t* b, uint64_t inv2,
                                            void* __restrict__ z, long long off) {
  float o[2 * NP];
#pragma unroll
  for (int q = 0; q < NP; ++q) f2_unpack(f2_fma(a[q], f2_mul(v[q], inv2), b[q]), o[2 * q], o[2 * q + 1]);
  if constexpr (OUT_F32) {
#pragma unroll
    for (int q = 0; q < NP; q += 2)
      *reinterpret_cast<float4*>(static_cast<float*>(z) + off + 2 * q) =
          make_float4(o[2 * q], o[2 * q + 1], o[2 * q + 2], o[2 * q + 3]);
  } else if constexpr (NP == 2) {
    uint2 w;
    w.x = pack_bf16x2(o[0], o[1]);
    w.y = pack_bf16x2(o[2], o[3]);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(z) + off) = w;
  } else {
#pragma unroll
    for (int q = 0; q < NP; q += 4) {
      uint4 w;
      w.x = pack_bf16x2(o[2 * q], o[2 * q + 1]);
      w.y = pack_bf16x2(o[2 * q + 2], o[2 * q + 3]);
      w.z = pack_bf16x2(o[2 * q + 4], o[2 * q + 5]);
      w.w = pack_bf16x2(o[2 * q + 6], o[2 * q + 7]);
      *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(z) + off + 2 * q) = w;
    }
  }
}

__device__ __forceinline__ void load_pairs4(const float* __restrict__ p, uint64_t* d) {
  const ulonglong2 t = *reinterpret_cast<const ulonglong2*>(p);
  d[0] = t.x;
  d[1] = t.y;
}

template <int LOGN, bool OUT_F32>
__global__ void __launch_bounds__(HadCfg<LOGN>::CTA)
    swa_hadamard_kernel(const __nv_bfloat16* __restrict__ y, const float* __restrict__ alpha,
                        const float* __restrict__ beta, void* __restrict__ z, long long n_rows) {
  using Cfg = HadCfg<LOGN>;
  constexpr int N = Cfg::N, E = Cfg::E, J = Cfg::J, NT = Cfg::NT, TB = Cfg::TB, P2 = Cfg::P2,
                R = Cfg::R, ROWS = Cfg::ROWS;
  extern __shared__ __align__(16) float xs[];             // ROWS x XROW, when TB > 0
  const int tr = threadIdx.x % NT;                        // thread within its row
  const int rr = threadIdx.x / NT;                        // row within the CTA
  const long long row = static_cast<long long>(blockIdx.x) * ROWS + rr;
  const bool live = row < n_rows;
  const long long row_off = row * N;
  const float inv = rsqrtf(static_cast<float>(N));
  const uint64_t inv2 = f2_pack(inv, inv);

  // pass 1: bits of e and j.  p[k] holds elements (2k, 2k+1) of the thread's
  // list x[j * 8 + e]: bit 0 inside the pair, the other bits along k.
  uint64_t p[E / 2];
  {
    uint4 w[J];
#pragma unroll
    for (int j = 0; j < J; ++j)
      w[j] = live ? ld_nc_v4(y + row_off + (j * NT + tr) * 8) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const uint32_t u[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float lo = __uint_as_float(u[q] << 16), hi = __uint_as_float(u[q] & 0xffff0000u);
        p[j * 4 + q] = f2_pack(lo + hi, lo - hi);         // the bit-0 stage, scalar
      }
    }
  }
  fwht_pairs<E / 2>(p);

  if constexpr (TB == 0) {
    if (!live) return;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      const int e0 = (j * NT + tr) * 8;
      uint64_t av[4], bv[4];
      load_pairs4(alpha + e0, av);
      load_pairs4(alpha + e0 + 4, av + 2);
      load_pairs4(beta + e0, bv);
      load_pairs4(beta + e0 + 4, bv + 2);
      store_pairs<OUT_F32, 4>(&p[j * 4], av, bv, inv2, z, row_off + e0);
    }
  } else {
    float* buf = xs + rr * Cfg::XROW;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      ulonglong2* c = reinterpret_cast<ulonglong2*>(buf + xpos<P2>((j * NT + tr) * 8));
      c[0] = make_ulonglong2(p[j * 4 + 0], p[j * 4 + 1]);
      c[1] = make_ulonglong2(p[j * 4 + 2], p[j * 4 + 3]);
    }
    __syncthreads();

    // pass 2: bits 3 .. 3+P2-1 on pairs (i, i+1); each group is read and written
    // back by the same thread
    constexpr int M2 = 1 << P2;
#pragma unroll
    for (int k = 0; k < E / (2 * M2); ++k) {
      const int g = k * NT + tr;
      const int base = ((g & 3) << 1) | ((g >> 2) << (3 + P2));
      uint64_t v[M2];
      if constexpr (P2 >= 2) {
        uint64_t* b = reinterpret_cast<uint64_t*>(buf + xpos<P2>(base));
#pragma unroll
        for (int m = 0; m < M2; ++m) v[m] = b[(8 * m + 4 * (m >> 2)) / 2];
        fwht_pairs<M2>(v);
#pragma unroll
        for (int m = 0; m < M2; ++m) b[(8 * m + 4 * (m >> 2)) / 2] = v[m];
      } else {
#pragma unroll
        for (int m = 0; m < M2; ++m) v[m] = *reinterpret_cast<uint64_t*>(buf + xpos<P2>(base + (m << 3)));
        fwht_pairs<M2>(v);
#pragma unroll
        for (int m = 0; m < M2; ++m) *reinterpret_cast<uint64_t*>(buf + xpos<P2>(base + (m << 3))) = v[m];
      }
    }
    __syncthreads();

    // pass 3: the remaining R bits on quads of consecutive elements; thread tau
    // takes quad groups lg, lg + GW, ... of rows team, team + TEAMS, ...
    // a row has GPR quad groups, covered by GW threads; the CTA's threads form
    // TEAMS teams and each thread applies one load of its alpha/beta to RPT rows
    constexpr int M3 = 1 << R;
    constexpr int GPR = N / (4 * M3);
    constexpr int GW = GPR < Cfg::CTA ? GPR : Cfg::CTA;
    constexpr int TEAMS = Cfg::CTA / GW;
    constexpr int GQ = GPR / GW;
    constexpr int RPT = ROWS / TEAMS;
    const int team = static_cast<int>(threadIdx.x) / GW, lg = static_cast<int>(threadIdx.x) % GW;
    const long long row0 = static_cast<long long>(blockIdx.x) * ROWS;
#pragma unroll
    for (int k = 0; k < GQ; ++k) {
      const int g = lg + k * GW;
      const int base = ((g & 1) << 2) | (((g >> 1) & ((1 << P2) - 1)) << 3) | ((g >> (1 + P2)) << (3 + TB));
      uint64_t av[M3][2], bv[M3][2];
#pragma unroll
      for (int w = 0; w < M3; ++w) {
        load_pairs4(alpha + base + (w << (3 + P2)), av[w]);
        load_pairs4(beta + base + (w << (3 + P2)), bv[w]);
      }
#pragma unroll 1
      for (int m = 0; m < RPT; ++m) {
        const int r = team + m * TEAMS;
        if (row0 + r >= n_rows) break;                    // rows of a team ascend
        const float* rb = xs + r * Cfg::XROW;
        uint64_t c[2][M3];                                // c[q][w]: pair q of quad w
#pragma unroll
        for (int w = 0; w < M3; ++w) {
          const ulonglong2 t = *reinterpret_cast<const ulonglong2*>(rb + xpos<P2>(base + (w << (3 + P2))));
          c[0][w] = t.x;
          c[1][w] = t.y;
        }
        fwht_pairs<M3>(c[0]);
        fwht_pairs<M3>(c[1]);
#pragma unroll
        for (int w = 0; w < M3; ++w) {
          const uint64_t o[2] = {c[0][w], c[1][w]};
          store_pairs<OUT_F32, 2>(o, av[w], bv[w], inv2, z, (row0 + r) * N + base + (w << (3 + P2)));
        }
      }
    }
  }
}

template <int LOGN, bool OUT_F32>
cudaError_t launch_hadamard_impl(const HadamardArgs& a, cudaStream_t stream) {
  using Cfg = HadCfg<LOGN>;
  const long long blocks = (a.n_rows + Cfg::ROWS - 1) / Cfg::ROWS;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  auto kern = swa_hadamard_kernel<LOGN, OUT_F32>;
  if (Cfg::SMEM > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Cfg::SMEM));
    if (e != cudaSuccess) return e;
  }
  kern<<<static_cast<unsigned>(blocks), Cfg::CTA, Cfg::SMEM, stream>>>(
      static_cast<const __nv_bfloat16*>(a.y), a.alpha, a.beta, a.z, a.n_rows);
  return cudaGetLastError();
}

template <bool OUT_F32>
cudaError_t dispatch(int logn, const HadamardArgs& a, cudaStream_t stream) {
  switch (logn) {
    case 5: return launch_hadamard_impl<5, OUT_F32>(a, stream);
    case 6: return launch_hadamard_impl<6, OUT_F32>(a, stream);
    case 7: return launch_hadamard_impl<7, OUT_F32>(a, stream);
    case 8: return launch_hadamard_impl<8, OUT_F32>(a, stream);
    case 9: return launch_hadamard_impl<9, OUT_F32>(a, stream);
    case 10: return launch_hadamard_impl<10, OUT_F32>(a, stream);
    case 11: return launch_hadamard_impl<11, OUT_F32>(a, stream);
    case 12: return launch_hadamard_impl<12, OUT_F32>(a, stream);
    case 13: return launch_hadamard_impl<13, OUT_F32>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_hadamard(const HadamardArgs& a, int n, bool out_f32, int sms, cudaStream_t stream) {
  int logn = 0;
  while ((1 << logn) < n) ++logn;
  (void)sms;
  return out_f32 ? dispatch<true>(logn, a, stream) : dispatch<false>(logn, a, stream);
}

}  // namespace swa
