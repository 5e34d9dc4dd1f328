// Prefill of the Based linear branch on the tensor cores (tcgen05, bf16
// operands, fp32 accumulators in tensor memory).  The method is the second-order
// Taylor linear attention described in swa_based_linear.cu ("Simple linear
// attention language models balance the recall-throughput tradeoff", proposed
// method): out_t = phi(q_t) S_t / phi(q_t).z_t with S_t = sum_{s<=t} phi(k_s) v_s^T.
//
// One CTA per (sequence, head) walks the sequence in chunks of 128 tokens.  With
// V1 = [V | 1 | 0...] (80 columns: the values, a column of ones that turns the
// same products into the normaliser, zero padding) a chunk is
//   X  = phi_lin(Q) phi_lin(K)^T                       (= scale q.k, K = 16)
//   O  = phi(Q) S_bf16  +  kappa_causal(X) V1           (S from earlier chunks)
//   S += phi(K)^T V1
// where kappa(x) = 1 + x + x^2/2 with the causal mask applied, and out = O[:, :64]
// / O[:, 64].  Features are kept in an internal order: the 256 products
// u_a u_b (a-major), then the 16 linear terms, then the constant, then zeros up to
// 384 = 3 x 128 feature rows, so that S is three 128-row accumulators.
//
// Roles (288 threads):
//   warps 0-3  token rows: q/k loads, phi(Q) and phi_lin(K) into shared memory,
//              kappa of X into P (bf16, over X's own tensor-memory columns),
//              phi(K), the output epilogue;
//   warps 4-7  state: V loads into V1, S (tensor memory, fp32) -> S_bf16 (shared,
//              the B operand of the next chunk), the final state;
//   warp 8     one thread issues every MMA.
// All waits on mbarriers are bounded; on a time-out the CTA stops, drains its
// MMAs, frees its tensor memory and records the status.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "based_linear.h"
#include "ptx.cuh"

namespace swa {
namespace {

namespace bl {
constexpr int kChunk = 128;                  // tokens per chunk (MMA M)
constexpr int kDK = 16, kDV = 64;
constexpr int kF = 1 + kDK + kDK * kDK;      // 273 features
constexpr int kNV = 80;                      // V1 columns: 64 values, the ones column, padding
constexpr int kQSteps = 18;                  // phi(Q) S_bf16 over features 0 .. 287 (K steps of 16)
constexpr int kThreads = 288;
constexpr int kMmaWarp = 8;
constexpr uint32_t kCh = kChunk * 128;       // one 64-column chunk of a 128-row operand: 16 KB
constexpr uint32_t kSbCh = kNV * 128;        // one 64-column chunk of S_bf16 (80 rows): 10 KB
constexpr uint32_t OFF_PHI = 0;              // [128 tokens x 384 features], 6 chunks
constexpr uint32_t OFF_KLIN = 6 * kCh;       // [128 tokens x 64]: phi_lin(K) in columns 0 .. 15
constexpr uint32_t OFF_V1 = 7 * kCh;         // values chunk, then the ones chunk
constexpr uint32_t OFF_SB = 9 * kCh;         // S_bf16 [80 columns of S x 384 features], 6 chunks
constexpr uint32_t OFF_BAR = OFF_SB + 6 * kSbCh;
enum { B_PHIQ, B_V1, B_X, B_O1, B_P, B_PHIK, B_OFULL, B_OFREE, B_SFULL, B_SB, B_DRAIN, kNumBars };
constexpr uint32_t OFF_TMEMPTR = OFF_BAR + kNumBars * 8;
constexpr uint32_t OFF_ABORT = OFF_TMEMPTR + 4;
constexpr uint32_t kSmemUsed = OFF_ABORT + 4;
constexpr uint32_t kSmem = kSmemUsed + 1024;  // slack to align the base to 1024 bytes
static_assert(kSmem <= 232448, "shared memory");
// tensor-memory columns
constexpr uint32_t T_X = 0;                  // X (fp32, 128 columns); P (bf16 pairs) over its first 64
constexpr uint32_t T_O = 128;                // O (80 columns)
constexpr uint32_t T_S = 256;                // S tile j at T_S + 80 j, j = 0 .. 2
// instruction descriptors (bf16 x bf16 -> fp32); bit 15 makes A MN-major
constexpr uint32_t IDESC_X = make_idesc(1, 128, 128, false);
constexpr uint32_t IDESC_QS = make_idesc(1, 128, kNV, false);
constexpr uint32_t IDESC_PV = make_idesc(1, 128, kNV, true);
constexpr uint32_t IDESC_KV = make_idesc(1, 128, kNV, true) | (1u << 15);
constexpr int kStatusTimeout = 4;            // SWA_ERR_DEVICE_TIMEOUT
}  // namespace bl

// K-major operand with 128-byte rows in 64-column chunks of `chunk` bytes: K step kk (16 columns).
__device__ __forceinline__ uint64_t bl_kdesc(uint32_t base, uint32_t chunk, int kk) {
  return smem_desc(base + (kk >> 2) * chunk + (kk & 3) * 32, 16, 1024, kLayoutSw128);
}
// MN-major operand (rows = K, 64-element chunks along M or N, `chunk` bytes apart): K step kk (16 rows).
__device__ __forceinline__ uint64_t bl_mndesc(uint32_t base, uint32_t chunk, int kk) {
  return smem_desc(base + kk * 16 * 128, chunk, 1024, kLayoutSw128);
}
// 16-byte granule g of row r in a 128-byte-swizzled chunk.
__device__ __forceinline__ uint32_t gran(uint32_t chunk_base, int r, int g) {
  return chunk_base + r * 128 + (((g ^ r) & 7) << 4);
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t a) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(a) : "memory");
}
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

struct BlCtl {
  volatile int* abort_flag;
  const BasedLinearArgs* a;
};
// Bounded wait; false on time-out (which starts the CTA's abort) or once another
// thread has started it (unless honor_abort is false, as in the teardown).
__device__ __forceinline__ bool bl_wait(uint32_t bar, uint32_t parity, const BlCtl& c, bool honor_abort = true) {
  for (int i = 0; i < 128; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honor_abort && *c.abort_flag) return false;
    if (globaltimer_ns() - t0 > c.a->timeout_ns) {
      *c.abort_flag = 1;
      atomicCAS(c.a->err, 0, bl::kStatusTimeout);
      return false;
    }
  }
}

// The same wait taken by a whole warp: true only if every lane's wait succeeded, so
// that the warp-collective tensor-memory loads that follow run converged.
__device__ __forceinline__ bool bl_warp_wait(uint32_t bar, uint32_t parity, const BlCtl& c) {
  const bool ok = bl_wait(bar, parity, c);
  return __all_sync(0xffffffffu, ok);
}

// Row t of phi(u) (internal order) into the K-major feature operand; `keep` = 0
// writes a zero row (tokens past the end of the sequence).
__device__ __forceinline__ void write_phi_row(uint32_t phi, int t, const float* u, float c2, float rs, bool keep) {
  using namespace bl;
#pragma unroll
  for (int a = 0; a < kDK; ++a) {
    const float ca = keep ? c2 * u[a] : 0.f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float* ub = u + 8 * h;
      sts128(gran(phi + (a >> 2) * kCh, t, (a & 3) * 2 + h), pack_bf16x2(ca * ub[0], ca * ub[1]),
             pack_bf16x2(ca * ub[2], ca * ub[3]), pack_bf16x2(ca * ub[4], ca * ub[5]),
             pack_bf16x2(ca * ub[6], ca * ub[7]));
    }
  }
  const float r = keep ? rs : 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float* ub = u + 8 * h;
    sts128(gran(phi + 4 * kCh, t, h), pack_bf16x2(r * ub[0], r * ub[1]), pack_bf16x2(r * ub[2], r * ub[3]),
           pack_bf16x2(r * ub[4], r * ub[5]), pack_bf16x2(r * ub[6], r * ub[7]));
  }
  sts128(gran(phi + 4 * kCh, t, 2), keep ? 0x3F80u : 0u, 0u, 0u, 0u);   // the constant feature (1.0)
}

__device__ __forceinline__ void unpack16(const uint4& lo, const uint4& hi, float* u) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    u[2 * i] = bf_lo(w[i]);
    u[2 * i + 1] = bf_hi(w[i]);
  }
}

// Internal feature row -> position in the state layout [1, linear (16), products (256)].
__device__ __forceinline__ int abi_feature(int f) { return f < 256 ? 17 + f : (f < 272 ? 1 + (f - 256) : 0); }

__global__ void __launch_bounds__(bl::kThreads, 1)
    swa_based_linear_tc_kernel(const __grid_constant__ BasedLinearArgs a) {
  using namespace bl;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  auto bar = [&](int i) { return base + OFF_BAR + 8u * i; };
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(gbase + OFF_TMEMPTR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + OFF_ABORT);
  const BlCtl ctl{abort_flag, &a};

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x, b = bh / a.H, h = bh % a.H;
  const int nc = (a.L + kChunk - 1) / kChunk;

  // zero the feature operand (its padding stays zero), S_bf16 (features past 272
  // stay zero) and the ones chunk of V1, then put the ones in place
  for (uint32_t o = tid * 16; o < 6 * kCh; o += kThreads * 16) sts128(base + OFF_PHI + o, 0, 0, 0, 0);
  for (uint32_t o = tid * 16; o < 6 * kSbCh; o += kThreads * 16) sts128(base + OFF_SB + o, 0, 0, 0, 0);
  for (uint32_t o = tid * 16; o < kCh; o += kThreads * 16) sts128(base + OFF_V1 + kCh + o, 0, 0, 0, 0);
  __syncthreads();
  if (tid < kChunk) sts32(gran(base + OFF_V1 + kCh, tid, 0), 0x3F80u);   // column 64 of V1 = 1.0
  fence_proxy_async_smem();
  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(bar(i), (i == B_PHIQ || i == B_V1 || i == B_P || i == B_PHIK ||
                                                          i == B_OFREE || i == B_SB) ? 128 : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_ptr), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const float c2 = a.scale * 0.70710678118654752f, rs = sqrtf(a.scale);

  if (warp < 4) {
    // ---------------------------------------------------------------- token rows
    const int t = tid;                                   // row of the chunk = tensor-memory lane
    const uint32_t lane_t = static_cast<uint32_t>(warp * 32) << 16;
    const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(a.q);
    const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(a.k);
    auto load_qk = [&](int i, uint4* r) {
      const int tok = i * kChunk + t;
      if (i < nc && tok < a.L) {
        const long long row = (static_cast<long long>(b) * a.L + tok) * a.H + h;
        const uint4* pq = reinterpret_cast<const uint4*>(qg + row * kDK);
        const uint4* pk = reinterpret_cast<const uint4*>(kg + row * kDK);
        r[0] = __ldg(pq);
        r[1] = __ldg(pq + 1);
        r[2] = __ldg(pk);
        r[3] = __ldg(pk + 1);
      } else {
        r[0] = r[1] = r[2] = r[3] = make_uint4(0, 0, 0, 0);
      }
    };
    uint4 cur[4], nxt[4];
    load_qk(0, cur);
    bool ok = true;
    for (int i = 0; i < nc && ok; ++i) {
      const int n = min(kChunk, a.L - i * kChunk);
      load_qk(i + 1, nxt);
      float u[16];
      // phi(Q) and phi_lin(K) once the previous chunk's MMAs are done with the operand
      if (i > 0 && !(ok = bl_warp_wait(bar(B_SFULL), (i - 1) & 1, ctl))) break;
      unpack16(cur[0], cur[1], u);
      write_phi_row(base + OFF_PHI, t, u, c2, rs, true);
      unpack16(cur[2], cur[3], u);
      {
        const bool keep = t < n;
        const float r = keep ? rs : 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const float* ub = u + 8 * hh;
          sts128(gran(base + OFF_KLIN, t, hh), pack_bf16x2(r * ub[0], r * ub[1]), pack_bf16x2(r * ub[2], r * ub[3]),
                 pack_bf16x2(r * ub[4], r * ub[5]), pack_bf16x2(r * ub[6], r * ub[7]));
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(B_PHIQ));
      // kappa(X) with the causal mask -> P (bf16 pairs over X's first 64 columns)
      if (!(ok = bl_warp_wait(bar(B_X), i & 1, ctl))) break;
      __syncwarp();
      tc_fence_after();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t xr[64], pr[32];
        tmem_ld32_wait(tmem + lane_t + T_X + 64 * half, xr);
        tmem_ld32_wait(tmem + lane_t + T_X + 64 * half + 32, xr + 32);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int s0 = 64 * half + 2 * j;
          const float x0 = __uint_as_float(xr[2 * j]), x1 = __uint_as_float(xr[2 * j + 1]);
          const float k0 = s0 <= t ? fmaf(x0, fmaf(0.5f, x0, 1.f), 1.f) : 0.f;
          const float k1 = s0 + 1 <= t ? fmaf(x1, fmaf(0.5f, x1, 1.f), 1.f) : 0.f;
          pr[j] = pack_bf16x2(k0, k1);
        }
        tmem_st32(tmem + lane_t + T_X + 32 * half, pr);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(B_P));
      // phi(K) over phi(Q) once O = phi(Q) S_bf16 has read it
      if (!(ok = bl_warp_wait(bar(B_O1), i & 1, ctl))) break;
      write_phi_row(base + OFF_PHI, t, u, c2, rs, t < n);
      fence_proxy_async_smem();
      mbar_arrive(bar(B_PHIK));
      // epilogue: out = O[:, :64] / O[:, 64]
      if (!(ok = bl_warp_wait(bar(B_OFULL), i & 1, ctl))) break;
      __syncwarp();
      tc_fence_after();
      uint32_t orr[96];
      tmem_ld32_wait(tmem + lane_t + T_O, orr);
      tmem_ld32_wait(tmem + lane_t + T_O + 32, orr + 32);
      tmem_ld32_wait(tmem + lane_t + T_O + 64, orr + 64);
      tc_fence_before();
      mbar_arrive(bar(B_OFREE));
      if (t < n) {
        const float inv = 1.0f / __uint_as_float(orr[64]);
        const long long row = (static_cast<long long>(b) * a.L + i * kChunk + t) * a.H + h;
        if (a.out_f32) {
          float4* o = reinterpret_cast<float4*>(static_cast<float*>(a.out) + row * kDV);
#pragma unroll
          for (int c = 0; c < 16; ++c)
            o[c] = make_float4(__uint_as_float(orr[4 * c]) * inv, __uint_as_float(orr[4 * c + 1]) * inv,
                               __uint_as_float(orr[4 * c + 2]) * inv, __uint_as_float(orr[4 * c + 3]) * inv);
        } else {
          uint4* o = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + row * kDV);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t* w = orr + 8 * c;
            o[c] = make_uint4(pack_bf16x2(__uint_as_float(w[0]) * inv, __uint_as_float(w[1]) * inv),
                              pack_bf16x2(__uint_as_float(w[2]) * inv, __uint_as_float(w[3]) * inv),
                              pack_bf16x2(__uint_as_float(w[4]) * inv, __uint_as_float(w[5]) * inv),
                              pack_bf16x2(__uint_as_float(w[6]) * inv, __uint_as_float(w[7]) * inv));
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) cur[j] = nxt[j];
    }
  } else if (warp < 8) {
    // ---------------------------------------------------------------- state
    const int r = tid - 128;                             // token row for V loads
    const int w = warp - 4;                              // tensor-memory lane quarter
    const uint32_t lane_t = static_cast<uint32_t>(w * 32) << 16;
    const __nv_bfloat16* vg = static_cast<const __nv_bfloat16*>(a.v);
    auto load_v = [&](int i, uint4* dst) {
      const int tok = i * kChunk + r;
      if (i < nc && tok < a.L) {
        const uint4* pv = reinterpret_cast<const uint4*>(
            vg + ((static_cast<long long>(b) * a.L + tok) * a.H + h) * kDV);
#pragma unroll
        for (int g = 0; g < 8; ++g) dst[g] = __ldg(pv + g);
      } else {
#pragma unroll
        for (int g = 0; g < 8; ++g) dst[g] = make_uint4(0, 0, 0, 0);
      }
    };
    uint4 vr[8];
    load_v(0, vr);
    bool ok = true;
    for (int i = 0; i < nc && ok; ++i) {
      if (i > 0) {
        if (!(ok = bl_warp_wait(bar(B_SFULL), (i - 1) & 1, ctl))) break;
        __syncwarp();
        tc_fence_after();
      }
      // this chunk's values into V1 (the previous chunk's MMAs are done with it)
#pragma unroll
      for (int g = 0; g < 8; ++g) sts128(gran(base + OFF_V1, r, g), vr[g].x, vr[g].y, vr[g].z, vr[g].w);
      fence_proxy_async_smem();
      mbar_arrive(bar(B_V1));
      load_v(i + 1, vr);
      if (i > 0) {
        // S after chunk i-1 -> S_bf16, the K-major B operand [80 x 384] of phi(Q) S:
        // thread = feature row f; lanes f, f^1 swap values so that each stores a pair
        const bool odd = lane & 1;
#pragma unroll 1
        for (int j = 0; j < 3; ++j) {
          if (j == 2 && w > 0) break;                    // features 288 .. 383 are zero
          const int f = 128 * j + 32 * w + lane;
          uint32_t sr[96];
          tmem_ld32_wait(tmem + lane_t + T_S + 80 * j, sr);
          tmem_ld32_wait(tmem + lane_t + T_S + 80 * j + 32, sr + 32);
          tmem_ld32_wait(tmem + lane_t + T_S + 80 * j + 64, sr + 64);
          const int fe = (f & ~1) & 63;                  // even feature of the pair, within its chunk
          const uint32_t cb = base + OFF_SB + (f >> 6) * kSbCh;
#pragma unroll
          for (int m = 0; m < kNV / 2; ++m) {
            const float mine0 = __uint_as_float(sr[2 * m]), mine1 = __uint_as_float(sr[2 * m + 1]);
            const float other = __shfl_xor_sync(0xffffffffu, odd ? mine0 : mine1, 1);
            const int row = 2 * m + (odd ? 1 : 0);
            const uint32_t val = odd ? pack_bf16x2(other, mine1) : pack_bf16x2(mine0, other);
            sts32(cb + row * 128 + ((((fe >> 3) ^ row) & 7) << 4) + (fe & 7) * 2, val);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(B_SB));
      }
    }
    // final state, in the layout [1, linear, products] x (64 values | z)
    if (ok && a.state != nullptr) {
      const long long sb = static_cast<long long>(bh) * kF;
      if (nc == 0) {
        for (int f = r; f < kF; f += 128) {
          float4* dst = reinterpret_cast<float4*>(a.state + (sb + f) * kDV);
#pragma unroll
          for (int c = 0; c < 16; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
          a.zsum[sb + f] = 0.f;
        }
      } else if (bl_warp_wait(bar(B_SFULL), (nc - 1) & 1, ctl)) {
        __syncwarp();
        tc_fence_after();
#pragma unroll 1
        for (int j = 0; j < 3; ++j) {
          if (j == 2 && w > 0) break;
          const int f = 128 * j + 32 * w + lane;
          uint32_t sr[96];
          tmem_ld32_wait(tmem + lane_t + T_S + 80 * j, sr);
          tmem_ld32_wait(tmem + lane_t + T_S + 80 * j + 32, sr + 32);
          tmem_ld32_wait(tmem + lane_t + T_S + 80 * j + 64, sr + 64);
          if (f < kF) {
            const long long fa = sb + abi_feature(f);
            float4* dst = reinterpret_cast<float4*>(a.state + fa * kDV);
#pragma unroll
            for (int c = 0; c < 16; ++c)
              dst[c] = make_float4(__uint_as_float(sr[4 * c]), __uint_as_float(sr[4 * c + 1]),
                                   __uint_as_float(sr[4 * c + 2]), __uint_as_float(sr[4 * c + 3]));
            a.zsum[fa] = __uint_as_float(sr[64]);
          }
        }
      }
    }
  } else {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && (a.debug_flags & 1) == 0) {
      bool ok = true;
      for (int i = 0; i < nc && ok; ++i) {
        if (!(ok = bl_wait(bar(B_PHIQ), i & 1, ctl))) break;
        if (!(ok = bl_wait(bar(B_V1), i & 1, ctl))) break;
        if (i > 0) {
          if (!(ok = bl_wait(bar(B_SB), (i - 1) & 1, ctl))) break;
          if (!(ok = bl_wait(bar(B_OFREE), (i - 1) & 1, ctl))) break;
        }
        tc_fence_after();
        // X = phi_lin(Q) phi_lin(K)^T: features 256 .. 271 of phi(Q), columns 0 .. 15 of phi_lin(K)
        umma_ss<false>(tmem + T_X, bl_kdesc(base + OFF_PHI, kCh, 16), bl_kdesc(base + OFF_KLIN, kCh, 0), IDESC_X, 0u);
        tc_commit(bar(B_X));
        if (i > 0) {
#pragma unroll 1
          for (int kk = 0; kk < kQSteps; ++kk)
            umma_ss<false>(tmem + T_O, bl_kdesc(base + OFF_PHI, kCh, kk), bl_kdesc(base + OFF_SB, kSbCh, kk),
                           IDESC_QS, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_O1));
        if (!(ok = bl_wait(bar(B_P), i & 1, ctl))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          umma_ts<false>(tmem + T_O, tmem + T_X + kk * 8, bl_mndesc(base + OFF_V1, kCh, kk), IDESC_PV,
                         (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(B_OFULL));
        if (!(ok = bl_wait(bar(B_PHIK), i & 1, ctl))) break;
        tc_fence_after();
#pragma unroll 1
        for (int j = 0; j < 3; ++j)
#pragma unroll
          for (int kk = 0; kk < kChunk / 16; ++kk)
            umma_ss<false>(tmem + T_S + 80 * j, bl_mndesc(base + OFF_PHI + 2 * j * kCh, kCh, kk),
                           bl_mndesc(base + OFF_V1, kCh, kk), IDESC_KV, (i > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(B_SFULL));
      }
      // let every issued MMA finish before the tensor memory is freed
      tc_commit(bar(B_DRAIN));
      bl_wait(bar(B_DRAIN), 0, ctl, false);
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace

cudaError_t launch_based_linear_fwd(const BasedLinearArgs& a, cudaStream_t stream) {
  if (a.debug_flags & 8) return launch_based_linear_fwd_simt(a, stream);
  cudaError_t e = cudaFuncSetAttribute(swa_based_linear_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(bl::kSmem));
  if (e != cudaSuccess) return e;
  swa_based_linear_tc_kernel<<<a.B * a.H, bl::kThreads, bl::kSmem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace swa
